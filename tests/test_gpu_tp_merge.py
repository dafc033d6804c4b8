"""The statistics-merge form of the vocabulary-parallel forward, on one GPU:
the shards' stages run one after another and their records are combined with
torch ops standing in for the collectives (max, sum, min, concatenation in
rank order), so no kernel waits on another. The merged result must take the
same support decisions as the unsharded forward (support size, cut id and
logit, flags) on every row it does not hand to the gather form, with logprobs
within float64 summation order; the plan must be the same on every rank; and
against the float64 oracle the usual contract holds."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import (bf16_tensor, compare_logprob, f32_values, near_gap_rows, row_tensors,
                     small_case)

pytestmark = pytest.mark.gpu

DECISIONS = ("support_size", "cut_id", "cut_logit", "flags")


def merge_emulated(sts, shards, V, meta):
    """The four stages of every shard with in-process combination."""
    Vl = shards[0].shape[1]
    m = torch.stack([sts.sts_tp_row_max(S) for S in shards]).max(0).values
    counts = torch.stack([sts.sts_tp_count(S, m) for S in shards]).sum(0, dtype=torch.int32)
    recs = [sts.sts_tp_exact(S, r * Vl, V, *meta, m, counts) for r, S in enumerate(shards)]
    for rec in recs[1:]:
        assert torch.equal(rec["plan"], recs[0]["plan"])  # every rank plans alike
    merged = {"plan": recs[0]["plan"],
              "sums": torch.stack([r["sums"] for r in recs]).sum(0),
              "keys": torch.stack([r["keys"] for r in recs]).min(0).values,
              "ylogit": torch.stack([r["ylogit"] for r in recs]).sum(0)}
    assert bool((merged["ylogit"][:, 1] == 1.0).all())  # the target's owner contributed once
    cand = torch.stack([r["cand"] for r in recs])
    ncand = torch.stack([r["ncand"] for r in recs])
    lp, saved, need, ws = sts.sts_tp_finish(V, *meta, m, merged["plan"], merged["sums"],
                                            merged["keys"], merged["ylogit"], cand, ncand)
    st, bad = sts.sts_get_status(ws)
    return lp, saved, need.bool(), st


def shard_logits(sts, Hd, Wd, tau, world):
    V = Wd.shape[0]
    vl = V // world
    return [sts.sts_scaled_logits(Hd, Wd[r * vl:(r + 1) * vl].contiguous(), tau).contiguous()
            for r in range(world)]


def check_against_forward(sts, Hd, Wd, meta, world, max_need=0):
    V = Wd.shape[0]
    lp0, saved0, _ = sts.sts_forward(Hd, Wd, *meta, check=True, entropy=True)  # float64 masses
    lp, saved, need, st = merge_emulated(sts, shard_logits(sts, Hd, Wd, meta[1], world), V, meta)
    assert st == 0
    keep = ~need
    assert int(need.sum()) <= max_need, int(need.sum())
    for key in DECISIONS:
        assert torch.equal(saved[key][keep], saved0[key][keep]), key
    assert torch.equal(saved["row_max"][keep], saved0["row_max"][keep])
    fin = torch.isfinite(lp0) & keep
    assert torch.equal(torch.isfinite(lp) & keep, fin)
    assert (lp[fin] - lp0[fin]).abs().max().item() < 1e-5
    assert (saved["lse_support"][keep] - saved0["lse_support"][keep]).abs().max().item() < 1e-5
    return lp, saved, need


@pytest.mark.parametrize("world", [2, 4])
def test_merge_matches_unsharded_forward(cuda_lib, world):
    sts = cuda_lib
    T, d, V = 300, 136, 4096
    H, W, meta, u = small_case(31, T, d, V, k_choices=(0, 1, 7, 50, 3000),
                               p_choices=(1.0, 0.95, 0.9, 0.5), mu_choices=(0.0, 0.05, 0.3))
    Hf, Wf = f32_values(H), f32_values(W)
    s = oracle.scaled_logits(Hf, Wf, meta["temperature"])
    y = oracle.sample_rows(s, dict(meta, target=np.zeros(T, np.int64)), u)
    rows = dict(meta, target=y)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    lp, saved, need = check_against_forward(sts, Hd, Wd, row_tensors(rows), world)
    # and the float64 oracle's contract
    ref = oracle.forward(Hf, Wf, rows, s=s)
    flagged = near_gap_rows(s, rows)
    n_bad, _, _ = compare_logprob(lp.cpu().numpy(), saved["support_size"].cpu().numpy(), s, rows,
                                  ref, flagged)
    assert n_bad == 0


def test_merge_identity_ties_and_invalid_rows(cuda_lib):
    """Identity rows, duplicated tokens (equal logits: the lower id first) and
    invalid metadata (NaN row, status word) through the merge."""
    sts = cuda_lib
    T, d, V = 140, 64, 2048
    H, W, meta, u = small_case(32, T, d, V, k_choices=(0, 5), p_choices=(1.0, 0.8),
                               mu_choices=(0.0, 0.1))
    W[1024:1536] = W[0:512]  # every token of the second quarter duplicates one of the first
    meta["top_k"][::4] = 0
    meta["top_p"][::4] = 1.0
    meta["min_p"][::4] = 0.0
    y = np.random.Generator(np.random.PCG64(3)).integers(0, V, T)
    rows = dict(meta, target=y)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    check_against_forward(sts, Hd, Wd, row_tensors(rows), 2)
    bad = dict(rows, top_p=rows["top_p"].copy())
    bad["top_p"][5] = 0.0
    meta_t = row_tensors(bad)
    lp, saved, need, st = merge_emulated(sts, shard_logits(sts, Hd, Wd, meta_t[1], 2), V, meta_t)
    assert st != 0 and torch.isnan(lp[5]) and int(saved["flags"][5]) & 2
    others = torch.ones(T, dtype=torch.bool, device="cuda")
    others[5] = False
    lp0, saved0, _ = sts.sts_forward(Hd, Wd, *row_tensors(rows), entropy=True)
    assert torch.equal(saved["cut_id"][others], saved0["cut_id"][others])


@pytest.mark.parametrize("index", [4, 5])
def test_merge_full_vocabulary(cuda_lib, index):
    """128 rows of workload 4 / 5 at their full vocabulary over 2 shards: flat
    rows with wide top-p brackets and top-k = 1 / duplicated-token rows. Rows
    whose bracket exceeds one sort go to the gather form (counted)."""
    sts = cuda_lib
    data = workloads.make(index, T=128)
    rows = dict({k: data[k] for k in ("temperature", "top_k", "top_p", "min_p")},
                target=np.random.Generator(np.random.PCG64(5)).integers(0, data["W"].shape[0], 128))
    Hd, Wd = bf16_tensor(data["H"]), bf16_tensor(data["W"])
    _, _, need = check_against_forward(sts, Hd, Wd, row_tensors(rows), 2, max_need=128)
    print(f"workload {index}: {int(need.sum())} of 128 rows handed to the gather form")


def test_vocab_parallel_merge_single_rank_nccl(cuda_lib):
    """VocabParallel's merge over a one-rank NCCL group: the decisions of
    sts_forward (fp32-mass mode, as both skip the entropy), logprob within the
    fp32 mass bound."""
    import datetime
    import socket

    import torch.distributed as dist

    from helpers import assert_same_decisions
    from sampling_transform_lm_b200.tp import VocabParallel

    sts = cuda_lib
    T, d, V = 300, 64, 2048
    H, W, meta, u = small_case(33, T, d, V)
    rows = dict(meta, target=np.random.Generator(np.random.PCG64(6)).integers(0, V, T))
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp0, saved0, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, check=True)
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        tp = VocabParallel(row_chunk=128)
        lp, saved = tp.forward(Hd, Wd, y, tau, k, p, mu)
        g = torch.ones(T, dtype=torch.float32, device="cuda")
        dH, dW = tp.backward(Hd, Wd, y, tau, k, p, mu, saved, g)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert_same_decisions(lp0, saved0, lp, saved)
    dH0, dW0 = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved0, g, check=True)
    assert torch.allclose(dH, dH0, rtol=1e-4, atol=1e-6) and torch.allclose(dW, dW0, rtol=1e-4,
                                                                              atol=1e-6)

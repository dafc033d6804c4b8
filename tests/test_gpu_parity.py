"""End-to-end parity of sts_forward / sts_backward / sts_sample with the
float64 oracle, through the C ABI, on seeded inputs that span several tiles
and ragged tails, plus the edge cases of the method."""

import math
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads
from sampling_transform_lm_b200.dp import SliceAllReduce
from helpers import (GRAD_RTOL, assert_same_decisions, bf16_tensor, compare_logprob, f32_values,
                     grad_rows, near_gap_rows, rel_fro, row_tensors, small_case)

pytestmark = pytest.mark.gpu

ENT_ATOL = 1e-3  # entropy from fp32-accumulated logits against float64 ones


def _run(sts, H, W, rows, grad=None, row_chunk=0, vocab_chunk=0):
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp, saved, ws = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, row_chunk=row_chunk, entropy=True)
    status, bad = sts.sts_get_status(ws)
    # the same rows without the entropy output take fp32 masses where no mass
    # comparison decides: identical decisions, logprob within the mass bound
    lp2, saved2, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, row_chunk=row_chunk)
    assert_same_decisions(lp, saved, lp2, saved2)
    out = {"logprob": lp.cpu().numpy(), "saved": {k_: v.cpu().numpy() for k_, v in saved.items()},
           "status": status, "bad_row": bad}
    if grad is not None:
        g = torch.from_numpy(np.asarray(grad, np.float32)).cuda()
        dH, dW = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved, g, vocab_chunk=vocab_chunk,
                                  check=True)
        out["dH"] = dH.cpu().numpy()
        out["dW"] = dW.cpu().numpy()
    return out


def _oracle_case(H, W, rows_meta, u):
    Hf, Wf = f32_values(H), f32_values(W)
    s = oracle.scaled_logits(Hf, Wf, rows_meta["temperature"])
    y = oracle.sample_rows(s, dict(rows_meta, target=np.zeros(len(u), np.int64)), u)
    rows = dict(rows_meta, target=y)
    return Hf, Wf, s, rows


def _check_forward(sts_out, s, rows, ref):
    """Forward contract; returns the rows whose gradients are comparable."""
    flagged = near_gap_rows(s, rows)
    size = sts_out["saved"]["support_size"]
    bad, ndiff, max_err = compare_logprob(sts_out["logprob"], size, s, rows, ref, flagged)
    print(f"{len(flagged)} rows, logprob compared on all (max |dlogprob| {max_err:.2e}); "
          f"{int(flagged.sum())} near-gap, {ndiff} of them with another valid support size")
    assert sts_out["status"] == 0
    assert bad == 0, (bad, ndiff, max_err)
    # entropy of the filtered distribution on the GPU's support
    ent = oracle.entropy(s, rows, sizes=size)
    np.testing.assert_allclose(sts_out["saved"]["entropy"], ent, rtol=0, atol=ENT_ATOL)
    # gradients are comparable where the support is the oracle's
    return grad_rows(sts_out["saved"]["flags"], ref["in_support"]) & (size == ref["size"])


@pytest.mark.parametrize("grad_kind", ["ones", "normal"])
def test_workload1_forward_backward(cuda_lib, grad_kind):
    """The tiny oracle-check workload (T=64, d=128, V=1024): every row."""
    data = workloads.make(1)
    meta = {k: data[k] for k in ("temperature", "top_k", "top_p", "min_p")}
    Hf, Wf, s, rows = _oracle_case(data["H"], data["W"], meta, data["u"])
    g = data["g"] if grad_kind == "ones" else workloads.extra_grad(1, 64)
    ref = oracle.forward(Hf, Wf, rows, s=s)
    fwd = _run(cuda_lib, data["H"], data["W"], rows)
    same = _check_forward(fwd, s, rows, ref)
    gm = np.where(same, g, 0.0).astype(np.float32)
    out = _run(cuda_lib, data["H"], data["W"], rows, grad=gm)
    dH, dW = oracle.backward(Hf, Wf, rows, gm, s=s)
    assert rel_fro(out["dH"], dH) < GRAD_RTOL
    assert rel_fro(out["dW"], dW) < GRAD_RTOL


@pytest.mark.parametrize("seed,T,d,V", [(1, 300, 136, 1000), (2, 257, 256, 4100), (3, 130, 64, 5)])
def test_ragged_shapes_forward_backward(cuda_lib, seed, T, d, V):
    H, W, meta, u = small_case(seed, T, d, V, k_choices=(0, 1, 3, 50), p_choices=(1.0, 0.9, 0.6),
                               mu_choices=(0.0, 0.05, 0.2))
    Hf, Wf, s, rows = _oracle_case(H, W, meta, u)
    g = np.random.Generator(np.random.PCG64(seed)).standard_normal(T).astype(np.float32)
    ref = oracle.forward(Hf, Wf, rows, s=s)
    same = _check_forward(_run(cuda_lib, H, W, rows), s, rows, ref)
    gm = np.where(same, g, 0.0).astype(np.float32)
    out = _run(cuda_lib, H, W, rows, grad=gm)
    dH, dW = oracle.backward(Hf, Wf, rows, gm, s=s)
    assert rel_fro(out["dH"], dH) < GRAD_RTOL
    assert rel_fro(out["dW"], dW) < GRAD_RTOL


def test_chunking_does_not_change_results(cuda_lib):
    """Several forward row chunks and backward vocab chunks (ragged last chunk)
    give the same logprobs and cuts bit for bit, dW bit for bit, dH to fp32
    reduction order."""
    sts = cuda_lib
    T, d, V = 300, 128, 1000
    H, W, meta, u = small_case(9, T, d, V)
    rows = dict(meta, target=np.zeros(T, np.int64))
    g = np.ones(T, np.float32)
    a = _run(sts, H, W, rows, grad=g)
    b = _run(sts, H, W, rows, grad=g, row_chunk=128, vocab_chunk=256)
    assert np.array_equal(a["logprob"], b["logprob"])
    for key in ("support_size", "cut_id", "cut_logit", "lse_support", "flags"):
        assert np.array_equal(a["saved"][key], b["saved"][key]), key
    assert np.array_equal(a["dW"], b["dW"])
    assert rel_fro(b["dH"], a["dH"]) < 1e-5  # fp32 reduce-add across chunks vs one K loop


def test_identity_rows_match_plain_softmax(cuda_lib):
    """Identity metadata is the plain temperature log-softmax of the GPU's own
    fp32 logits ('Testing': identity metadata collapses to the untouched path)."""
    sts = cuda_lib
    T, d, V = 256, 256, 3000
    H, W, meta, u = small_case(11, T, d, V, k_choices=(0, V, -1), p_choices=(1.0,), mu_choices=(0.0,))
    y = np.random.Generator(np.random.PCG64(5)).integers(0, V, T)
    rows = dict(meta, target=y)
    out = _run(sts, H, W, rows)
    S = sts.sts_scaled_logits(bf16_tensor(H), bf16_tensor(W),
                              torch.from_numpy(meta["temperature"]).cuda()).double()
    plain = (S[torch.arange(T), torch.from_numpy(y).cuda()] - torch.logsumexp(S, dim=1)).cpu().numpy()
    assert np.abs(out["logprob"] - plain).max() < 1e-5
    assert (out["saved"]["support_size"] == V).all()
    assert ((out["saved"]["flags"] & 4) != 0).all()


def test_forward_cuts_equal_filter_hook_on_own_logits(cuda_lib):
    """The forward's resolver and the filter hook agree exactly on the GPU's
    own fp32 logits, and the oracle filter on those same fp32 logits agrees
    with both (the bit-exact contract)."""
    sts = cuda_lib
    T, d, V = 200, 192, 6000
    H, W, meta, u = small_case(12, T, d, V, k_choices=(0, 1, 20, 700), p_choices=(1.0, 0.95, 0.5),
                               mu_choices=(0.0, 0.02, 0.3))
    rows = dict(meta, target=np.zeros(T, np.int64))
    out = _run(sts, H, W, rows)
    S = sts.sts_scaled_logits(bf16_tensor(H), bf16_tensor(W), torch.from_numpy(meta["temperature"]).cuda())
    _, k, p, mu = row_tensors(rows)[1:]
    hook = sts.sts_filter_logits(S.contiguous(), k, p, mu, check=True)
    assert np.array_equal(hook["size"].cpu().numpy(), out["saved"]["support_size"])
    assert np.array_equal(hook["cut_id"].cpu().numpy(), out["saved"]["cut_id"])
    Sn = S.cpu().numpy()
    ref = oracle.filter_rows(Sn, rows)
    gaps = oracle.row_gaps(Sn, rows).min(axis=1)
    mism = (ref["size"] != out["saved"]["support_size"]) & (gaps > 1e-12)
    assert not mism.any(), np.flatnonzero(mism)
    assert np.array_equal(ref["row_max"].astype(np.float32), out["saved"]["row_max"])


def test_sampler_matches_oracle_inverse_cdf(cuda_lib):
    sts = cuda_lib
    T, d, V = 256, 128, 2000
    H, W, meta, u = small_case(13, T, d, V, k_choices=(0, 1, 10, 500), p_choices=(1.0, 0.9, 0.5),
                               mu_choices=(0.0, 0.05))
    _, tau, k, p, mu = row_tensors(dict(meta, target=np.zeros(T, np.int64)))
    y = sts.sts_sample(bf16_tensor(H), bf16_tensor(W), tau, k, p, mu,
                       torch.from_numpy(u).cuda(), check=True).cpu().numpy()
    S = sts.sts_scaled_logits(bf16_tensor(H), bf16_tensor(W), tau).cpu().numpy()
    rows = dict(meta, target=np.zeros(T, np.int64))
    ref = oracle.sample_rows(S, rows, u)
    gaps = oracle.row_gaps(S, rows).min(axis=1)
    mism = (y != ref) & (gaps > 1e-9)
    assert mism.sum() <= 1, np.flatnonzero(mism)  # a draw landing within rounding of a CDF step
    # every draw lies inside its row's support
    f = oracle.filter_rows(S, rows, want_mask=True)
    assert f["mask"][np.arange(T), y].all()


def test_out_of_support_target_scores_minus_inf_with_zero_grad(cuda_lib):
    """'What this PR does', item 4."""
    sts = cuda_lib
    T, d, V = 128, 64, 512
    H, W, meta, u = small_case(14, T, d, V, k_choices=(1,), p_choices=(1.0,), mu_choices=(0.0,))
    S = sts.sts_scaled_logits(bf16_tensor(H), bf16_tensor(W), torch.from_numpy(meta["temperature"]).cuda())
    S = S.cpu().numpy()
    top = np.argmax(S, axis=1)
    y = np.where(np.arange(T) % 2 == 0, top, (top + 1) % V)
    rows = dict(meta, target=y)
    out = _run(sts, H, W, rows, grad=np.ones(T, np.float32))
    lp = out["logprob"]
    assert (lp[0::2] == 0.0).all()  # single-token support, the target is it
    assert np.isneginf(lp[1::2]).all()
    assert (out["dH"][1::2] == 0).all() and (out["dH"][0::2] == 0).all()  # p = onehot -> zero
    assert not out["dW"].any()


def test_invalid_rows_report_status_and_stay_isolated(cuda_lib):
    sts = cuda_lib
    T, d, V = 8, 64, 300
    H, W, meta, u = small_case(15, T, d, V, k_choices=(0,), p_choices=(1.0,), mu_choices=(0.0,))
    y = np.arange(T, dtype=np.int64)
    meta["temperature"][2] = 0.0          # STS_ERR_TEMPERATURE
    meta["top_p"][4] = 1.5                 # STS_ERR_TOP_P
    meta["min_p"][5] = -0.5                # STS_ERR_MIN_P
    y[6] = V                               # STS_ERR_TARGET
    meta["temperature"][7] = float("nan")  # STS_ERR_TEMPERATURE
    rows = dict(meta, target=y)
    out = _run(sts, H, W, rows)
    assert (out["status"], out["bad_row"]) == (4, 2)
    lp = out["logprob"]
    bad = [2, 4, 5, 6, 7]
    assert np.isnan(lp[bad]).all()
    good = [0, 1, 3]
    assert np.isfinite(lp[good]).all()
    assert ((out["saved"]["flags"][bad] & 2) != 0).all()
    # the backward leaves invalid rows out
    y2, tau, k, p, mu = row_tensors(rows)
    y2[6] = 0
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    lp2, saved, _ = sts.sts_forward(Hd, Wd, y2, tau, k, p, mu)
    dH, dW = sts.sts_backward(Hd, Wd, y2, tau, k, p, mu, saved, torch.ones(T, device="cuda"))
    assert (dH[[2, 4, 5, 7]] == 0).all()
    assert torch.isfinite(dW).all()


def test_accumulate_dw(cuda_lib):
    sts = cuda_lib
    T, d, V = 256, 128, 700
    H, W, meta, u = small_case(16, T, d, V)
    rows = dict(meta, target=np.zeros(T, np.int64))
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp, saved, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu)
    g = torch.ones(T, device="cuda")
    _, dW = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved, g)
    base = torch.full((V, d), 0.5, device="cuda")
    _, acc = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved, g, dW=base.clone(), accumulate_dW=True)
    assert torch.allclose(acc, dW + 0.5, atol=1e-6, rtol=0)


def test_single_token_vocab(cuda_lib):
    sts = cuda_lib
    T, d, V = 3, 8, 1
    H, W, meta, u = small_case(17, T, d, V, k_choices=(0, 1), p_choices=(1.0, 0.5), mu_choices=(0.0, 1.0))
    rows = dict(meta, target=np.zeros(T, np.int64))
    out = _run(sts, H, W, rows, grad=np.ones(T, np.float32))
    assert (out["logprob"] == 0).all()
    assert not out["dH"].any() and not out["dW"].any()


def test_workload2_forward_all_rows(cuda_lib):
    """T=4096, d=2048, V=32768, rows split in thirds top_k=20 / top_p=0.95 /
    min_p=0.1; forward only; every row against the oracle."""
    data = workloads.make(2)
    meta = {k: data[k] for k in ("temperature", "top_k", "top_p", "min_p")}
    Hf, Wf, s, rows = _oracle_case(data["H"], data["W"], meta, data["u"])
    out = _run(cuda_lib, data["H"], data["W"], rows)
    ref = oracle.forward(Hf, Wf, rows, s=s)
    _check_forward(out, s, rows, ref)
    flagged = near_gap_rows(s, rows)
    print(f"workload 2: {int(flagged.sum())} near-gap rows of {len(flagged)}")


@pytest.mark.parametrize("objective", ["cispo", "clipped"])
def test_policy_grad_matches_oracle(cuda_lib, objective):
    """The policy-gradient coefficient, elementwise against the oracle."""
    sts = cuda_lib
    rng = np.random.Generator(np.random.PCG64(40))
    T = 5003  # several blocks and a ragged tail
    lp = (-rng.exponential(2.0, T)).astype(np.float32)
    old = (lp + rng.normal(0.0, 0.4, T)).astype(np.float32)
    adv = rng.normal(0.0, 1.0, T).astype(np.float32)
    lp[::97] = -np.inf  # replayed token outside the support
    lp[5::211] = np.nan  # invalid rows
    adv[::13] = 0.0
    old[7::301] = np.nan  # a missing behaviour logprob: no signal
    adv[11::307] = np.inf  # a non-finite advantage: no signal
    old[3::401] = -1000.0  # the ratio overflows float64
    cu = lambda a: torch.from_numpy(a).cuda()
    got = sts.sts_policy_grad(cu(lp), cu(old), cu(adv), objective=objective, eps_low=0.2,
                              eps_high=0.28, scale=1.0 / T).cpu().numpy()
    ref = oracle.policy_grad(lp, old, adv, objective, np.float32(0.2), np.float32(0.28),
                             np.float32(1.0 / T))
    rr = np.exp(lp.astype(np.float64) - old)
    near = (np.abs(rr - (1 + np.float32(0.28))) < 1e-12) | (np.abs(rr - (1 - np.float32(0.2))) < 1e-12)
    assert not near.any()  # no clip decision rests on rounding
    np.testing.assert_allclose(got, ref, rtol=2e-7, atol=1e-30)
    assert (got[::97] == 0).all() and (got[5::211] == 0).all()
    assert (got[7::301] == 0).all() and (got[11::307] == 0).all()
    assert np.isfinite(got[3::401]).all() if objective == "cispo" else True
    with pytest.raises(sts.StsError):
        sts.sts_policy_grad(cu(lp), cu(old), cu(adv), objective="ppo")


def test_policy_gradient_through_the_backward(cuda_lib):
    """CISPO end to end on the tiny workload: the coefficient formed from the
    GPU's fresh logprobs drives the backward; dH and dW match the oracle's
    backward driven by the oracle's coefficient from its own logprobs."""
    data = workloads.make(1)
    meta = {k: data[k] for k in ("temperature", "top_k", "top_p", "min_p")}
    Hf, Wf, s, rows = _oracle_case(data["H"], data["W"], meta, data["u"])
    ref = oracle.forward(Hf, Wf, rows, s=s)
    rng = np.random.Generator(np.random.PCG64(41))
    T = len(rows["target"])
    old = (np.where(np.isfinite(ref["logprob"]), ref["logprob"], -5.0) + rng.normal(0, 0.3, T))
    old = old.astype(np.float32)
    adv = rng.normal(0.0, 1.0, T).astype(np.float32)
    fwd = _run(cuda_lib, data["H"], data["W"], rows)
    same = _check_forward(fwd, s, rows, ref)
    lp_gpu = torch.from_numpy(fwd["logprob"]).cuda()
    g = cuda_lib.sts_policy_grad(lp_gpu, torch.from_numpy(old).cuda(), torch.from_numpy(adv).cuda(),
                                 objective="cispo", eps_high=0.28, scale=1.0 / T).cpu().numpy()
    g_ref = oracle.policy_grad(ref["logprob"], old, adv, "cispo", 0.2, np.float32(0.28),
                               np.float32(1.0 / T))
    assert np.abs(g - g_ref)[same].max() <= 1e-2 * np.abs(g_ref).max()
    gm = np.where(same, g, 0.0).astype(np.float32)
    out = _run(cuda_lib, data["H"], data["W"], rows, grad=gm)
    dH, dW = oracle.backward(Hf, Wf, rows, np.where(same, g_ref, 0.0), s=s)
    assert rel_fro(out["dH"], dH) < GRAD_RTOL
    assert rel_fro(out["dW"], dW) < GRAD_RTOL


def test_sliced_backward_allreduce_single_rank(cuda_lib):
    """sts_backward_sliced through SliceAllReduce on a one-rank NCCL group:
    the hook sees every vocabulary slice once in increasing order, the result
    equals the plain backward bit for bit (a one-rank sum is the identity),
    and leaving SMs to the exchange does not change it either."""
    import datetime
    import socket

    import torch.distributed as dist

    sts = cuda_lib
    H, W, meta, u = small_case(21, 300, 136, 2500)
    Hf, Wf, s, rows = _oracle_case(H, W, meta, u)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp, saved, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, check=True)
    g = torch.ones(300, dtype=torch.float32, device="cuda")
    dH0, dW0 = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved, g, vocab_chunk=512, check=True)
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        red = SliceAllReduce()
        dH1, dW1 = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved, g, vocab_chunk=512,
                                    on_dw_slice=red, comm_sms=16, check=True)
        order = red.finish()
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert order == [(v0, min(512, 2500 - v0)) for v0 in range(0, 2500, 512)]
    assert torch.equal(dW1, dW0) and torch.equal(dH1, dH0)


def test_vocab_shards_reproduce_the_unsharded_path(cuda_lib):
    """Two vocabulary shards on one GPU, without collectives: the shards'
    logits (sts_scaled_logits) interleaved in rank order by
    sts_gather_vocab_shards equal the full projection bit for bit, the support
    program on them (sts_resolve_logits) gives sts_forward's logprob and saved
    scalars bit for bit, each shard's backward (sts_backward_shard) gives its
    rows of dW bit for bit, and the two partial dH add up to dH."""
    sts = cuda_lib
    T, d, V = 260, 136, 2 * 1280
    H, W, meta, u = small_case(23, T, d, V)
    Hf, Wf, s, rows = _oracle_case(H, W, meta, u)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp0, saved0, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, check=True, entropy=True)
    g = torch.from_numpy(np.asarray(workloads.extra_grad(23, T))).cuda()
    dH0, dW0 = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved0, g, vocab_chunk=512, check=True)
    vl = V // 2
    blocks = torch.stack([sts.sts_scaled_logits(Hd, Wd[r * vl:(r + 1) * vl].contiguous(), tau)
                          for r in range(2)])
    full = torch.empty((T, V), dtype=torch.float32, device="cuda")
    sts.sts_gather_vocab_shards(blocks.contiguous(), full)
    assert torch.equal(full, sts.sts_scaled_logits(Hd, Wd, tau))
    lp1, saved1, _ = sts.sts_resolve_logits(full, y, tau, k, p, mu, check=True, entropy=True)
    assert torch.equal(lp1, lp0)
    for key in ("row_max", "lse_support", "cut_logit", "cut_id", "support_size", "flags",
                "entropy"):
        assert torch.equal(saved1[key], saved0[key]), key
    parts = [sts.sts_backward_shard(Hd, Wd[r * vl:(r + 1) * vl].contiguous(), y, tau, k, p, mu,
                                    saved1, g, vocab_offset=r * vl, vocab_chunk=512, check=True)
             for r in range(2)]
    assert torch.equal(torch.cat([parts[0][1], parts[1][1]]), dW0)
    dH = parts[0][0] + parts[1][0]
    assert rel_fro(dH.cpu().numpy(), dH0.cpu().numpy()) < 1e-6


def test_vocab_parallel_single_rank_nccl(cuda_lib):
    """VocabParallel's gather form over a one-rank NCCL group (the collectives
    are the identity): the same logprobs, dH and dW as the unsharded path."""
    import datetime

    import torch.distributed as dist

    from sampling_transform_lm_b200.tp import VocabParallel

    sts = cuda_lib
    T, d, V = 300, 64, 1024
    H, W, meta, u = small_case(24, T, d, V)
    Hf, Wf, s, rows = _oracle_case(H, W, meta, u)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    y, tau, k, p, mu = row_tensors(rows)
    lp0, saved0, _ = sts.sts_forward(Hd, Wd, y, tau, k, p, mu, check=True)
    g = torch.ones(T, dtype=torch.float32, device="cuda")
    dH0, dW0 = sts.sts_backward(Hd, Wd, y, tau, k, p, mu, saved0, g, check=True)
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        tp = VocabParallel(row_chunk=128, mode="gather")
        lp, saved = tp.forward(Hd, Wd, y, tau, k, p, mu)
        dH, dW = tp.backward(Hd, Wd, y, tau, k, p, mu, saved, g)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(lp, lp0) and torch.equal(dW, dW0) and torch.equal(dH, dH0)

"""Host logic of the vocabulary-parallel path (VocabParallel), on CPU with two
gloo ranks and per-rank stand-ins for the kernels built from the float64
oracle, in both forms: the gather (the shards' logits gathered in rank order
reproduce the full rows) and the statistics merge (the collectives of every
stage in order -- max, sum, sum / min / sum, two all-gathers -- with stand-in
stages whose merged keys rebuild the rows, and rows handed to the gather form
where the merge flags them). Either way the support program gives the
unsharded oracle's logprobs, each rank keeps its own dW shard and the summed
dH equals the unsharded one. The library's kernels take the same steps in the
GPU tests."""

import math
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
for p in (ROOT, os.path.join(ROOT, "tests")):
    if p not in sys.path:
        sys.path.insert(0, p)

import oracle  # noqa: E402
from sampling_transform_lm_b200.tp import VocabParallel  # noqa: E402


class OracleOps:
    """Per-rank steps as float64 oracle calls on CPU tensors."""

    def empty(self, shape, like):
        return torch.empty(shape, dtype=torch.float32)

    def shard_logits(self, H, W_shard, temperature, t0, rows, out):
        s = oracle.scaled_logits(H[t0:t0 + rows].numpy(), W_shard.numpy(),
                                 temperature[t0:t0 + rows].numpy())
        out.copy_(torch.from_numpy(s.astype(np.float32)))

    def gather(self, blocks, out):
        world, _, vl = blocks.shape
        for k in range(world):
            out[:, k * vl:(k + 1) * vl] = blocks[k]

    def resolve(self, S, V, target, temperature, top_k, top_p, min_p, entropy):
        rows = {"target": target.numpy(), "temperature": temperature.numpy(),
                "top_k": top_k.numpy(), "top_p": top_p.numpy(), "min_p": min_p.numpy()}
        ref = oracle.forward(None, None, rows, s=S[:, :V].double().numpy())
        saved = {"S": S[:, :V].clone(), "size": torch.from_numpy(ref["size"])}
        return torch.from_numpy(ref["logprob"]), saved

    # statistics-merge stand-ins: each rank's "gathered keys" are all of its
    # keys, so the merged keys rebuild the full rows; every seventh row is
    # flagged for the gather form
    def row_max(self, local):
        return local.max(dim=1).values.clone()

    def count(self, local, m):
        f = (m[:, None].numpy() - local.numpy()).astype(np.float32) * np.float32(128.0)
        b = np.clip(np.floor(f), 0, 4095).astype(np.int64)
        out = np.zeros((local.shape[0], 4096), np.int32)
        for r in range(local.shape[0]):
            out[r] = np.bincount(b[r], minlength=4096)
        return torch.from_numpy(out)

    @staticmethod
    def _keys(vals, ids):
        u = vals.astype(np.float32).view(np.uint32).astype(np.uint64)
        u[u == 0x80000000] = 0
        k32 = np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000)
        return (k32 << np.uint64(32)) | (np.uint64(0xFFFFFFFF) - ids.astype(np.uint64))

    def sort_cap(self):
        return 8192

    def exact(self, local, vocab_offset, V, target, temperature, top_k, top_p, min_p, m, counts,
              cap):
        rows, vl = local.shape
        s = local.numpy()
        K = self._keys(s, np.arange(vocab_offset, vocab_offset + vl)[None, :].repeat(rows, 0))
        y = target.numpy()
        mine = (y >= vocab_offset) & (y < vocab_offset + vl)
        yl = np.zeros((rows, 2), np.float32)
        yl[mine, 0] = s[mine, y[mine] - vocab_offset]
        yl[mine, 1] = 1.0
        flip = np.uint64(1 << 63)
        return {"plan": torch.zeros((rows, 8), dtype=torch.int32),
                "sums": torch.from_numpy(np.exp(s.astype(np.float64) - m.numpy()[:, None].astype(
                    np.float64)).sum(1, keepdims=True).repeat(5, 1)),
                "keys": torch.from_numpy((K.min(1) ^ flip).view(np.int64)[:, None].repeat(2, 1)),
                "ylogit": torch.from_numpy(yl),
                "cand": torch.from_numpy(K.view(np.int64)),
                "ncand": torch.full((rows,), vl, dtype=torch.int32)}

    def finish(self, V, target, temperature, top_k, top_p, min_p, m, rec, cand, ncand):
        world, rows, cap = cand.shape
        assert (ncand.numpy() == cap).all() and world * cap == V
        K = cand.numpy().view(np.uint64).transpose(1, 0, 2).reshape(rows, V)
        k32 = (K >> np.uint64(32)).astype(np.uint32)
        u = np.where(k32 & 0x80000000, k32 & 0x7FFFFFFF, (~k32) & 0xFFFFFFFF).astype(np.uint32)
        ids = (np.uint64(0xFFFFFFFF) - (K & np.uint64(0xFFFFFFFF))).astype(np.int64)
        S = np.zeros((rows, V), np.float32)
        np.put_along_axis(S, ids, u.view(np.float32), axis=1)
        # the merged records hold each rank's contribution exactly once
        assert np.allclose(rec["ylogit"].numpy()[:, 1], 1.0)
        lp, saved = self.resolve(torch.from_numpy(S), V, target, temperature, top_k, top_p,
                                 min_p, False)
        need = torch.zeros(rows, dtype=torch.int32)
        need[::7] = 1
        lp = torch.where(need.bool(), torch.full_like(lp, float("nan")), lp)
        return lp, saved, need

    def backward_shard(self, H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad,
                       vocab_offset):
        rows = {"target": target.numpy(), "temperature": temperature.numpy(),
                "top_k": top_k.numpy(), "top_p": top_p.numpy(), "min_p": min_p.numpy()}
        dZ = oracle.logit_grad(saved["S"].double().numpy(), rows, grad.numpy())
        vl = W_shard.shape[0]
        dz = dZ[:, vocab_offset:vocab_offset + vl]
        return (torch.from_numpy(dz @ W_shard.double().numpy()),
                torch.from_numpy(dz.T @ H.double().numpy()))


def _case(T=300, d=24, V=512):
    rng = np.random.Generator(np.random.PCG64(17))
    H = rng.standard_normal((T, d)).astype(np.float32)
    W = (rng.standard_normal((V, d)) / math.sqrt(d)).astype(np.float32)
    meta = {"temperature": rng.uniform(0.5, 1.5, T).astype(np.float32),
            "top_k": rng.choice(np.array([0, 7, 50], np.int32), T).astype(np.int32),
            "top_p": rng.choice(np.array([1.0, 0.9, 0.6], np.float32), T).astype(np.float32),
            "min_p": rng.choice(np.array([0.0, 0.05], np.float32), T).astype(np.float32)}
    s = oracle.scaled_logits(H, W, meta["temperature"]).astype(np.float32)
    y = oracle.sample_rows(s.astype(np.float64), dict(meta, target=np.zeros(T, np.int64)),
                           rng.random(T))
    g = rng.standard_normal(T)
    return H, W, dict(meta, target=y), g, s


def _worker(rank, world, port, q, mode="gather"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, W, rows, g, _ = _case()
        vl = W.shape[0] // world
        Ws = torch.from_numpy(W[rank * vl:(rank + 1) * vl])
        t = {k: torch.from_numpy(np.asarray(v)) for k, v in rows.items()}
        tp = VocabParallel(ops=OracleOps(), row_chunk=128, mode=mode)
        lp, saved = tp.forward(torch.from_numpy(H), Ws, t["target"], t["temperature"], t["top_k"],
                               t["top_p"], t["min_p"])
        dH, dW = tp.backward(torch.from_numpy(H), Ws, t["target"], t["temperature"], t["top_k"],
                             t["top_p"], t["min_p"], saved, torch.from_numpy(g))
        q.put((rank, lp.numpy(), dH.numpy(), dW.numpy(), tp.gathered_rows))
    finally:
        dist.destroy_process_group()


def _run_two_ranks(mode):
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=180) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    H, W, rows, g, s = _case()
    ref = oracle.forward(None, None, rows, s=s.astype(np.float64))
    dZ = oracle.logit_grad(s.astype(np.float64), rows, g)
    dH_ref = dZ @ W.astype(np.float64)
    dW_ref = dZ.T @ H.astype(np.float64)
    vl = W.shape[0] // 2
    for rank, lp, dH, dW, gathered in got:
        np.testing.assert_array_equal(lp, ref["logprob"])  # same fp32 rows, same program
        np.testing.assert_allclose(dH, dH_ref, rtol=1e-12, atol=1e-12)  # partial sums added
        np.testing.assert_allclose(dW, dW_ref[rank * vl:(rank + 1) * vl], rtol=1e-12, atol=1e-12)
    return [x[4] for x in got]


def test_vocab_parallel_two_gloo_ranks():
    _run_two_ranks("gather")


def test_vocab_parallel_statistics_merge_two_gloo_ranks():
    """The merge's collectives in order, and the rows it flags (every seventh
    here) taken from the gather form on both ranks alike."""
    gathered = _run_two_ranks("merge")
    T = 300
    flagged = sum(len(range(0, min(128, T - t0), 7)) for t0 in range(0, T, 128))
    assert gathered == [flagged, flagged]

"""Host logic of the vocabulary-parallel path (VocabParallel), on CPU with two
gloo ranks and per-rank stand-ins for the kernels built from the float64
oracle: the shards' logits gathered in rank order reproduce the full rows,
the support program on them gives the unsharded oracle's logprobs, each rank
keeps its own dW shard and the summed dH equals the unsharded one. The
library's kernels take the same steps in the GPU tests."""

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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, W, rows, g, _ = _case()
        vl = W.shape[0] // world
        Ws = torch.from_numpy(W[rank * vl:(rank + 1) * vl])
        t = {k: torch.from_numpy(np.asarray(v)) for k, v in rows.items()}
        tp = VocabParallel(ops=OracleOps(), row_chunk=128)
        lp, saved = tp.forward(torch.from_numpy(H), Ws, t["target"], t["temperature"], t["top_k"],
                               t["top_p"], t["min_p"])
        dH, dW = tp.backward(torch.from_numpy(H), Ws, t["target"], t["temperature"], t["top_k"],
                             t["top_p"], t["min_p"], saved, torch.from_numpy(g))
        q.put((rank, lp.numpy(), dH.numpy(), dW.numpy()))
    finally:
        dist.destroy_process_group()


def test_vocab_parallel_two_gloo_ranks():
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
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
    for rank, lp, dH, dW in got:
        np.testing.assert_array_equal(lp, ref["logprob"])  # same fp32 rows, same program
        np.testing.assert_allclose(dH, dH_ref, rtol=1e-12, atol=1e-12)  # partial sums added
        np.testing.assert_allclose(dW, dW_ref[rank * vl:(rank + 1) * vl], rtol=1e-12, atol=1e-12)

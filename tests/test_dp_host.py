"""Host logic of the data-parallel weight-gradient sum, on CPU with two gloo
ranks: the slices the backward hands out (the library's own vocabulary
chunking, read from its host-side sts_vocab_chunk) are all-reduced one by one
as they arrive, and after ``finish`` every rank holds the sum of all ranks'
partial dW. Nothing here needs a GPU; the CUDA path of the same callback runs
in the GPU tests."""

import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import sampling_transform_lm_b200 as sts  # noqa: E402
from sampling_transform_lm_b200.dp import SliceAllReduce  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _slices(T, d, V, vocab_chunk):
    vc = sts.sts_vocab_chunk(T, d, V, vocab_chunk)
    return [(v0, min(vc, V - v0)) for v0 in range(0, V, vc)]


def _worker(rank, world, port, q, T, d, V, vocab_chunk):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank's partial dW: a seeded draw per rank
        g = torch.Generator().manual_seed(100 + rank)
        partial = torch.randn(V, d, generator=g)
        dW = torch.zeros(V, d)
        red = SliceAllReduce()
        # the backward writes slice i, then hands it out, then goes on
        for v0, n in _slices(T, d, V, vocab_chunk):
            dW[v0:v0 + n] = partial[v0:v0 + n]
            red(v0, n, dW[v0:v0 + n])
        order = red.finish()
        q.put((rank, order, dW.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("V,vocab_chunk", [(1000, 256), (4100, 0), (300, 512)])
def test_slice_allreduce_two_gloo_ranks(V, vocab_chunk):
    T, d = 64, 8
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, T, d, V, vocab_chunk))
             for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=120) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    want = sum(torch.randn(V, d, generator=torch.Generator().manual_seed(100 + r)).numpy()
               for r in range(2))
    expected_slices = _slices(T, d, V, vocab_chunk)
    for rank, order, dW in got:
        assert order == expected_slices  # increasing v0, covering [0, V) once
        np.testing.assert_allclose(dW, want, rtol=1e-6, atol=1e-6)


def test_slices_cover_the_vocabulary_once():
    for T, d, V, vc in [(7, 8, 1, 0), (7, 8, 255, 0), (7, 8, 257, 256), (7, 8, 152064, 0),
                        (7, 8, 151936, 8192)]:
        s = _slices(T, d, V, vc)
        assert s[0][0] == 0 and sum(n for _, n in s) == V
        assert all(a[0] + a[1] == b[0] for a, b in zip(s, s[1:]))

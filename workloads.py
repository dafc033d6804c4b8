"""Seeded synthetic workloads for the sampling-transform scoring core.

This module only draws inputs. It holds none of the method's arithmetic (no
logits, filters, logprobs or gradients), so both the float64 oracle and the
CUDA path can consume exactly the same data without sharing code.

Recipe (all draws from ``numpy.random.Generator(PCG64(seed))``, seed = 1000 +
the 1-based workload index, in this order):

1. H [T, d]: standard normal float32, rounded to nearest-even bf16.
2. W [V, d]: standard normal float32 times float32(1/sqrt(d)), rounded to bf16
   (so each logit is ~N(0, 1) and rows are flat, the hard case for top-p).
   The stress workload then overwrites a seeded 5% of vocabulary rows with
   exact copies of random lower-index rows, which forces exact logit ties.
3. per-row temperature, top_k, top_p, min_p as each workload states.
4. u [T] uniform in [0, 1): the uniforms a sampler uses to draw the replayed
   token from the filtered distribution (the draw itself is done by the caller).
5. g [T]: the upstream gradient, 1 for every row; a second seeded N(0, 1) draw
   (seed 2000 + index) is available for the two small workloads.

bf16 tensors are returned as uint16 bit patterns; ``bf16_to_f32`` widens them
exactly for float64 consumers.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

_CHUNK = 1 << 24  # elements per generation chunk (bounds host memory)


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    T: int
    d: int
    V: int
    vocab_chunk: int  # 0: library default
    backward: bool
    desc: str


WORKLOADS = {
    1: Workload(1, "tiny-oracle-check", 64, 128, 1024, 0, True,
                "T=64 d=128 V=1024; tau~U[0.5,1.5]; top_k in {off,50}, top_p in {1.0,0.9}, "
                "min_p in {0,0.05} independent 50/50; g=1"),
    2: Workload(2, "fwd-T4096-d2048-V32768", 4096, 2048, 32768, 0, False,
                "T=4096 d=2048 V=32768; tau~U[0.6,1.2]; rows split in thirds: top_k=20 / "
                "top_p=0.95 / min_p=0.1; forward only"),
    3: Workload(3, "T8192-d4096-V151936", 8192, 4096, 151936, 8192, True,
                "T=8192 d=4096 V=151936, vocab chunk 8192; tau~U[0.7,1.0]; every row top_k=50, "
                "top_p=0.9, min_p=0.02; forward+backward"),
    4: Workload(4, "T16384-d5120-V152064", 16384, 5120, 152064, 0, True,
                "T=16384 d=5120 V=152064; tau~U[0.5,1.5]; top_p~U[0.8,1.0] with 10% rows exactly "
                "1.0; min_p in {0,0.05}; top_k off; forward+backward (headline roofline workload)"),
    5: Workload(5, "stress-T32768-d4096-V262144", 32768, 4096, 262144, 0, True,
                "T=32768 d=4096 V=262144; 5% duplicated W rows (exact ties); top_k in {V,1}, "
                "top_p in {1.0,0.5}; tau~U[0.3,2.0]; min_p=0; forward+backward"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite float32 values to nearest-even bf16; return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to the float32 values they denote."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(rng, n_rows, n_cols, scale):
    out = np.empty((n_rows, n_cols), dtype=np.uint16)
    flat = out.reshape(-1)
    total = n_rows * n_cols
    sc = np.float32(scale)
    for lo in range(0, total, _CHUNK):
        hi = min(total, lo + _CHUNK)
        x = rng.standard_normal(hi - lo, dtype=np.float32)
        if scale != 1.0:
            x *= sc
        flat[lo:hi] = f32_to_bf16_bits(x)
    return out


def _thirds(rng, T):
    perm = rng.permutation(T)
    a = T // 3
    return perm[:a], perm[a:2 * a], perm[2 * a:]


def _redraw_rows(index, rng, T, V, top_k, top_p, min_p):
    """Fill the per-row metadata arrays in place; return the temperatures."""
    top_k[:] = 0
    top_p[:] = 1.0
    min_p[:] = 0.0
    if index == 1:
        tau = rng.uniform(0.5, 1.5, T).astype(np.float32)
        top_k[:] = np.where(rng.integers(0, 2, T) == 1, 50, 0)
        top_p[:] = np.where(rng.integers(0, 2, T) == 1, np.float32(0.9), np.float32(1.0))
        min_p[:] = np.where(rng.integers(0, 2, T) == 1, np.float32(0.05), np.float32(0.0))
    elif index == 2:
        tau = rng.uniform(0.6, 1.2, T).astype(np.float32)
        a, b, c = _thirds(rng, T)
        top_k[a] = 20
        top_p[b] = np.float32(0.95)
        min_p[c] = np.float32(0.1)
    elif index == 3:
        tau = rng.uniform(0.7, 1.0, T).astype(np.float32)
        top_k[:] = 50
        top_p[:] = np.float32(0.9)
        min_p[:] = np.float32(0.02)
    elif index == 4:
        tau = rng.uniform(0.5, 1.5, T).astype(np.float32)
        top_p[:] = rng.uniform(0.8, 1.0, T).astype(np.float32)
        ident = rng.permutation(T)[: int(round(0.1 * T))]
        top_p[ident] = np.float32(1.0)
        min_p[:] = np.where(rng.integers(0, 2, T) == 1, np.float32(0.05), np.float32(0.0))
    elif index == 5:
        tau = rng.uniform(0.3, 2.0, T).astype(np.float32)
        top_k[:] = np.where(rng.integers(0, 2, T) == 1, 1, V)
        top_p[:] = np.where(rng.integers(0, 2, T) == 1, np.float32(0.5), np.float32(1.0))
    else:
        raise ValueError(f"unknown workload {index}")
    return tau



def make(index: int, T: int | None = None, with_weights: bool = True, batch: int = 0,
         V: int | None = None):
    """Draw workload ``index`` (1..5). ``T`` overrides the row count (the
    per-row distributions are unchanged) for reduced-size test cases.
    ``batch`` > 0 draws another batch of rows (H, metadata, u) from a second
    generator seeded (1000 + index, batch) while W stays the workload's own --
    one batch per data-parallel rank. ``V`` overrides the vocabulary size
    (reduced cases for profiling captures only).

    Returns a dict with ``H`` (uint16 [T, d]), ``W`` (uint16 [V, d], or None
    when ``with_weights`` is false), ``temperature`` (f32), ``top_k`` (i32),
    ``top_p`` (f32), ``min_p`` (f32), ``u`` (f64) and ``g`` (f32), plus the
    ``workload`` record.
    """
    wl = WORKLOADS[index]
    T = wl.T if T is None else int(T)
    d = wl.d
    V = wl.V if V is None else int(V)
    rng = np.random.Generator(np.random.PCG64(1000 + index))

    H = _normal_bf16(rng, T, d, 1.0)
    W = None
    if with_weights:
        W = _normal_bf16(rng, V, d, 1.0 / np.sqrt(d))
    else:
        # keep the stream position identical whether or not W is materialised
        total = V * d
        for lo in range(0, total, _CHUNK):
            rng.standard_normal(min(total, lo + _CHUNK) - lo, dtype=np.float32)
    if index == 5:
        n_dup = int(round(0.05 * V))
        dst = np.sort(rng.choice(np.arange(1, V), size=n_dup, replace=False))
        src = np.array([rng.integers(0, i) for i in dst], dtype=np.int64)
        if W is not None:
            for i, j in zip(dst, src):
                W[i] = W[j]
    else:
        dst = src = np.zeros(0, dtype=np.int64)

    top_k = np.zeros(T, dtype=np.int32)
    top_p = np.ones(T, dtype=np.float32)
    min_p = np.zeros(T, dtype=np.float32)
    tau = _redraw_rows(index, rng, T, V, top_k, top_p, min_p)

    if batch:
        rng_b = np.random.Generator(np.random.PCG64([1000 + index, int(batch)]))
        H = _normal_bf16(rng_b, T, d, 1.0)
        tau = _redraw_rows(index, rng_b, T, V, top_k, top_p, min_p)
        u = rng_b.random(T)
    else:
        u = rng.random(T)
    g = np.ones(T, dtype=np.float32)
    return {
        "workload": wl,
        "H": H,
        "W": W,
        "dup_dst": dst,
        "dup_src": src,
        "temperature": tau,
        "top_k": top_k,
        "top_p": top_p,
        "min_p": min_p,
        "u": u,
        "g": g,
    }


def extra_grad(index: int, T: int) -> np.ndarray:
    """The second upstream-gradient draw: N(0, 1) float32, seed 2000 + index."""
    rng = np.random.Generator(np.random.PCG64(2000 + index))
    return rng.standard_normal(T, dtype=np.float32)


def rows_dict(data, target):
    """Bundle per-row metadata with the replayed tokens ``target``."""
    return {
        "target": np.asarray(target, dtype=np.int64),
        "temperature": data["temperature"],
        "top_k": data["top_k"],
        "top_p": data["top_p"],
        "min_p": data["min_p"],
    }

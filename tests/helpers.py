"""Shared test helpers: move seeded workloads to the GPU, run the oracle on
the same values, and compare with the tolerances of the parity contract
(logprob 2e-3 absolute, gradients 1e-2 relative Frobenius, support cuts
bit-exact when both sides filter the same fp32 logits; rows whose oracle
threshold gap is below 1e-4 are counted and reported rather than failed)."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import workloads

LOGPROB_ATOL = 2e-3
GRAD_RTOL = 1e-2
GAP_EPS = 1e-4


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def f32_values(bits: np.ndarray) -> np.ndarray:
    return workloads.bf16_to_f32(bits)


def row_tensors(rows: dict, device="cuda"):
    return (
        torch.from_numpy(np.asarray(rows["target"], np.int64)).to(device),
        torch.from_numpy(np.asarray(rows["temperature"], np.float32)).to(device),
        torch.from_numpy(np.asarray(rows["top_k"], np.int32)).to(device),
        torch.from_numpy(np.asarray(rows["top_p"], np.float32)).to(device),
        torch.from_numpy(np.asarray(rows["min_p"], np.float32)).to(device),
    )


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def near_gap_rows(s: np.ndarray, rows: dict, eps: float = GAP_EPS) -> np.ndarray:
    return oracle.row_gaps(s, rows).min(axis=1) < eps


def compare_logprob(gpu_lp: np.ndarray, ora_lp: np.ndarray, flagged: np.ndarray):
    """Returns (n_bad, n_flagged_mismatch, max_abs_err_on_unflagged_finite).

    A row mismatches when the GPU value is NaN, when a finite pair is further
    apart than LOGPROB_ATOL, or when the target is inside the support on one
    side only. Mismatches on rows whose oracle thresholds sit within GAP_EPS
    of a decision boundary are counted and reported (the fp32 logits may
    legitimately cross such a boundary); any other mismatch is a failure.
    """
    gpu_lp = np.asarray(gpu_lp, np.float64)
    gi = np.isneginf(gpu_lp)
    oi = np.isneginf(ora_lp)
    both = ~gi & ~oi
    err = np.where(both, np.abs(gpu_lp - ora_lp), 0.0)
    mism = (both & (err > LOGPROB_ATOL)) | np.isnan(gpu_lp) | (gi != oi)
    n_bad = int((mism & ~flagged).sum())
    sel = both & ~flagged
    max_err = float(err[sel].max()) if sel.any() else 0.0
    return n_bad, int((mism & flagged).sum()), max_err


def grad_rows(gpu_flags: np.ndarray, ref_in_support: np.ndarray) -> np.ndarray:
    """Rows whose target is in (or out of) the support on both sides: only
    these carry comparable gradients."""
    return ((np.asarray(gpu_flags) & 1) != 0) == np.asarray(ref_in_support)


def small_case(seed, T, d, V, tau=(0.5, 1.5), k_choices=(0, 50), p_choices=(1.0, 0.9),
               mu_choices=(0.0, 0.05)):
    """A config-1-style random case of any size (H ~ N(0,1), W ~ N(0,1/d))."""
    rng = np.random.Generator(np.random.PCG64(seed))
    H = workloads.f32_to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))
    W = workloads.f32_to_bf16_bits(rng.standard_normal((V, d), dtype=np.float32)
                                   * np.float32(1 / math.sqrt(d)))
    rows = {
        "temperature": rng.uniform(*tau, T).astype(np.float32),
        "top_k": rng.choice(np.asarray(k_choices, np.int32), T).astype(np.int32),
        "top_p": rng.choice(np.asarray(p_choices, np.float32), T).astype(np.float32),
        "min_p": rng.choice(np.asarray(mu_choices, np.float32), T).astype(np.float32),
    }
    u = rng.random(T)
    return H, W, rows, u

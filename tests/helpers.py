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


def compare_logprob(gpu_lp, gpu_size, s, rows, ref, flagged):
    """Returns (n_bad, n_size_diff, max_abs_err). Every row is compared.

    The expected logprob of a row is the oracle's, or -- where the GPU's
    support size differs from the oracle's, which is only allowed on a row
    whose oracle threshold lies within GAP_EPS of a decision boundary -- the
    oracle's logprob on the GPU's support (``oracle.logprob_on_prefix``): the
    order of the row is unique, so a support is a prefix length, and the
    logprob follows from it. On every row the target membership must agree
    with that expectation and finite values must agree within LOGPROB_ATOL;
    a NaN is always a failure.
    """
    gpu_lp = np.asarray(gpu_lp, np.float64)
    gpu_size = np.asarray(gpu_size, np.int64)
    want = np.array(ref["logprob"], np.float64)
    diff = gpu_size != np.asarray(ref["size"])
    if diff.any():
        idx = np.flatnonzero(diff)
        sub = {k: np.asarray(v)[idx] for k, v in rows.items()}
        want[idx] = oracle.logprob_on_prefix(np.asarray(s)[idx], sub, gpu_size[idx])[0]
    gi = np.isneginf(gpu_lp)
    wi = np.isneginf(want)
    both = ~gi & ~wi & ~np.isnan(gpu_lp)
    err = np.where(both, np.abs(gpu_lp - want), 0.0)
    bad = (both & (err > LOGPROB_ATOL)) | np.isnan(gpu_lp) | (gi != wi) | (diff & ~flagged)
    max_err = float(err[both].max()) if both.any() else 0.0
    return int(bad.sum()), int(diff.sum()), max_err


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


# --------------------------------------------------------------------------
# the oracle's per-row loops over a process pool (spawn: the parent may
# already hold a CUDA context, and a forked child of it would hang)


def _oracle_call(name, args, kwargs):
    return getattr(oracle, name)(*args, **kwargs)


class OraclePool:
    """Runs an oracle function on row slices in parallel and joins the
    results in row order. The oracle itself is unchanged: each worker calls
    the same function on a contiguous block of rows."""

    def __init__(self, workers=None):
        import concurrent.futures
        import multiprocessing
        import os

        n = workers or max(1, min(16, (os.cpu_count() or 2) - 1))
        self.n = n
        self.ex = concurrent.futures.ProcessPoolExecutor(
            max_workers=n, mp_context=multiprocessing.get_context("spawn"))

    def close(self):
        self.ex.shutdown(wait=True, cancel_futures=True)

    def _slices(self, T):
        step = max(1, -(-T // (2 * self.n)))
        return [(a, min(T, a + step)) for a in range(0, T, step)]

    @staticmethod
    def _rows_slice(rows, a, b):
        return {k: np.asarray(v)[a:b] for k, v in rows.items()}

    def map_rows(self, name, s, rows, *extra, per_row_extra=()):
        """oracle.<name>(s[a:b], rows[a:b], *extra[a:b] ...) for row blocks;
        returns the per-block results in order."""
        T = s.shape[0]
        futs = []
        for a, b in self._slices(T):
            args = [s[a:b], self._rows_slice(rows, a, b)]
            args += [np.asarray(e)[a:b] for e in per_row_extra]
            args += list(extra)
            futs.append(self.ex.submit(_oracle_call, name, tuple(args), {}))
        return [f.result() for f in futs]

    def forward(self, s, rows):
        futs = []
        for a, b in self._slices(s.shape[0]):
            futs.append(self.ex.submit(_oracle_call, "forward",
                                       (None, None, self._rows_slice(rows, a, b)), {"s": s[a:b]}))
        parts = [f.result() for f in futs]
        return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}

    def filter_rows(self, s, rows):
        parts = self.map_rows("filter_rows", s, rows)
        return {k: np.concatenate([p[k] for p in parts]) for k in parts[0]}

    def row_gaps(self, s, rows):
        return np.concatenate(self.map_rows("row_gaps", s, rows))

    def sample_rows(self, s, rows, u):
        return np.concatenate(self.map_rows("sample_rows", s, rows, per_row_extra=(u,)))

    def logit_grad(self, s, rows, g):
        return np.concatenate(self.map_rows("logit_grad", s, rows, per_row_extra=(g,)))


F32_MASS_LP_ATOL = 3e-5  # logprob of the fp32-mass forward against the float64-mass one


def assert_same_decisions(lp_a, saved_a, lp_b, saved_b):
    """Two forwards of the same rows, one with the entropy output (float64
    masses) and one without (fp32 masses where no mass comparison decides the
    support): identical support decisions, logprobs within the fp32 mass
    bound (relative 2e-5 on the support mass, so 2e-5 on its log, plus the
    fp32 rounding of LSE_S)."""
    for key in ("support_size", "cut_id", "cut_logit", "flags"):
        a, b = saved_a[key], saved_b[key]
        same = (a == b) | (torch.isnan(a) & torch.isnan(b)) if a.is_floating_point() else a == b
        assert bool(same.all()), key
    fin = torch.isfinite(lp_a)
    assert torch.equal(fin, torch.isfinite(lp_b))
    assert torch.equal(torch.isnan(lp_a), torch.isnan(lp_b))
    assert torch.equal(lp_a[~fin & ~torch.isnan(lp_a)], lp_b[~fin & ~torch.isnan(lp_b)])
    if bool(fin.any()):
        assert (lp_a[fin] - lp_b[fin]).abs().max().item() < F32_MASS_LP_ATOL

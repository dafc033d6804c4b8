"""Float64 CPU oracle for the chunked sampling-transform scoring core.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this module. The CUDA
product path (``sampling_transform_lm_b200``) never imports it, and this module
imports nothing from the product path: the two share no code.

What it computes, and where the pages define it
-----------------------------------------------
Sources (cited by page title and section):

* [xorl#74] "Consolidate sampling-transform scoring on one shared chunked core;
  implement top-k/top-p/min-p replay for generic ce_modes" (togethercomputer/xorl,
  pull request 74).
  - "What this PR does", item 1: the pinned program -- temperature first,
    stable token-ID tie-break, inclusive top-p crossing, min-p against the
    original row maximum, top_p == 1.0 an exact identity even where an fp32
    cumulative sum overshoots.
  - item 2: chunked projection -> temperature -> support program -> selected
    logprob; closed-form recompute VJP that keeps only per-row scalars; the
    generic lane computes chunk logits with an fp32-output GEMM.
  - item 4: a replayed token outside its row's support scores -inf logprob
    (+inf CE) and receives zero gradient.
  - "Self-review pass (second commit)": per-row temperature is applied after
    the GEMM; the selected score is clamped to <= 0; metadata whose length
    differs from the row count is rejected.
* [align-v2] "align architecture v2: proposal", section 5.4 A "Fused head +
  policy-gradient token loss": the head needs fp32 *logits* from bf16
  operands, and the logit gradient of a selected-token logprob is
  (onehot - softmax) scaled per token; "Why the in-chunk form works for this
  loss" gives that per-token coefficient for CISPO and the clipped surrogate
  (``policy_grad``).

Readings taken where the pages are silent (each is a deliberate choice):

* Filter composition: top-k, then top-p measured on the top-k-renormalised
  distribution, then min-p. Min-p is a threshold relative to the unfiltered
  (temperature-scaled) row maximum, so the final support is the shortest of
  the three prefixes of the (logit desc, token id asc) order.
* Inclusive crossing: sorted position j is kept iff the exclusive running mass
  C_j is strictly below p * Z_k, where Z_k is the top-k mass. The token whose
  mass first brings the running sum to >= p * Z_k is therefore kept.
* Min-p: token i is kept iff exp(s_i - m) >= min_p (float64), m the row max of
  the temperature-scaled logits; min_p == 0 switches it off.
* top_k <= 0 or top_k >= V switches top-k off; top_p >= 1 is the identity.
* Temperature: s = z / tau with tau per row; no gradient flows to tau or
  through the thresholds (the support is piecewise constant).
* Sampling (used to draw the replayed token of the synthetic workloads): the
  inverse CDF of the filtered distribution walked in the support's sorted
  order, driven by a caller-supplied uniform u in [0, 1).

Arithmetic: float64 throughout. Logits are z = H . W^T on the float64 values
of the bf16 operands; sorting is numpy's stable argsort of -s; the top-p
running mass is a sequential float64 cumulative sum in sorted order; Z_k and
the support mass are exactly rounded sums (math.fsum).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "RowFilter",
    "scaled_logits",
    "filter_row",
    "filter_rows",
    "forward",
    "backward",
    "sample_rows",
    "row_gaps",
    "logprob_on_prefix",
    "entropy",
    "logit_grad",
    "policy_grad",
]


@dataclass
class RowFilter:
    """Result of the support program on one row (positions refer to the
    (s desc, id asc) order)."""

    order: np.ndarray  # int64 [V], token ids in sorted order
    m: float  # unfiltered row max of the scaled logits
    k_eff: int  # effective top-k size
    m_p: int  # top-p prefix length (k_eff when top-p is off)
    m_mu: int  # min-p prefix length (V when min-p is off)
    size: int  # final support size = min(k_eff, m_p, m_mu)
    Z_k: float  # top-k mass sum exp(s - m) (nan when top-p is off)

    @property
    def cut_id(self) -> int:
        """Token id of the last kept position."""
        return int(self.order[self.size - 1])


def scaled_logits(H, W, temperature, vocab_slice=None) -> np.ndarray:
    """s = (H . W^T) / tau in float64.

    [xorl#74] "What this PR does", item 2 (chunked projection, fp32-output GEMM
    on the generic lane) and "Self-review pass" (per-row temperature applied
    after the GEMM). The oracle keeps the full float64 product of the bf16
    operand values, which is the exact logit up to one float64 rounding per
    accumulation step. ``vocab_slice`` only bounds host memory: W is widened
    to float64 that many rows at a time; every logit is the same dot product.
    """
    H = np.asarray(H, dtype=np.float64)
    tau = np.asarray(temperature, dtype=np.float64)
    V = W.shape[0]
    step = V if vocab_slice is None else int(vocab_slice)
    z = np.empty((H.shape[0], V), dtype=np.float64)
    for a in range(0, V, step):
        z[:, a:a + step] = H @ np.asarray(W[a:a + step], dtype=np.float64).T
    return z / tau[:, None]


def filter_row(s, top_k: int, top_p: float, min_p: float) -> RowFilter:
    """The pinned support program on one row of scaled logits.

    [xorl#74] "What this PR does", item 1: stable token-ID tie-break (a stable
    sort of -s keeps equal logits in increasing id order), inclusive top-p
    crossing, min-p against the original row maximum, top_p == 1.0 exact
    identity.
    """
    s = np.asarray(s, dtype=np.float64)
    V = s.shape[0]
    order = np.argsort(-s, kind="stable")
    ss = s[order]
    m = float(ss[0])

    k_eff = V if (top_k <= 0 or top_k >= V) else int(top_k)

    p = float(top_p)
    Z_k = float("nan")
    if p >= 1.0:
        m_p = k_eff  # exact identity, no cumulative sum is formed at all
    else:
        q = np.exp(ss[:k_eff] - m)
        Z_k = math.fsum(q)
        C = np.empty(k_eff, dtype=np.float64)  # exclusive running mass
        C[0] = 0.0
        if k_eff > 1:
            np.cumsum(q[:-1], out=C[1:])
        m_p = int(np.count_nonzero(C < p * Z_k))

    mu = float(min_p)
    if mu > 0.0:
        # exp(s - m) is non-increasing along the sorted order, so this count is
        # the length of a prefix.
        m_mu = int(np.count_nonzero(np.exp(ss - m) >= mu))
    else:
        m_mu = V

    size = min(k_eff, m_p, m_mu)
    return RowFilter(order=order, m=m, k_eff=k_eff, m_p=m_p, m_mu=m_mu, size=size, Z_k=Z_k)


def _row_meta(rows, t):
    return (
        int(rows["top_k"][t]),
        float(np.float32(rows["top_p"][t])),
        float(np.float32(rows["min_p"][t])),
    )


def filter_rows(s, rows, want_mask: bool = False):
    """Run the support program on every row of ``s`` [T, V].

    Returns a dict with per-row ``size`` (int64), ``cut_id`` (int64),
    ``cut_value`` (the scaled logit at the cut, float64), ``row_max``
    (float64) and, when asked, the boolean support ``mask`` [T, V].
    Used on float32 logits for the bit-exact check of the GPU filter: the
    float32 values are widened exactly and every decision is taken in float64.
    """
    s = np.asarray(s)
    T, V = s.shape
    out = {
        "size": np.zeros(T, dtype=np.int64),
        "cut_id": np.zeros(T, dtype=np.int64),
        "cut_value": np.zeros(T, dtype=np.float64),
        "row_max": np.zeros(T, dtype=np.float64),
    }
    if want_mask:
        out["mask"] = np.zeros((T, V), dtype=bool)
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        out["size"][t] = f.size
        out["cut_id"][t] = f.cut_id
        out["cut_value"][t] = float(s[t, f.cut_id])
        out["row_max"][t] = f.m
        if want_mask:
            out["mask"][t, f.order[: f.size]] = True
    return out


def _support_lse(ss, m, size):
    """LSE over the first ``size`` sorted logits: m + log(sum exp(s - m))."""
    return m + math.log(math.fsum(np.exp(ss[:size] - m)))


def forward(H, W, rows, s=None):
    """Selected-token logprob on the filtered support, per row.

    [xorl#74] item 2 (selected logprob on the filtered support), item 4
    (out-of-support target -> -inf) and "Self-review pass" (<= 0 clamp).

    logprob_t = min(s_y - LSE_S, 0) if y in S else -inf, with
    LSE_S = m + log(sum_{i in S} exp(s_i - m)).

    Returns a dict: ``logprob``, ``lse_support``, ``row_max``, ``size``,
    ``cut_id``, ``in_support`` (bool) -- all float64 / int64 per row.
    ``s`` may be passed to reuse already computed scaled logits.
    """
    if s is None:
        s = scaled_logits(H, W, rows["temperature"])
    T, V = s.shape
    y = np.asarray(rows["target"], dtype=np.int64)
    res = {
        "logprob": np.zeros(T, dtype=np.float64),
        "lse_support": np.zeros(T, dtype=np.float64),
        "row_max": np.zeros(T, dtype=np.float64),
        "size": np.zeros(T, dtype=np.int64),
        "cut_id": np.zeros(T, dtype=np.int64),
        "in_support": np.zeros(T, dtype=bool),
    }
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        ss = s[t, f.order]
        lse = _support_lse(ss, f.m, f.size)
        rank = np.empty(V, dtype=np.int64)
        rank[f.order] = np.arange(V)
        inside = bool(rank[y[t]] < f.size)
        res["lse_support"][t] = lse
        res["row_max"][t] = f.m
        res["size"][t] = f.size
        res["cut_id"][t] = f.cut_id
        res["in_support"][t] = inside
        res["logprob"][t] = min(float(s[t, y[t]]) - lse, 0.0) if inside else -math.inf
    return res


def entropy(s, rows, sizes=None):
    """Entropy of each row's filtered (renormalised) distribution, in nats:
    H_t = -sum_{i in S_t} p_i ln p_i with p_i = exp(s_i - LSE_S). ``sizes``
    (optional) gives each row's support size instead of deriving it, as
    ``logprob_on_prefix`` does.

    [align-v2] section 5.4 A names the per-token entropy as one of the
    statistics of the fused head ("entropy from the same sweep"); the
    distribution is the one the selected logprob is scored on ([xorl#74]
    item 2): the support of item 1, renormalised. Written as the sum of the
    non-negative terms p_i (LSE_S - s_i), exactly rounded (math.fsum).
    """
    s = np.asarray(s, dtype=np.float64)
    T = s.shape[0]
    out = np.zeros(T, dtype=np.float64)
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        size = f.size if sizes is None else int(sizes[t])
        ss = s[t, f.order[:size]]
        lse = _support_lse(ss, f.m, size)
        pr = np.exp(ss - lse)
        out[t] = math.fsum(pr * (lse - ss))
    return out


def logprob_on_prefix(s, rows, sizes):
    """Selected-token logprob when row t's support is the first sizes[t]
    positions of its (s desc, id asc) order; returns (logprob, in_support).

    The same definition as ``forward`` ([xorl#74] item 2, item 4, the <= 0
    clamp of "Self-review pass") with the support size given instead of
    derived. A result whose support differs from the oracle's at a near-tie
    boundary is a valid alternative; its logprob is then fixed by that
    support, and this gives it.
    """
    s = np.asarray(s, dtype=np.float64)
    T, V = s.shape
    y = np.asarray(rows["target"], dtype=np.int64)
    lp = np.zeros(T, dtype=np.float64)
    inside = np.zeros(T, dtype=bool)
    for t in range(T):
        size = int(sizes[t])
        order = np.argsort(-s[t], kind="stable")
        ss = s[t, order]
        lse = _support_lse(ss, float(ss[0]), size)
        rank = np.empty(V, dtype=np.int64)
        rank[order] = np.arange(V)
        inside[t] = bool(rank[y[t]] < size)
        lp[t] = min(float(s[t, y[t]]) - lse, 0.0) if inside[t] else -math.inf
    return lp, inside


def logit_grad(s, rows, grad_logprob):
    """dlogprob/dz per row: g * (onehot(y) - p_S) / tau, or a zero row when
    y is outside the support.

    [xorl#74] item 2 (closed-form VJP) and item 4 (zero gradient out of
    support); [align-v2] 5.4 A (logit gradient of a selected-token logprob is
    onehot minus the softmax, times the token's coefficient). Here the softmax
    is the renormalised support distribution p_i = exp(s_i - LSE_S) 1[i in S]
    and the 1/tau factor is the derivative of s = z / tau.
    """
    s = np.asarray(s, dtype=np.float64)
    T, V = s.shape
    y = np.asarray(rows["target"], dtype=np.int64)
    tau = np.asarray(rows["temperature"], dtype=np.float64)
    g = np.asarray(grad_logprob, dtype=np.float64)
    dZ = np.zeros((T, V), dtype=np.float64)
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        ss = s[t, f.order]
        support = f.order[: f.size]
        rank = np.empty(V, dtype=np.int64)
        rank[f.order] = np.arange(V)
        if rank[y[t]] >= f.size:
            continue
        lse = _support_lse(ss, f.m, f.size)
        row = np.zeros(V, dtype=np.float64)
        row[support] = -np.exp(s[t, support] - lse)
        row[y[t]] += 1.0
        dZ[t] = g[t] * row / tau[t]
    return dZ


def backward(H, W, rows, grad_logprob, s=None, vocab_rows=None, vocab_slice=None, dZ=None):
    """Closed-form VJP: dH = dZ . W and dW = dZ^T . H in float64.

    [xorl#74] item 2 (recompute closed-form VJP) and "Acceptance criteria"
    (hidden and weight gradients). ``vocab_rows`` restricts dW to the listed
    vocabulary rows (the full [V, d] float64 matrix of the large workloads
    does not fit comfortably in host memory); ``vocab_slice`` widens W to
    float64 that many rows at a time for dH = sum over vocabulary slices.
    ``dZ`` may pass the logit gradient already formed by ``logit_grad`` on the
    same rows (for example row slice by row slice, in parallel).
    """
    H = np.asarray(H, dtype=np.float64)
    if dZ is None:
        if s is None:
            s = scaled_logits(H, W, rows["temperature"], vocab_slice=vocab_slice)
        dZ = logit_grad(s, rows, grad_logprob)
    V = W.shape[0]
    step = V if vocab_slice is None else int(vocab_slice)
    dH = np.zeros((H.shape[0], H.shape[1]), dtype=np.float64)
    for a in range(0, V, step):
        dH += dZ[:, a:a + step] @ np.asarray(W[a:a + step], dtype=np.float64)
    if vocab_rows is None:
        dW = dZ.T @ H
    else:
        dW = dZ[:, vocab_rows].T @ H
    return dH, dW


def sample_rows(s, rows, u):
    """Draw one token per row from the filtered distribution.

    Inverse CDF in the support's sorted order: with I_j the inclusive running
    mass of the j-th kept token and Z_S the support mass, the draw is the
    first sorted position with I_j > u * Z_S (u in [0, 1) supplied by the
    caller). The rule follows from the program of [xorl#74] item 1; the pages
    fix no sampler, so this one only generates replayed tokens for tests.
    """
    s = np.asarray(s, dtype=np.float64)
    T, V = s.shape
    y = np.zeros(T, dtype=np.int64)
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        q = np.exp(s[t, f.order[: f.size]] - f.m)
        inc = np.cumsum(q)
        j = int(np.searchsorted(inc, float(u[t]) * inc[-1], side="right"))
        y[t] = int(f.order[min(j, f.size - 1)])
    return y


def row_gaps(s, rows):
    """Distance of each threshold that can move the support from its decision
    boundary, per row: columns (gap_k, gap_p, gap_mu).

    gap_k: s_(k-1) - s_(k) in scaled-logit units (exact ties report +inf: they
    are decided by token id, not by rounding). gap_p: min(p Z_k - C_(m_p - 1),
    C_(m_p) - p Z_k) / Z_k, C the exclusive running mass (the first term only
    when m_p > 1, the second only when m_p < k_eff: the first position is
    always kept and a crossing cannot pass the last top-k position; +inf when
    neither boundary exists). gap_mu: the distance in logit units of the min-p
    threshold t = m + ln(min_p) from the last kept logit (unless that one ties
    the row max, which min_p <= 1 always keeps) and from the first dropped one.

    A rule reports its gap only where it can move the result: its prefix
    length is within one position of the support size (m_r <= size + 1; the
    support is the shortest of the prefixes, so crossing one boundary moves
    m_r by one and can change the support only then). Rules that are off, or
    whose prefix ends two or more positions after the support's, report +inf.
    A row whose smallest gap is tiny can legitimately resolve differently
    under float32 logits or another summation order ([xorl#74] item 1 fixes
    the program; this measure only sorts rows for reporting).
    """
    s = np.asarray(s, dtype=np.float64)
    T, V = s.shape
    out = np.full((T, 3), np.inf)
    for t in range(T):
        k, p, mu = _row_meta(rows, t)
        f = filter_row(s[t], k, p, mu)
        ss = s[t, f.order]
        live = f.size + 1
        if f.k_eff < V and f.k_eff <= live:
            g = ss[f.k_eff - 1] - ss[f.k_eff]
            out[t, 0] = g if g > 0 else np.inf
        if p < 1.0 and f.m_p <= live:
            q = np.exp(ss[: f.k_eff] - f.m)
            C = np.concatenate(([0.0], np.cumsum(q)))
            target = p * f.Z_k
            # no boundary below when only the first position is kept (C_0 = 0 <
            # p Z_k for every p > 0), none above when every top-k position is
            lo = target - C[f.m_p - 1] if f.m_p > 1 else np.inf
            hi = C[f.m_p] - target if f.m_p < f.k_eff else np.inf
            out[t, 1] = min(lo, hi) / f.Z_k
        if mu > 0.0 and f.m_mu <= live:
            thr = f.m + math.log(mu)
            # the last kept logit bounds it from above unless it ties the max
            # (min_p <= 1 always keeps the max); the first dropped one from below
            up = ss[f.m_mu - 1] - thr if ss[f.m_mu - 1] < f.m else np.inf
            down = thr - ss[f.m_mu] if f.m_mu < V else np.inf
            out[t, 2] = min(up, down)
    return out


# ---------------------------------------------------------------- policy-gradient coefficient

def policy_grad(logprob, old_logprob, advantage, objective="cispo", eps_low=0.2, eps_high=0.2,
                scale=1.0):
    """Upstream gradient g_t = dL/dlogprob_t of a policy-gradient token loss,
    to be fed to the backward as grad_logprob.

    [align-v2] section 5.4 A, "Why the in-chunk form works for this loss": the
    per-token logit gradient of the objective J is c_t (softmax - onehot) with a
    token coefficient known from the fresh logprob; the loss the optimiser
    minimises is L = -J. With r_t = exp(logprob_t - old_logprob_t):

    * "cispo" (CISPO, cited there as arXiv:2506.13585 Sec. 3.1 Eq. 4-5): J =
      sum_t sg(min(r_t, 1 + eps_high)) A_t logprob_t, the importance weight a
      stop-gradient constant with no lower bound, so
      g_t = -scale * A_t * min(r_t, 1 + eps_high).
    * "clipped" (the clipped surrogate of the same passage): J = sum_t
      min(r_t A_t, clip(r_t, 1 - eps_low, 1 + eps_high) A_t); where the clip
      binds the term is constant in logprob, elsewhere d(r_t A_t)/dlogprob_t =
      r_t A_t, so g_t = -scale * A_t * r_t * 1[not clipped], clipped meaning
      r_t > 1 + eps_high for A_t >= 0 and r_t < 1 - eps_low for A_t < 0.

    ``scale`` carries the loss normalisation (for example 1 / tokens). Rows
    whose logprob is -inf (replayed token outside the support) or NaN (an
    invalid row), or whose old logprob or advantage is not finite, get
    g_t = 0; so do rows with scale * A_t == 0 (no signal). The ratio r_t is
    +inf where exp overflows (logprob - old_logprob above ~709.8): the CISPO
    weight is then 1 + eps_high, the clipped surrogate is clipped for A_t >= 0
    and its gradient is infinite for A_t < 0. Float64 throughout.
    """
    lp = np.asarray(logprob, dtype=np.float64)
    old = np.asarray(old_logprob, dtype=np.float64)
    adv = np.asarray(advantage, dtype=np.float64)
    out = np.zeros(lp.shape, dtype=np.float64)
    for t in range(lp.shape[0]):
        if not (np.isfinite(lp[t]) and np.isfinite(old[t]) and np.isfinite(adv[t])):
            continue
        if scale * adv[t] == 0.0:
            continue
        try:
            r = math.exp(lp[t] - old[t])
        except OverflowError:
            r = math.inf
        if objective == "cispo":
            out[t] = -scale * adv[t] * min(r, 1.0 + eps_high)
        elif objective == "clipped":
            clipped = r > 1.0 + eps_high if adv[t] >= 0 else r < 1.0 - eps_low
            out[t] = 0.0 if clipped else -scale * adv[t] * r
        else:
            raise ValueError(f"unknown objective {objective!r}")
    return out


"""Pins for the float64 oracle: every check compares it with something other
than itself -- hand-worked cases, closed forms, a brute-force formulation,
torch autograd, finite differences and structural invariants.

The pinned program is the one of "Consolidate sampling-transform scoring on one
shared chunked core; implement top-k/top-p/min-p replay for generic ce_modes"
(xorl pull request 74), section "What this PR does", items 1, 2 and 4.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import workloads

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _rows(T, target, tau=1.0, k=0, p=1.0, mu=0.0):
    return {
        "target": np.full(T, target, dtype=np.int64) if np.isscalar(target) else np.asarray(target),
        "temperature": np.full(T, tau, dtype=np.float32) if np.isscalar(tau) else np.asarray(tau, np.float32),
        "top_k": np.full(T, k, dtype=np.int32) if np.isscalar(k) else np.asarray(k, np.int32),
        "top_p": np.full(T, p, dtype=np.float32) if np.isscalar(p) else np.asarray(p, np.float32),
        "min_p": np.full(T, mu, dtype=np.float32) if np.isscalar(mu) else np.asarray(mu, np.float32),
    }


# --------------------------------------------------------------------------
# hand-worked golden cases


def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_worked_case(case):
    if "H" in case:
        H = np.array(case["H"], dtype=np.float64)
        W = np.array(case["W"], dtype=np.float64)
        tau = np.array([case["temperature"]], dtype=np.float32)
        s = oracle.scaled_logits(H, W, tau)
    else:
        row = np.log(np.array(case["weights"], dtype=np.float64)) if "weights" in case else \
            np.array(case["logits"], dtype=np.float64)
        s = row[None, :] / np.float64(case["temperature"])
        H = W = None
    rows = _rows(1, case["target"], case["temperature"], case["top_k"], case["top_p"], case["min_p"])
    f = oracle.filter_rows(s, rows, want_mask=True)
    assert sorted(np.flatnonzero(f["mask"][0]).tolist()) == case["support"]
    res = oracle.forward(H, W, rows, s=s)
    want = case["logprob"]
    if want == "-inf":
        assert res["logprob"][0] == -math.inf
        dZ = oracle.logit_grad(s, rows, np.ones(1))
        assert not dZ.any()
    else:
        assert abs(res["logprob"][0] - want) < 1e-12


# --------------------------------------------------------------------------
# closed form: identity metadata is the temperature log-softmax


def test_identity_rows_equal_log_softmax():
    rng = np.random.default_rng(7)
    T, V = 32, 257
    s = rng.standard_normal((T, V)) * 3
    y = rng.integers(0, V, T)
    for k, p, mu in [(0, 1.0, 0.0), (V, 1.0, 0.0), (-5, 1.0, 0.0), (V + 9, 1.0, 0.0)]:
        rows = _rows(T, y, 1.0, k, p, mu)
        res = oracle.forward(None, None, rows, s=s)
        want = s[np.arange(T), y] - scipy.special.logsumexp(s, axis=1)
        np.testing.assert_allclose(res["logprob"], want, rtol=0, atol=1e-12)
        assert (res["size"] == V).all()


def test_temperature_matches_scaled_cross_entropy_torch():
    """Per-row temperature equals scaled CE ('Testing' section)."""
    rng = np.random.default_rng(8)
    T, d, V = 16, 24, 97
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) / np.sqrt(d)
    tau = rng.uniform(0.3, 2.0, T).astype(np.float32)
    y = rng.integers(0, V, T)
    rows = _rows(T, y, tau)
    res = oracle.forward(H, W, rows)
    z = torch.tensor(H) @ torch.tensor(W).T
    ce = torch.nn.functional.cross_entropy(z / torch.tensor(tau, dtype=torch.float64)[:, None],
                                           torch.tensor(y), reduction="none")
    np.testing.assert_allclose(res["logprob"], -ce.numpy(), rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# brute force on tiny vocabularies


def _bruteforce_support(s, k, p, mu):
    """Pairwise-rank formulation with a subset enumeration for top-p.

    rank_i = #{j : s_j > s_i or (s_j == s_i and j < i)}; top-k keeps rank < k;
    top-p keeps the smallest upward-closed subset (in rank order) of the top-k
    set whose mass reaches p * Z_k, found by enumerating all subsets; min-p
    keeps exp(s_i - max) >= mu. The support is the intersection.
    """
    V = len(s)
    rank = np.array([sum(1 for j in range(V) if s[j] > s[i] or (s[j] == s[i] and j < i))
                     for i in range(V)])
    kk = V if (k <= 0 or k >= V) else k
    topk = {i for i in range(V) if rank[i] < kk}
    m = max(s)
    q = {i: math.exp(s[i] - m) for i in range(V)}
    if p >= 1.0:
        topp = set(topk)
    else:
        Zk = math.fsum(q[i] for i in topk)
        best = None
        members = sorted(topk)
        for r in range(1, len(members) + 1):
            for sub in itertools.combinations(members, r):
                sub = set(sub)
                worst = max(rank[i] for i in sub)
                closed = all(j in sub for j in topk if rank[j] < worst)
                if not closed:
                    continue
                if math.fsum(q[i] for i in sub) >= p * Zk:
                    best = sub
                    break
            if best is not None:
                break
        topp = best
    minp = {i for i in range(V) if mu <= 0 or q[i] >= mu}
    return topk & topp & minp


@pytest.mark.parametrize("seed", range(40))
def test_bruteforce_small_vocab(seed):
    rng = np.random.default_rng(100 + seed)
    V = int(rng.integers(2, 13))
    # coarse grid so exact ties are frequent
    s = rng.integers(-4, 5, V).astype(np.float64) * 0.5
    k = int(rng.choice([0, 1, 2, 3, V, V + 1, -1]))
    p = float(np.float32(rng.choice([1.0, 0.9, 0.5, 0.3, 0.75])))
    mu = float(np.float32(rng.choice([0.0, 0.05, 0.3, 1.0])))
    rows = _rows(1, 0, 1.0, k, p, mu)
    f = oracle.filter_rows(s[None], rows, want_mask=True)
    want = _bruteforce_support(s.tolist(), k, p, mu)
    assert set(np.flatnonzero(f["mask"][0]).tolist()) == want


def test_bruteforce_v16_random_reals():
    rng = np.random.default_rng(5)
    for _ in range(6):
        V = 16
        s = rng.standard_normal(V)
        for k, p, mu in [(0, 0.7, 0.0), (6, 0.6, 0.0), (0, 1.0, 0.2), (9, 0.85, 0.1)]:
            rows = _rows(1, 0, 1.0, k, p, mu)
            f = oracle.filter_rows(s[None], rows, want_mask=True)
            assert set(np.flatnonzero(f["mask"][0]).tolist()) == _bruteforce_support(s.tolist(), k, p, mu)


# --------------------------------------------------------------------------
# structural invariants


def test_support_invariants_and_monotonicity():
    rng = np.random.default_rng(11)
    V = 300
    for _ in range(20):
        s = rng.standard_normal(V) * rng.uniform(0.5, 4)
        s[rng.integers(0, V, 20)] = s[rng.integers(0, V, 20)]  # ties
        key = sorted(range(V), key=lambda i: (-s[i], i))
        prev = None
        for k in [0, 200, 100, 50, 10, 1]:
            for p in [1.0, 0.95, 0.8, 0.5, 0.1]:
                for mu in [0.0, 0.01, 0.1, 0.5]:
                    f = oracle.filter_row(s, k, p, mu)
                    S = set(f.order[: f.size].tolist())
                    # argmax (lowest id among maxima) always kept
                    assert key[0] in S
                    # a prefix of the (s desc, id asc) order
                    assert S == set(key[: f.size])
                    # renormalised support mass is one
                    lse = f.m + math.log(math.fsum(np.exp(s[list(S)] - f.m)))
                    assert abs(math.fsum(np.exp(s[list(S)] - lse)) - 1.0) < 1e-12
        # size is non-increasing as k/p shrink and mu grows
        for mu in [0.0, 0.02, 0.2]:
            sizes = [oracle.filter_row(s, 0, p, mu).size for p in [1.0, 0.9, 0.6, 0.3]]
            assert sizes == sorted(sizes, reverse=True)
        for p in [1.0, 0.7]:
            sizes = [oracle.filter_row(s, k, p, 0.0).size for k in [0, 150, 40, 3, 1]]
            assert sizes == sorted(sizes, reverse=True)
            sizes = [oracle.filter_row(s, 0, p, mu).size for mu in [0.0, 0.01, 0.1, 0.9]]
            assert sizes == sorted(sizes, reverse=True)
        prev = s
    assert prev is not None


def test_min_p_commutes_with_top_k():
    """min-p is a logit-space threshold against the unfiltered max, so cutting
    the row to its min-p survivors first and applying top-k afterwards gives
    the same support as the program."""
    rng = np.random.default_rng(12)
    for _ in range(30):
        V = 200
        s = rng.standard_normal(V) * 2
        mu = float(np.float32(rng.choice([0.01, 0.05, 0.3])))
        k = int(rng.integers(1, V))
        f = oracle.filter_row(s, k, 1.0, mu)
        keep_mu = np.flatnonzero(np.exp(s - s.max()) >= mu)
        sub = s[keep_mu]
        g = oracle.filter_row(sub, k, 1.0, 0.0)
        assert set(keep_mu[g.order[: g.size]].tolist()) == set(f.order[: f.size].tolist())


def test_top_p_one_identity_despite_fp32_cumulative_overshoot():
    """'What this PR does', item 1: top_p == 1.0 keeps the full support even
    where a float32 cumulative sum of the probabilities reaches 1 early."""
    V = 4096
    s = np.full(V, -30.0)
    s[0] = 0.0
    s[1:8] = -0.1
    p32 = (np.exp(s - s.max()) / np.exp(s - s.max()).sum()).astype(np.float32)
    excl32 = np.concatenate(([np.float32(0)], np.cumsum(p32, dtype=np.float32)[:-1]))
    # the premise: a float32 exclusive cumsum reaches >= 1.0 before the end
    assert (excl32 >= np.float32(1.0)).any()
    f = oracle.filter_row(s, 0, 1.0, 0.0)
    assert f.size == V
    # the just-below-one top_p does cut the float64 tail
    g = oracle.filter_row(s, 0, float(np.nextafter(np.float32(1), np.float32(0))), 0.0)
    assert g.size < V


def test_top_k_one_logprob():
    rng = np.random.default_rng(13)
    V = 50
    s = rng.standard_normal((4, V))
    s[:, 7] = s.max(axis=1) + 1.0
    s[:, 30] = s[:, 7]  # tied maximum, higher id
    rows = _rows(4, [7, 30, 7, 3], 1.0, 1)
    res = oracle.forward(None, None, rows, s=s)
    assert res["logprob"][0] == 0.0 and res["logprob"][2] == 0.0
    assert res["logprob"][1] == -math.inf and res["logprob"][3] == -math.inf


def test_logprob_clamped_to_nonpositive():
    """'Self-review pass': the selected score is clamped to <= 0."""
    rng = np.random.default_rng(14)
    V = 64
    s = rng.standard_normal((200, V)) * 20  # sharp rows: support often one token
    rows = _rows(200, np.argmax(s, axis=1), 1.0, 0, 0.3, 0.0)
    res = oracle.forward(None, None, rows, s=s)
    assert (res["logprob"] <= 0).all()
    assert (res["logprob"][res["size"] == 1] == 0).all()


# --------------------------------------------------------------------------
# gradients


def _torch_filtered_logprob_grad(H, W, tau, rows):
    """torch float64 autograd of s_y - logsumexp(s[S]) with S held fixed."""
    Ht = torch.tensor(H, requires_grad=True)
    Wt = torch.tensor(W, requires_grad=True)
    s = (Ht @ Wt.T) / torch.tensor(tau, dtype=torch.float64)[:, None]
    s_np = s.detach().numpy()
    f = oracle.filter_rows(s_np, rows, want_mask=True)
    mask = torch.tensor(f["mask"])
    y = torch.tensor(rows["target"])
    masked = torch.where(mask, s, torch.tensor(-math.inf, dtype=torch.float64))
    lp = s[torch.arange(len(y)), y] - torch.logsumexp(masked, dim=1)
    inside = mask[torch.arange(len(y)), y]
    total = torch.where(inside, lp, torch.zeros_like(lp)).sum()
    total.backward()
    return Ht.grad.numpy(), Wt.grad.numpy()


def test_vjp_matches_torch_autograd_support_fixed():
    rng = np.random.default_rng(21)
    T, d, V = 24, 16, 120
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) / np.sqrt(d) * 2
    tau = rng.uniform(0.5, 1.5, T).astype(np.float32)
    s = oracle.scaled_logits(H, W, tau)
    k = rng.choice([0, 5, 40], T)
    p = rng.choice([1.0, 0.9, 0.6], T).astype(np.float32)
    mu = rng.choice([0.0, 0.05], T).astype(np.float32)
    rows0 = _rows(T, 0, tau, k, p, mu)
    y = oracle.sample_rows(s, rows0, rng.random(T))
    y[:3] = np.argsort(s[:3], axis=1)[:, 0]  # some rows out of support
    rows = _rows(T, y, tau, k, p, mu)
    dH, dW = oracle.backward(H, W, rows, np.ones(T))
    tH, tW = _torch_filtered_logprob_grad(H, W, tau, rows)
    np.testing.assert_allclose(dH, tH, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dW, tW, rtol=0, atol=1e-12)


def test_unfiltered_vjp_is_teach_signal_form():
    """For unfiltered rows with tau = 1 and g = -1/n the hidden gradient is the
    mean-CE teaching signal (softmax - onehot) . W / n of the nested-learning
    trainer page ('compute_teach_signal')."""
    rng = np.random.default_rng(22)
    T, d, V = 10, 12, 40
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d))
    y = rng.integers(0, V, T)
    rows = _rows(T, y)
    dH, _ = oracle.backward(H, W, rows, np.full(T, -1.0 / T))
    logits = torch.tensor(H) @ torch.tensor(W).T
    probs = torch.softmax(logits, dim=-1)
    resid = probs.clone()
    resid[torch.arange(T), torch.tensor(y)] -= 1.0
    want = (resid @ torch.tensor(W)).numpy() / T
    np.testing.assert_allclose(dH, want, rtol=0, atol=1e-12)


def test_vjp_central_finite_differences():
    rng = np.random.default_rng(23)
    T, d, V = 6, 8, 60
    H = rng.standard_normal((T, d))
    W = rng.standard_normal((V, d)) / np.sqrt(d) * 2
    tau = rng.uniform(0.6, 1.4, T).astype(np.float32)
    k = np.array([0, 10, 0, 30, 0, 0])
    p = np.array([0.8, 1.0, 0.7, 0.9, 1.0, 1.0], dtype=np.float32)
    mu = np.array([0.0, 0.0, 0.05, 0.0, 0.1, 0.0], dtype=np.float32)
    s = oracle.scaled_logits(H, W, tau)
    rows = _rows(T, 0, tau, k, p, mu)
    y = oracle.sample_rows(s, rows, np.full(T, 0.3))
    rows["target"] = y
    gaps = oracle.row_gaps(s, rows)
    assert gaps.min() > 1e-3, "pick a seed whose thresholds are far from ties"
    g = rng.standard_normal(T)
    dH, dW = oracle.backward(H, W, rows, g)

    def loss(Hx, Wx):
        r = oracle.forward(Hx, Wx, rows)
        return float(np.dot(g, r["logprob"]))

    h = 1e-6
    for (t, j) in [(0, 1), (1, 3), (2, 0), (3, 7), (5, 5)]:
        Hp, Hm = H.copy(), H.copy()
        Hp[t, j] += h
        Hm[t, j] -= h
        fd = (loss(Hp, W) - loss(Hm, W)) / (2 * h)
        assert abs(fd - dH[t, j]) <= 1e-6 * max(1.0, abs(dH[t, j]))
    for (v, j) in [(int(y[0]), 2), (int(y[3]), 4), (11, 1), (59, 7)]:
        Wp, Wm = W.copy(), W.copy()
        Wp[v, j] += h
        Wm[v, j] -= h
        fd = (loss(H, Wp) - loss(H, Wm)) / (2 * h)
        assert abs(fd - dW[v, j]) <= 1e-6 * max(1.0, abs(dW[v, j]))


# --------------------------------------------------------------------------
# sampler and gaps


def test_sampler_inverse_cdf_frequencies():
    """Draws follow the renormalised support distribution."""
    s = np.log(np.array([[4.0, 2.0, 1.0, 1.0, 0.5]]))
    rows = _rows(1, 0, 1.0, 0, 0.9, 0.0)  # support {0,1,2,3}
    u = (np.arange(20000) + 0.5) / 20000
    ys = np.array([oracle.sample_rows(s, rows, [ui])[0] for ui in u[::10]])
    freq = np.bincount(ys, minlength=5) / len(ys)
    np.testing.assert_allclose(freq, [0.5, 0.25, 0.125, 0.125, 0.0], atol=2e-3)


def test_row_gaps_detect_near_ties():
    s = np.array([[3.0, 2.0, 2.0 - 1e-9, 0.0]])
    rows = _rows(1, 0, 1.0, 2, 1.0, 0.0)
    assert oracle.row_gaps(s, rows)[0, 0] < 1e-8
    rows = _rows(1, 0, 1.0, 1, 1.0, 0.0)
    assert oracle.row_gaps(s, rows)[0, 0] == pytest.approx(1.0)


GAPS = os.path.join(os.path.dirname(__file__), "golden", "threshold_gaps.json")


def _gap_cases():
    with open(GAPS) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _gap_cases(), ids=lambda c: c["name"])
def test_row_gaps_hand_worked(case):
    """gap_k, gap_p and gap_mu of hand-worked rows, including the rule that a
    gap only counts where its prefix ends within one position of the support."""
    s = np.log(np.array([case["weights"]], dtype=np.float64))
    rows = _rows(1, 0, 1.0, case["top_k"], case["top_p"], case["min_p"])
    assert oracle.filter_rows(s, rows)["size"][0] == case["size"]
    got = oracle.row_gaps(s, rows)[0]
    for g, want in zip(got, case["gaps"]):
        if want == "inf":
            assert g == math.inf
        else:
            assert abs(g - want) < 1e-12, (g, want)


def _distance_to_change(f, x0, lo, hi):
    """Distance from x0 to the nearest x in [lo, hi] where the integer
    function f changes value, by bisection on each side (inf if none)."""
    v0 = f(x0)
    best = math.inf
    for end in (lo, hi):
        if f(end) == v0:
            continue
        a, b = x0, end  # f(a) == v0, f(b) != v0
        for _ in range(200):
            mid = 0.5 * (a + b)
            if mid == a or mid == b:
                break
            if f(mid) == v0:
                a = mid
            else:
                b = mid
        best = min(best, abs(b - x0))
    return best


def test_row_gaps_match_bisection_on_random_rows():
    """An independent formulation of the gaps on random rows (V <= 12): the
    distance, found by bisection, by which p (in units of the top-k mass) or
    ln(min_p) (in logit units) must move before the rule's own prefix length
    m_p or m_mu changes -- compared with the closed forms of row_gaps wherever
    the rule can move the support (its prefix within one position of it)."""
    rng = np.random.default_rng(11)
    checked = {"p": 0, "mu": 0}
    for _ in range(400):
        V = int(rng.integers(3, 12))
        s = rng.standard_normal(V) * 2
        k = int(rng.choice([0, 2, 3, V]))
        p = float(np.float32(rng.choice([1.0, 0.5, 0.75, 0.9, 0.3])))
        mu = float(np.float32(rng.choice([0.0, 0.1, 0.3, 0.6])))
        rows = _rows(1, 0, 1.0, k, p, mu)
        base = oracle.filter_row(s, k, p, mu)
        gaps = oracle.row_gaps(s[None, :], rows)[0]
        live = base.size + 1
        if p < 1.0:
            want = _distance_to_change(lambda x: oracle.filter_row(s, k, x, mu).m_p, p, 1e-12, 1.0 - 1e-15)
            if base.m_p <= live:
                assert abs(gaps[1] - want) < 1e-9, (gaps, want, s, k, p, mu)
                checked["p"] += 1
            else:
                assert gaps[1] == math.inf
        if mu > 0.0:
            lm = math.log(mu)
            want = _distance_to_change(
                lambda x: oracle.filter_row(s, k, p, math.exp(x)).m_mu, lm, lm - 60.0, 0.0)
            if base.m_mu <= live:
                assert abs(gaps[2] - want) < 1e-9, (gaps, want, s, k, p, mu)
                checked["mu"] += 1
            else:
                assert gaps[2] == math.inf
    assert checked["p"] > 50 and checked["mu"] > 50, checked


def test_workload_inputs_are_bf16_and_seeded():
    a = workloads.make(1)
    b = workloads.make(1)
    assert np.array_equal(a["H"], b["H"]) and np.array_equal(a["W"], b["W"])
    Hf = workloads.bf16_to_f32(a["H"])
    assert np.array_equal(workloads.f32_to_bf16_bits(Hf), a["H"])
    assert abs(Hf.std() - 1.0) < 0.05
    Wf = workloads.bf16_to_f32(a["W"])
    assert abs(Wf.std() * np.sqrt(128) - 1.0) < 0.05
    # round-to-nearest-even on a hand-picked tie: 1 + 2^-8 is halfway between
    # bf16 1.0 and 1 + 2^-7 and rounds to the even mantissa (1.0)
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    assert workloads.bf16_to_f32(workloads.f32_to_bf16_bits(x)).tolist() == [1.0, 1.0 + 2.0 ** -6]


def test_stress_workload_duplicates_rows():
    d = workloads.make(5, T=8, with_weights=False)
    assert len(d["dup_dst"]) == round(0.05 * 262144)
    assert (d["dup_src"] < d["dup_dst"]).all()


# ---------------------------------------------------------------- policy-gradient coefficient

def _pg_inputs(n=400, seed=31):
    rng = np.random.Generator(np.random.PCG64(seed))
    lp = -rng.exponential(2.0, n)
    old = lp + rng.normal(0.0, 0.4, n)  # ratios spread around 1, many clipped
    adv = rng.normal(0.0, 1.0, n)
    adv[::17] = 0.0
    return lp, old, adv


@pytest.mark.parametrize("objective", ["cispo", "clipped"])
def test_policy_grad_is_the_autograd_of_the_loss(objective):
    """The coefficient is the float64 autograd of the loss written out as the
    passage defines it: L = -sum sg(min(r, 1+eh)) A logprob (CISPO) or
    L = -sum min(r A, clip(r, 1-el, 1+eh) A) (clipped surrogate)."""
    lp, old, adv = _pg_inputs()
    el, eh, scale = 0.2, 0.28, 1.0 / 400
    x = torch.tensor(lp, dtype=torch.float64, requires_grad=True)
    o = torch.tensor(old, dtype=torch.float64)
    a = torch.tensor(adv, dtype=torch.float64)
    r = torch.exp(x - o)
    if objective == "cispo":
        loss = -(torch.clamp(r, max=1 + eh).detach() * a * x).sum() * scale
    else:
        loss = -torch.minimum(r * a, torch.clamp(r, 1 - el, 1 + eh) * a).sum() * scale
    loss.backward()
    got = oracle.policy_grad(lp, old, adv, objective, el, eh, scale)
    rr = np.exp(lp - old)
    # away from the clip boundaries, where the loss is not differentiable
    ok = (np.abs(rr - (1 + eh)) > 1e-9) & (np.abs(rr - (1 - el)) > 1e-9)
    assert ok.sum() > 350
    np.testing.assert_allclose(got[ok], x.grad.numpy()[ok], rtol=1e-12, atol=1e-15)
    # both clip regimes occur in the sample
    assert (rr > 1 + eh).any() and (rr < 1 - el).any()


def test_policy_grad_special_rows():
    lp = np.array([-np.inf, np.nan, -1.0, -1.0, -1.0, -1.0])
    old = np.array([-2.0, -2.0, -1.0, -1.5, -0.5, -1.5])
    adv = np.array([1.0, 1.0, 0.0, 2.0, -2.0, -2.0])
    c = oracle.policy_grad(lp, old, adv, "cispo", 0.2, 0.3, 1.0)
    assert c[0] == 0.0 and c[1] == 0.0 and c[2] == 0.0  # out of support, invalid, A = 0
    assert c[3] == -2.0 * 1.3  # r = e^0.5 > 1.3: the weight saturates at 1 + eps_high
    assert c[4] == pytest.approx(2.0 * np.exp(-0.5), rel=1e-15)  # no lower bound for CISPO
    k = oracle.policy_grad(lp, old, adv, "clipped", 0.2, 0.3, 1.0)
    assert k[3] == 0.0  # A > 0, r above 1 + eps_high: clipped
    assert k[4] == 0.0  # A < 0, r = e^-0.5 below 1 - eps_low: clipped
    assert k[5] == pytest.approx(2.0 * np.exp(0.5), rel=1e-15)  # A < 0, r above 1: not clipped
    with pytest.raises(ValueError):
        oracle.policy_grad(lp, old, adv, "ppo")


def test_policy_grad_non_finite_inputs_and_overflowing_ratio():
    """Rows with a non-finite old logprob or advantage carry no signal (0); a
    ratio that overflows float64 saturates the CISPO weight at 1 + eps_high,
    is clipped for A >= 0 and gives an infinite gradient for A < 0 in the
    clipped surrogate (d(r A)/dlogprob = r A is unbounded there)."""
    lp = np.array([-1.0, -1.0, -1.0, -1.0, -0.5, -0.5])
    old = np.array([np.nan, -np.inf, -1.0, -2.0, -1000.0, -1000.0])
    adv = np.array([1.0, 1.0, np.inf, np.nan, 1.0, -1.0])
    c = oracle.policy_grad(lp, old, adv, "cispo", 0.2, 0.3, 1.0)
    assert c.tolist()[:4] == [0.0, 0.0, 0.0, 0.0]
    assert c[4] == -1.3 and c[5] == 1.3  # r = e^999.5 overflows: weight 1 + eps_high
    k = oracle.policy_grad(lp, old, adv, "clipped", 0.2, 0.3, 1.0)
    assert k.tolist()[:5] == [0.0, 0.0, 0.0, 0.0, 0.0]
    assert k[5] == math.inf
    z = oracle.policy_grad(lp, old, adv, "clipped", 0.2, 0.3, 0.0)  # scale 0: no signal
    assert not z.any()

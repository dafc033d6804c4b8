"""Kernel-level GPU tests through the C ABI: the tcgen05 logits GEMM (first
pass of the forward) and the exact support resolver (filter hook), each
against an independent reference on the same inputs."""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import bf16_tensor, f32_values

pytestmark = pytest.mark.gpu


def _rand_hw(seed, T, d, V):
    rng = np.random.Generator(np.random.PCG64(seed))
    H = workloads.f32_to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))
    W = workloads.f32_to_bf16_bits(rng.standard_normal((V, d), dtype=np.float32)
                                   * np.float32(1 / math.sqrt(d)))
    tau = rng.uniform(0.5, 1.5, T).astype(np.float32)
    return H, W, tau


@pytest.mark.parametrize("T,d,V", [(128, 64, 256), (300, 136, 1000), (513, 1024, 4100), (64, 8, 7),
                                   (1, 2048, 300)])
def test_scaled_logits_against_float64(cuda_lib, T, d, V):
    """S = (H . W^T) / tau with fp32 accumulation against the float64 product of
    the same bf16 values (ragged M, N and K tails included)."""
    sts = cuda_lib
    H, W, tau = _rand_hw(10 + T + d + V, T, d, V)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    taud = torch.from_numpy(tau).cuda()
    S = sts.sts_scaled_logits(Hd, Wd, taud).cpu().numpy()
    ref = oracle.scaled_logits(f32_values(H), f32_values(W), tau)
    # fp32 accumulation of d products of magnitude ~1/sqrt(d): error ~ sqrt(d) ulp
    err = np.abs(S - ref).max()
    assert err < 2e-5 * max(1.0, math.sqrt(d) / 8), err
    # the division is the IEEE fp32 quotient of the fp32 accumulator: re-dividing
    # the recovered product reproduces S exactly for the vast majority of entries
    assert np.isfinite(S).all()


def test_scaled_logits_sub_block_is_bit_identical(cuda_lib):
    """A tile computed inside a sub-block launch equals the same tile of the full
    launch bit for bit: the backward's recompute can trust the forward's cuts."""
    sts = cuda_lib
    T, d, V = 384, 520, 1300
    H, W, tau = _rand_hw(3, T, d, V)
    Hd, Wd = bf16_tensor(H), bf16_tensor(W)
    taud = torch.from_numpy(tau).cuda()
    full = sts.sts_scaled_logits(Hd, Wd, taud)
    sub = sts.sts_scaled_logits(Hd, Wd, taud, t0=128, rows=200, v0=256, cols=700)
    assert torch.equal(full[128:328, 256:956], sub)
    sub2 = sts.sts_scaled_logits(Hd, Wd, taud, t0=256, rows=128, v0=1024, cols=276)
    assert torch.equal(full[256:384, 1024:1300], sub2)


def test_scaled_logits_large_k(cuda_lib):
    """Long K loop (d = 5120, the headline hidden size) over several M/N tiles."""
    sts = cuda_lib
    T, d, V = 256, 5120, 768
    H, W, tau = _rand_hw(4, T, d, V)
    S = sts.sts_scaled_logits(bf16_tensor(H), bf16_tensor(W), torch.from_numpy(tau).cuda())
    ref = oracle.scaled_logits(f32_values(H), f32_values(W), tau)
    assert np.abs(S.cpu().numpy() - ref).max() < 1e-4


# --------------------------------------------------------------------------
# the support program on given fp32 logits: bit-exact against the oracle


def _filter_case():
    """Rows built to reach every branch of the resolver (V = 20000 > the
    4096-entry candidate buffer)."""
    rng = np.random.Generator(np.random.PCG64(77))
    V = 20000
    rows, meta = [], []

    def add(s, k, p, mu):
        rows.append(np.asarray(s, np.float32))
        meta.append((k, p, mu))

    for i in range(12):  # flat random rows, mixed filters
        s = rng.standard_normal(V).astype(np.float32) / np.float32(rng.uniform(0.4, 1.6))
        add(s, [0, 20, 50, 3000][i % 4], [1.0, 0.9, 0.5, 0.95][(i // 4) % 4], [0.0, 0.05, 0.1][i % 3])
    for k in (1, 5, 50, 7000):  # coarse grid: many exact ties
        s = (rng.integers(-20, 5, V) * 0.25).astype(np.float32)
        add(s, k, 0.8, 0.0)
    z = np.zeros(V, np.float32)  # one giant tie group: top-k and top-p inside it
    add(z, 3, 1.0, 0.0)
    add(z, 0, 0.5, 0.0)
    add(z, 12345, 0.7, 0.0)
    dense = (1.0 + np.arange(V) * 2.0 ** -20).astype(np.float32)[rng.permutation(V)]
    add(dense, 10000, 0.5, 0.0)  # distinct values packed into very few buckets
    add(dense, 0, 0.3, 0.0)
    tie_max = rng.standard_normal(V).astype(np.float32)
    tie_max[[5, 900, 19999]] = tie_max.max() + 1.0
    add(tie_max, 1, 1.0, 0.0)
    add(tie_max, 0, 1.0, 1.0)
    signed0 = np.where(rng.random(V) < 0.5, np.float32(0.0), np.float32(-0.0)).astype(np.float32)
    signed0[:100] = 1.0
    add(signed0, 150, 1.0, 0.0)
    tail = rng.standard_normal(V).astype(np.float32)
    tail[V // 2:] -= 80.0  # far tail beyond the level-0 bucket range
    add(tail, 0, 0.9999, 0.0)
    add(tail, 15000, 1.0, 0.0)
    add(rng.standard_normal(V).astype(np.float32) * 6, 0, 1e-6, 0.0)
    add(rng.standard_normal(V).astype(np.float32), 0, float(np.nextafter(np.float32(1), np.float32(0))), 0.0)
    add(rng.standard_normal(V).astype(np.float32), V, 1.0, 0.0)
    add(rng.standard_normal(V).astype(np.float32), -3, 1.0, 0.01)
    # the planning sample reads float4 sweeps 0, 8, 16, ... of 512 float4s:
    # elements [0, 2048) and [16384, 18432) here. Rows whose sample is
    # unrepresentative must still resolve exactly (the plan is only checked).
    skew = rng.standard_normal(V).astype(np.float32)
    skew[:2048] -= 6.0
    skew[16384:18432] -= 6.0
    add(skew, 0, 0.9, 0.0)
    add(skew, 30, 0.9, 0.05)
    add(skew, 0, 1.0, 0.2)
    hot = rng.standard_normal(V).astype(np.float32) - 4.0
    hot[:2048] += 6.0  # the sample sees only the top of the row
    add(hot, 0, 0.7, 0.0)
    add(hot, 100, 1.0, 0.0)
    add(rng.standard_normal(V).astype(np.float32), 0, 1.0, 1e-30)  # threshold in the far tail
    peaked = (rng.standard_normal(V) * 0.01 - 30.0).astype(np.float32)
    peaked[123] = 0.0  # min-p keeps the max alone; no sampled bucket before it
    add(peaked, 0, 1.0, 0.5)
    add(peaked, 0, 0.5, 0.5)
    # large top-k (more than the 4096-entry sort up to the k-th element's
    # bucket): the k-th element inside its own bucket, then top-p on the
    # top-k mass and min-p before, at or after that bucket
    for kk in (6000, 9000, 15000):
        for pp, mm in ((1.0, 0.0), (0.9, 0.0), (1.0, 0.02), (0.95, 0.3)):
            add(rng.standard_normal(V).astype(np.float32), kk, pp, mm)
    S = np.stack(rows)
    T = S.shape[0]
    md = {
        "top_k": np.array([m[0] for m in meta], np.int32),
        "top_p": np.array([m[1] for m in meta], np.float32),
        "min_p": np.array([m[2] for m in meta], np.float32),
        "temperature": np.ones(T, np.float32),
        "target": np.zeros(T, np.int64),
    }
    return S, md


ENT_RTOL, ENT_ATOL = 2e-6, 1e-6  # fp32 output of a float64 sum on the same fp32 logits


def _check_entropy(got, S, md):
    want = oracle.entropy(S, md)
    np.testing.assert_allclose(got.cpu().numpy(), want, rtol=ENT_RTOL, atol=ENT_ATOL)


def test_filter_bit_exact_against_oracle(cuda_lib):
    sts = cuda_lib
    S, md = _filter_case()
    T, V = S.shape
    out = sts.sts_filter_logits(torch.from_numpy(S).cuda(), torch.from_numpy(md["top_k"]).cuda(),
                                torch.from_numpy(md["top_p"]).cuda(),
                                torch.from_numpy(md["min_p"]).cuda(), want_mask=True,
                                want_entropy=True, check=True)
    ref = oracle.filter_rows(S, md, want_mask=True)
    size = out["size"].cpu().numpy()
    cid = out["cut_id"].cpu().numpy()
    cval = out["cut_logit"].cpu().numpy()
    mask = out["mask"].cpu().numpy().astype(bool)
    bad = [t for t in range(T) if size[t] != ref["size"][t] or cid[t] != ref["cut_id"][t]]
    assert not bad, [(t, size[t], ref["size"][t], cid[t], ref["cut_id"][t]) for t in bad]
    assert np.array_equal(cval, S[np.arange(T), ref["cut_id"]])
    assert np.array_equal(mask, ref["mask"])
    # the entropy of each filtered distribution, every resolver path included
    _check_entropy(out["entropy"], S, md)


def test_filter_odd_vocab_scalar_path(cuda_lib):
    """A row stride that is not a multiple of four floats takes the scalar
    load path of every pass (planning sample included): bit-exact too."""
    sts = cuda_lib
    rng = np.random.Generator(np.random.PCG64(81))
    T, V = 40, 7001
    S = (rng.standard_normal((T, V), dtype=np.float32)
         / rng.uniform(0.4, 1.6, T).astype(np.float32)[:, None])
    S[5:10, ::7] = S[5:10, :1]  # exact ties
    md = {
        "top_k": rng.choice(np.array([0, 1, 20, 700, 7001], np.int32), T).astype(np.int32),
        "top_p": rng.choice(np.array([1.0, 0.95, 0.6, 0.2], np.float32), T).astype(np.float32),
        "min_p": rng.choice(np.array([0.0, 0.02, 0.3], np.float32), T).astype(np.float32),
        "temperature": np.ones(T, np.float32),
        "target": np.zeros(T, np.int64),
    }
    out = sts.sts_filter_logits(torch.from_numpy(S).cuda(), torch.from_numpy(md["top_k"]).cuda(),
                                torch.from_numpy(md["top_p"]).cuda(),
                                torch.from_numpy(md["min_p"]).cuda(), want_mask=True,
                                want_entropy=True, check=True)
    ref = oracle.filter_rows(S, md, want_mask=True)
    assert np.array_equal(out["size"].cpu().numpy(), ref["size"])
    assert np.array_equal(out["cut_id"].cpu().numpy(), ref["cut_id"])
    assert np.array_equal(out["mask"].cpu().numpy().astype(bool), ref["mask"])
    _check_entropy(out["entropy"], S, md)


def test_filter_flat_rows_full_vocab(cuda_lib):
    """Headline-shaped flat rows (V = 152064, s ~ N(0, 1/tau^2)): top-p keeps
    tens of thousands of tokens; the cut must still be exact."""
    sts = cuda_lib
    rng = np.random.Generator(np.random.PCG64(78))
    T, V = 24, 152064
    S = (rng.standard_normal((T, V), dtype=np.float32)
         / rng.uniform(0.5, 1.5, T).astype(np.float32)[:, None])
    md = {
        "top_k": np.where(np.arange(T) % 3 == 0, 50, 0).astype(np.int32),
        "top_p": rng.uniform(0.8, 1.0, T).astype(np.float32),
        "min_p": np.where(np.arange(T) % 2 == 0, 0.05, 0.0).astype(np.float32),
        "temperature": np.ones(T, np.float32),
        "target": np.zeros(T, np.int64),
    }
    md["top_p"][::5] = 1.0
    ws = torch.empty(sts.sts_workspace_bytes(T, 8, V, 2), dtype=torch.uint8, device="cuda")
    out = sts.sts_filter_logits(torch.from_numpy(S).cuda(), torch.from_numpy(md["top_k"]).cuda(),
                                torch.from_numpy(md["top_p"]).cuda(),
                                torch.from_numpy(md["min_p"]).cuda(), ws=ws, check=True)
    paths = sts.sts_path_counts(ws)
    print("resolver paths:", paths)
    assert sum(paths.values()) == T
    # top-k rows are decided by the sampled plan and one gathering pass
    assert paths["planned"] >= int((md["top_k"] > 0).sum()), paths
    ref = oracle.filter_rows(S, md)
    gaps = oracle.row_gaps(S, md).min(axis=1)
    size = out["size"].cpu().numpy()
    cid = out["cut_id"].cpu().numpy()
    mism = (size != ref["size"]) | (cid != ref["cut_id"])
    # a mismatch is only acceptable where float64 summation order could decide it
    assert not (mism & (gaps > 1e-12)).any(), np.flatnonzero(mism)


def test_large_top_k_takes_the_direct_path(cuda_lib):
    """Headline-shaped rows with top-k between 4096 and V: decided by the
    count pass and one exact pass (the k-th element located in its bucket),
    not by the exact search; bit-exact against the oracle."""
    sts = cuda_lib
    rng = np.random.Generator(np.random.PCG64(82))
    T, V = 12, 152064
    S = (rng.standard_normal((T, V), dtype=np.float32)
         / rng.uniform(0.6, 1.4, T).astype(np.float32)[:, None])
    md = {
        "top_k": np.array([5000, 20000, 70000, 150000] * 3, np.int32),
        "top_p": np.array([1.0] * 8 + [0.9] * 4, np.float32),
        "min_p": np.array([0.0] * 4 + [0.05] * 4 + [0.0] * 4, np.float32),
        "temperature": np.ones(T, np.float32),
        "target": np.zeros(T, np.int64),
    }
    ws = torch.empty(sts.sts_workspace_bytes(T, 8, V, 2), dtype=torch.uint8, device="cuda")
    out = sts.sts_filter_logits(torch.from_numpy(S).cuda(), torch.from_numpy(md["top_k"]).cuda(),
                                torch.from_numpy(md["top_p"]).cuda(),
                                torch.from_numpy(md["min_p"]).cuda(), ws=ws, want_entropy=True,
                                check=True)
    paths = sts.sts_path_counts(ws)
    print("resolver paths:", paths)
    assert paths["exact"] == 0, paths
    ref = oracle.filter_rows(S, md)
    gaps = oracle.row_gaps(S, md).min(axis=1)
    size = out["size"].cpu().numpy()
    cid = out["cut_id"].cpu().numpy()
    mism = (size != ref["size"]) | (cid != ref["cut_id"])
    assert not (mism & (gaps > 1e-12)).any(), np.flatnonzero(mism)
    ok = ~mism
    np.testing.assert_allclose(out["entropy"].cpu().numpy()[ok], oracle.entropy(S, md)[ok],
                               rtol=ENT_RTOL, atol=ENT_ATOL)


def _estimate_defeating_rows():
    """Rows whose logits sit on bucket edges, so that weighting every element
    by its bucket's mid-point mass (the resolver's planning estimate) is off
    by up to 0.39 % per bucket: the top-p crossing lands outside the planned
    window (a retry with the wider window, or the exact search). The rows'
    min-p alternates between off and 0.01."""
    rng = np.random.Generator(np.random.PCG64(79))
    V = 152064
    rows, ps = [], []
    # a heavy bucket at its top edge followed by one at its bottom edge: the
    # crossing's bucket is misjudged by one. With 1300 logits per bucket the
    # 3-bucket retry holds it; with 6000 the window exceeds the candidate
    # buffer and the exact search decides.
    for n, p_list in ((1300, (0.5026, 0.5032)), (6000, (0.5025,))):
        s = np.full(V, -40.0, np.float32)
        s[0] = 0.0
        s[1:n + 1] = np.float32(-10 / 128)
        s[n + 1:2 * n + 1] = np.float32(-12 / 128 + 2.0 ** -20)
        s[2 * n + 1:2 * n + 8000] = (rng.standard_normal(7999) * 0.5 - 8).astype(np.float32)
        for p in p_list:
            rows.append(s)
            ps.append(p)
    # 600 light buckets of three equal logits, then 150,000 logits on one
    # bucket edge: the mass estimate shifts the crossing by >10 buckets
    s = np.empty(V, np.float32)
    s[0] = 0.0
    for b in range(1, 601):
        s[3 * b - 2:3 * b + 1] = np.float32(-(b + 0.5) / 128)
    s[1801:] = np.float32(-700 / 128)
    for p in (0.3411794900894165, 0.36984652280807495):
        rows.append(s)
        ps.append(p)
    S = np.stack(rows)
    T = S.shape[0]
    md = {
        "top_k": np.zeros(T, np.int32),
        "top_p": np.array(ps, np.float32),
        "min_p": np.where(np.arange(T) % 2 == 1, 0.01, 0.0).astype(np.float32),
        "temperature": np.ones(T, np.float32),
        "target": np.zeros(T, np.int64),
    }
    return S, md


def test_filter_when_the_planning_estimate_is_wrong(cuda_lib):
    sts = cuda_lib
    S, md = _estimate_defeating_rows()
    T, V = S.shape
    ws = torch.empty(sts.sts_workspace_bytes(T, 8, V, 2), dtype=torch.uint8, device="cuda")
    out = sts.sts_filter_logits(torch.from_numpy(S).cuda(), torch.from_numpy(md["top_k"]).cuda(),
                                torch.from_numpy(md["top_p"]).cuda(),
                                torch.from_numpy(md["min_p"]).cuda(), ws=ws, want_entropy=True,
                                check=True)
    paths = sts.sts_path_counts(ws)
    print("resolver paths:", paths)
    assert paths["fast"] + paths["exact"] > 0  # the fallbacks are exercised
    _check_entropy(out["entropy"], S, md)
    ref = oracle.filter_rows(S, md)
    assert oracle.row_gaps(S, md).min() > 1e-6  # no near-tie decides these rows
    T = S.shape[0]
    size = out["size"].cpu().numpy()
    cid = out["cut_id"].cpu().numpy()
    assert np.array_equal(size, ref["size"]) and np.array_equal(cid, ref["cut_id"]), (size, ref["size"])
    assert np.array_equal(out["cut_logit"].cpu().numpy(), S[np.arange(T), ref["cut_id"]])


def test_filter_rejects_bad_rows(cuda_lib):
    sts = cuda_lib
    T, V = 4, 100
    S = torch.randn(T, V, device="cuda")
    k = torch.zeros(T, dtype=torch.int32, device="cuda")
    p = torch.tensor([1.0, 0.0, 0.5, 1.5], device="cuda")
    mu = torch.tensor([0.0, 0.0, -0.1, 0.0], device="cuda")
    ws = torch.empty(sts.sts_workspace_bytes(T, 8, V, 2), dtype=torch.uint8, device="cuda")
    out = sts.sts_filter_logits(S, k, p, mu, ws=ws)
    status, row = sts.sts_get_status(ws)
    assert (status, row) == (6, 1)  # STS_ERR_TOP_P, reported at the first bad row
    size = out["size"].cpu().tolist()
    assert size[0] == V and size[1] == 0 and size[2] == 0 and size[3] == 0


def test_table_driven_mass_exp_against_library_and_numpy(cuda_lib):
    """The resolver's float64 token mass (table-driven exp, Tang 1989) agrees
    with the CUDA library exp and with numpy's exp to a few ulp over the whole
    bucket range, including the clamped far tail."""
    sts = cuda_lib
    rng = np.random.Generator(np.random.PCG64(5))
    m = np.float32(3.7)
    gaps = np.concatenate([np.linspace(0, 40, 400001), rng.uniform(0, 33, 200000),
                           np.arange(0, 4096) / 128.0])
    s = (m - gaps).astype(np.float32)
    mine, lib = sts.sts_probe_mass_exp(torch.from_numpy(s).cuda(), float(m))
    mine = mine.cpu().numpy()
    lib = lib.cpu().numpy()
    ref = np.exp(s.astype(np.float64) - np.float64(m))
    ulp = np.spacing(ref)
    assert np.abs(mine - ref).max() <= 4 * ulp.max() and (np.abs(mine - ref) <= 4 * ulp).all()
    assert (np.abs(mine - lib) <= 4 * np.spacing(lib)).all()

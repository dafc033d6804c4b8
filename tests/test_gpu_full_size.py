"""Parity at the full sizes of the three large workloads, in the launch
configuration the benchmark times (default row chunk, the workload's vocabulary
chunk, all rows on the GPU), on a seeded sample of N_TILES whole 128-row tiles
(512 rows) that the float64 oracle computes row by row.

Checks, each able to fail on any sampled row:
  1. support size equal to the oracle's on every row that is not near-gap
     (every threshold that can move the support further than 1e-4 from its
     boundary); a near-gap row may take another valid size (counted);
  2. logprob and target membership on every row: against the oracle's, or,
     where the support size legitimately differs, against the oracle's
     logprob on the GPU's support (within 2e-3);
  2b. the forward without the entropy output (the benchmark's, with fp32
     masses where no mass comparison decides the support): the same support
     decisions on every row and its logprob within 3e-5 of the other's;
  3. the forward's cuts (support size, cut id, cut logit) bit-exact against
     the oracle's support program run on the GPU's own fp32 logits of the
     same rows (same fp32 values, every decision in float64 on both sides);
     a difference is only allowed where that row's top-p crossing is within
     1e-12 of a boundary (float64 summation order);
  4. the entropy of each filtered distribution (the forward's optional
     output) against the oracle's: within 1e-3 on the float64 logits and the
     GPU's support, and to fp32 rounding on the GPU's own fp32 logits;
  5. dH on the sampled rows and dW on ~1000 sampled vocabulary rows (the
     upstream gradient is 1 on the sampled rows whose support equals the
     oracle's, 0 elsewhere, so dW stays comparable): relative Frobenius
     error < 1e-2.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import (GAP_EPS, GRAD_RTOL, OraclePool, assert_same_decisions, bf16_tensor,
                     compare_logprob, f32_values, grad_rows, rel_fro)

pytestmark = pytest.mark.gpu

N_TILES = 4  # 128-row tiles: 512 sampled rows
N_VOCAB = 1024


@pytest.fixture(scope="module")
def pool():
    p = OraclePool()
    yield p
    p.close()


@pytest.mark.parametrize("index", [3, 4, 5])
def test_full_size_workload(cuda_lib, pool, index):
    sts = cuda_lib
    data = workloads.make(index)
    wl = data["workload"]
    T, d, V = wl.T, wl.d, wl.V
    rng = np.random.Generator(np.random.PCG64(3000 + index))
    tiles = np.sort(rng.choice(T // 128, N_TILES, replace=False))
    sel = (tiles[:, None] * 128 + np.arange(128)[None, :]).reshape(-1)
    meta_sel = {k: data[k][sel] for k in ("temperature", "top_k", "top_p", "min_p")}

    # the oracle: float64 logits of the sampled rows, replayed tokens drawn
    # from its own filtered distribution, forward and threshold gaps
    Hf_sel = f32_values(data["H"][sel])
    Wf = f32_values(data["W"])
    s_sel = oracle.scaled_logits(Hf_sel, Wf, meta_sel["temperature"], vocab_slice=16384)
    rows0 = dict(meta_sel, target=np.zeros(len(sel), np.int64))
    y_sel = pool.sample_rows(s_sel, rows0, data["u"][sel])
    rows_sel = dict(meta_sel, target=y_sel)
    ref = pool.forward(s_sel, rows_sel)
    flagged = pool.row_gaps(s_sel, rows_sel).min(axis=1) < GAP_EPS

    # the GPU forward on every row (targets outside the sample are token 0)
    target = np.zeros(T, np.int64)
    target[sel] = y_sel
    Hd, Wd = bf16_tensor(data["H"]), bf16_tensor(data["W"])
    dev = lambda a, dt: torch.from_numpy(np.asarray(a, dt)).cuda()  # noqa: E731
    y_t = dev(target, np.int64)
    tau, k, p, mu = (dev(data["temperature"], np.float32), dev(data["top_k"], np.int32),
                     dev(data["top_p"], np.float32), dev(data["min_p"], np.float32))
    lp, saved, _ = sts.sts_forward(Hd, Wd, y_t, tau, k, p, mu, check=True, entropy=True)
    lp_sel = lp.cpu().numpy()[sel]
    sv = {n: v.cpu().numpy()[sel] for n, v in saved.items()}
    # the benchmark's forward (no entropy output: fp32 masses where no mass
    # comparison decides the support): the same decisions on every row, its
    # logprob within the fp32 mass bound of the float64-mass one, and within
    # the oracle tolerance on the sampled rows
    lp32, saved32, _ = sts.sts_forward(Hd, Wd, y_t, tau, k, p, mu, check=True)
    assert_same_decisions(lp, saved, lp32, saved32)
    bad32, _, err32 = compare_logprob(lp32.cpu().numpy()[sel], sv["support_size"], s_sel, rows_sel,
                                      ref, flagged)
    assert bad32 == 0, (bad32, err32)

    # 1 and 2: against the float64 oracle
    bad, ndiff, max_err = compare_logprob(lp_sel, sv["support_size"], s_sel, rows_sel, ref, flagged)
    dsize = np.abs(sv["support_size"] - ref["size"])
    # 3: the forward's cuts against the oracle's program on the GPU's logits
    S_gpu = torch.cat([sts.sts_scaled_logits(Hd, Wd, tau, t0=int(t) * 128, rows=128)
                       for t in tiles]).cpu().numpy()
    own = pool.filter_rows(S_gpu, rows_sel)
    own_gap_p = pool.row_gaps(S_gpu, rows_sel)[:, 1]
    cut_diff = ((sv["support_size"] != own["size"]) | (sv["cut_id"] != own["cut_id"])
                | (sv["cut_logit"] != own["cut_value"].astype(np.float32)))
    n = len(sel)
    print(f"workload {index}: {n} rows; logprob compared on all {n} (max |dlogprob| "
          f"{max_err:.2e}); {int((~flagged).sum())} rows with every threshold further than "
          f"{GAP_EPS:g} from its boundary, {int(flagged.sum())} near-gap ({ndiff} with another "
          f"valid support size, at most {int(dsize.max(initial=0))} tokens apart); "
          f"cuts bit-exact against the oracle on the GPU's fp32 logits on "
          f"{int((~cut_diff).sum())} of {n} rows")
    assert bad == 0
    assert not (cut_diff & ~(own_gap_p < 1e-12)).any(), np.flatnonzero(cut_diff)
    # entropy of the filtered distribution: against the oracle's on the GPU's
    # support (float64 logits) and on the GPU's own fp32 logits
    ent_ref = np.concatenate(pool.map_rows("entropy", s_sel, rows_sel,
                                           per_row_extra=(sv["support_size"],)))
    assert np.abs(sv["entropy"] - ent_ref).max() < 1e-3
    ent_own = np.concatenate(pool.map_rows("entropy", S_gpu, rows_sel))
    same_cut = ~cut_diff
    np.testing.assert_allclose(sv["entropy"][same_cut], ent_own[same_cut], rtol=2e-6, atol=1e-6)

    # 5: gradients on the rows whose support equals the oracle's; zero elsewhere
    same = grad_rows(sv["flags"], ref["in_support"]) & (dsize == 0)
    g = np.zeros(T, np.float32)
    g[sel[same]] = 1.0
    dH, dW = sts.sts_backward(Hd, Wd, y_t, tau, k, p, mu, saved, dev(g, np.float32),
                              vocab_chunk=wl.vocab_chunk, check=True)
    vocab = np.unique(np.concatenate([rng.choice(V, N_VOCAB, replace=False), y_sel]))
    if index == 5:
        vocab = np.unique(np.concatenate([vocab, data["dup_dst"][:64], data["dup_src"][:64]]))
    dZ = pool.logit_grad(s_sel, rows_sel, same.astype(np.float64))
    dH_ref, dW_ref = oracle.backward(Hf_sel, Wf, rows_sel, None, vocab_rows=vocab,
                                     vocab_slice=16384, dZ=dZ)
    assert rel_fro(dH.cpu().numpy()[sel], dH_ref) < GRAD_RTOL
    dW_sub = dW[torch.from_numpy(vocab).cuda()].cpu().numpy()
    assert rel_fro(dW_sub, dW_ref) < GRAD_RTOL

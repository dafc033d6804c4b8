"""Parity at the full sizes of the three large workloads, in the launch
configuration the benchmark times (default row and vocabulary chunks, all
rows on the GPU), checked on a seeded sample of rows the oracle computes one
by one: logprobs, support sizes, dH rows and dW on a sample of vocabulary rows
(the upstream gradient is zero outside the sampled rows so dW stays
comparable)."""

import numpy as np
import pytest
import torch

import oracle
import workloads
from helpers import (GRAD_RTOL, bf16_tensor, compare_logprob, f32_values, grad_rows,
                     near_gap_rows, rel_fro)

pytestmark = pytest.mark.gpu

N_ROWS = 48
N_VOCAB = 1024


def _sample_rows(data, T, rng):
    idx = set(rng.choice(T, N_ROWS, replace=False).tolist())
    # make sure each metadata class appears
    for key in ("top_k", "top_p", "min_p"):
        vals = data[key]
        for v in np.unique(vals)[:4]:
            hits = np.flatnonzero(vals == v)
            idx.add(int(hits[rng.integers(0, len(hits))]))
    return np.array(sorted(idx), dtype=np.int64)


@pytest.mark.parametrize("index", [3, 4, 5])
def test_full_size_workload(cuda_lib, index):
    sts = cuda_lib
    data = workloads.make(index)
    wl = data["workload"]
    T, d, V = wl.T, wl.d, wl.V
    rng = np.random.Generator(np.random.PCG64(3000 + index))
    sel = _sample_rows(data, T, rng)
    meta_sel = {k: data[k][sel] for k in ("temperature", "top_k", "top_p", "min_p")}

    Hf_sel = f32_values(data["H"][sel])
    Wf = f32_values(data["W"])
    s_sel = oracle.scaled_logits(Hf_sel, Wf, meta_sel["temperature"], vocab_slice=16384)
    y_sel = oracle.sample_rows(s_sel, dict(meta_sel, target=np.zeros(len(sel), np.int64)),
                               data["u"][sel])
    rows_sel = dict(meta_sel, target=y_sel)
    ref = oracle.forward(None, None, rows_sel, s=s_sel)

    target = np.zeros(T, np.int64)
    target[sel] = y_sel

    Hd, Wd = bf16_tensor(data["H"]), bf16_tensor(data["W"])
    dev = lambda a, dt: torch.from_numpy(np.asarray(a, dt)).cuda()  # noqa: E731
    y_t = dev(target, np.int64)
    tau, k, p, mu = (dev(data["temperature"], np.float32), dev(data["top_k"], np.int32),
                     dev(data["top_p"], np.float32), dev(data["min_p"], np.float32))
    lp, saved, _ = sts.sts_forward(Hd, Wd, y_t, tau, k, p, mu, check=True)

    lp_sel = lp.cpu().numpy()[sel]
    flagged = near_gap_rows(s_sel, rows_sel)
    bad, flagged_mism, max_err = compare_logprob(lp_sel, ref["logprob"], flagged)
    size = saved["support_size"].cpu().numpy()[sel]
    dsize = np.abs(size - ref["size"])
    print(f"workload {index}: {len(sel)} rows, {int(flagged.sum())} near-gap, "
          f"{flagged_mism} near-gap membership flips, max |dlogprob| {max_err:.2e}, "
          f"max support-size difference {int(dsize.max())} tokens")
    assert bad == 0
    assert not ((dsize != 0) & ~flagged).any()

    # gradients on the rows whose target membership agrees; zero elsewhere
    same = grad_rows(saved["flags"].cpu().numpy()[sel], ref["in_support"])
    g = np.zeros(T, np.float32)
    g[sel[same]] = 1.0
    dH, dW = sts.sts_backward(Hd, Wd, y_t, tau, k, p, mu, saved, dev(g, np.float32),
                              vocab_chunk=wl.vocab_chunk, check=True)
    vocab = np.unique(np.concatenate([rng.choice(V, N_VOCAB, replace=False), y_sel]))
    if index == 5:
        vocab = np.unique(np.concatenate([vocab, data["dup_dst"][:64], data["dup_src"][:64]]))
    dH_ref, dW_ref = oracle.backward(Hf_sel, Wf, rows_sel, same.astype(np.float64), s=s_sel,
                                     vocab_rows=vocab, vocab_slice=16384)
    dH_sel = dH.cpu().numpy()[sel]
    assert rel_fro(dH_sel, dH_ref) < GRAD_RTOL
    dW_sub = dW[torch.from_numpy(vocab).cuda()].cpu().numpy()
    assert rel_fro(dW_sub, dW_ref) < GRAD_RTOL

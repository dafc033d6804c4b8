"""sts_filter_logits_noalloc: the filter path for callers that cannot allocate
device memory (a fixed device-memory reservation, or code inside an allocator
or framework callback). It must give the same results as sts_filter_logits
on two calls in a row, reject row counts beyond its fixed scratch array, and
leave the device's free memory unchanged. Collected last on purpose."""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

MAX_ROWS = 65536


def _case(seed, T, V):
    rng = np.random.Generator(np.random.PCG64(seed))
    S = (rng.standard_normal((T, V), dtype=np.float32)
         / rng.uniform(0.5, 1.5, T).astype(np.float32)[:, None])
    S[3, ::7] = S[3, 0]  # exact ties
    k = rng.choice(np.array([0, 1, 20, 500], np.int32), T).astype(np.int32)
    p = rng.choice(np.array([1.0, 0.9, 0.5], np.float32), T).astype(np.float32)
    mu = rng.choice(np.array([0.0, 0.05], np.float32), T).astype(np.float32)
    p[5] = 1.5  # an invalid row
    dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    return dev(S), dev(k), dev(p), dev(mu)


def _noalloc(sts, S, k, p, mu):
    T, V = S.shape
    out = {
        "size": torch.full((T,), -7, dtype=torch.int32, device="cuda"),
        "cut_logit": torch.zeros(T, dtype=torch.float32, device="cuda"),
        "cut_id": torch.full((T,), -7, dtype=torch.int32, device="cuda"),
        "mask": torch.zeros((T, V), dtype=torch.uint8, device="cuda"),
    }
    sts.sts_filter_logits_noalloc(S, k, p, mu, support_size=out["size"], cut_logit=out["cut_logit"],
                                  cut_id=out["cut_id"], mask=out["mask"])
    torch.cuda.synchronize()
    return out


def test_noalloc_matches_workspace_filter_twice(cuda_lib):
    sts = cuda_lib
    for seed, (T, V) in ((1, (64, 9000)), (2, (300, 32768))):
        S, k, p, mu = _case(seed, T, V)
        ref = sts.sts_filter_logits(S, k, p, mu, want_mask=True)
        torch.cuda.synchronize()
        for _ in range(2):  # the shared scratch keeps the previous call's contents
            got = _noalloc(sts, S, k, p, mu)
            assert torch.equal(got["size"], ref["size"])
            assert torch.equal(got["cut_id"], ref["cut_id"])
            assert torch.equal(got["mask"], ref["mask"])
            ok = ref["size"] > 0
            assert torch.equal(got["cut_logit"][ok], ref["cut_logit"][ok])
        assert got["size"][5].item() == 0 and got["cut_id"][5].item() == -1


def test_noalloc_allocates_nothing_and_bounds_rows(cuda_lib):
    sts = cuda_lib
    S, k, p, mu = _case(3, 128, 4096)
    _noalloc(sts, S, k, p, mu)  # first call on the device resolves the scratch address
    free0, _ = torch.cuda.mem_get_info()
    _noalloc(sts, S, k, p, mu)
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    T = MAX_ROWS + 1
    big = torch.zeros((T, 8), dtype=torch.float32, device="cuda")
    kk = torch.zeros(T, dtype=torch.int32, device="cuda")
    pp = torch.ones(T, dtype=torch.float32, device="cuda")
    mm = torch.zeros(T, dtype=torch.float32, device="cuda")
    outs = [torch.zeros(T, dtype=dt, device="cuda") for dt in (torch.int32, torch.float32, torch.int32)]
    with pytest.raises(sts.StsError) as ei:
        sts.sts_filter_logits_noalloc(big, kk, pp, mm, support_size=outs[0], cut_logit=outs[1],
                                      cut_id=outs[2])
    assert ei.value.status == 2  # STS_ERR_SHAPE: beyond the fixed scratch array

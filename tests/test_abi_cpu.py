"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function that include/sts.h declares, sizes workspaces, and rejects bad
arguments before touching the device."""

import ctypes
import os
import re

import pytest

import sampling_transform_lm_b200 as sts
from sampling_transform_lm_b200 import _Rows, _Saved, _Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "sts.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sts_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return sts.load()


def test_library_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "sts_forward" in names and "sts_backward" in names
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(sts.EXPORTED_SYMBOLS)
    assert lib.sts_abi_version() == 3


def test_status_strings(lib):
    for code in range(14):
        assert lib.sts_status_string(code)
    assert b"unknown" in lib.sts_status_string(99)


def _shape(T=256, d=64, V=1000, vc=0, rc=0):
    return _Shape(T, d, V, vc, rc)


def test_workspace_sizes(lib):
    sh = _shape(T=1000, d=128, V=50000)
    fwd = lib.sts_workspace_bytes(ctypes.byref(sh), 0)
    bwd = lib.sts_workspace_bytes(ctypes.byref(sh), 1)
    flt = lib.sts_workspace_bytes(ctypes.byref(sh), 2)
    # forward: header + flags + one row chunk of fp32 logits (row stride padded to 4)
    assert fwd >= 1024 * 50000 * 4 and fwd % 1024 == 0
    # backward: one vocab chunk (default 28416 columns) of bf16 dZ for all rows,
    # and H^T in bf16 (rows padded to 8 elements)
    assert lib.sts_vocab_chunk(ctypes.byref(sh)) == 28416
    assert bwd >= 1000 * 28416 * 2 + 128 * 1000 * 2
    assert flt >= 1000 * 4
    sh2 = _shape(T=1000, d=128, V=50000, vc=8192, rc=256)
    assert lib.sts_workspace_bytes(ctypes.byref(sh2), 1) < bwd
    assert lib.sts_workspace_bytes(ctypes.byref(sh2), 0) < fwd
    assert lib.sts_workspace_bytes(ctypes.byref(sh), 7) == 0


@pytest.mark.parametrize("bad", [
    dict(T=0), dict(d=0), dict(d=12), dict(V=0), dict(vc=100), dict(rc=64), dict(T=-5),
])
def test_bad_shapes_rejected(lib, bad):
    kw = dict(T=256, d=64, V=1000, vc=0, rc=0)
    kw.update(bad)
    sh = _shape(**kw)
    assert lib.sts_workspace_bytes(ctypes.byref(sh), 0) == 0
    rows = _Rows(kw["T"], 16, 16, 16, 16, 16)
    saved = _Saved(16, 16, 16, 16, 16, 16)
    st = lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(rows), 16, None, ctypes.byref(saved),
                         4096, 1 << 40, None)
    assert st == 2  # STS_ERR_SHAPE


def test_null_and_length_and_workspace_errors(lib):
    sh = _shape()
    saved = _Saved(16, 16, 16, 16, 16, 16)
    good_rows = _Rows(256, 16, 16, 16, 16, 16)
    big = 1 << 40
    # null operands
    assert lib.sts_forward(ctypes.byref(sh), None, 4096, ctypes.byref(good_rows), 16, None,
                           ctypes.byref(saved), 4096, big, None) == 1
    # metadata length differs from T: rejected, not truncated
    for n in (255, 257, 512):
        rows = _Rows(n, 16, 16, 16, 16, 16)
        assert lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(rows), 16, None,
                               ctypes.byref(saved), 4096, big, None) == 2
    # missing per-row array
    rows = _Rows(256, 16, None, 16, 16, 16)
    assert lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(rows), 16, None,
                           ctypes.byref(saved), 4096, big, None) == 1
    # workspace: null, misaligned, too small
    assert lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(good_rows), 16, None,
                           ctypes.byref(saved), None, big, None) == 9
    assert lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(good_rows), 16, None,
                           ctypes.byref(saved), 4096 + 16, big, None) == 9
    assert lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(good_rows), 16, None,
                           ctypes.byref(saved), 4096, 1024, None) == 9
    # sliced backward: a negative SM reservation is a shape error
    SLICE = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                             ctypes.c_void_p, ctypes.c_void_p)
    lib.sts_backward_sliced.argtypes = [ctypes.c_void_p] * 12 + [SLICE, ctypes.c_void_p,
                                                                 ctypes.c_int]
    assert lib.sts_backward_sliced(ctypes.byref(sh), 4096, 4096, ctypes.byref(good_rows),
                                   ctypes.byref(saved), 4096, 4096, 4096, 0, 4096, big, None,
                                   SLICE(0), None, -1) == 2
    # backward: null gradient
    assert lib.sts_backward(ctypes.byref(sh), 4096, 4096, ctypes.byref(good_rows),
                            ctypes.byref(saved), None, 4096, 4096, 0, 4096, big, None) == 1
    # scaled-logits hook: t0 off the 128-row grid
    assert lib.sts_scaled_logits(ctypes.byref(sh), 4096, 4096, 16, 64, 10, 0, 10, 4096, 12,
                                 None) == 2
    assert lib.sts_get_status(None, None, None) == 9


def test_valid_call_without_gpu_reports_cuda_error(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("this checks the no-GPU behaviour")
    sh = _shape()
    saved = _Saved(16, 16, 16, 16, 16, 16)
    rows = _Rows(256, 16, 16, 16, 16, 16)
    st = lib.sts_forward(ctypes.byref(sh), 4096, 4096, ctypes.byref(rows), 16, None, ctypes.byref(saved),
                         4096, 1 << 40, None)
    assert st in (12, 13)  # no device: CUDA error, never a CPU fallback


def test_binding_rejects_non_bf16_head():
    import torch

    H = torch.zeros(4, 8, dtype=torch.float32)
    W = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(sts.StsError) as ei:
        sts._hw(H, W)
    assert ei.value.status == 3
    if hasattr(torch, "float8_e4m3fn"):
        W8 = torch.zeros(4, 8, dtype=torch.float8_e4m3fn)
        with pytest.raises(sts.StsError) as ei:
            sts._hw(W.clone(), W8)
        assert ei.value.status == 3


def test_binding_rejects_wrong_metadata_length():
    import torch

    t = torch.ones(5, dtype=torch.float32)
    k = torch.zeros(6, dtype=torch.int32)
    with pytest.raises(sts.StsError):
        sts._rows(5, None, t, k, t, t)


def test_vocab_chunk_choice():
    for T, d, V in [(16384, 5120, 152064), (8192, 4096, 151936), (32768, 4096, 262144),
                    (4096, 2048, 32768), (300, 64, 100000)]:
        vc = sts.sts_vocab_chunk(T, d, V)
        assert vc == min(28416, (V + 255) // 256 * 256)
        assert sts.sts_vocab_chunk(T, d, V, vocab_chunk=8192) == 8192  # an explicit chunk is kept
        assert sts.sts_workspace_bytes(T, d, V, 1) >= T * vc * 2  # the workspace follows it
    assert sts.sts_vocab_chunk(64, 128, 1000) == 1024
    assert sts.sts_vocab_chunk(64, 128, 1000, vocab_chunk=8192) == 1024
    with pytest.raises(sts.StsError):
        sts.sts_vocab_chunk(64, 128, 1000, vocab_chunk=100)  # not a multiple of 256


def test_policy_grad_host_checks(lib):
    """Argument errors return before any device work (no GPU needed)."""
    null = ctypes.c_void_p(0)
    assert lib.sts_policy_grad(-1, null, null, null, 0, 0.2, 0.2, 1.0, null, null) == 2
    assert lib.sts_policy_grad(4, null, null, null, 7, 0.2, 0.2, 1.0, null, null) == 2
    assert lib.sts_policy_grad(4, null, null, null, 0, -0.1, 0.2, 1.0, null, null) == 2
    assert lib.sts_policy_grad(4, null, null, null, 1, 0.2, float("nan"), 1.0, null, null) == 2
    assert lib.sts_policy_grad(4, null, null, null, 0, 0.2, 0.2, float("inf"), null, null) == 2
    assert lib.sts_policy_grad(4, null, null, null, 0, 0.2, 0.2, 1.0, null, null) == 1
    assert lib.sts_policy_grad(0, null, null, null, 1, 0.2, 0.2, 1.0, null, null) == 0


def test_statistics_merge_host_checks(lib):
    """The vocabulary-parallel merge stages: their record sizes, and argument
    errors returned before any device work (no GPU needed)."""
    c = sts.sts_tp_constants()
    assert c == {"buckets": 4096, "plan_fields": 8, "sum_fields": 5, "key_fields": 2,
                 "sort_cap": 8192}
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(4096)  # never dereferenced: the checks fail first
    assert lib.sts_tp_row_max(null, 4, 8, 8, fake, None) == 1
    assert lib.sts_tp_row_max(fake, 4, 8, 7, fake, None) == 2      # ld < Vl
    assert lib.sts_tp_row_max(fake, 0, 8, 8, fake, None) == 2      # no rows
    assert lib.sts_tp_count(fake, 4, 8, 8, null, fake, None) == 1
    assert lib.sts_tp_count(fake, 4, -1, 8, fake, fake, None) == 2
    rows = _Rows(4, fake, fake, fake, fake, fake)
    short = _Rows(3, fake, fake, fake, fake, fake)
    bad_off = [fake, 4, 8, 8, 12, 16, ctypes.byref(rows)] + [fake] * 8
    assert lib.sts_tp_exact(*bad_off, 4096, None) == 2           # offset + Vl > V
    assert lib.sts_tp_exact(*([fake, 4, 8, 8, 0, 16, ctypes.byref(short)] + [fake] * 8),
                            4096, None) == 2                     # metadata length != T
    assert lib.sts_tp_exact(*([fake, 4, 8, 8, 0, 16, ctypes.byref(rows)] + [fake] * 8),
                            0, None) == 2                        # cap < 1
    saved = _Saved(fake, fake, fake, fake, fake, fake)
    fin = [4, 16, 2, ctypes.byref(rows)] + [fake] * 7 + [4096, fake, ctypes.byref(saved), fake]
    assert lib.sts_tp_finish(*fin, null, 256, None) == 9          # no workspace
    assert lib.sts_tp_finish(*fin, fake, 100, None) == 9          # short workspace
    fin0 = [4, 16, 0, ctypes.byref(rows)] + [fake] * 7 + [4096, fake, ctypes.byref(saved), fake]
    assert lib.sts_tp_finish(*fin0, fake, 256, None) == 2         # world < 1

"""B200 (sm_100a) sampling-transform scoring core: thin Python binding.

Each function marshals torch tensors into the C ABI of ``libsts.so``
(declared in ``include/sts.h``) and calls the entry point of the same name.
Every step of the computation runs in the library's CUDA kernels; there is
no Python or CPU fallback, and a missing library raises ``StsError``.

The operation ("Consolidate sampling-transform scoring on one shared chunked
core; implement top-k/top-p/min-p replay for generic ce_modes", xorl PR 74,
"What this PR does", items 1, 2 and 4): per row, logits z = H . W^T with fp32
accumulation, s = z / temperature, the support program top-k -> top-p ->
min-p with token-id tie-break, and the selected token's logprob on the
filtered support; the backward recomputes the logits and forms
dz = g (onehot - p_support) / temperature inside the GEMM epilogue.
"""

from __future__ import annotations

import ctypes
import os

import torch

from .dp import SliceAllReduce  # noqa: E402
from .tp import VocabParallel  # noqa: E402

__all__ = [
    "StsError",
    "load",
    "library_path",
    "sts_workspace_bytes",
    "sts_vocab_chunk",
    "sts_forward",
    "sts_backward",
    "sts_backward_shard",
    "sts_resolve_logits",
    "sts_gather_vocab_shards",
    "sts_tp_constants",
    "sts_tp_row_max",
    "sts_tp_count",
    "sts_tp_exact",
    "sts_tp_finish",
    "VocabParallel",
    "SliceAllReduce",
    "sts_sample",
    "sts_filter_logits",
    "sts_scaled_logits",
    "sts_policy_grad",
    "sts_get_status",
    "sts_path_counts",
    "sts_status_string",
    "sts_probe_mass_exp",
    "sts_launch_count",
    "sts_timing_enable",
    "sts_timing_read",
    "sts_filter_logits_noalloc",
    "KERNEL_KINDS",
    "ROW_TARGET_IN_SUPPORT",
    "ROW_INVALID",
    "ROW_IDENTITY",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsts.so")

STS_OK = 0
STS_ERR_NULL = 1
STS_ERR_SHAPE = 2
STS_ERR_DTYPE = 3
STS_ERR_WORKSPACE = 9
ROW_TARGET_IN_SUPPORT = 1
ROW_INVALID = 2
ROW_IDENTITY = 4

KERNEL_KINDS = ("validate", "logits_gemm", "resolve", "dz_gemm", "dw_gemm", "dh_gemm")

EXPORTED_SYMBOLS = (
    "sts_workspace_bytes",
    "sts_vocab_chunk",
    "sts_forward",
    "sts_backward",
    "sts_sample",
    "sts_filter_logits",
    "sts_scaled_logits",
    "sts_get_status",
    "sts_status_string",
    "sts_abi_version",
    "sts_probe_mass_exp",
    "sts_launch_count",
    "sts_timing_enable",
    "sts_timing_read",
    "sts_filter_logits_noalloc",
    "sts_policy_grad",
    "sts_path_counts",
    "sts_backward_sliced",
    "sts_backward_shard",
    "sts_resolve_logits",
    "sts_gather_vocab_shards",
    "sts_tp_constants",
    "sts_tp_row_max",
    "sts_tp_count",
    "sts_tp_exact",
    "sts_tp_finish",
)


class StsError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = int(status)
        msg = _status_text(self.status)
        super().__init__(f"{what}: {msg} (status {self.status})" if what else msg)


class _Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int64), ("V", ctypes.c_int64),
                ("vocab_chunk", ctypes.c_int64), ("row_chunk", ctypes.c_int64)]


class _Rows(ctypes.Structure):
    _fields_ = [("len", ctypes.c_int64), ("target", ctypes.c_void_p),
                ("temperature", ctypes.c_void_p), ("top_k", ctypes.c_void_p),
                ("top_p", ctypes.c_void_p), ("min_p", ctypes.c_void_p)]


_SLICE_FN = ctypes.CFUNCTYPE(None, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                             ctypes.c_void_p)


class _Saved(ctypes.Structure):
    _fields_ = [("row_max", ctypes.c_void_p), ("lse_support", ctypes.c_void_p),
                ("cut_logit", ctypes.c_void_p), ("cut_id", ctypes.c_void_p),
                ("support_size", ctypes.c_void_p), ("flags", ctypes.c_void_p)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load ``libsts.so`` (raises StsError / OSError when it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise OSError(f"{_LIB_PATH} is missing: build it with "
                      "`python -m sampling_transform_lm_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, S, I64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int64
    lib.sts_workspace_bytes.argtypes = [ctypes.POINTER(_Shape), ctypes.c_int]
    lib.sts_workspace_bytes.restype = S
    lib.sts_vocab_chunk.argtypes = [ctypes.POINTER(_Shape)]
    lib.sts_vocab_chunk.restype = ctypes.c_int64
    lib.sts_forward.argtypes = [ctypes.POINTER(_Shape), P, P, ctypes.POINTER(_Rows), P, P,
                                ctypes.POINTER(_Saved), P, S, P]
    lib.sts_forward.restype = ctypes.c_int
    lib.sts_backward.argtypes = [ctypes.POINTER(_Shape), P, P, ctypes.POINTER(_Rows),
                                 ctypes.POINTER(_Saved), P, P, P, ctypes.c_int, P, S, P]
    lib.sts_backward.restype = ctypes.c_int
    lib.sts_backward_sliced.argtypes = [ctypes.POINTER(_Shape), P, P, ctypes.POINTER(_Rows),
                                        ctypes.POINTER(_Saved), P, P, P, ctypes.c_int, P, S, P,
                                        _SLICE_FN, P, ctypes.c_int]
    lib.sts_backward_sliced.restype = ctypes.c_int
    lib.sts_backward_shard.argtypes = [ctypes.POINTER(_Shape), P, P, ctypes.POINTER(_Rows),
                                       ctypes.POINTER(_Saved), P, P, P, ctypes.c_int, I64, P, S, P]
    lib.sts_backward_shard.restype = ctypes.c_int
    lib.sts_resolve_logits.argtypes = [ctypes.POINTER(_Shape), P, I64, ctypes.POINTER(_Rows), P, P,
                                       ctypes.POINTER(_Saved), P, S, P]
    lib.sts_resolve_logits.restype = ctypes.c_int
    lib.sts_gather_vocab_shards.argtypes = [P, I64, I64, I64, P, I64, P]
    lib.sts_gather_vocab_shards.restype = ctypes.c_int
    PI64 = ctypes.POINTER(ctypes.c_int64)
    lib.sts_tp_constants.argtypes = [PI64, PI64, PI64, PI64, PI64]
    lib.sts_tp_constants.restype = ctypes.c_int
    lib.sts_tp_row_max.argtypes = [P, I64, I64, I64, P, P]
    lib.sts_tp_row_max.restype = ctypes.c_int
    lib.sts_tp_count.argtypes = [P, I64, I64, I64, P, P, P]
    lib.sts_tp_count.restype = ctypes.c_int
    lib.sts_tp_exact.argtypes = [P, I64, I64, I64, I64, I64, ctypes.POINTER(_Rows), P, P, P, P, P,
                                 P, P, P, I64, P]
    lib.sts_tp_exact.restype = ctypes.c_int
    lib.sts_tp_finish.argtypes = [I64, I64, I64, ctypes.POINTER(_Rows), P, P, P, P, P, P, P, I64, P,
                                  ctypes.POINTER(_Saved), P, P, S, P]
    lib.sts_tp_finish.restype = ctypes.c_int
    lib.sts_sample.argtypes = [ctypes.POINTER(_Shape), P, P, ctypes.POINTER(_Rows), P, P, P, S, P]
    lib.sts_sample.restype = ctypes.c_int
    lib.sts_filter_logits.argtypes = [ctypes.POINTER(_Shape), P, ctypes.POINTER(_Rows), P, P, P, P,
                                      P, P, S, P]
    lib.sts_filter_logits.restype = ctypes.c_int
    lib.sts_scaled_logits.argtypes = [ctypes.POINTER(_Shape), P, P, P, I64, I64, I64, I64, P, I64, P]
    lib.sts_scaled_logits.restype = ctypes.c_int
    lib.sts_get_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.sts_get_status.restype = ctypes.c_int
    lib.sts_path_counts.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    lib.sts_path_counts.restype = ctypes.c_int
    lib.sts_status_string.argtypes = [ctypes.c_int]
    lib.sts_status_string.restype = ctypes.c_char_p
    lib.sts_probe_mass_exp.argtypes = [P, ctypes.c_float, P, P, I64, P]
    lib.sts_probe_mass_exp.restype = ctypes.c_int
    lib.sts_policy_grad.argtypes = [I64, P, P, P, ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                    ctypes.c_float, P, P]
    lib.sts_policy_grad.restype = ctypes.c_int
    lib.sts_launch_count.argtypes = [ctypes.c_int]
    lib.sts_launch_count.restype = ctypes.c_int64
    lib.sts_timing_enable.argtypes = [ctypes.c_int]
    lib.sts_timing_enable.restype = ctypes.c_int
    lib.sts_timing_read.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64)]
    lib.sts_timing_read.restype = ctypes.c_int
    lib.sts_filter_logits_noalloc.argtypes = [ctypes.POINTER(_Shape), P, ctypes.POINTER(_Rows), P, P,
                                              P, P, P]
    lib.sts_filter_logits_noalloc.restype = ctypes.c_int
    lib.sts_abi_version.argtypes = []
    lib.sts_abi_version.restype = ctypes.c_int
    _lib = lib
    return lib


def _status_text(status: int) -> str:
    try:
        return load().sts_status_string(int(status)).decode()
    except OSError:
        return f"status {status}"


def sts_status_string(status: int) -> str:
    return _status_text(status)


def _check(status: int, what: str):
    if status != STS_OK:
        raise StsError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _shape(T, d, V, vocab_chunk=0, row_chunk=0):
    return _Shape(int(T), int(d), int(V), int(vocab_chunk), int(row_chunk))


def _need(t, dtype, name, shape=None):
    if t.dtype != dtype:
        status = STS_ERR_DTYPE if dtype == torch.bfloat16 else STS_ERR_SHAPE
        raise StsError(status, f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise StsError(STS_ERR_SHAPE, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise StsError(STS_ERR_SHAPE, f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise StsError(STS_ERR_SHAPE, f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _rows(T, target, temperature, top_k, top_p, min_p):
    for name, t, dt in (("temperature", temperature, torch.float32), ("top_k", top_k, torch.int32),
                        ("top_p", top_p, torch.float32), ("min_p", min_p, torch.float32)):
        _need(t, dt, name)
        if t.dim() != 1:
            raise StsError(STS_ERR_SHAPE, f"{name} must be 1-D")
        if t.shape[0] != T:  # over- or under-length metadata is rejected, never truncated
            raise StsError(STS_ERR_SHAPE, f"{name} has {t.shape[0]} rows, expected {T}")
    if target is not None:
        _need(target, torch.int64, "target", (T,))
    return _Rows(T, _ptr(target), _ptr(temperature), _ptr(top_k), _ptr(top_p), _ptr(min_p))


def sts_workspace_bytes(T, d, V, pass_, vocab_chunk=0, row_chunk=0) -> int:
    sh = _shape(T, d, V, vocab_chunk, row_chunk)
    n = load().sts_workspace_bytes(ctypes.byref(sh), int(pass_))
    if n == 0:
        raise StsError(STS_ERR_SHAPE, "sts_workspace_bytes")
    return int(n)


def sts_vocab_chunk(T, d, V, vocab_chunk=0) -> int:
    """The backward's vocabulary chunk for this shape (28416 when
    ``vocab_chunk`` is 0; clamped to V rounded up to 256)."""
    sh = _shape(T, d, V, vocab_chunk, 0)
    n = load().sts_vocab_chunk(ctypes.byref(sh))
    if n < 0:
        raise StsError(STS_ERR_SHAPE, "sts_vocab_chunk")
    return int(n)


def _workspace(nbytes, device, ws=None):
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise StsError(STS_ERR_WORKSPACE, f"workspace holds {ws.numel()} bytes, needs {nbytes}")
        return ws
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _hw(H, W):
    for name, t in (("H", H), ("W", W)):  # dtype first: an fp8 head is a dtype error
        if t.dtype != torch.bfloat16:
            raise StsError(STS_ERR_DTYPE, f"{name} must be torch.bfloat16, got {t.dtype}")
    _need(H, torch.bfloat16, "H")
    _need(W, torch.bfloat16, "W")
    if H.dim() != 2 or W.dim() != 2 or H.shape[1] != W.shape[1]:
        raise StsError(STS_ERR_SHAPE, "H must be [T, d] and W [V, d]")
    return H.shape[0], H.shape[1], W.shape[0]


def sts_forward(H, W, target, temperature, top_k, top_p, min_p, *, row_chunk=0, ws=None,
                stream=None, check=False, entropy=False):
    """Filtered-support logprob per row plus the saved per-row scalars.

    Returns ``(logprob [T] fp32, saved dict, workspace)``. With ``entropy``
    the dict also holds ``"entropy"`` [T] fp32, the entropy (nats) of each
    row's filtered distribution. With ``check`` the call synchronises and
    raises on a row-value error.
    """
    lib = load()
    T, d, V = _hw(H, W)
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    sh = _shape(T, d, V, 0, row_chunk)
    dev = H.device
    ws = _workspace(sts_workspace_bytes(T, d, V, 0, 0, row_chunk), dev, ws)
    logprob = torch.empty(T, dtype=torch.float32, device=dev)
    saved = {
        "row_max": torch.empty(T, dtype=torch.float32, device=dev),
        "lse_support": torch.empty(T, dtype=torch.float32, device=dev),
        "cut_logit": torch.empty(T, dtype=torch.float32, device=dev),
        "cut_id": torch.empty(T, dtype=torch.int32, device=dev),
        "support_size": torch.empty(T, dtype=torch.int32, device=dev),
        "flags": torch.empty(T, dtype=torch.int32, device=dev),
    }
    sv = _Saved(*(_ptr(saved[k]) for k in ("row_max", "lse_support", "cut_logit", "cut_id",
                                            "support_size", "flags")))
    ent = torch.empty(T, dtype=torch.float32, device=dev) if entropy else None
    st = lib.sts_forward(ctypes.byref(sh), _ptr(H), _ptr(W), ctypes.byref(rows), _ptr(logprob),
                         _ptr(ent), ctypes.byref(sv), _ptr(ws), ws.numel(), _stream(stream))
    if ent is not None:
        saved["entropy"] = ent
    _check(st, "sts_forward")
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return logprob, saved, ws


def sts_backward(H, W, target, temperature, top_k, top_p, min_p, saved, grad_logprob, *,
                 dW=None, dH=None, accumulate_dW=False, vocab_chunk=0, ws=None, stream=None,
                 check=False, on_dw_slice=None, comm_sms=0):
    """dH [T, d] and dW [V, d] (fp32) of sum_t g_t * logprob_t.

    ``on_dw_slice(v0, rows, dW_slice)`` (optional) is called on this thread,
    in increasing v0, right after the GEMM that writes dW[v0:v0 + rows] has
    been enqueued (``sts_backward_sliced``): a data-parallel caller starts the
    slice's cross-rank sum there (see ``SliceAllReduce``). ``comm_sms`` SMs are
    left free of the persistent GEMMs for the exchange kernels."""
    lib = load()
    T, d, V = _hw(H, W)
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    _need(grad_logprob, torch.float32, "grad_logprob", (T,))
    sh = _shape(T, d, V, vocab_chunk, 0)
    dev = H.device
    ws = _workspace(sts_workspace_bytes(T, d, V, 1, vocab_chunk, 0), dev, ws)
    if dH is None:
        dH = torch.empty((T, d), dtype=torch.float32, device=dev)
    else:
        _need(dH, torch.float32, "dH", (T, d))
    if dW is None:
        if accumulate_dW:
            raise StsError(STS_ERR_NULL, "accumulate_dW needs a dW tensor")
        dW = torch.empty((V, d), dtype=torch.float32, device=dev)
    else:
        _need(dW, torch.float32, "dW", (V, d))
    sv = _Saved(*(_ptr(saved[k]) for k in ("row_max", "lse_support", "cut_logit", "cut_id",
                                            "support_size", "flags")))
    if on_dw_slice is None and not comm_sms:
        st = lib.sts_backward(ctypes.byref(sh), _ptr(H), _ptr(W), ctypes.byref(rows),
                              ctypes.byref(sv), _ptr(grad_logprob), _ptr(dH), _ptr(dW),
                              1 if accumulate_dW else 0, _ptr(ws), ws.numel(), _stream(stream))
        _check(st, "sts_backward")
    else:
        errors = []

        def hook(_user, v0, n, _ptr_slice, _st):
            try:
                if on_dw_slice is not None:
                    on_dw_slice(int(v0), int(n), dW[v0:v0 + n])
            except BaseException as e:  # noqa: BLE001  (re-raised after the call)
                errors.append(e)

        cb = _SLICE_FN(hook)
        st = lib.sts_backward_sliced(ctypes.byref(sh), _ptr(H), _ptr(W), ctypes.byref(rows),
                                     ctypes.byref(sv), _ptr(grad_logprob), _ptr(dH), _ptr(dW),
                                     1 if accumulate_dW else 0, _ptr(ws), ws.numel(),
                                     _stream(stream), cb, None, int(comm_sms))
        if errors:
            raise errors[0]
        _check(st, "sts_backward_sliced")
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return dH, dW


def sts_sample(H, W, temperature, top_k, top_p, min_p, u, *, row_chunk=0, ws=None, stream=None,
               check=False):
    """One token per row drawn from the filtered distribution with uniforms u."""
    lib = load()
    T, d, V = _hw(H, W)
    rows = _rows(T, None, temperature, top_k, top_p, min_p)
    _need(u, torch.float64, "u", (T,))
    sh = _shape(T, d, V, 0, row_chunk)
    ws = _workspace(sts_workspace_bytes(T, d, V, 0, 0, row_chunk), H.device, ws)
    out = torch.empty(T, dtype=torch.int64, device=H.device)
    st = lib.sts_sample(ctypes.byref(sh), _ptr(H), _ptr(W), ctypes.byref(rows), _ptr(u), _ptr(out),
                        _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "sts_sample")
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return out


def sts_filter_logits(S, top_k, top_p, min_p, *, want_mask=False, want_entropy=False, ws=None,
                      stream=None, check=False):
    """The support program alone on fp32 scaled logits S [T, V] (with
    ``want_entropy`` also the entropy of each row's filtered distribution)."""
    lib = load()
    _need(S, torch.float32, "S")
    T, V = S.shape
    for name, t, dt in (("top_k", top_k, torch.int32), ("top_p", top_p, torch.float32),
                        ("min_p", min_p, torch.float32)):
        _need(t, dt, name, (T,))
    rows = _Rows(T, None, None, _ptr(top_k), _ptr(top_p), _ptr(min_p))
    sh = _shape(T, 8, V)
    ws = _workspace(sts_workspace_bytes(T, 8, V, 2), S.device, ws)
    size = torch.empty(T, dtype=torch.int32, device=S.device)
    cut_logit = torch.empty(T, dtype=torch.float32, device=S.device)
    cut_id = torch.empty(T, dtype=torch.int32, device=S.device)
    mask = torch.empty((T, V), dtype=torch.uint8, device=S.device) if want_mask else None
    ent = torch.empty(T, dtype=torch.float32, device=S.device) if want_entropy else None
    st = lib.sts_filter_logits(ctypes.byref(sh), _ptr(S), ctypes.byref(rows), _ptr(size),
                               _ptr(cut_logit), _ptr(cut_id), _ptr(mask), _ptr(ent), _ptr(ws),
                               ws.numel(), _stream(stream))
    _check(st, "sts_filter_logits")
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return {"size": size, "cut_logit": cut_logit, "cut_id": cut_id, "mask": mask, "entropy": ent}


def sts_filter_logits_noalloc(S, top_k, top_p, min_p, *, support_size, cut_logit, cut_id,
                              mask=None, stream=None):
    """sts_filter_logits without a workspace, for callers that cannot allocate
    device memory: every output is caller-provided and the C entry point
    allocates nothing (its scratch is a fixed device array, T <= 65,536)."""
    lib = load()
    _need(S, torch.float32, "S")
    T, V = S.shape
    for name, t, dt in (("top_k", top_k, torch.int32), ("top_p", top_p, torch.float32),
                        ("min_p", min_p, torch.float32), ("support_size", support_size, torch.int32),
                        ("cut_logit", cut_logit, torch.float32), ("cut_id", cut_id, torch.int32)):
        _need(t, dt, name, (T,))
    if mask is not None:
        _need(mask, torch.uint8, "mask", (T, V))
    rows = _Rows(T, None, None, _ptr(top_k), _ptr(top_p), _ptr(min_p))
    sh = _shape(T, 8, V)
    _check(lib.sts_filter_logits_noalloc(ctypes.byref(sh), _ptr(S), ctypes.byref(rows),
                                         _ptr(support_size), _ptr(cut_logit), _ptr(cut_id),
                                         _ptr(mask), _stream(stream)), "sts_filter_logits_noalloc")


PG_OBJECTIVES = {"cispo": 0, "clipped": 1}


def sts_policy_grad(logprob, old_logprob, advantage, *, objective="cispo", eps_low=0.2,
                    eps_high=0.2, scale=1.0, out=None, stream=None):
    """grad_logprob [T] (fp32) of a policy-gradient token loss from the fresh
    logprobs, to pass to sts_backward: CISPO (-scale A min(r, 1 + eps_high))
    or the clipped surrogate (-scale A r where the clip does not bind)."""
    lib = load()
    if objective not in PG_OBJECTIVES:
        raise StsError(STS_ERR_SHAPE, f"objective must be one of {sorted(PG_OBJECTIVES)}")
    T = logprob.shape[0]
    for name, t in (("logprob", logprob), ("old_logprob", old_logprob), ("advantage", advantage)):
        _need(t, torch.float32, name, (T,))
    if out is None:
        out = torch.empty(T, dtype=torch.float32, device=logprob.device)
    _need(out, torch.float32, "out", (T,))
    st = lib.sts_policy_grad(int(T), _ptr(logprob), _ptr(old_logprob), _ptr(advantage),
                             PG_OBJECTIVES[objective], float(eps_low), float(eps_high), float(scale),
                             _ptr(out), _stream(stream))
    if st != STS_OK:
        raise StsError(st, "sts_policy_grad")
    return out


def sts_scaled_logits(H, W, temperature, t0=0, rows=None, v0=0, cols=None, *, out=None,
                      stream=None):
    """The forward's first pass alone: S = (H . W^T) / temperature (fp32)."""
    lib = load()
    T, d, V = _hw(H, W)
    _need(temperature, torch.float32, "temperature", (T,))
    rows = T - t0 if rows is None else rows
    cols = V - v0 if cols is None else cols
    ld = (cols + 3) // 4 * 4
    if out is None:
        out = torch.empty((rows, ld), dtype=torch.float32, device=H.device)
    sh = _shape(T, d, V)
    st = lib.sts_scaled_logits(ctypes.byref(sh), _ptr(H), _ptr(W), _ptr(temperature), int(t0),
                               int(rows), int(v0), int(cols), _ptr(out), int(out.stride(0)),
                               _stream(stream))
    _check(st, "sts_scaled_logits")
    return out[:, :cols]


def sts_probe_mass_exp(s, m, *, stream=None):
    """The resolver's float64 token mass exp(s - m) next to the CUDA library exp."""
    lib = load()
    _need(s, torch.float32, "s")
    n = s.numel()
    mass = torch.empty(n, dtype=torch.float64, device=s.device)
    ref = torch.empty(n, dtype=torch.float64, device=s.device)
    _check(lib.sts_probe_mass_exp(_ptr(s), float(m), _ptr(mass), _ptr(ref), n, _stream(stream)),
           "sts_probe_mass_exp")
    return mass, ref


def sts_launch_count(kind=None):
    """Kernels launched by the library in this process (one kind, or all)."""
    lib = load()
    if kind is None:
        return sum(int(lib.sts_launch_count(i)) for i in range(len(KERNEL_KINDS)))
    return int(lib.sts_launch_count(KERNEL_KINDS.index(kind) if isinstance(kind, str) else kind))


def sts_timing_enable(on=True):
    _check(load().sts_timing_enable(1 if on else 0), "sts_timing_enable")


def sts_timing_read():
    """{kind: (total_ms, launches)} over the records since timing was enabled."""
    lib = load()
    out = {}
    for i, name in enumerate(KERNEL_KINDS):
        ms = ctypes.c_double(0.0)
        n = ctypes.c_int64(0)
        _check(lib.sts_timing_read(i, ctypes.byref(ms), ctypes.byref(n)), "sts_timing_read")
        out[name] = (float(ms.value), int(n.value))
    return out


def sts_get_status(ws, stream=None, raise_on_error=False):
    """Synchronise and read the status word left in ``ws``: (status, first_bad_row)."""
    lib = load()
    row = ctypes.c_int64(-1)
    st = lib.sts_get_status(_ptr(ws), _stream(stream), ctypes.byref(row))
    if raise_on_error and st != STS_OK:
        raise StsError(st, f"row {row.value}" if row.value >= 0 else "device status")
    return int(st), int(row.value)


RESOLVE_PATHS = ("planned", "fast", "exact", "identity")


def sts_path_counts(ws, stream=None):
    """Rows the support resolver decided by each path since ``ws`` was last
    reset by a forward / sample / filter call: {path: rows}. Synchronises."""
    lib = load()
    counts = (ctypes.c_int64 * 4)()
    _check(lib.sts_path_counts(_ptr(ws), _stream(stream), counts), "sts_path_counts")
    return {name: int(counts[i]) for i, name in enumerate(RESOLVE_PATHS)}


def _saved_tensors(T, dev):
    return {
        "row_max": torch.empty(T, dtype=torch.float32, device=dev),
        "lse_support": torch.empty(T, dtype=torch.float32, device=dev),
        "cut_logit": torch.empty(T, dtype=torch.float32, device=dev),
        "cut_id": torch.empty(T, dtype=torch.int32, device=dev),
        "support_size": torch.empty(T, dtype=torch.int32, device=dev),
        "flags": torch.empty(T, dtype=torch.int32, device=dev),
    }


def _saved_struct(saved):
    return _Saved(*(_ptr(saved[k]) for k in ("row_max", "lse_support", "cut_logit", "cut_id",
                                              "support_size", "flags")))


def sts_resolve_logits(S, target, temperature, top_k, top_p, min_p, *, V=None, entropy=False,
                       ws=None, stream=None, check=False):
    """The support program, logprob and saved scalars on fp32 scaled logits
    S [T, ld] (the first V columns of each row; V defaults to ld)."""
    lib = load()
    _need(S, torch.float32, "S")
    T, ld = S.shape
    V = ld if V is None else int(V)
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    sh = _shape(T, 8, V)
    ws = _workspace(sts_workspace_bytes(T, 8, V, 2), S.device, ws)
    logprob = torch.empty(T, dtype=torch.float32, device=S.device)
    saved = _saved_tensors(T, S.device)
    ent = torch.empty(T, dtype=torch.float32, device=S.device) if entropy else None
    st = lib.sts_resolve_logits(ctypes.byref(sh), _ptr(S), ld, ctypes.byref(rows), _ptr(logprob),
                                _ptr(ent), ctypes.byref(_saved_struct(saved)), _ptr(ws), ws.numel(),
                                _stream(stream))
    _check(st, "sts_resolve_logits")
    if ent is not None:
        saved["entropy"] = ent
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return logprob, saved, ws


def sts_backward_shard(H, W_shard, target, temperature, top_k, top_p, min_p, saved, grad_logprob,
                       *, vocab_offset, dW=None, dH=None, accumulate_dW=False, vocab_chunk=0,
                       ws=None, stream=None, check=False):
    """One vocabulary shard's backward: (dH_partial [T, d], dW_shard [Vl, d])."""
    lib = load()
    T, d, Vl = _hw(H, W_shard)
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    _need(grad_logprob, torch.float32, "grad_logprob", (T,))
    sh = _shape(T, d, Vl, vocab_chunk, 0)
    dev = H.device
    ws = _workspace(sts_workspace_bytes(T, d, Vl, 1, vocab_chunk, 0), dev, ws)
    dH = torch.empty((T, d), dtype=torch.float32, device=dev) if dH is None else dH
    if dW is None:
        if accumulate_dW:
            raise StsError(STS_ERR_NULL, "accumulate_dW needs a dW tensor")
        dW = torch.empty((Vl, d), dtype=torch.float32, device=dev)
    _need(dH, torch.float32, "dH", (T, d))
    _need(dW, torch.float32, "dW", (Vl, d))
    st = lib.sts_backward_shard(ctypes.byref(sh), _ptr(H), _ptr(W_shard), ctypes.byref(rows),
                                ctypes.byref(_saved_struct(saved)), _ptr(grad_logprob), _ptr(dH),
                                _ptr(dW), 1 if accumulate_dW else 0, int(vocab_offset), _ptr(ws),
                                ws.numel(), _stream(stream))
    _check(st, "sts_backward_shard")
    if check:
        sts_get_status(ws, stream, raise_on_error=True)
    return dH, dW


def sts_tp_constants():
    """Sizes of the statistics-merge stages' per-row records."""
    lib = load()
    v = [ctypes.c_int64() for _ in range(5)]
    _check(lib.sts_tp_constants(*(ctypes.byref(x) for x in v)), "sts_tp_constants")
    return dict(zip(("buckets", "plan_fields", "sum_fields", "key_fields", "sort_cap"),
                    (int(x.value) for x in v)))


def _shard_view(S):
    _need(S, torch.float32, "S")
    if S.dim() != 2 or S.stride(1) != 1:
        raise StsError(STS_ERR_SHAPE, "S must be [T, Vl] with unit column stride")
    return S.shape[0], S.shape[1], S.stride(0)


def sts_tp_row_max(S, *, stream=None):
    """Stage 1 of the statistics merge: this shard's row maxima [T]."""
    lib = load()
    T, Vl, ld = _shard_view(S)
    out = torch.empty(T, dtype=torch.float32, device=S.device)
    _check(lib.sts_tp_row_max(_ptr(S), T, Vl, ld, _ptr(out), _stream(stream)), "sts_tp_row_max")
    return out


def sts_tp_count(S, m, *, stream=None):
    """Stage 2: this shard's bucket counts [T, buckets] against the merged row max m."""
    lib = load()
    T, Vl, ld = _shard_view(S)
    _need(m, torch.float32, "m", (T,))
    nb = sts_tp_constants()["buckets"]
    out = torch.empty((T, nb), dtype=torch.int32, device=S.device)
    _check(lib.sts_tp_count(_ptr(S), T, Vl, ld, _ptr(m), _ptr(out), _stream(stream)),
           "sts_tp_count")
    return out


def sts_tp_exact(S, vocab_offset, V, target, temperature, top_k, top_p, min_p, m, counts, *,
                 cap=None, stream=None):
    """Stage 3: the row plans, float64 sums, smallest keys, target logit and
    gathered composite keys of this shard (a dict of tensors)."""
    lib = load()
    T, Vl, ld = _shard_view(S)
    c = sts_tp_constants()
    cap = c["sort_cap"] if cap is None else int(cap)
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    _need(m, torch.float32, "m", (T,))
    _need(counts, torch.int32, "counts", (T, c["buckets"]))
    dev = S.device
    out = {
        "plan": torch.empty((T, c["plan_fields"]), dtype=torch.int32, device=dev),
        "sums": torch.empty((T, c["sum_fields"]), dtype=torch.float64, device=dev),
        "keys": torch.empty((T, c["key_fields"]), dtype=torch.int64, device=dev),
        "ylogit": torch.empty((T, 2), dtype=torch.float32, device=dev),
        "cand": torch.empty((T, cap), dtype=torch.int64, device=dev),
        "ncand": torch.empty(T, dtype=torch.int32, device=dev),
    }
    st = lib.sts_tp_exact(_ptr(S), T, Vl, ld, int(vocab_offset), int(V), ctypes.byref(rows), _ptr(m),
                          _ptr(counts), _ptr(out["plan"]), _ptr(out["sums"]), _ptr(out["keys"]),
                          _ptr(out["ylogit"]), _ptr(out["cand"]), _ptr(out["ncand"]), cap,
                          _stream(stream))
    _check(st, "sts_tp_exact")
    return out


def sts_tp_finish(V, target, temperature, top_k, top_p, min_p, m, plan, sums, keys, ylogit, cand,
                  ncand, *, ws=None, stream=None):
    """Stage 4: logprob and saved scalars from the merged stage-3 records
    (cand [world, T, cap] and ncand [world, T] in rank order). Returns
    (logprob, saved, need_gather, ws)."""
    lib = load()
    world, T, cap = cand.shape
    rows = _rows(T, target, temperature, top_k, top_p, min_p)
    dev = m.device
    _need(ncand, torch.int32, "ncand", (world, T))
    ws = _workspace(256, dev, ws)
    logprob = torch.empty(T, dtype=torch.float32, device=dev)
    saved = _saved_tensors(T, dev)
    need = torch.empty(T, dtype=torch.int32, device=dev)
    st = lib.sts_tp_finish(T, int(V), world, ctypes.byref(rows), _ptr(m), _ptr(plan), _ptr(sums),
                           _ptr(keys), _ptr(ylogit), _ptr(cand), _ptr(ncand), cap, _ptr(logprob),
                           ctypes.byref(_saved_struct(saved)), _ptr(need), _ptr(ws), ws.numel(),
                           _stream(stream))
    _check(st, "sts_tp_finish")
    return logprob, saved, need, ws


def sts_gather_vocab_shards(src, dst, *, stream=None):
    """dst [T, ld] <- the rank-order interleave of src [world, T, Vl]."""
    lib = load()
    _need(src, torch.float32, "src")
    _need(dst, torch.float32, "dst")
    world, T, Vl = src.shape
    if dst.shape[0] != T:
        raise StsError(STS_ERR_SHAPE, "dst rows must equal the shards' rows")
    _check(lib.sts_gather_vocab_shards(_ptr(src), world, T, Vl, _ptr(dst), dst.shape[1],
                                       _stream(stream)), "sts_gather_vocab_shards")
    return dst

"""Gated DeltaNet token mixer forward pass for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libgdn.so`` (declared in ``include/gdn.h``):
argument marshalling only -- every step of the computation runs in the CUDA
kernels of the library. PyTorch provides device memory and streams. There is
no CPU fallback: if the library is missing the import of an op fails loudly.

    o, state_out = prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None)
    o = decode(q, k, v, g, beta, state)          # state updated in place

q, k and v may be bf16, f16 or fp32 (all three the same); g, beta and the
prefill states are fp32.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = ["prefill", "prefill_noalloc", "decode", "prefill_workspace_bytes", "prefill_plan", "device_error",
           "wait_selftest",
           "GdnError",
           "lib", "debug_lib", "library_path", "debug_library_path", "GDN_BF16", "GDN_F32", "GDN_F16"]

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libgdn.so")
debug_library_path = os.path.join(_PKG, "libgdn_debug.so")   # GDN_DEBUG build: device-side index checks

(GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_CUDA, GDN_ERR_DEVICE_TIMEOUT,
 GDN_ERR_DEVICE_CHECK) = range(6)
GDN_BF16, GDN_F32, GDN_F16 = 0, 1, 2
STATUS_NAMES = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED",
                3: "GDN_ERR_CUDA", 4: "GDN_ERR_DEVICE_TIMEOUT", 5: "GDN_ERR_DEVICE_CHECK"}


class GdnPlan(ctypes.Structure):
    """struct gdn_plan: the tensor-core prefill's launch plan (0 = the library's choice)."""
    _fields_ = [("dvp", ctypes.c_int), ("n_chain_ctas", ctypes.c_int)]


def _plan_arg(plan):
    """A (dvp, n_chain_ctas) pair (None or 0 per field: the library's choice) as a
    gdn_plan pointer, or None."""
    if plan is None:
        return None
    dvp, nc = plan
    return ctypes.byref(GdnPlan(int(dvp or 0), int(nc or 0)))


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lock = threading.Lock()
_lib = None

_vp, _fp, _i32p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
_i, _i64, _f, _sz = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t

SIGNATURES = {
    "gdn_version": (_i, []),
    "gdn_last_error": (ctypes.c_char_p, []),
    "gdn_prefill_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "gdn_prefill": (_i, [_vp, _vp, _vp, _fp, _fp, _fp, _i32p, _i, _i64, _i, _i, _i, _i, _f, _i, _i,
                         _vp, _fp, _vp, _sz, _vp]),
    "gdn_decode": (_i, [_vp, _vp, _vp, _fp, _fp, _fp, _i, _i, _i, _i, _i, _f, _i, _vp, _vp]),
    "gdn_decode_bf16_state": (_i, [_vp, _vp, _vp, _fp, _fp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp, _vp]),
    "gdn_prefill_noalloc": (_i, [_vp, _vp, _vp, _fp, _fp, _fp, _i32p, _i, _i64, _i, _i, _i, _i, _f, _i, _i,
                                 _vp, _fp, _vp]),
    "gdn_device_error": (_i, [_vp]),
    "gdn_wait_selftest": (_i, [_i, _vp]),
    "gdn_prefill_ex": (_i, [_vp, _vp, _vp, _fp, _fp, _fp, _i32p, _i, _i64, _i, _i, _i, _i, _f, _i, _i,
                            _vp, _fp, _vp, _sz, _vp, _vp]),
    "gdn_prefill_plan": (_i, [_i, _i64, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp]),
    "gdn_debug_checks": (_i, []),
}


def _open(path):
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with "
            "`python -m gated_deltanet_linear_21_b200.build` (there is no CPU fallback)")
    handle = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype, fn.argtypes = res, args
    return handle


def lib():
    """Load libgdn.so (built in-tree); raises if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = _open(library_path)
    return _lib


_debug_lib = None


def debug_lib():
    """Load libgdn_debug.so, the GDN_DEBUG build (same C ABI, device-side index
    checks reported as GDN_ERR_DEVICE_CHECK by its gdn_device_error); a ctypes
    handle for direct calls. The Python wrappers above always use libgdn.so."""
    global _debug_lib
    with _lock:
        if _debug_lib is None:
            _debug_lib = _open(debug_library_path)
    return _debug_lib


def _check(status: int):
    if status != GDN_OK:
        raise GdnError(status, lib().gdn_last_error().decode())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float16:
        return GDN_F16
    if t.dtype == torch.float32:
        return GDN_F32
    raise TypeError(f"q, k, v must be bf16, f16 or fp32, got {t.dtype}")


def _torch_dtype_code(dtype) -> int:
    return {torch.bfloat16: GDN_BF16, torch.float16: GDN_F16, torch.float32: GDN_F32}[dtype]


def _shape(t, name, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _prefill_args(q, k, v, g, beta, state_in, cu_seqlens, o, state_out):
    """Checks and default outputs shared by the prefill entry points."""
    _dev(q, "q"); _dev(k, "k", q.dtype); _dev(v, "v", q.dtype)
    _dev(g, "g", torch.float32); _dev(beta, "beta", torch.float32)
    if q.dim() != 3 or v.dim() != 3:
        raise ValueError("q, k must be [T, Hqk, dk] and v [T, Hv, dv]")
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    _shape(k, "k", (T, Hqk, dk)); _shape(v, "v", (T, Hv, dv))
    _shape(g, "g", (T, Hv)); _shape(beta, "beta", (T, Hv))
    if cu_seqlens is None:
        cu_seqlens = torch.tensor([0, T], dtype=torch.int32, device=q.device)
    _dev(cu_seqlens, "cu_seqlens", torch.int32)
    N = cu_seqlens.numel() - 1
    if state_in is not None:
        _dev(state_in, "state_in", torch.float32)
        _shape(state_in, "state_in", (N, Hv, dv, dk))
    if o is None:
        o = torch.empty(T, Hv, dv, dtype=q.dtype, device=q.device)
    _dev(o, "o", q.dtype); _shape(o, "o", (T, Hv, dv))
    if state_out is None:
        state_out = torch.empty(N, Hv, dv, dk, dtype=torch.float32, device=q.device)
    _dev(state_out, "state_out", torch.float32); _shape(state_out, "state_out", (N, Hv, dv, dk))
    return T, Hqk, dk, Hv, dv, N, cu_seqlens, o, state_out


def _dev(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def prefill_workspace_bytes(n_seqs, Hv, dk, dv, dtype=torch.bfloat16) -> int:
    return int(lib().gdn_prefill_workspace_bytes(n_seqs, Hv, dk, dv, _torch_dtype_code(dtype)))


def prefill_plan(n_seqs, total_T, Hv, dk=128, dv=128, dtype=torch.bfloat16, sm_count=0, requested=None):
    """(dvp, n_chain_ctas, rounds): the launch plan the tensor-core prefill would
    use for this problem, given a `requested` (dvp, n_chain_ctas) plan or None;
    host only. sm_count=0 asks the current device."""
    out = [ctypes.c_int(0) for _ in range(3)]
    _check(lib().gdn_prefill_plan(int(n_seqs), int(total_T), int(Hv), int(dk), int(dv), _torch_dtype_code(dtype),
                                  int(sm_count), _plan_arg(requested), *[ctypes.byref(x) for x in out]))
    return tuple(x.value for x in out)


def prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, scale=None, chunk=0,
            o=None, state_out=None, workspace=None, plan=None, stream=None):
    """Chunked prefill over packed sequences.

    q, k [T, Hqk, dk]; v [T, Hv, dv] (bf16, f16 or fp32, same dtype); g, beta
    [T, Hv] fp32; state_in [N, Hv, dv, dk] fp32 or None; cu_seqlens [N+1] int32
    (None = one sequence of T tokens). `plan` = (dvp, n_chain_ctas) for the
    tensor-core kernel (gdn_prefill_ex; None or 0: the library's choice).
    Returns (o [T, Hv, dv], state_out [N, Hv, dv, dk]).
    """
    T, Hqk, dk, Hv, dv, N, cu_seqlens, o, state_out = _prefill_args(q, k, v, g, beta, state_in, cu_seqlens,
                                                                    o, state_out)
    need = prefill_workspace_bytes(N, Hv, dk, dv, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().gdn_prefill_ex(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
        state_in.data_ptr() if state_in is not None else None, cu_seqlens.data_ptr(),
        N, T, Hqk, Hv, dk, dv, float(scale or 0.0), int(chunk), _dtype_code(q),
        o.data_ptr(), state_out.data_ptr(), ws_ptr, ws_bytes, _plan_arg(plan), _stream_handle(stream)))
    return o, state_out


def prefill_noalloc(q, k, v, g, beta, state_in=None, cu_seqlens=None, *, scale=None, o=None,
                    state_out=None, stream=None):
    """gdn_prefill_noalloc: the prefill with the library's built-in scratch
    instead of a workspace (for callers that cannot allocate device memory).
    Outputs are allocated here only if not given."""
    T, Hqk, dk, Hv, dv, N, cu_seqlens, o, state_out = _prefill_args(q, k, v, g, beta, state_in, cu_seqlens,
                                                                    o, state_out)
    _check(lib().gdn_prefill_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
        state_in.data_ptr() if state_in is not None else None, cu_seqlens.data_ptr(),
        N, T, Hqk, Hv, dk, dv, float(scale or 0.0), 0, _dtype_code(q),
        o.data_ptr(), state_out.data_ptr(), _stream_handle(stream)))
    return o, state_out


def decode(q, k, v, g, beta, state, *, scale=None, o=None, stream=None):
    """One decode step: q, k [B, Hqk, dk]; v [B, Hv, dv]; g, beta [B, Hv];
    state [B, Hv, dv, dk] updated in place -- fp32 (gdn_decode) or bf16
    (gdn_decode_bf16_state: fp32 arithmetic, stored rounded to nearest even).
    Returns o [B, Hv, dv]."""
    _dev(q, "q"); _dev(k, "k", q.dtype); _dev(v, "v", q.dtype)
    _dev(g, "g", torch.float32); _dev(beta, "beta", torch.float32)
    _dev(state, "state")
    if state.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"state must be fp32 or bf16, got {state.dtype}")
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if o is None:
        o = torch.empty(B, Hv, dv, dtype=q.dtype, device=q.device)
    fn = lib().gdn_decode if state.dtype == torch.float32 else lib().gdn_decode_bf16_state
    _check(fn(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(), state.data_ptr(),
        B, Hqk, Hv, dk, dv, float(scale or 0.0), _dtype_code(q), o.data_ptr(),
        _stream_handle(stream)))
    return o


def wait_selftest(max_wait_us: int = 2000, stream=None) -> None:
    """Enqueue the bounded-wait self test (gdn_wait_selftest): a following
    device_error() raises GdnError with GDN_ERR_DEVICE_TIMEOUT."""
    _check(lib().gdn_wait_selftest(int(max_wait_us), _stream_handle(stream)))


def device_error(stream=None) -> None:
    """Synchronise and raise GdnError if a bounded device wait ran out."""
    _check(lib().gdn_device_error(_stream_handle(stream)))

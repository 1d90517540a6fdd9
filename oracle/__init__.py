"""fp64 sequential CPU oracle for the Gated DeltaNet token mixer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package; the product library
never does. It shares no code with the CUDA path.

The arithmetic lives in ``gdn_oracle.c`` (plain C, fp64, no fast-math); this
module compiles it with gcc and marshals numpy arrays through ctypes. The
definition it follows is written out in the header of ``gdn_oracle.c``: the
gated delta rule S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t
k_t^T, o_t = S_t q_t, with q and k L2-normalised and q scaled, which the
Herbert pages name as the Gated DeltaNet mixer recurrence ("On descend d'un
cran : #001 un compilateur pour moteur de LLM", section "Un compilateur, pas
une bibliothèque de kernels") without printing it.

Pins (tests/test_oracle.py): an explicit-matrix brute force, an independent
chunked formulation, closed forms and a hand-worked example
(tests/golden/handworked_d2_t2.json).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

EPS = 1e-6  # L2-normalisation epsilon, added inside the square root


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so (gcc, fp64, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.gdn_oracle_prefill.restype = ctypes.c_int
            lib.gdn_oracle_prefill.argtypes = [
                dp, dp, dp, dp, dp, dp, ctypes.POINTER(ctypes.c_int64),
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                dp, dp, ctypes.c_int]
            lib.gdn_oracle_decode.restype = ctypes.c_int
            lib.gdn_oracle_decode.argtypes = [
                dp, dp, dp, dp, dp, dp,
                ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_double, ctypes.c_double, ctypes.c_int, ctypes.c_int,
                dp, ctypes.c_int]
            lib.gdn_oracle_decode_ex.restype = ctypes.c_int
            lib.gdn_oracle_decode_ex.argtypes = lib.gdn_oracle_decode.argtypes + [ctypes.c_int]
            lib.gdn_oracle_round_bf16.restype = None
            lib.gdn_oracle_round_bf16.argtypes = [dp, dp, ctypes.c_long]
            lib.gdn_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Widen a numpy array or CPU torch tensor (any float dtype) to contiguous fp64."""
    if hasattr(x, "detach"):  # torch tensor: widen through torch (bf16 has no numpy type)
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().gdn_oracle_max_threads())


def prefill(q, k, v, g, beta, state_in, cu_seqlens, scale=None, eps=EPS,
            heads=None, n_threads=None):
    """Sequential fp64 prefill.

    q, k [T, Hqk, dk]; v [T, Hv, dv]; g, beta [T, Hv]; state_in [N, Hv, dv, dk]
    or None (zero state); cu_seqlens [N+1]. ``heads`` = (h_lo, h_hi) restricts
    the value heads computed (others stay NaN). Returns (o [T, Hv, dv],
    state_out [N, Hv, dv, dk]) as fp64 numpy arrays.
    """
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    cu = np.ascontiguousarray(np.asarray(
        cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
    T, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    N = cu.shape[0] - 1
    if scale is None:
        scale = dk ** -0.5
    h_lo, h_hi = heads if heads is not None else (0, Hv)
    o = np.full((T, Hv, dv), np.nan)
    s_out = np.full((N, Hv, dv, dk), np.nan)
    s_in = None if state_in is None else _f64(state_in)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    rc = _load().gdn_oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
        None if s_in is None else _ptr(s_in),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        N, Hqk, Hv, dk, dv, float(scale), float(eps), h_lo, h_hi,
        _ptr(o), _ptr(s_out), int(n_threads))
    if rc != 0:
        raise ValueError("gdn_oracle_prefill rejected its arguments")
    return o, s_out


def round_bf16(x) -> np.ndarray:
    """fp64 values rounded to the nearest bfloat16 (ties to even) by way of the
    nearest float, as the bf16-state decode stores them."""
    x = _f64(x)
    out = np.empty_like(x)
    _load().gdn_oracle_round_bf16(_ptr(x), _ptr(out), x.size)
    return out


def decode(q, k, v, g, beta, state, scale=None, eps=EPS, heads=None, n_threads=None, state_bf16=False):
    """One fp64 decode step. ``state`` [B, Hv, dv, dk] (fp64 numpy) is updated in
    place and also returned; returns (o [B, Hv, dv], state). With ``state_bf16``
    the updated state is stored rounded to bfloat16 (o is read before that)."""
    q, k, v, g, beta = (_f64(a) for a in (q, k, v, g, beta))
    if not (isinstance(state, np.ndarray) and state.dtype == np.float64
            and state.flags.c_contiguous):
        raise TypeError("state must be a C-contiguous fp64 numpy array (updated in place)")
    B, Hqk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    if scale is None:
        scale = dk ** -0.5
    h_lo, h_hi = heads if heads is not None else (0, Hv)
    o = np.full((B, Hv, dv), np.nan)
    if n_threads is None:
        n_threads = os.cpu_count() or 1
    rc = _load().gdn_oracle_decode_ex(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state),
        B, Hqk, Hv, dk, dv, float(scale), float(eps), h_lo, h_hi, _ptr(o), int(n_threads),
        1 if state_bf16 else 0)
    if rc != 0:
        raise ValueError("gdn_oracle_decode rejected its arguments")
    return o, state

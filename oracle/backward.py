"""fp64 CPU oracle for the gradients of the GLA forward pass (dq, dk, dv,
dlog_alpha).

TEST INFRASTRUCTURE ONLY: used by tests/; the CUDA library never imports it.

The arithmetic lives in ``gla_backward.c``: reverse mode through the
recurrence S_t = diag(alpha_t) S_{t-1} + k_t^T v_t, o_t = q_t S_t of "GTR:
Gated Token Recurrence for Efficient Dense Prediction" (x-techcon article,
section 架构), in the scan order of the chosen direction.  This file builds
and loads it and marshals numpy arrays.  Array convention as in oracle.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_backward.c")
_LIB_PATH = os.path.join(_HERE, "libgla_backward.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile gla_backward.c into oracle/libgla_backward.so (gcc, -O2, every
    multiply and add rounded separately)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        lib.gla_oracle_backward.argtypes = [dp] * 10 + [ctypes.c_int] * 7
        lib.gla_oracle_backward.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def backward(q, k, v, log_alpha, d_out, direction: int, d_final_state=None):
    """Gradients of L = sum(d_out * out) + sum(d_final_state * final_state)
    with respect to q, k, v and log_alpha.  Returns (dq, dk, dv, dlog_alpha)."""
    q, k, v, la, dO = (_f64(a) for a in (q, k, v, log_alpha, d_out))
    if q.ndim != 5 or k.shape != q.shape or la.shape != q.shape:
        raise ValueError("q, k, log_alpha must share shape [B,H,grid_h,grid_w,d_k]")
    if v.ndim != 5 or v.shape[:4] != q.shape[:4] or dO.shape != v.shape:
        raise ValueError("v and d_out must be [B,H,grid_h,grid_w,d_v]")
    B, H, gh, gw, dk = q.shape
    dv = v.shape[-1]
    dS = None if d_final_state is None else _f64(d_final_state)
    if dS is not None and dS.shape != (B, H, dk, dv):
        raise ValueError("d_final_state must be [B,H,d_k,d_v]")
    gq, gk, gla = np.empty_like(q), np.empty_like(k), np.empty_like(la)
    gv = np.empty_like(v)
    rc = _load().gla_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(dO), _ptr(dS),
                                     _ptr(gq), _ptr(gk), _ptr(gv), _ptr(gla), B, H, gh, gw, dk, dv,
                                     int(direction))
    if rc != 0:
        raise ValueError(f"gla_oracle_backward rejected its arguments (code {rc})")
    return gq, gk, gv, gla

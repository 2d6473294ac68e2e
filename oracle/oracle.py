"""fp64 CPU oracle for the GTR key-gated linear attention forward pass.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by the cpu_baseline / reference legs of ``bench.py``.  The product path
(the CUDA library and its Python binding) never imports this module.

The arithmetic lives in ``gla_oracle.c`` (plain C, fp64, OpenMP over the B*H
planes); this file only builds/loads it and marshals numpy arrays.

Source of the method: "GTR: Gated Token Recurrence for Efficient Dense
Prediction" (x-techcon article, section 架构 for the recurrence and the four
scan directions, section 算子 for the chunkwise reorganisation).

Array convention: q, k, log_alpha are [B, H, grid_h, grid_w, d_k]; v and the
output are [B, H, grid_h, grid_w, d_v]; the final state is [B, H, d_k, d_v].
Everything is converted to contiguous float64 before the call, so fp16 inputs
enter as their exactly-representable rounded values.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgla_oracle.so")
_lib = None

DIRECTIONS = {0: "L->R", 1: "R->L", 2: "T->B", 3: "B->T"}


def build(force: bool = False) -> str:
    """Compile gla_oracle.c into oracle/libgla_oracle.so (gcc, -O2, OpenMP).

    -ffp-contract=off keeps every multiply and add separately rounded, so the
    oracle's fp64 results do not depend on the host's FMA support.
    """
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.gla_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp] + [i] * 8
        lib.gla_oracle_forward.restype = i
        lib.gla_oracle_chunkwise.argtypes = [dp, dp, dp, dp, dp, dp] + [i] * 9
        lib.gla_oracle_chunkwise.restype = i
        lib.gla_oracle_max_threads.argtypes = []
        lib.gla_oracle_max_threads.restype = i
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: upcast on the CPU
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _prep(q, k, v, log_alpha):
    q, k, v, la = _f64(q), _f64(k), _f64(v), _f64(log_alpha)
    if q.ndim != 5 or k.shape != q.shape or la.shape != q.shape:
        raise ValueError("q, k, log_alpha must share shape [B,H,grid_h,grid_w,d_k]")
    if v.ndim != 5 or v.shape[:4] != q.shape[:4]:
        raise ValueError("v must be [B,H,grid_h,grid_w,d_v]")
    return q, k, v, la


def forward(q, k, v, log_alpha, direction: int, n_threads: int = 0):
    """Token-by-token recurrence in fp64.  Returns (out, final_state)."""
    q, k, v, la = _prep(q, k, v, log_alpha)
    B, H, gh, gw, dk = q.shape
    dv = v.shape[-1]
    out = np.empty((B, H, gh, gw, dv), np.float64)
    fs = np.empty((B, H, dk, dv), np.float64)
    rc = _load().gla_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(out),
                                    _ptr(fs), B, H, gh, gw, dk, dv, int(direction),
                                    int(n_threads))
    if rc != 0:
        raise ValueError(f"gla_oracle_forward rejected its arguments (code {rc})")
    return out, fs


def chunkwise(q, k, v, log_alpha, direction: int, chunk: int, n_threads: int = 0):
    """The chunkwise reorganisation written out in fp64.  Returns (out, final_state)."""
    q, k, v, la = _prep(q, k, v, log_alpha)
    B, H, gh, gw, dk = q.shape
    dv = v.shape[-1]
    out = np.empty((B, H, gh, gw, dv), np.float64)
    fs = np.empty((B, H, dk, dv), np.float64)
    rc = _load().gla_oracle_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(out),
                                      _ptr(fs), B, H, gh, gw, dk, dv, int(direction),
                                      int(chunk), int(n_threads))
    if rc != 0:
        raise ValueError(f"gla_oracle_chunkwise rejected its arguments (code {rc})")
    return out, fs


def max_threads() -> int:
    return int(_load().gla_oracle_max_threads())


def rel_err(got, ref) -> float:
    """max|got - ref| / max|ref| over the whole tensor (the parity metric)."""
    got = _f64(got)
    ref = _f64(ref)
    denom = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    if denom == 0.0:
        return num
    return num / denom

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


def _scan_order(gh: int, gw: int, direction: int) -> np.ndarray:
    """Raster token index at each scan position."""
    rows = np.arange(gh * gw)
    cols = np.array([y * gw + x for x in range(gw) for y in range(gh)])
    return {0: rows, 1: rows[::-1], 2: cols, 3: cols[::-1]}[int(direction)]


def chunkwise_backward(q, k, v, log_alpha, d_out, direction: int, chunk: int, d_final_state=None):
    """The same gradients as backward(), reorganised by chunks of `chunk`
    tokens as a chunked kernel computes them (fp64, numpy):

    1. forward over chunks: boundary states S_in(c), with b the inclusive
       in-chunk log-gate sum and g its value at the chunk's end:
       S_in(c+1) = diag(e^g) S_in(c) + sum_s (k_s . e^{g - b_s})^T v_s;
    2. backward over chunks: dS_out of the last chunk is dS_final, and
       dS_out(c-1) = dS_in(c) = diag(e^g) dS_out(c) + sum_t (q_t . e^{b_t})^T dO_t;
    3. in every chunk, with A[t,s] = sum_i q_ti k_si e^{b_ti - b_si} (s <= t)
       and W[t,s] = dO_t . v_s (s <= t):
         dq_t = e^{b_t} . (dO_t S_in^T) + sum_{s<=t} W[t,s] k_s . e^{b_t - b_s}
         dk_s = sum_{t>=s} W[t,s] q_t . e^{b_t - b_s} + e^{g - b_s} . (dS_out v_s)
         dv_s = sum_{t>=s} A[t,s] dO_t + (k_s . e^{g - b_s}) dS_out;
    4. the log-gates: with B the log-gate sum from the start of the scan,
       o_t depends on B only through q_t e^{B_t} and k_s e^{-B_s}, and S_final
       through e^{B_last - B_s}, so dL/dB_t = q_t . dq_t - k_t . dk_t (plus
       rowsum(dS_final . S_final) at the last token), and dlog_alpha_u is the
       sum of dL/dB_t over t >= u.
    Returns (dq, dk, dv, dlog_alpha)."""
    q, k, v, la, dO = (_f64(a) for a in (q, k, v, log_alpha, d_out))
    B, H, gh, gw, dk_ = q.shape
    dv_ = v.shape[-1]
    n = gh * gw
    order = _scan_order(gh, gw, direction)
    dS_all = None if d_final_state is None else _f64(d_final_state)
    outs = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(la)]
    for b in range(B):
        for h in range(H):
            Q = q[b, h].reshape(n, dk_)[order]
            K = k[b, h].reshape(n, dk_)[order]
            V = v[b, h].reshape(n, dv_)[order]
            L = la[b, h].reshape(n, dk_)[order]
            G = dO[b, h].reshape(n, dv_)[order]
            starts = list(range(0, n, chunk))
            # 1. boundary states
            S_in = [np.zeros((dk_, dv_))]
            for t0 in starts:
                sl = slice(t0, min(t0 + chunk, n))
                bb = np.cumsum(L[sl], axis=0)
                g = bb[-1]
                S_in.append(np.exp(g)[:, None] * S_in[-1] + (K[sl] * np.exp(g - bb)).T @ V[sl])
            S_final = S_in[-1]
            # 2. state gradients, last chunk first
            dS_out = [None] * len(starts)
            cur = np.zeros((dk_, dv_)) if dS_all is None else dS_all[b, h].copy()
            for ci in range(len(starts) - 1, -1, -1):
                t0 = starts[ci]
                sl = slice(t0, min(t0 + chunk, n))
                bb = np.cumsum(L[sl], axis=0)
                g = bb[-1]
                dS_out[ci] = cur
                cur = np.exp(g)[:, None] * cur + (Q[sl] * np.exp(bb)).T @ G[sl]
            # 3. per-chunk gradients
            dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
            for ci, t0 in enumerate(starts):
                sl = slice(t0, min(t0 + chunk, n))
                m = sl.stop - sl.start
                bb = np.cumsum(L[sl], axis=0)
                g = bb[-1]
                mask = np.tril(np.ones((m, m)))
                E = np.exp(bb[:, None, :] - bb[None, :, :]) * mask[:, :, None]  # [t, s, i]
                A = np.einsum("ti,si,tsi->ts", Q[sl], K[sl], E)
                W = (G[sl] @ V[sl].T) * mask
                dQ[sl] = np.exp(bb) * (G[sl] @ S_in[ci].T) + np.einsum("ts,si,tsi->ti", W, K[sl], E)
                kt = K[sl] * np.exp(g - bb)
                dK[sl] = np.einsum("ts,ti,tsi->si", W, Q[sl], E) + np.exp(g - bb) * (V[sl] @ dS_out[ci].T)
                dV[sl] = A.T @ G[sl] + kt @ dS_out[ci]
            # 4. log-gates
            dBt = Q * dQ - K * dK
            dBt[-1] += np.sum(dS_all[b, h] * S_final, axis=1) if dS_all is not None else 0.0
            dL = np.cumsum(dBt[::-1], axis=0)[::-1]
            for arr, src, d in ((outs[0], dQ, dk_), (outs[1], dK, dk_), (outs[2], dV, dv_), (outs[3], dL, dk_)):
                flat = np.empty((n, d))
                flat[order] = src
                arr[b, h] = flat.reshape(gh, gw, d)
    return tuple(outs)

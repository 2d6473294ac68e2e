"""ctypes binding of the library's tensor-core GEMM (gtr_gemm_fwd; argument
marshalling only).  See ``include/gtr_gemm.h``: out[M, N] = in[M, K] .
W[N, K]^T (+ bias[N]) (+ resid[M, N]), fp16 or bf16, row-major."""
from __future__ import annotations

import ctypes

import torch

from . import gla as _gla

_lib = _gla._lib
_vp = ctypes.c_void_p
_lib.gtr_gemm_fwd.argtypes = [_vp] * 5 + [ctypes.c_longlong, ctypes.c_int, ctypes.c_int, ctypes.c_int, _vp]
_lib.gtr_gemm_fwd.restype = ctypes.c_int


def gtr_gemm_fwd(x, w, bias=None, resid=None, out=None, stream=None):
    """x [..., K] . w[N, K]^T (+ bias[N]) (+ resid[..., N]) in x's dtype.
    resid may be out (accumulate in place).  Returns out."""
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("x must be fp16 or bf16")
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    N = w.shape[0]
    dev = x.device
    _gla._check("x", x, tuple(x.shape), x.dtype, dev)
    _gla._check("w", w, (N, K), x.dtype, dev)
    if bias is not None:
        _gla._check("bias", bias, (N,), x.dtype, dev)
    oshape = tuple(x.shape[:-1]) + (N,)
    if resid is not None:
        _gla._check("resid", resid, oshape, x.dtype, dev)
    if out is None:
        out = torch.empty(oshape, dtype=x.dtype, device=dev)
    _gla._check("out", out, oshape, x.dtype, dev)
    rc = _lib.gtr_gemm_fwd(_gla._ptr(x), _gla._ptr(w), _gla._ptr(bias), _gla._ptr(resid), _gla._ptr(out),
                           M, N, K, _gla._DTYPE_CODE[x.dtype], _vp(_gla._stream_handle(stream)))
    if rc != 0:
        raise _gla.GlaError(rc)
    return out

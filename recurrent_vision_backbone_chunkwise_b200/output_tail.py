"""ctypes binding of the token mixer's output tail in libgtr_gla.so (argument
marshalling only; the arithmetic runs in the library's kernel).  See
``include/gtr_output_tail.h`` for the contract.

Tensors are torch CUDA tensors, contiguous: o [B, H, grid_h, grid_w, d_v] (the
attention's output), z [B, grid_h, grid_w, H * d_v] and the output in fp16 or
bf16, w [H, d_v] in fp32.
"""
from __future__ import annotations

import ctypes

import torch

from . import gla as _gla

_lib = _gla._lib
_vp, _int, _flt = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_lib.gtr_output_tail_fwd.argtypes = [_vp] * 4 + [_int] * 5 + [_flt, _int, _vp]
_lib.gtr_output_tail_fwd.restype = _int


def gtr_output_tail_fwd(o, z, w, eps: float = 1e-5, out=None, stream=None):
    """y = per-head RMS norm of o (weight w) times SiLU(z), heads merged
    channels-last.  Returns y [B, grid_h, grid_w, H * d_v]."""
    if o.dim() != 5:
        raise ValueError("o must be [B, H, grid_h, grid_w, d_v]")
    if o.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("o must be fp16 or bf16")
    B, H, gh, gw, dv = o.shape
    if out is None:
        out = torch.empty((B, gh, gw, H * dv), dtype=o.dtype, device=o.device)
    rc = _lib.gtr_output_tail_fwd(_gla._ptr(o), _gla._ptr(z), _gla._ptr(w), _gla._ptr(out), B, H, gh,
                                  gw, dv, float(eps), _gla._DTYPE_CODE[o.dtype],
                                  _vp(_gla._stream_handle(stream)))
    if rc != 0:
        raise _gla.GlaError(rc)
    return out

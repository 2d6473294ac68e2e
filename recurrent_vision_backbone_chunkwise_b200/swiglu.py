"""ctypes binding of the Spatial SwiGLU entry points of libgtr_gla.so
(argument marshalling only; the arithmetic runs in the library's kernels: its
tensor-core GEMM for the two projections, its fused kernel for the rest).  See
``include/gtr_swiglu.h`` for the contract.

Tensors are torch CUDA tensors, contiguous: x [B, grid_h, grid_w, C] and the
output in fp16 or bf16, w_gu [2F, C] and w_down [C, F] in the same dtype,
b_gu [2F], w_dw [F, 3, 3], b_dw [F], b_down [C] in fp32.
"""
from __future__ import annotations

import ctypes

import torch

from . import gla as _gla

_lib = _gla._lib
_vp, _int, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.gtr_swiglu_fwd.argtypes = [_vp] * 8 + [_int] * 6 + [_vp, _sz, _vp]
_lib.gtr_swiglu_fwd.restype = _int
_lib.gtr_swiglu_workspace_size.argtypes = [_int] * 6
_lib.gtr_swiglu_workspace_size.restype = _sz

_workspaces = {}


def gtr_swiglu_workspace_size(B, grid_h, grid_w, C, F, dtype=_gla.F16) -> int:
    return int(_lib.gtr_swiglu_workspace_size(B, grid_h, grid_w, C, F, dtype))


def gtr_swiglu_fwd(x, w_gu, b_gu, w_dw, b_dw, w_down, b_down, out=None, workspace=None,
                   stream=None):
    """y = Spatial SwiGLU(x).  A workspace is taken from a per-device cache
    when none is given.  Returns y."""
    if x.dim() != 4:
        raise ValueError("x must be [B, grid_h, grid_w, C]")
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("x must be fp16 or bf16")
    B, gh, gw, C = x.shape
    F = w_gu.shape[0] // 2
    dtype = _gla._DTYPE_CODE[x.dtype]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        need = gtr_swiglu_workspace_size(B, gh, gw, C, F, dtype)
        key = (x.device.index, need)
        workspace = _workspaces.get(key)
        if workspace is None:
            workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=x.device)
            _workspaces[key] = workspace
    rc = _lib.gtr_swiglu_fwd(_gla._ptr(x), _gla._ptr(w_gu), _gla._ptr(b_gu), _gla._ptr(w_dw),
                             _gla._ptr(b_dw), _gla._ptr(w_down), _gla._ptr(b_down),
                             _gla._ptr(out), B, gh, gw, C, F, dtype, _gla._ptr(workspace),
                             workspace.numel(), _vp(_gla._stream_handle(stream)))
    if rc != 0:
        raise _gla.GlaError(rc)
    return out

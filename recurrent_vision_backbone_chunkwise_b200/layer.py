"""ctypes binding of the backbone entry points of libgtr_gla.so (argument
marshalling only): one GTR layer (gtr_layer_fwd) and the direction-cycled
stack (gtr_backbone_fwd).  See ``include/gtr_layer.h`` for the contract.

Activations x [B, grid_h, grid_w, C] in fp16 or bf16, updated in place.  One
layer's parameters come as the dict that ``inputs.make_backbone_params`` gives
(the oracle's names and shapes); ``pack_weights`` puts them on the device, with
W_q, W_k, W_v, W_a, W_z stacked into the fused projection w_proj [5C, C].
"""
from __future__ import annotations

import ctypes

import torch

from . import gla as _gla

_lib = _gla._lib
_vp, _int, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

_FIELDS = ("ln1_w", "ln1_b", "w_proj", "b_a", "w_n", "w_o", "ln2_w", "ln2_b", "w_gu", "b_gu", "w_dw",
           "b_dw", "w_down", "b_down")


class GtrLayerWeights(ctypes.Structure):
    _fields_ = [(n, _vp) for n in _FIELDS]


_lib.gtr_layer_fwd.argtypes = [_vp, ctypes.POINTER(GtrLayerWeights)] + [_int] * 7 + [_vp, _sz, _vp]
_lib.gtr_layer_fwd.restype = _int
_lib.gtr_backbone_fwd.argtypes = [_vp, ctypes.POINTER(GtrLayerWeights)] + [_int] * 7 + [_vp, _sz, _vp]
_lib.gtr_backbone_fwd.restype = _int
_lib.gtr_layer_workspace_size.argtypes = [_int] * 6
_lib.gtr_layer_workspace_size.restype = _sz


def _shapes(C: int, F: int) -> dict:
    H = C // 64
    return {"ln1_w": (C,), "ln1_b": (C,), "w_proj": (5 * C, C), "b_a": (C,), "w_n": (H, 64),
            "w_o": (C, C), "ln2_w": (C,), "ln2_b": (C,), "w_gu": (2 * F, C), "b_gu": (2 * F,),
            "w_dw": (F, 3, 3), "b_dw": (F,), "w_down": (C, F), "b_down": (C,)}


_MATRICES = ("w_proj", "w_o", "w_gu", "w_down")


class LayerWeights:
    """One layer's parameters on the device and the struct that points at them
    (the tensors stay alive as long as this object)."""

    def __init__(self, tensors: dict, C: int, F: int):
        self.tensors, self.C, self.F = tensors, C, F
        self.struct = GtrLayerWeights(*[_vp(tensors[n].data_ptr()) for n in _FIELDS])

    def check(self, dtype, device):
        for name, shape in _shapes(self.C, self.F).items():
            t = self.tensors[name]
            _gla._check(name, t, shape, dtype if name in _MATRICES else torch.float32, device)


def pack_weights(p: dict, device, dtype=torch.float16) -> LayerWeights:
    """Device copies of one layer's parameters, with the five projections of
    the token mixer stacked into w_proj."""
    d = {}
    for k, t in p.items():
        d[k] = t.to(device=device, dtype=dtype if k.startswith("w_") and k not in ("w_n", "w_dw")
                    else torch.float32).contiguous()
    d["w_proj"] = torch.cat([d.pop(n) for n in ("w_q", "w_k", "w_v", "w_a", "w_z")], 0).contiguous()
    C = d["ln1_w"].shape[0]
    F = d["b_dw"].shape[0]
    return LayerWeights(d, C, F)


def gtr_layer_workspace_size(B, grid_h, grid_w, C, F, dtype=_gla.F16) -> int:
    return int(_lib.gtr_layer_workspace_size(B, grid_h, grid_w, C, F, dtype))


def _check_x(x, weights):
    if not isinstance(x, torch.Tensor) or x.dim() != 4:
        raise ValueError("x must be a 4-D tensor [B, grid_h, grid_w, C]")
    if x.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("x must be fp16 or bf16")
    if not x.is_contiguous() or x.device.type != "cuda":
        raise ValueError("x must be a contiguous CUDA tensor")
    for w in weights:
        if w.C != x.shape[-1]:
            raise ValueError(f"weights are for C = {w.C}, x has C = {x.shape[-1]}")
        if w.F != weights[0].F:
            raise ValueError("all layers must have the same F")
        w.check(x.dtype, x.device)


def _workspace(x, F, workspace):
    B, gh, gw, C = x.shape
    need = gtr_layer_workspace_size(B, gh, gw, C, F, _gla._DTYPE_CODE[x.dtype])
    if workspace is None:
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=x.device)
    _gla._check("workspace", workspace, (workspace.numel(),), torch.uint8, x.device)
    return workspace


def gtr_layer_fwd(x, weights: LayerWeights, direction: int, workspace=None, stream=None):
    """One layer applied to x in place.  A given workspace must be zero-filled
    before its first use.  Returns x."""
    _check_x(x, [weights])
    workspace = _workspace(x, weights.F, workspace)
    B, gh, gw, C = x.shape
    rc = _lib.gtr_layer_fwd(_gla._ptr(x), ctypes.byref(weights.struct), B, gh, gw, C, weights.F,
                            int(direction), _gla._DTYPE_CODE[x.dtype], _gla._ptr(workspace),
                            workspace.numel(), _vp(_gla._stream_handle(stream)))
    if rc != 0:
        raise _gla.GlaError(rc)
    return x


def gtr_backbone_fwd(x, layers: list, workspace=None, stream=None):
    """len(layers) layers applied to x in place, layer l scanning in direction
    l mod 4.  Returns x."""
    if not layers:
        raise ValueError("at least one layer")
    _check_x(x, layers)
    workspace = _workspace(x, layers[0].F, workspace)
    arr = (GtrLayerWeights * len(layers))(*[w.struct for w in layers])
    B, gh, gw, C = x.shape
    rc = _lib.gtr_backbone_fwd(_gla._ptr(x), arr, len(layers), B, gh, gw, C, layers[0].F,
                               _gla._DTYPE_CODE[x.dtype], _gla._ptr(workspace), workspace.numel(),
                               _vp(_gla._stream_handle(stream)))
    if rc != 0:
        raise _gla.GlaError(rc)
    return x

"""ctypes binding of libgtr_gla.so (argument marshalling only).

Every function here has the name of the C entry point it forwards to (see
``include/gtr_gla.h``); the arithmetic runs in the library's CUDA kernels.
If the library is missing or cannot be loaded, importing this module raises:
there is no CPU fallback.

Tensors are torch CUDA tensors, contiguous, laid out [B, H, grid_h, grid_w, d]
(q, k, log_alpha with d = d_k; v, out with d = d_v); the final state is
[B, H, d_k, d_v] fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgtr_gla.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m recurrent_vision_backbone_chunkwise_b200.build` (needs nvcc)")

_lib = ctypes.CDLL(LIB_PATH)

_vp, _int, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.gtr_gla_fwd.argtypes = [_vp] * 6 + [_int] * 7 + [_vp]
_lib.gtr_gla_fwd.restype = _int
_lib.gtr_gla_fwd_ex.argtypes = [_vp] * 6 + [_int] * 9 + [_vp, _sz, _vp]
_lib.gtr_gla_fwd_ex.restype = _int
_lib.gtr_gla_fwd_noalloc.argtypes = [_vp] * 6 + [_int] * 7 + [_vp]
_lib.gtr_gla_fwd_noalloc.restype = _int
_lib.gtr_gla_fwd_tail.argtypes = [_vp] * 6 + [ctypes.c_float] + [_vp] * 2 + [_int] * 8 + [_vp, _sz, _vp]
_lib.gtr_gla_fwd_tail.restype = _int
_lib.gtr_gla_tail_workspace_size.argtypes = [_int] * 7
_lib.gtr_gla_tail_workspace_size.restype = _sz
_lib.gtr_gla_workspace_size.argtypes = [_int] * 8
_lib.gtr_gla_workspace_size.restype = _sz
_lib.gtr_gla_status.argtypes = [_vp]
_lib.gtr_gla_status.restype = _int
_lib.gtr_gla_strerror.argtypes = [_int]
_lib.gtr_gla_strerror.restype = ctypes.c_char_p
_lib.gtr_gla_release.argtypes = []
_lib.gtr_gla_release.restype = None
_lib.gtr_gla_launch_count.argtypes = []
_lib.gtr_gla_launch_count.restype = ctypes.c_ulonglong

# enums of include/gtr_gla.h
L2R, R2L, T2B, B2T = 0, 1, 2, 3
F16, BF16, F32 = 0, 1, 2
_DTYPE_CODE = {torch.float16: F16, torch.bfloat16: BF16, torch.float32: F32}


class GlaError(RuntimeError):
    def __init__(self, code: int):
        self.code = code
        super().__init__(f"gtr_gla error {code}: {gtr_gla_strerror(code)}")


def gtr_gla_strerror(code: int) -> str:
    return _lib.gtr_gla_strerror(int(code)).decode()


def gtr_gla_launch_count() -> int:
    return int(_lib.gtr_gla_launch_count())


def gtr_gla_release() -> None:
    _lib.gtr_gla_release()


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def gtr_gla_status(stream=None) -> int:
    return int(_lib.gtr_gla_status(_vp(_stream_handle(stream))))


def gtr_gla_workspace_size(B, H, grid_h, grid_w, d_k, d_v, dtype=F16, chunk=64) -> int:
    return int(_lib.gtr_gla_workspace_size(B, H, grid_h, grid_w, d_k, d_v, dtype, chunk))


def _ptr(t):
    return None if t is None else _vp(t.data_ptr())


def _shape(q, v):
    if q.dim() != 5 or v.dim() != 5:
        raise ValueError("q and v must be 5-D [B,H,grid_h,grid_w,d]")
    B, H, gh, gw, dk = q.shape
    return B, H, gh, gw, dk, v.shape[-1]


def _check(name, t, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} (got {t.dtype})")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != "cuda" or t.device != device:
        raise ValueError(f"{name} must be on the CUDA device of q (got {t.device})")


def _validate(q, k, v, log_alpha, out, final_state):
    """Host-side checks before any call: the library reads and writes the
    tensors through raw pointers, so a wrong shape, dtype, layout or device
    would make it touch memory outside them."""
    B, H, gh, gw, dk, dv = _shape(q, v)
    dev = q.device
    _check("q", q, (B, H, gh, gw, dk), q.dtype, dev)
    _check("k", k, (B, H, gh, gw, dk), q.dtype, dev)
    _check("v", v, (B, H, gh, gw, dv), q.dtype, dev)
    _check("log_alpha", log_alpha, (B, H, gh, gw, dk), torch.float32, dev)
    if out is not None:
        _check("out", out, (B, H, gh, gw, dv), q.dtype, dev)
    if final_state is not None:
        _check("final_state", final_state, (B, H, dk, dv), torch.float32, dev)


def _alloc_out(q, v, out, final_state, want_state):
    B, H, gh, gw, dk, dv = _shape(q, v)
    if out is None:
        out = torch.empty((B, H, gh, gw, dv), dtype=v.dtype, device=v.device)
    if final_state is None and want_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=v.device)
    return out, final_state


def gtr_gla_fwd(q, k, v, log_alpha, direction, out=None, final_state=None,
                want_state=True, stream=None):
    """fp16 forward, chunk 64, library-owned workspace.  Returns (out, final_state)."""
    if q.dtype != torch.float16 or k.dtype != torch.float16 or v.dtype != torch.float16:
        raise ValueError("gtr_gla_fwd takes fp16 q, k, v (use gtr_gla_fwd_ex for others)")
    _validate(q, k, v, log_alpha, out, final_state)
    out, final_state = _alloc_out(q, v, out, final_state, want_state)
    B, H, gh, gw, dk, dv = _shape(q, v)
    rc = _lib.gtr_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(out),
                          _ptr(final_state), B, H, gh, gw, dk, dv, int(direction),
                          _vp(_stream_handle(stream)))
    if rc != 0:
        raise GlaError(rc)
    return out, final_state


def gtr_gla_fwd_ex(q, k, v, log_alpha, direction, chunk=64, workspace=None, out=None,
                   final_state=None, want_state=True, stream=None):
    """Forward with the dtype taken from q and a caller workspace (allocated here
    as a zero-filled uint8 CUDA tensor if not given).  Returns (out, final_state)."""
    _validate(q, k, v, log_alpha, out, final_state)
    out, final_state = _alloc_out(q, v, out, final_state, want_state)
    B, H, gh, gw, dk, dv = _shape(q, v)
    dtype = _DTYPE_CODE.get(q.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    need = gtr_gla_workspace_size(B, H, gh, gw, dk, dv, dtype, chunk)
    if workspace is not None and (workspace.device != q.device or not workspace.is_contiguous()):
        raise ValueError("workspace must be a contiguous tensor on q's device")
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = _lib.gtr_gla_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(out),
                             _ptr(final_state), B, H, gh, gw, dk, dv, int(direction),
                             dtype, int(chunk), _ptr(workspace), ws_bytes,
                             _vp(_stream_handle(stream)))
    if rc != 0:
        raise GlaError(rc)
    return out, final_state


def gtr_gla_fwd_noalloc(q, k, v, log_alpha, direction, out, final_state=None, stream=None):
    """fp16 forward that allocates nothing: the caller passes ``out`` (and
    optionally ``final_state``); the scratch is the library's fixed device
    array.  Returns (out, final_state)."""
    if q.dtype != torch.float16 or k.dtype != torch.float16 or v.dtype != torch.float16:
        raise ValueError("gtr_gla_fwd_noalloc takes fp16 q, k, v")
    if out is None:
        raise ValueError("gtr_gla_fwd_noalloc needs a caller-given out")
    _validate(q, k, v, log_alpha, out, final_state)
    B, H, gh, gw, dk, dv = _shape(q, v)
    rc = _lib.gtr_gla_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(out),
                                  _ptr(final_state), B, H, gh, gw, dk, dv, int(direction),
                                  _vp(_stream_handle(stream)))
    if rc != 0:
        raise GlaError(rc)
    return out, final_state


def gtr_gla_tail_workspace_size(B, H, grid_h, grid_w, d_k, d_v, dtype=F16) -> int:
    return int(_lib.gtr_gla_tail_workspace_size(B, H, grid_h, grid_w, d_k, d_v, dtype))


def gtr_gla_fwd_tail(q, k, v, log_alpha, z, w_n, direction, eps=1e-5, y=None, final_state=None,
                     want_state=True, workspace=None, stream=None):
    """Forward pass with the output tail fused into its stores: y [B, grid_h,
    grid_w, H*d_v] = RMSNorm_head(o) * w_n * SiLU(z), fp16 or bf16 (dtype of q).
    A workspace is allocated (zero-filled) if not given.  Returns (y, final_state)."""
    _validate(q, k, v, log_alpha, None, final_state)
    B, H, gh, gw, dk, dv = _shape(q, v)
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("gtr_gla_fwd_tail takes fp16 or bf16 q, k, v")
    dev = q.device
    _check("z", z, (B, gh, gw, H * dv), q.dtype, dev)
    _check("w_n", w_n, (H, dv), torch.float32, dev)
    if y is None:
        y = torch.empty((B, gh, gw, H * dv), dtype=q.dtype, device=dev)
    _check("y", y, (B, gh, gw, H * dv), q.dtype, dev)
    if final_state is None and want_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    dtype = _DTYPE_CODE[q.dtype]
    need = gtr_gla_tail_workspace_size(B, H, gh, gw, dk, dv, dtype)
    if workspace is None:
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=dev)
    _check("workspace", workspace, (workspace.numel(),), torch.uint8, dev)
    rc = _lib.gtr_gla_fwd_tail(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(z), _ptr(w_n),
                               float(eps), _ptr(y), _ptr(final_state), B, H, gh, gw, dk, dv,
                               int(direction), dtype, _ptr(workspace), workspace.numel(),
                               _vp(_stream_handle(stream)))
    if rc != 0:
        raise GlaError(rc)
    return y, final_state


_lib.gtr_gla_bwd.argtypes = [_vp] * 10 + [_int] * 8 + [_vp, _sz, _vp]
_lib.gtr_gla_bwd.restype = _int
_lib.gtr_gla_bwd_workspace_size.argtypes = [_int] * 6
_lib.gtr_gla_bwd_workspace_size.restype = _sz


def gtr_gla_bwd_workspace_size(B, H, grid_h, grid_w, d_k=64, d_v=64) -> int:
    return int(_lib.gtr_gla_bwd_workspace_size(B, H, grid_h, grid_w, d_k, d_v))


def gtr_gla_bwd(q, k, v, log_alpha, d_out, direction, d_final_state=None, workspace=None, stream=None):
    """Gradients (dq, dk, dv, dlog_alpha) of sum(d_out * out) + sum(d_final_state *
    final_state) for the forward pass with the same arguments; see
    ``include/gtr_gla_bwd.h``.  dq, dk, dv in q's dtype, dlog_alpha fp32."""
    _validate(q, k, v, log_alpha, d_out, d_final_state)
    B, H, gh, gw, dk_, dv_ = _shape(q, v)
    dtype = _DTYPE_CODE.get(q.dtype)
    if dtype is None:
        raise ValueError(f"unsupported dtype {q.dtype}")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dla = torch.empty_like(log_alpha)
    need = gtr_gla_bwd_workspace_size(B, H, gh, gw, dk_, dv_)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _check("workspace", workspace, (workspace.numel(),), torch.uint8, q.device)
    rc = _lib.gtr_gla_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(d_out), _ptr(d_final_state),
                          _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dla), B, H, gh, gw, dk_, dv_, int(direction), dtype,
                          _ptr(workspace), workspace.numel(), _vp(_stream_handle(stream)))
    if rc != 0:
        raise GlaError(rc)
    return dq, dk, dv, dla

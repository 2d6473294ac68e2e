"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA path.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, imports neither the oracle nor the CUDA binding, and is
the only code the two sides have in common.

Recipe (stands in for the GLA inputs of GTR's backbone at the 640x640
detection, 1024x1024 segmentation and 2048x2048 high-resolution patch grids,
stride-16 patch tokens; "GTR: Gated Token Recurrence for Efficient Dense
Prediction", x-techcon article, sections 架构 and 算子):

* one CPU ``torch.Generator`` seeded with ``seed``;
* draw order q, k, v, then the gate pre-activations, each ``randn`` in fp32;
* k is divided by sqrt(d_k) (no scale is applied inside the operator);
* gates: ``logsigmoid(x) / 16`` ("normal") or ``logsigmoid(x + 2)``
  ("stress": near-1 gates, long memory); every log-gate is finite and <= 0;
* q, k, v are then cast to the I/O dtype; log_alpha stays fp32.

Tensors come back on the CPU with layout [B, H, grid_h, grid_w, d].
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

DTYPES = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@dataclass(frozen=True)
class Shape:
    B: int
    H: int
    grid_h: int
    grid_w: int
    d_k: int
    d_v: int

    @property
    def tokens(self) -> int:
        return self.grid_h * self.grid_w


def make_inputs(shape: Shape, dtype: str = "f16", seed: int = 0, gates: str = "normal"):
    """Return (q, k, v, log_alpha) CPU tensors for ``shape``."""
    if dtype not in DTYPES:
        raise ValueError(f"dtype must be one of {sorted(DTYPES)}")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    s = shape
    qk_shape = (s.B, s.H, s.grid_h, s.grid_w, s.d_k)
    v_shape = (s.B, s.H, s.grid_h, s.grid_w, s.d_v)
    q = torch.randn(qk_shape, generator=g, dtype=torch.float32)
    k = torch.randn(qk_shape, generator=g, dtype=torch.float32)
    v = torch.randn(v_shape, generator=g, dtype=torch.float32)
    x = torch.randn(qk_shape, generator=g, dtype=torch.float32)
    k = k / math.sqrt(s.d_k)
    if gates == "normal":
        log_alpha = torch.nn.functional.logsigmoid(x) / 16.0
    elif gates == "stress":
        log_alpha = torch.nn.functional.logsigmoid(x + 2.0)
    else:
        raise ValueError("gates must be 'normal' or 'stress'")
    dt = DTYPES[dtype]
    return (q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(),
            log_alpha.contiguous())


def make_swiglu_inputs(B: int, grid_h: int, grid_w: int, C: int, F: int, dtype: str = "f16",
                       seed: int = 0):
    """Seeded synthetic input and weights of the Spatial SwiGLU block (no
    trained weights exist here).  One CPU generator; draw order x, w_gu, b_gu,
    w_dw, b_dw, w_down, b_down, each randn in fp32, then scaled: x ~ N(0, 1),
    linear maps ~ N(0, 1/fan_in), biases ~ 0.1 N(0, 1), depthwise taps
    ~ N(0, 1/9).  x, w_gu, w_down are cast to the I/O dtype (tensor-core
    operands); biases and depthwise taps stay fp32.  Layouts: x [B, grid_h,
    grid_w, C], w_gu [2F, C] (gate rows first), b_gu [2F], w_dw [F, 3, 3],
    b_dw [F], w_down [C, F], b_down [C]."""
    if dtype not in DTYPES or dtype == "f32":
        raise ValueError("dtype must be f16 or bf16")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))

    def rn(*shape):
        return torch.randn(shape, generator=g, dtype=torch.float32)

    x = rn(B, grid_h, grid_w, C)
    w_gu = rn(2 * F, C) / math.sqrt(C)
    b_gu = 0.1 * rn(2 * F)
    w_dw = rn(F, 3, 3) / 3.0
    b_dw = 0.1 * rn(F)
    w_down = rn(C, F) / math.sqrt(F)
    b_down = 0.1 * rn(C)
    dt = DTYPES[dtype]
    return (x.to(dt).contiguous(), w_gu.to(dt).contiguous(), b_gu.contiguous(),
            w_dw.contiguous(), b_dw.contiguous(), w_down.to(dt).contiguous(),
            b_down.contiguous())



def make_tail_inputs(B: int, H: int, grid_h: int, grid_w: int, d_v: int, dtype: str = "f16",
                     seed: int = 0, o_scale: float = 1.0):
    """Seeded synthetic inputs of the attention's output tail.  One CPU
    generator; draw order o, z, w, each randn in fp32: o ~ o_scale * N(0, 1)
    (the attention output, [B, H, grid_h, grid_w, d_v]), z ~ N(0, 1) (the
    output-gate projection, [B, grid_h, grid_w, H * d_v]), w ~ 1 + 0.1 N(0, 1)
    (per-head norm weights, [H, d_v], fp32).  o and z are cast to the I/O
    dtype."""
    if dtype not in DTYPES or dtype == "f32":
        raise ValueError("dtype must be f16 or bf16")
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))

    def rn(*shape):
        return torch.randn(shape, generator=g, dtype=torch.float32)

    o = o_scale * rn(B, H, grid_h, grid_w, d_v)
    z = rn(B, grid_h, grid_w, H * d_v)
    w = 1.0 + 0.1 * rn(H, d_v)
    dt = DTYPES[dtype]
    return o.to(dt).contiguous(), z.to(dt).contiguous(), w.contiguous()


def make_backbone_params(C: int, F: int, n_layers: int, dtype: str = "f16", seed: int = 0):
    """Seeded synthetic weights of n_layers backbone layers (no trained weights
    exist here).  One CPU generator; per layer, in this order, each randn in
    fp32 then scaled: ln1_w, ln1_b, w_q, w_k, w_v, w_a, b_a, w_z, w_n, w_o,
    ln2_w, ln2_b, then the Spatial SwiGLU weights as make_swiglu_inputs draws
    them (w_gu, b_gu, w_dw, b_dw, w_down, b_down).  LayerNorm weights
    1 + 0.1 N(0, 1) and biases 0.1 N(0, 1); linear maps N(0, 1/fan_in); gate
    bias b_a ~ N(0, 1); norm weights w_n ~ 1 + 0.1 N(0, 1).  The projection
    matrices are in the I/O dtype (tensor-core operands), the rest fp32.
    Shapes: see oracle/backbone.py."""
    if dtype not in DTYPES or dtype == "f32":
        raise ValueError("dtype must be f16 or bf16")
    if C % 64:
        raise ValueError("C must be a multiple of 64")
    H = C // 64
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    dt = DTYPES[dtype]

    def rn(*shape):
        return torch.randn(shape, generator=g, dtype=torch.float32)

    layers = []
    for _ in range(n_layers):
        p = {}
        p["ln1_w"] = 1.0 + 0.1 * rn(C)
        p["ln1_b"] = 0.1 * rn(C)
        for name in ("w_q", "w_k", "w_v", "w_a"):
            p[name] = (rn(H * 64, C) / math.sqrt(C)).to(dt)
        p["b_a"] = rn(H * 64)
        p["w_z"] = (rn(H * 64, C) / math.sqrt(C)).to(dt)
        p["w_n"] = 1.0 + 0.1 * rn(H, 64)
        p["w_o"] = (rn(C, H * 64) / math.sqrt(H * 64)).to(dt)
        p["ln2_w"] = 1.0 + 0.1 * rn(C)
        p["ln2_b"] = 0.1 * rn(C)
        p["w_gu"] = (rn(2 * F, C) / math.sqrt(C)).to(dt)
        p["b_gu"] = 0.1 * rn(2 * F)
        p["w_dw"] = rn(F, 3, 3) / 3.0
        p["b_dw"] = 0.1 * rn(F)
        p["w_down"] = (rn(C, F) / math.sqrt(F)).to(dt)
        p["b_down"] = 0.1 * rn(C)
        layers.append({k: v.contiguous() for k, v in p.items()})
    return layers

# The workloads named for this operator: (name, Shape, dtype, directions).
CONFIGS = {
    "tiny": (Shape(1, 2, 16, 16, 64, 64), "f32"),
    "640_b1": (Shape(1, 6, 40, 40, 64, 64), "f16"),
    "640_b8": (Shape(8, 12, 40, 40, 64, 64), "f16"),
    "1024_b1": (Shape(1, 12, 64, 64, 64, 64), "f16"),
    "1024_b4": (Shape(4, 12, 64, 64, 64, 64), "f16"),
    "16k_d64": (Shape(1, 12, 128, 128, 64, 64), "f16"),
    "16k_d128": (Shape(1, 12, 128, 128, 128, 128), "f16"),
}

"""fp64 CPU oracle for a GTR backbone layer and the direction-cycled stack.

TEST INFRASTRUCTURE ONLY: used by tests/ and the CPU legs of ``bench.py``; the
CUDA library never imports it.

Source: "GTR: Gated Token Recurrence for Efficient Dense Prediction"
(x-techcon article, section 架构).  The backbone turns the image into patch
tokens at stride 16 and runs 12 layers on the fixed grid.  Every layer has a
GLA token mixer for long-range context and a Spatial SwiGLU for neighbouring
patches.  The scan direction cycles over consecutive layers (left to right,
right to left, top to bottom, bottom to top; four layers per round), and each
layer restores the grid order after its scan.  The pages give no projections,
norms or residual layout.  The plainest reading, the pre-norm residual layer
of a vision transformer with the attention replaced, is used here:

    x1 = LayerNorm_1(x)
    q = x1 W_q^T,  k = x1 W_k^T / sqrt(d_k),  v = x1 W_v^T,
    log alpha = logsigmoid(x1 W_a^T + b_a) / tau,  z = x1 W_z^T  (heads of d = 64)
    o = GLA(q, k, v, log alpha, direction)         (oracle.forward)
    x = x + OutputTail(o, z, w_n) W_o^T            (oracle.output_tail)
    x = x + SpatialSwiGLU(LayerNorm_2(x))          (oracle.swiglu)

Here direction = layer index mod 4 (0 L->R, 1 R->L, 2 T->B, 3 B->T), tau = 16,
LayerNorm has eps 1e-6 with a weight and a bias, and the output tail has
eps 1e-5.  The patch embedding and the task head are not part of the stack.

Arrays (any float dtype, upcast to float64): x [B, grid_h, grid_w, C] with
C = H * 64.  Each layer's parameters are a dict: ln1_w, ln1_b, ln2_w, ln2_b [C];
w_q, w_k, w_v, w_a, w_z [H*64, C]; b_a [H*64]; w_n [H, 64]; w_o [C, H*64];
w_gu [2F, C]; b_gu [2F]; w_dw [F, 3, 3]; b_dw [F]; w_down [C, F]; b_down [C].
"""
from __future__ import annotations

import numpy as np

from . import output_tail as _tail
from . import swiglu as _swiglu
from .oracle import forward as _gla_forward

HEAD_DIM = 64
TAU = 16.0
LN_EPS = 1e-6
TAIL_EPS = 1e-5


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def layer_norm(x, w, b, eps: float = LN_EPS):
    """Normalise over the last axis (mean and biased variance), then w * . + b."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(w) + _f64(b)


def _heads(t, H):
    """[B, gh, gw, H*d] -> [B, H, gh, gw, d]."""
    B, gh, gw, HD = t.shape
    return np.ascontiguousarray(np.transpose(t.reshape(B, gh, gw, H, HD // H), (0, 3, 1, 2, 4)))


def _logsigmoid(a):
    # log(1 / (1 + e^{-a})) = -log(1 + e^{-a}), computed without overflow
    return -np.logaddexp(0.0, -a)


def layer_forward(x, p: dict, direction: int, parts: bool = False):
    """One layer (see the module docstring).  Returns the new x, or with
    parts=True a dict of the intermediate tensors as well."""
    x = _f64(x)
    P = {k: _f64(v) for k, v in p.items()}
    C = x.shape[-1]
    if C % HEAD_DIM:
        raise ValueError("C must be a multiple of 64")
    H = C // HEAD_DIM
    x1 = layer_norm(x, P["ln1_w"], P["ln1_b"])
    q = _heads(x1 @ P["w_q"].T, H)
    k = _heads(x1 @ P["w_k"].T, H) / np.sqrt(HEAD_DIM)
    v = _heads(x1 @ P["w_v"].T, H)
    la = _heads(_logsigmoid(x1 @ P["w_a"].T + P["b_a"]), H) / TAU
    z = x1 @ P["w_z"].T
    o, _ = _gla_forward(q, k, v, la, direction)
    t = _tail.forward(o, z, P["w_n"], TAIL_EPS)
    xm = x + t @ P["w_o"].T
    x2 = layer_norm(xm, P["ln2_w"], P["ln2_b"])
    y = xm + _swiglu.forward(x2, P["w_gu"], P["b_gu"], P["w_dw"], P["b_dw"], P["w_down"], P["b_down"])
    if parts:
        return y, {"x1": x1, "q": q, "k": k, "v": v, "log_alpha": la, "z": z, "o": o, "tail": t,
                   "x_mid": xm, "x2": x2}
    return y


def backbone_forward(x, layers):
    """The stack: layer l scans in direction l mod 4."""
    for l, p in enumerate(layers):
        x = layer_forward(x, p, l % 4)
    return x

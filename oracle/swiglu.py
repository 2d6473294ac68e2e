"""fp64 CPU oracle for GTR's Spatial SwiGLU block.

TEST INFRASTRUCTURE ONLY: used by tests/, by ``__graft_entry__.smoke()`` and by
the CPU legs of ``bench.py``; the CUDA library never imports it.

Source: "GTR: Gated Token Recurrence for Efficient Dense Prediction"
(x-techcon article, section 架构): the channel mixer of every GTR layer is a
SwiGLU whose value branch gets a 3 x 3 per-channel convolution, so that
neighbouring patches exchange information directly (this replaces a position
embedding).  The pages give no formula; the plainest reading, used here:

* gate and value: g = x W_g^T + b_g,  u = x W_u^T + b_u  (one linear map to 2F
  channels, rows 0..F-1 the gate, F..2F-1 the value);
* value branch: v = DWConv3x3(u) + b_dw, a per-channel 3 x 3 cross-correlation
  (the usual depthwise convolution), stride 1, zero padding of one patch
  around the grid:  v[y, x, f] = b_dw[f] + sum_{a, c in 0..2} w_dw[f, a, c] *
  u[y + a - 1, x + c - 1, f]  with u = 0 outside the grid;
* gated product with the Swish / SiLU gate: h = SiLU(g) * v,
  SiLU(z) = z / (1 + e^{-z});
* down projection: y = h W_d^T + b_d.

Arrays (any float dtype, upcast to float64): x [B, grid_h, grid_w, C];
w_gu [2F, C]; b_gu [2F]; w_dw [F, 3, 3]; b_dw [F]; w_down [C, F]; b_down [C].
Output y [B, grid_h, grid_w, C].
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def forward(x, w_gu, b_gu, w_dw, b_dw, w_down, b_down, parts: bool = False):
    """The block in fp64.  Returns y, or (g, u, v, h, y) with parts=True."""
    x, w_gu, b_gu, w_dw, b_dw, w_down, b_down = (
        _f64(a) for a in (x, w_gu, b_gu, w_dw, b_dw, w_down, b_down))
    if x.ndim != 4:
        raise ValueError("x must be [B, grid_h, grid_w, C]")
    B, gh, gw, C = x.shape
    F2 = w_gu.shape[0]
    if F2 % 2 or w_gu.shape != (F2, C) or b_gu.shape != (F2,):
        raise ValueError("w_gu must be [2F, C] and b_gu [2F]")
    F = F2 // 2
    if w_dw.shape != (F, 3, 3) or b_dw.shape != (F,):
        raise ValueError("w_dw must be [F, 3, 3] and b_dw [F]")
    if w_down.shape != (C, F) or b_down.shape != (C,):
        raise ValueError("w_down must be [C, F] and b_down [C]")
    gu = x @ w_gu.T + b_gu
    g, u = gu[..., :F], gu[..., F:]
    # the 3 x 3 cross-correlation as nine shifted, weighted copies of the
    # zero-padded value field
    up = np.zeros((B, gh + 2, gw + 2, F))
    up[:, 1:gh + 1, 1:gw + 1, :] = u
    v = np.broadcast_to(b_dw, u.shape).copy()
    for a in range(3):
        for c in range(3):
            v += w_dw[:, a, c] * up[:, a:a + gh, c:c + gw, :]
    h = g / (1.0 + np.exp(-g)) * v
    y = h @ w_down.T + b_down
    if parts:
        return g, u, v, h, y
    return y

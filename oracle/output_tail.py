"""fp64 CPU oracle for the output tail of GTR's GLA token mixer.

TEST INFRASTRUCTURE ONLY: used by tests/, by ``__graft_entry__.smoke()`` and by
the CPU legs of ``bench.py``; the CUDA library never imports it.

Source: "GTR: Gated Token Recurrence for Efficient Dense Prediction"
(x-techcon article, section 算子): the operator benchmark leaves out the
fusion of the operator's output tail, and the pages say no more about what
that tail is.  The plainest reading, the per-token epilogue that gated linear
attention layers put between the recurrence and the output projection, is
used here:

* per head h and token t, RMS normalisation of the head's output row
  o[t, h, :] (d_v values) with a learned per-channel weight w[h, :]:
  n = o / sqrt(mean_j o_j^2 + eps) * w;
* an output gate from a separate projection z of the layer input, applied
  with SiLU: n * SiLU(z), SiLU(z) = z / (1 + e^{-z});
* the heads merged channels-last, channel h * d_v + j of the token, the
  layout the output projection (and the channel mixer) read.

Arrays (any float dtype, upcast to float64): o [B, H, grid_h, grid_w, d_v]
(the attention's output layout), z [B, grid_h, grid_w, H * d_v], w [H, d_v].
Output y [B, grid_h, grid_w, H * d_v].
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().double().numpy()
    return np.asarray(a, dtype=np.float64)


def forward(o, z, w, eps: float = 1e-5):
    """The output tail in fp64 (see the module docstring)."""
    o, z, w = _f64(o), _f64(z), _f64(w)
    if o.ndim != 5:
        raise ValueError("o must be [B, H, grid_h, grid_w, d_v]")
    B, H, gh, gw, dv = o.shape
    if z.shape != (B, gh, gw, H * dv):
        raise ValueError("z must be [B, grid_h, grid_w, H * d_v]")
    if w.shape != (H, dv):
        raise ValueError("w must be [H, d_v]")
    # heads to the channel axis: [B, gh, gw, H, d_v]
    oh = np.transpose(o, (0, 2, 3, 1, 4))
    ms = np.mean(oh * oh, axis=-1, keepdims=True)
    n = oh / np.sqrt(ms + eps) * w
    zh = z.reshape(B, gh, gw, H, dv)
    y = n * (zh / (1.0 + np.exp(-zh)))
    return y.reshape(B, gh, gw, H * dv)

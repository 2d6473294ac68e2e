"""GPU parity of the forward pass with the output tail fused into its stores
(gtr_gla_fwd_tail, through the C ABI) against the fp64 oracles: the token
recurrence (oracle.forward) followed by the tail (oracle/output_tail.py).

Tolerances are the ones of the unfused tail (5e-3 of max|ref| for fp16 I/O,
1e-2 for bf16): the fused path takes the norm of the fp32 attention output,
so its only rounding of note is y's single rounding to the I/O dtype plus the
attention's own error (<= 5e-3 of max|o|, the parity bound), which the norm
carries over as a relative error of the same size.  final_state is held to
the attention's own bound.
"""
import numpy as np
import pytest
import torch

import oracle
import oracle.output_tail as otail
from recurrent_vision_backbone_chunkwise_b200.inputs import Shape, make_inputs, make_tail_inputs

pytestmark = pytest.mark.gpu

TOL = {"f16": 5e-3, "bf16": 1e-2}


def rel(a, ref):
    a = a.double().cpu().numpy() if hasattr(a, "cpu") else a
    return float(np.max(np.abs(a - ref)) / np.max(np.abs(ref)))


def run(shape, dtype, direction, seed=0, eps=1e-5):
    from recurrent_vision_backbone_chunkwise_b200 import gla

    q, k, v, la = make_inputs(shape, dtype, seed)
    _, z, w = make_tail_inputs(shape.B, shape.H, shape.grid_h, shape.grid_w, shape.d_v, dtype, seed + 1)
    y, fs = gla.gtr_gla_fwd_tail(*(t.cuda() for t in (q, k, v, la, z, w)), direction, eps=eps)
    assert gla.gtr_gla_status() == 0
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.forward(q, k, v, la, direction)
    y_ref = otail.forward(o_ref, z, w, eps)
    return y, fs, y_ref, s_ref


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_640_b1_matches_oracle(direction):
    y, fs, y_ref, s_ref = run(Shape(1, 6, 40, 40, 64, 64), "f16", direction)
    assert torch.isfinite(y).all()
    assert rel(y, y_ref) <= TOL["f16"]
    assert rel(fs, s_ref) <= TOL["f16"]


@pytest.mark.parametrize("shape,dtype,direction", [
    (Shape(2, 3, 7, 37, 64, 64), "f16", 2),    # column scan through four-row gathers, ragged tail
    (Shape(2, 3, 7, 37, 64, 64), "f16", 1),    # reversed row scan, ragged tail at raster start
    (Shape(1, 2, 1, 1, 64, 64), "f16", 0),     # one token
    (Shape(3, 4, 24, 24, 64, 64), "bf16", 3),
    (Shape(1, 2, 12, 20, 128, 128), "f16", 0),  # head size 128: attention, then the tail kernel
    (Shape(1, 2, 12, 20, 128, 128), "bf16", 3),
])
def test_edge_cases_match_oracle(shape, dtype, direction):
    y, fs, y_ref, s_ref = run(shape, dtype, direction, seed=4)
    assert rel(y, y_ref) <= TOL[dtype]
    assert rel(fs, s_ref) <= TOL[dtype]


def test_many_segments_and_eps():
    """1024x1024 grid, batch 4: several segments per head, and eps = 1."""
    y, fs, y_ref, s_ref = run(Shape(4, 12, 64, 64, 64, 64), "f16", 2, seed=2, eps=1.0)
    assert rel(y, y_ref) <= TOL["f16"]
    assert rel(fs, s_ref) <= TOL["f16"]


def test_fused_equals_attention_then_tail():
    """The fused stores agree with the two-step path (attention output in fp16,
    then the tail kernel) to within the fp16 rounding of o that the fused path
    skips."""
    from recurrent_vision_backbone_chunkwise_b200 import gla, output_tail

    shape = Shape(1, 6, 40, 40, 64, 64)
    q, k, v, la = (t.cuda() for t in make_inputs(shape, "f16", 7))
    _, z, w = (t.cuda() for t in make_tail_inputs(1, 6, 40, 40, 64, "f16", 8))
    y, _ = gla.gtr_gla_fwd_tail(q, k, v, la, z, w, 0)
    o, _ = gla.gtr_gla_fwd_ex(q, k, v, la, 0)
    y2 = output_tail.gtr_output_tail_fwd(o, z, w, 1e-5)
    torch.cuda.synchronize()
    d = (y.float() - y2.float()).abs().max() / y2.float().abs().max()
    assert float(d) <= 4e-3


def test_binding_rejects_wrong_gate_shape():
    from recurrent_vision_backbone_chunkwise_b200 import gla

    shape = Shape(1, 2, 4, 4, 64, 64)
    q, k, v, la = (t.cuda() for t in make_inputs(shape, "f16", 0))
    z = torch.zeros(1, 4, 4, 64, dtype=torch.float16, device="cuda")  # H*d_v would be 128
    w = torch.ones(2, 64, device="cuda")
    with pytest.raises(ValueError):
        gla.gtr_gla_fwd_tail(q, k, v, la, z, w, 0)

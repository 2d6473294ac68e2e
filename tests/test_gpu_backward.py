"""GPU parity of the backward pass (gtr_gla_bwd, through the C ABI) against
the fp64 oracle (oracle/backward.py: reverse mode through the token
recurrence, itself pinned by finite differences of the forward oracle).

Tolerances per gradient tensor, max|err| / max|ref|: 1e-4 with fp32 I/O
(fp32 arithmetic; the dlog_alpha suffix sums over a few thousand tokens lose
well under that), 5e-3 with fp16 I/O (dq, dk, dv are rounded once to fp16, a
relative error of 2^-11 of an element; dlog_alpha stays fp32 and is taken from
the unrounded gradients), 1e-2 with bf16 (rounding 2^-8)."""
import numpy as np
import pytest
import torch

import oracle.backward as ob
from recurrent_vision_backbone_chunkwise_b200.inputs import Shape, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "f16": 5e-3, "bf16": 1e-2}
TDT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def rel(a, ref):
    a = a.double().cpu().numpy()
    return float(np.max(np.abs(a - ref)) / np.max(np.abs(ref)))


def run(shape, dtype, direction, with_final, seed=0):
    from recurrent_vision_backbone_chunkwise_b200 import gla

    q, k, v, la = make_inputs(shape, dtype, seed)
    g = torch.Generator().manual_seed(seed + 100)
    dO = torch.randn(v.shape, generator=g).to(TDT[dtype])
    dSf = torch.randn(shape.B, shape.H, shape.d_k, shape.d_v, generator=g) if with_final else None
    dev = [t.cuda() if t is not None else None for t in (q, k, v, la, dO, dSf)]
    got = gla.gtr_gla_bwd(*dev[:5], direction, d_final_state=dev[5])
    assert gla.gtr_gla_status() == 0
    ref = ob.backward(q, k, v, la, dO, direction, d_final_state=dSf)
    for name, a, r in zip(("dq", "dk", "dv", "dlog_alpha"), got, ref):
        assert torch.isfinite(a).all(), name
        if np.max(np.abs(r)) == 0.0:
            # an exactly zero gradient (the first token's gate multiplies the
            # zero initial state): held against the size of the products
            # q . dq and k . dk whose difference it is
            scale = max(np.max(np.abs(ref[0])) * float(q.abs().max()), np.max(np.abs(ref[1])) * float(k.abs().max()))
            e = float(a.abs().max()) / scale
        else:
            e = rel(a, r)
        assert e <= TOL[dtype], f"{name}: {e:.3e}"


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_backward_matches_oracle(direction, dtype):
    run(Shape(1, 2, 12, 20, 64, 64), dtype, direction, with_final=direction % 2 == 0, seed=direction)


@pytest.mark.parametrize("shape,dtype,direction", [
    (Shape(2, 3, 7, 37, 64, 64), "f16", 2),   # ragged last chunk in column order
    (Shape(1, 1, 1, 1, 64, 64), "f32", 1),    # one token
    (Shape(1, 6, 40, 40, 64, 64), "f16", 3),  # the 640x640 detection grid
    (Shape(1, 2, 16, 16, 64, 64), "bf16", 0),
    (Shape(4, 12, 24, 24, 64, 64), "f16", 1),  # 432 chunk CTAs: the 256-thread chunk kernels
])
def test_backward_edge_cases(shape, dtype, direction):
    run(shape, dtype, direction, with_final=True, seed=7)


def test_backward_rejects_head_size_128():
    from recurrent_vision_backbone_chunkwise_b200 import gla

    x = torch.zeros(1, 1, 4, 4, 128, dtype=torch.float16, device="cuda")
    la = torch.zeros(1, 1, 4, 4, 128, device="cuda")
    with pytest.raises(gla.GlaError) as e:
        gla.gtr_gla_bwd(x, x.clone(), x.clone(), la, x.clone(), 0)
    assert e.value.code == -3

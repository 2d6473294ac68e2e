"""GPU parity of the token mixer's output tail against the fp64 oracle
(oracle/output_tail.py), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle.output_tail as otail
from recurrent_vision_backbone_chunkwise_b200.inputs import make_tail_inputs

pytestmark = pytest.mark.gpu

TOL = {"f16": 5e-3, "bf16": 1e-2}


def rel(y, ref):
    y = y.double().cpu().numpy()
    return np.max(np.abs(y - ref)) / np.max(np.abs(ref))


def run(B, H, gh, gw, dv, dtype, eps=1e-5, seed=0, o_scale=1.0):
    from recurrent_vision_backbone_chunkwise_b200 import gla, output_tail

    o, z, w = make_tail_inputs(B, H, gh, gw, dv, dtype, seed, o_scale)
    y = output_tail.gtr_output_tail_fwd(o.cuda(), z.cuda(), w.cuda(), eps)
    assert gla.gtr_gla_status() == 0
    torch.cuda.synchronize()
    return y, otail.forward(o, z, w, eps)


@pytest.mark.parametrize("shape", [
    (1, 6, 40, 40, 64),     # 640x640 detection grid, 6 heads
    (2, 3, 5, 7, 64),       # ragged: the last warp only partly in range
    (1, 1, 1, 1, 128),      # one token, head size 128
    (1, 4, 16, 16, 128),
    (4, 12, 64, 64, 64),    # 1024x1024 grid, batch 4: more warps than the grid holds (grid-stride)
])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_tail_matches_oracle(shape, dtype):
    y, ref = run(*shape, dtype)
    assert torch.isfinite(y).all()
    e = rel(y, ref)
    assert e <= TOL[dtype], f"err {e:.3e} > {TOL[dtype]}"


@pytest.mark.parametrize("eps", [0.0, 1e-5, 1e-2])
def test_tail_eps_on_small_outputs(eps):
    """Head outputs of about 1e-3 (mean square 1e-6), where eps = 1e-5 and
    1e-2 dominate the norm and eps = 0 does not."""
    y, ref = run(2, 3, 6, 9, 64, "f16", eps=eps, seed=3, o_scale=1e-3)
    assert rel(y, ref) <= TOL["f16"]


def test_tail_zero_rows_give_zero():
    from recurrent_vision_backbone_chunkwise_b200 import output_tail

    o, z, w = make_tail_inputs(1, 2, 3, 4, 64, "f16", 5)
    o[:, 1] = 0
    y = output_tail.gtr_output_tail_fwd(o.cuda(), z.cuda(), w.cuda(), 1e-5).cpu()
    assert torch.all(y[..., 64:] == 0)
    assert torch.isfinite(y).all()


def test_tail_deterministic():
    from recurrent_vision_backbone_chunkwise_b200 import output_tail

    o, z, w = (t.cuda() for t in make_tail_inputs(2, 5, 7, 11, 64, "bf16", 9))
    a = output_tail.gtr_output_tail_fwd(o, z, w).clone()
    b = output_tail.gtr_output_tail_fwd(o, z, w)
    assert torch.equal(a, b)

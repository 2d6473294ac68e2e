"""GPU parity of the Spatial SwiGLU block (through the C ABI) against the fp64
oracle (oracle/swiglu.py) on the same seeded inputs and weights.

Metric: max|gpu - ref| / max|ref| over the whole output.  Bounds: 5e-3 for
fp16 I/O, 1e-2 for bf16 (the projected gate/value and the gated product are
stored in the I/O dtype between the three steps: three roundings of 2^-11,
resp. 2^-8, relative, under fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle.swiglu as osw
from recurrent_vision_backbone_chunkwise_b200.inputs import make_swiglu_inputs

pytestmark = pytest.mark.gpu

TOL = {"f16": 5e-3, "bf16": 1e-2}


def rel(got, ref):
    got = got.detach().cpu().double().numpy()
    d = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (d if d > 0 else 1.0)


def run(B, gh, gw, C, F, dtype, seed=0):
    from recurrent_vision_backbone_chunkwise_b200 import gla, swiglu

    ins = make_swiglu_inputs(B, gh, gw, C, F, dtype, seed)
    y = swiglu.gtr_swiglu_fwd(*(t.cuda() for t in ins))
    assert gla.gtr_gla_status() == 0
    torch.cuda.synchronize()
    return y, osw.forward(*ins)


@pytest.mark.parametrize("shape", [
    (1, 40, 40, 384, 1536),   # 640x640 detection grid, 6 heads of 64, hidden 4C
    (1, 5, 7, 16, 32),        # ragged: a partial channel block, rows shorter than a block
    (1, 1, 1, 8, 8),          # one token: only the centre tap
    (2, 16, 20, 64, 256),
    (1, 3, 64, 24, 72),       # a wide grid of three rows
    (1, 9, 1, 16, 64),        # a single column
    (2, 1024, 1040, 8, 8),    # more token tiles than one grid dimension holds
    (1, 4, 5, 8, 38400),      # more channel blocks than SMs: one launch per group of blocks
])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_swiglu_matches_oracle(shape, dtype):
    y, ref = run(*shape, dtype)
    assert torch.isfinite(y).all()
    e = rel(y, ref)
    assert e <= TOL[dtype], f"err {e:.3e} > {TOL[dtype]}"


def test_swiglu_1024_grid_batch4():
    """1024x1024 segmentation grid, batch 4, 12 heads of 64 (C = 768)."""
    y, ref = run(4, 64, 64, 768, 3072, "f16", seed=3)
    assert rel(y, ref) <= TOL["f16"]


def test_swiglu_deterministic():
    from recurrent_vision_backbone_chunkwise_b200 import swiglu

    ins = [t.cuda() for t in make_swiglu_inputs(1, 12, 9, 64, 128, "f16", 7)]
    a = swiglu.gtr_swiglu_fwd(*ins).clone()
    b = swiglu.gtr_swiglu_fwd(*ins)
    assert torch.equal(a, b)

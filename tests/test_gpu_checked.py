"""The bounds-checked build (libgtr_gla_checked.so, -DGTR_CHECKED) on tiny,
ragged and many-segment shapes: every computed global index and TMA
coordinate of the kernels is tested before use, a failed test is latched as
GTR_GLA_ERR_BOUNDS.  Each case must report status 0 (no failed check, no
timed-out wait) and match the fp64 oracle at the parity bounds.  This is the
project's stand-in for a memory checker (compute-sanitizer is closed on this
pool).  The library is loaded through its own ctypes handle, next to the
normal one: each keeps its own kernels and error word."""
import ctypes
import os

import numpy as np
import pytest
import torch

import oracle
from recurrent_vision_backbone_chunkwise_b200.inputs import Shape, make_inputs, make_tail_inputs

pytestmark = pytest.mark.gpu

TOL = {"f16": 5e-3, "bf16": 1e-2, "f32": 1e-4}  # the parity suite's bounds
CODE = {"f16": 0, "bf16": 1, "f32": 2}
vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t


@pytest.fixture(scope="module")
def lib():
    from recurrent_vision_backbone_chunkwise_b200 import build

    path = build.build(checked=True)
    assert os.path.basename(path) == "libgtr_gla_checked.so"
    L = ctypes.CDLL(path)
    L.gtr_gla_fwd_ex.argtypes = [vp] * 6 + [i32] * 9 + [vp, sz, vp]
    L.gtr_gla_fwd_tail.argtypes = [vp] * 6 + [ctypes.c_float] + [vp] * 2 + [i32] * 8 + [vp, sz, vp]
    L.gtr_gla_workspace_size.argtypes = [i32] * 8
    L.gtr_gla_workspace_size.restype = sz
    L.gtr_gla_tail_workspace_size.argtypes = [i32] * 7
    L.gtr_gla_tail_workspace_size.restype = sz
    L.gtr_gla_status.argtypes = [vp]
    return L


def rel(a, ref):
    a = a.double().cpu().numpy()
    return float(np.max(np.abs(a - ref)) / np.max(np.abs(ref)))


def p(t):
    return vp(t.data_ptr())


def run(lib, shape, dtype, direction, chunk=64, seed=0):
    q, k, v, la = make_inputs(shape, dtype, seed)
    qd, kd, vd, lad = (t.cuda() for t in (q, k, v, la))
    out = torch.full_like(vd, float("nan"))
    fs = torch.empty((shape.B, shape.H, shape.d_k, shape.d_v), device="cuda")
    need = lib.gtr_gla_workspace_size(shape.B, shape.H, shape.grid_h, shape.grid_w, shape.d_k, shape.d_v,
                                      CODE[dtype], chunk)
    ws = torch.zeros(max(need, 1), dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = lib.gtr_gla_fwd_ex(p(qd), p(kd), p(vd), p(lad), p(out), p(fs), shape.B, shape.H, shape.grid_h,
                            shape.grid_w, shape.d_k, shape.d_v, direction, CODE[dtype], chunk, p(ws), need,
                            vp(st))
    assert rc == 0
    assert lib.gtr_gla_status(vp(st)) == 0  # no index check failed, no wait gave up
    o_ref, s_ref = oracle.forward(q, k, v, la, direction)
    assert rel(out, o_ref) <= TOL[dtype]
    assert rel(fs, s_ref) <= TOL[dtype]


@pytest.mark.parametrize("grid", [(1, 1), (1, 77), (77, 1), (3, 200), (130, 2), (7, 37), (40, 40), (8, 24)])
@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_fused_edge_grids(lib, grid, direction):
    run(lib, Shape(1, 2, grid[0], grid[1], 64, 64), "f16", direction, seed=grid[0] + direction)


@pytest.mark.parametrize("shape,dtype,direction", [
    (Shape(8, 12, 12, 40, 64, 64), "f16", 1),   # many planes: several waves, per-segment folds
    (Shape(1, 6, 40, 40, 64, 64), "f16", 2),    # one wave of one-chunk segments: the transposed scan
    (Shape(1, 12, 64, 64, 64, 64), "bf16", 3),
    (Shape(1, 2, 20, 24, 128, 128), "f16", 0),  # head size 128 in four parts
    (Shape(1, 2, 20, 24, 64, 128), "f16", 3),
    (Shape(3, 16, 24, 40, 64, 64), "f16", 0),   # 48 planes x 3 segments of uneven length
    (Shape(3, 16, 24, 40, 64, 64), "bf16", 3),
])
def test_fused_plans_and_head_sizes(lib, shape, dtype, direction):
    run(lib, shape, dtype, direction, seed=9)


@pytest.mark.parametrize("chunk,dtype,direction", [(32, "f16", 2), (128, "f16", 1), (64, "f32", 3)])
def test_generic_path(lib, chunk, dtype, direction):
    run(lib, Shape(1, 2, 9, 21, 64, 64), dtype, direction, chunk=chunk, seed=5)


@pytest.mark.parametrize("direction", [0, 3])
def test_fused_tail(lib, direction):
    import oracle.output_tail as otail

    shape = Shape(2, 3, 7, 37, 64, 64)
    q, k, v, la = make_inputs(shape, "f16", 1)
    _, z, w = make_tail_inputs(2, 3, 7, 37, 64, "f16", 2)
    qd, kd, vd, lad, zd, wd = (t.cuda() for t in (q, k, v, la, z, w))
    y = torch.full_like(zd, float("nan"))
    need = lib.gtr_gla_tail_workspace_size(2, 3, 7, 37, 64, 64, 0)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    rc = lib.gtr_gla_fwd_tail(p(qd), p(kd), p(vd), p(lad), p(zd), p(wd), 1e-5, p(y), None, 2, 3, 7, 37, 64, 64,
                              direction, 0, p(ws), need, vp(st))
    assert rc == 0
    assert lib.gtr_gla_status(vp(st)) == 0
    o_ref, _ = oracle.forward(q, k, v, la, direction)
    assert rel(y, otail.forward(o_ref, z, w, 1e-5)) <= 5e-3


def _random_cases(n=24, seed=2024):
    import random

    rng = random.Random(seed)
    cases = []
    for _ in range(n):
        d_k, d_v = rng.choice([(64, 64), (64, 64), (64, 64), (128, 128), (64, 128), (128, 64)])
        dtype = rng.choice(["f16", "f16", "bf16"])
        chunk = 64 if rng.random() < 0.8 else rng.choice([32, 128 if d_k == 64 else 32])
        if chunk != 64:
            dtype = rng.choice(["f16", "f32"])
        cases.append((Shape(rng.randint(1, 4), rng.randint(1, 16), rng.randint(1, 48), rng.randint(1, 48), d_k, d_v),
                      dtype, rng.randint(0, 3), chunk))
    return cases


@pytest.mark.parametrize("shape,dtype,direction,chunk", _random_cases())
def test_random_shapes(lib, shape, dtype, direction, chunk):
    """Seeded random batches, head counts, grids, head sizes, directions,
    dtypes and chunk lengths: the plan's segment counts and lengths, the
    cooperative and folding boundary paths and both places of the leftover
    chunks all come up; every index check passes and the result matches."""
    run(lib, shape, dtype, direction, chunk=chunk, seed=shape.B * 7 + shape.grid_h)

"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Metric: err = max|gpu - ref| / max|ref| over a whole output tensor (and,
separately, over the final state) of one (config, direction, dtype) run.
Bounds: 5e-3 for fp16 I/O and 1e-4 for fp32 I/O (the stated tolerances),
1e-2 for bf16 I/O (bf16 output rounding alone is up to 2^-9 ~ 2e-3 of an
element, and the tensor-core operands are rounded to bf16 as well).
Inputs are the seeded synthetic ones; the oracle sees the dtype-rounded
values upcast to fp64.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS, Shape, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f16": 5e-3, "bf16": 1e-2, "f32": 1e-4}


@functools.lru_cache(maxsize=None)
def gla():
    from recurrent_vision_backbone_chunkwise_b200 import gla as g

    return g


def rel(got, ref):
    got = got.detach().cpu().double().numpy() if hasattr(got, "detach") else got
    d = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (d if d > 0 else 1.0)


@functools.lru_cache(maxsize=8)
def case(shape: Shape, dtype: str, seed: int, gates: str):
    return make_inputs(shape, dtype, seed, gates)


@functools.lru_cache(maxsize=16)
def reference(shape: Shape, dtype: str, seed: int, gates: str, direction: int):
    q, k, v, la = case(shape, dtype, seed, gates)
    return oracle.forward(q, k, v, la, direction)


def run_gpu(shape, dtype, seed, gates, direction, chunk=64, api="ex"):
    q, k, v, la = (t.cuda() for t in case(shape, dtype, seed, gates))
    g = gla()
    if api == "fwd":
        out, fs = g.gtr_gla_fwd(q, k, v, la, direction)
    else:
        out, fs = g.gtr_gla_fwd_ex(q, k, v, la, direction, chunk=chunk)
    assert g.gtr_gla_status() == 0
    torch.cuda.synchronize()
    return out, fs


def check(shape, dtype, direction, chunk=64, seed=0, gates="normal", api="ex"):
    out, fs = run_gpu(shape, dtype, seed, gates, direction, chunk, api)
    ref_o, ref_fs = reference(shape, dtype, seed, gates, direction)
    assert torch.isfinite(out).all()
    e_o, e_s = rel(out, ref_o), rel(fs, ref_fs)
    assert e_o <= TOL[dtype], f"out err {e_o:.3e} > {TOL[dtype]}"
    assert e_s <= TOL[dtype], f"final_state err {e_s:.3e} > {TOL[dtype]}"
    return e_o, e_s


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_tiny_fp32(direction):
    shape, dtype = CONFIGS["tiny"]
    check(shape, dtype, direction)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_640_b1_fp16_default_entry_point(direction):
    shape, dtype = CONFIGS["640_b1"]
    check(shape, dtype, direction, api="fwd")


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("cfg", ["640_b8", "1024_b1", "1024_b4", "16k_d64", "16k_d128"])
def test_configs_fp16(cfg, direction):
    shape, dtype = CONFIGS[cfg]
    check(shape, dtype, direction)


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_1024_b4_stress_gates(direction):
    shape, dtype = CONFIGS["1024_b4"]
    check(shape, dtype, direction, gates="stress")


@pytest.mark.parametrize("chunk", [32, 64, 128])
@pytest.mark.parametrize("direction", [0, 3])
def test_chunk_sweep_16k(chunk, direction):
    shape, dtype = CONFIGS["16k_d64"]
    check(shape, dtype, direction, chunk=chunk)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("direction", [1, 2])
def test_other_dtypes_640(dtype, direction):
    shape, _ = CONFIGS["640_b1"]
    check(shape, dtype, direction)


@pytest.mark.parametrize("dims", [(64, 128), (128, 64)])
def test_rectangular_head_dims(dims):
    shape = Shape(2, 3, 24, 40, dims[0], dims[1])
    for direction in range(4):
        check(shape, "f16", direction, seed=5)


@pytest.mark.parametrize("grid", [(1, 1), (1, 77), (77, 1), (5, 13), (7, 9), (3, 200), (130, 2)])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_edge_grids(grid, dtype):
    """Single token, single row/column, N < chunk, ragged tails in scan order."""
    shape = Shape(2, 2, grid[0], grid[1], 64, 64)
    for direction in range(4):
        check(shape, dtype, direction, seed=9)


def test_memoryless_gates_match():
    """log_alpha = -80 everywhere: the factors e^{-b} would overflow any
    factorised form; the path must still give o_t = (q_t.k_t) v_t."""
    shape = Shape(1, 2, 16, 20, 64, 64)
    q, k, v, _ = make_inputs(shape, "f16", 3)
    la = torch.full(q.shape, -80.0)
    g = gla()
    out, fs = g.gtr_gla_fwd_ex(q.cuda(), k.cuda(), v.cuda(), la.cuda(), 2)
    ref_o, ref_fs = oracle.forward(q, k, v, la, 2)
    assert rel(out, ref_o) <= 5e-3
    assert rel(fs, ref_fs) <= 5e-3


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_gates_one_is_causal_linear_attention(dtype):
    """log_alpha = 0 everywhere (no decay, the longest memory): the output is
    plain causal linear attention tril(Q K^T) V and the final state K^T V,
    written out with numpy matmuls; 1600 tokens in 13 segments (fp16, fused
    path) or one CUDA-core scan (fp32)."""
    shape = Shape(1, 3, 40, 40, 64, 64)
    q, k, v, _ = make_inputs(shape, dtype, 5)
    la = torch.zeros(q.shape)
    g = gla()
    out, fs = g.gtr_gla_fwd_ex(q.cuda(), k.cuda(), v.cuda(), la.cuda(), 0)
    assert g.gtr_gla_status() == 0
    Q, K, V = (t.double().numpy().reshape(1, 3, 1600, 64) for t in (q, k, v))
    ref_o = np.einsum("bhts,bhsd->bhtd", np.tril(np.einsum("bhtd,bhsd->bhts", Q, K)), V)
    ref_s = np.einsum("bhti,bhtj->bhij", K, V)
    assert rel(out.reshape(1, 3, 1600, 64), ref_o) <= TOL[dtype]
    assert rel(fs, ref_s) <= TOL[dtype]


def test_deterministic():
    shape, dtype = CONFIGS["1024_b1"]
    a, sa = run_gpu(shape, dtype, 0, "normal", 2)
    b, sb = run_gpu(shape, dtype, 0, "normal", 2)
    assert torch.equal(a, b) and torch.equal(sa, sb)


def test_final_state_optional_and_out_untouched_elsewhere():
    """final_state may be NULL; the call writes exactly the output tensor: a
    guard region of NaN sentinels on either side of it (one buffer three
    times its size, the middle third passed through the C ABI) is bitwise
    unchanged afterwards."""
    import ctypes

    shape, dtype = CONFIGS["640_b1"]
    q, k, v, la = (t.cuda() for t in case(shape, dtype, 0, "normal"))
    g = gla()
    out, fs = g.gtr_gla_fwd(q, k, v, la, 1, want_state=False)
    assert fs is None
    ref_o, _ = reference(shape, dtype, 0, "normal", 1)
    assert rel(out, ref_o) <= TOL[dtype]
    n = v.numel()
    buf = torch.full((3 * n,), float("nan"), dtype=v.dtype, device="cuda")
    guard = buf.clone()
    vp = ctypes.c_void_p
    rc = g._lib.gtr_gla_fwd(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(la.data_ptr()),
                            vp(buf[n:2 * n].data_ptr()), None, shape.B, shape.H, shape.grid_h,
                            shape.grid_w, shape.d_k, shape.d_v, 1,
                            vp(torch.cuda.current_stream().cuda_stream))
    assert rc == 0 and g.gtr_gla_status() == 0
    assert torch.equal(buf[:n].view(torch.int16), guard[:n].view(torch.int16))
    assert torch.equal(buf[2 * n:].view(torch.int16), guard[2 * n:].view(torch.int16))
    assert rel(buf[n:2 * n].view(v.shape), ref_o) <= TOL[dtype]


def test_workspace_shared_between_paths_and_left_clean():
    """The CUDA-core path (chunk 32) and the fused path (chunk 64) may share one
    workspace; the fused kernel's 64 KiB synchronisation header is zero after
    every call."""
    shape, dtype = CONFIGS["640_b1"]
    q, k, v, la = (t.cuda() for t in case(shape, dtype, 0, "normal"))
    g = gla()
    need = max(g.gtr_gla_workspace_size(1, 6, 40, 40, 64, 64, g.F16, c) for c in (32, 64))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ref_o, ref_s = reference(shape, dtype, 0, "normal", 3)
    for chunk in (32, 64, 32, 64):
        out, fs = g.gtr_gla_fwd_ex(q, k, v, la, 3, chunk=chunk, workspace=ws)
        assert g.gtr_gla_status() == 0
        assert rel(out, ref_o) <= TOL[dtype] and rel(fs, ref_s) <= TOL[dtype]
        assert int(ws[:65536].count_nonzero()) == 0


def test_cuda_graph_replay_matches_eager():
    shape, dtype = CONFIGS["1024_b1"]
    q, k, v, la = (t.cuda() for t in case(shape, dtype, 0, "normal"))
    g = gla()
    ws = torch.zeros(g.gtr_gla_workspace_size(1, 12, 64, 64, 64, 64, g.F16, 64),
                     dtype=torch.uint8, device="cuda")
    outs = [torch.empty_like(v) for _ in range(4)]
    fss = [torch.empty((1, 12, 64, 64), dtype=torch.float32, device="cuda") for _ in range(4)]
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for d in range(4):  # warm-up outside capture
            g.gtr_gla_fwd_ex(q, k, v, la, d, workspace=ws, out=outs[d], final_state=fss[d], stream=s)
    s.synchronize()
    eager = [o.clone() for o in outs]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for d in range(4):
            g.gtr_gla_fwd_ex(q, k, v, la, d, workspace=ws, out=outs[d], final_state=fss[d], stream=s)
    for _ in range(3):
        for o in outs:
            o.zero_()
        graph.replay()
        torch.cuda.synchronize()
        for d in range(4):
            assert torch.equal(outs[d], eager[d])
    assert g.gtr_gla_status() == 0


@pytest.mark.parametrize("direction", [0, 2])
def test_band_of_extreme_gates(direction):
    """Some chunks carry gate spans far beyond fp32 range of e^{-b}; those take
    the exact score path while the rest stay factorised."""
    shape = Shape(1, 3, 32, 48, 64, 64)
    q, k, v, la = make_inputs(shape, "f16", 4)
    la = la.clone()
    la[:, :, 10:14] = -60.0
    la[:, 1, :, 20:22] = -3.0
    g = gla()
    out, fs = g.gtr_gla_fwd_ex(q.cuda(), k.cuda(), v.cuda(), la.cuda(), direction)
    assert g.gtr_gla_status() == 0
    ref_o, ref_s = oracle.forward(q, k, v, la, direction)
    assert rel(out, ref_o) <= 5e-3
    assert rel(fs, ref_s) <= 5e-3


@pytest.mark.parametrize("direction", [1, 2])
def test_chunk_128_fp32_ragged(direction):
    """Chunk 128 on the 640x640 grid: 12 full chunks and a 64-token tail."""
    shape, _ = CONFIGS["640_b1"]
    check(shape, "f32", direction, chunk=128)


@pytest.mark.parametrize("direction", [0, 3])
def test_bf16_head_dim_128(direction):
    """bf16 with d = 128: four 64-wide fused launches, the second key half
    accumulating into the output."""
    shape = Shape(1, 4, 32, 40, 128, 128)
    check(shape, "bf16", direction, seed=11)


@pytest.mark.parametrize("dims", [(64, 128), (128, 64)])
def test_rectangular_head_dims_column_scans_edge_grid(dims):
    """Mixed head sizes on a grid whose height is not a multiple of 8 (the
    column scans take the row-gather path)."""
    shape = Shape(1, 3, 13, 9, dims[0], dims[1])
    for direction in (2, 3):
        check(shape, "f16", direction, seed=13)


@pytest.mark.parametrize("direction", [0, 3])
def test_many_segments_over_several_waves(direction):
    """B=2, H=20 on the 128x128 grid: the plan splits each (b,h) into 11
    segments, 440 CTAs in three waves on 148 SMs, with 440 segment flags
    (one cache line each) in the workspace header.  Later waves fold
    aggregates published by CTAs that have already exited."""
    shape = Shape(2, 20, 128, 128, 64, 64)
    check(shape, "f16", direction, seed=21)


def test_dirty_workspace_header_reports_and_recovers():
    """A workspace whose ticket counter is not zero at launch (as if two calls
    sharing it overlapped): one CTA draws a ticket past the last segment and
    reports GTR_GLA_ERR_WORKSPACE_STATE without touching memory; the segments
    of the first plane wait for a flag that nothing sets until their bounded
    wait (about 2 s) gives up.  The call returns, the error is reported, the
    header is clean again, and the next call on the same workspace is exact."""
    shape, dtype = CONFIGS["640_b1"]  # 13 segments per (b,h)
    q, k, v, la = (t.cuda() for t in case(shape, dtype, 0, "normal"))
    g = gla()
    need = g.gtr_gla_workspace_size(1, 6, 40, 40, 64, 64, g.F16, 64)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ws[:4].view(torch.int32)[0] = 1  # ticket counter
    out, fs = g.gtr_gla_fwd_ex(q, k, v, la, 0, workspace=ws)
    assert g.gtr_gla_status() == -12  # GTR_GLA_ERR_WORKSPACE_STATE, latched first
    assert g.gtr_gla_status() == 0   # status clears the latched error
    assert int(ws[:65536].count_nonzero()) == 0
    out, fs = g.gtr_gla_fwd_ex(q, k, v, la, 0, workspace=ws)
    assert g.gtr_gla_status() == 0
    ref_o, ref_s = reference(shape, dtype, 0, "normal", 0)
    assert rel(out, ref_o) <= TOL[dtype] and rel(fs, ref_s) <= TOL[dtype]


@pytest.mark.parametrize("direction", [1, 2])
def test_many_planes_single_segment(direction):
    """640 (b,h) planes of an 8x8 grid: more planes than segment flags fit in
    the workspace header, so every plane is one segment (no aggregates, no
    flags), 640 CTAs in five waves."""
    shape = Shape(40, 16, 8, 8, 64, 64)
    check(shape, "f16", direction, seed=23)

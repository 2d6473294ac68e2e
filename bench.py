#!/usr/bin/env python
"""Throughput of the chunkwise key-gated linear attention forward pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 640_b1] [--no-graph]

One step = the four scan directions (L->R, R->L, T->B, B->T, one call each,
as four consecutive GTR layers would issue them) over one batch of synthetic
input of the chosen workload.  Default workload: the 640x640 detection shape,
B=1, H=6, 40x40 patch grid (1600 tokens), d_k = d_v = 64, fp16.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronisation on both sides, timed with CUDA events on the
launching stream; the timed steps are replayed from one CUDA graph (per-call
events inside it give the per-launch durations).  Inputs rotate over enough
separate buffers that each step reads data that is not in L2.  Under torchrun
every rank runs its own replica (B*H planes are independent: no collective on
the data path) and rank 0 prints one JSON line with the max time over ranks.

--impl reference times the fp64 CPU oracle (the only other place this file
runs it) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from recurrent_vision_backbone_chunkwise_b200.inputs import CONFIGS, make_inputs  # noqa: E402
from recurrent_vision_backbone_chunkwise_b200.replicas import (  # noqa: E402
    aggregate_rate, max_over_ranks, rank_info, replica_seed)

METRIC = "GLA fwd tokens/s and µs at 1600/4096/16384 tokens; % of roofline (HBM or TC)"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s HBM3e figure the roofline is also quoted against
DIRECTIONS = (0, 1, 2, 3)
ESIZE = {"f16": 2, "bf16": 2, "f32": 4}


def workload_bytes(shape, dtype: str) -> int:
    """Algorithmic HBM bytes of one call: q,k,v read, log_alpha read (fp32),
    out written, final state written (fp32)."""
    tok = shape.B * shape.H * shape.tokens
    e = ESIZE[dtype]
    return (tok * (2 * shape.d_k + shape.d_v) * e + tok * shape.d_k * 4 + tok * shape.d_v * e
            + shape.B * shape.H * shape.d_k * shape.d_v * 4)


KERNEL_FILES = ("gla_fused.cu", "sm100.cuh", "gla_common.cuh", "gla_internal.h")
TAIL_FILES = ("output_tail.cu", "io_pack.cuh", "gla_common.cuh", "gla_internal.h")


def kernel_code_hash(files=KERNEL_FILES) -> str:
    """sha256 prefix of a kernel's code: its source and the headers it
    includes, with comments and whitespace removed (a comment edit does not
    make a profile stale; any code change does)."""
    import hashlib
    import re

    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "recurrent_vision_backbone_chunkwise_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(name.encode() + b"\0" + " ".join(text.split()).encode() + b"\0")
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, profile: str = "gla_fused_kernel.md", files=KERNEL_FILES):
    """DRAM bytes of one launch of a kernel for `workload`, from the committed
    ncu summary `profiles/<profile>`, if that summary was taken on the current
    kernel code (kernel_code_hash(files) matches); else None."""
    import re

    prof = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(prof):
        return None
    text = open(prof).read()
    m = re.search(r"kernel_code_sha256_16:\s*([0-9a-f]{16})", text)
    try:
        if not m or kernel_code_hash(files) != m.group(1):
            return None
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch\s+" + re.escape(workload) + r"\s+(\d+)", text)
    return int(m.group(1)) if m else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measured_tensor_peak():
    """Dense bf16 (= fp16) tensor-core TFLOP/s for a kernel timed on its own."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def swiglu_shape(workload: str):
    """The Spatial SwiGLU block on a workload's grid: C = 64 channels per head
    of the attention (H x 64) and a hidden width of 4C (the pages give no
    widths; 4C is the usual MLP ratio)."""
    shape, dtype = CONFIGS[workload]
    C = shape.H * 64
    return shape.B, shape.grid_h, shape.grid_w, C, 4 * C, ("f16" if dtype == "f32" else dtype)


def smi_index(local: int) -> int:
    """nvidia-smi index of this rank's GPU (the first visible device)."""
    first = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0]
    return int(first) if first.isdigit() else local


def dist_setup(ri, dev):
    """One NCCL process group over the ranks of a torchrun launch (None when
    the job has one rank)."""
    if ri.world <= 1:
        return None
    from datetime import timedelta

    import torch.distributed as dist

    dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    return dist


def dist_barrier(dist):
    if dist is not None:
        dist.barrier()


def run_swiglu(args):
    """Spatial SwiGLU leg (not the headline): tokens/s of the whole block, its
    tensor-core roofline fraction (6 M C F flops of the two projections), the
    fused kernel's share from the launch list, the fp64 oracle on the host."""
    import torch
    from recurrent_vision_backbone_chunkwise_b200 import gla, swiglu
    from recurrent_vision_backbone_chunkwise_b200.inputs import make_swiglu_inputs

    ri = rank_info()
    torch.cuda.set_device(ri.local_rank)
    dev = torch.device("cuda", ri.local_rank)
    dist = dist_setup(ri, dev)
    B, gh, gw, C, F, dtype = swiglu_shape(args.config)
    M = B * gh * gw
    ins = make_swiglu_inputs(B, gh, gw, C, F, dtype, seed=replica_seed(0, ri.rank))
    set_bytes = sum(t.numel() * t.element_size() for t in ins) + M * C * 2
    R = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    sets = [([t.to(dev) for t in ins], torch.empty_like(ins[0], device=dev)) for _ in range(R)]
    ws = torch.empty(swiglu.gtr_swiglu_workspace_size(B, gh, gw, C, F, gla._DTYPE_CODE[ins[0].dtype]),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, ev=None):
        t, y = sets[i % R]
        if ev is not None:
            ev[0].record(stream)
        swiglu.gtr_swiglu_fwd(*t, out=y, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    assert gla.gtr_gla_status(stream) == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
    launches0 = gla.gtr_gla_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            step(i, evs[i])
    launches = gla.gtr_gla_launch_count() - launches0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(ri.local_rank))
    sampler.start()
    time.sleep(0.2)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist_barrier(dist)
    clocks = sampler.stop(t0, t1)
    assert gla.gtr_gla_status(stream) == 0
    elapsed = max_over_ranks(start.elapsed_time(end), device=dev)
    call_ms = [e[0].elapsed_time(e[1]) for e in evs]
    del graph
    # end to end: x in from pinned host memory, y back, every step
    hx = ins[0].pin_memory()
    hy = torch.empty_like(ins[0]).pin_memory()
    K2 = min(K, 200)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K2):
            t, y = sets[i % R]
            t[0].copy_(hx, non_blocking=True)
            swiglu.gtr_swiglu_fwd(*t, out=y, workspace=ws, stream=stream)
            hy.copy_(y, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
    mean_s = statistics.mean(call_ms) / 1000.0
    flops = 6.0 * M * C * F
    peak, peak_kind = measured_tensor_peak()
    achieved = flops / mean_s / 1e12
    line = {
        "metric": "Spatial SwiGLU block tokens/s; % of tensor-core roofline", "value":
            aggregate_rate(ri.world, K, M, elapsed), "unit": "tokens/s", "n_gpus": ri.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": f"swiglu_{args.config}", "B": B, "grid": [gh, gw], "C": C, "F": F,
                   "l2": f"inputs and weights rotate over {R} sets "
                         f"({R * set_bytes / 2**20:.0f} MiB > 126 MiB L2)", "cuda_graph": True},
        "kernel_us_per_call": {"mean": 1e6 * mean_s, "median": 1e3 * statistics.median(call_ms),
                               "min": 1e3 * min(call_ms)},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peak_kind} dense bf16 burst",
                     "flops_per_call": flops,
                     "timed_unit": "one block: the two tensor-core GEMMs and the fused kernel"},
        "gpu_launches": int(launches),
        "e2e": {"value": aggregate_rate(ri.world, K2, M, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": M * C * 2, "d2h_bytes_per_step": M * C * 2, "steps": K2},
        "clocks": clocks,
    }
    if ri.rank == 0 and ri.world == 1 and not args.no_cpu_baseline:
        import oracle.swiglu as osw

        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 10.0 and reps < 1000:
            osw.forward(*ins)
            reps += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * M / el, "unit": "tokens/s", "cores": os.cpu_count(),
                                "kind": "oracle",
                                "sample": f"{reps} forwards of the full block (numpy fp64) in {el:.1f} s"}
    if ri.rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_backbone(args):
    """Backbone leg (not the headline): the 12-layer stack (direction = layer
    mod 4) on the workload's grid and batch, width C = 64 H and F = 4 C, all
    12 layers in one CUDA graph per step; images/s and the latency of one
    forward, the fp64 oracle's layers on the host as the CPU baseline."""
    import torch
    from recurrent_vision_backbone_chunkwise_b200 import gla, layer
    from recurrent_vision_backbone_chunkwise_b200.inputs import make_backbone_params

    ri = rank_info()
    torch.cuda.set_device(ri.local_rank)
    dev = torch.device("cuda", ri.local_rank)
    dist = dist_setup(ri, dev)
    shape, _ = CONFIGS[args.config]
    B, gh, gw, C = shape.B, shape.grid_h, shape.grid_w, 64 * shape.H
    F, n_layers = 4 * C, 12
    params = make_backbone_params(C, F, n_layers, "f16", seed=replica_seed(0, ri.rank))
    w_bytes = sum(t.numel() * t.element_size() for p in params for t in p.values())
    # weight sets rotate so that the weights a step reads exceed L2
    R = max(1, math.ceil(L2_BYTES / w_bytes) + (1 if w_bytes < L2_BYTES else 0))
    wsets = [[layer.pack_weights(p, dev) for p in params] for _ in range(R)]
    g = torch.Generator().manual_seed(replica_seed(1, ri.rank))
    x0 = torch.randn(B, gh, gw, C, generator=g).half()
    xs = [x0.to(dev) for _ in range(R)]
    ws = torch.zeros(layer.gtr_layer_workspace_size(B, gh, gw, C, F), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, ev=None):
        x = xs[i % R]
        if ev is not None:
            ev[0].record(stream)
        layer.gtr_backbone_fwd(x, wsets[i % R], workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    assert gla.gtr_gla_status(stream) == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
    launches0 = gla.gtr_gla_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            step(i, evs[i])
    launches = gla.gtr_gla_launch_count() - launches0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(ri.local_rank))
    sampler.start()
    time.sleep(0.2)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist_barrier(dist)
    clocks = sampler.stop(t0, t1)
    assert gla.gtr_gla_status(stream) == 0
    elapsed = max_over_ranks(start.elapsed_time(end), device=dev)
    call_ms = [e[0].elapsed_time(e[1]) for e in evs]
    del graph
    # end to end: the image's tokens in from pinned host memory, the features
    # back, every step, through the public entry point
    hx = x0.pin_memory()
    hy = torch.empty_like(x0).pin_memory()
    K2 = min(K, 100)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K2):
            x = xs[i % R]
            x.copy_(hx, non_blocking=True)
            layer.gtr_backbone_fwd(x, wsets[i % R], workspace=ws, stream=stream)
            hy.copy_(x, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
    line = {
        "metric": "GTR backbone (12 layers) images/s and ms per forward", "value":
            aggregate_rate(ri.world, K, B, elapsed), "unit": "images/s", "n_gpus": ri.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": f"backbone_{args.config}", "B": B, "grid": [gh, gw], "C": C, "F": F,
                   "layers": n_layers, "heads": C // 64,
                   "l2": f"weights rotate over {R} sets ({R * w_bytes / 2**20:.0f} MiB > 126 MiB L2)",
                   "cuda_graph": True},
        "ms_per_forward": {"mean": statistics.mean(call_ms), "median": statistics.median(call_ms),
                           "min": min(call_ms)},
        "gpu_launches": int(launches),
        "e2e": {"value": aggregate_rate(ri.world, K2, B, e2e_ms), "unit": "images/s",
                "h2d_bytes_per_step": x0.numel() * 2, "d2h_bytes_per_step": x0.numel() * 2, "steps": K2},
        "clocks": clocks,
    }
    if ri.rank == 0 and ri.world == 1 and not args.no_cpu_baseline:
        import oracle.backbone as obb

        reps, t0 = 0, time.perf_counter()
        x = x0
        while time.perf_counter() - t0 < 10.0 and reps < n_layers:
            x = obb.layer_forward(x, params[reps], reps % 4)
            reps += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": B * reps / n_layers / el, "unit": "images/s", "cores": host_threads(),
                                "kind": "oracle",
                                "sample": f"{reps} of the {n_layers} layers (fp64) in {el:.1f} s"}
    if ri.rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_bwd(args):
    """Backward leg (not the headline): the gradients of the attention on the
    workload (d = 64, chunk 64), image tokens/s per call (one direction per
    call, the four cycled) and its HBM roofline fraction: per token-head q, k,
    v, d_out read and dq, dk, dv written at 2 d bytes each, log_alpha read and
    dlog_alpha written at 4 d bytes each (1536 B at d = 64), plus the final-state
    gradient; the fp64 oracle on the host."""
    import torch
    from recurrent_vision_backbone_chunkwise_b200 import gla

    ri = rank_info()
    torch.cuda.set_device(ri.local_rank)
    dev = torch.device("cuda", ri.local_rank)
    dist = dist_setup(ri, dev)
    shape, dtype = CONFIGS[args.config]
    dtype = "f16" if dtype == "f32" else dtype
    if shape.d_k != 64 or shape.d_v != 64:
        raise SystemExit("the backward pass takes head size 64")
    B, H, gh, gw = shape.B, shape.H, shape.grid_h, shape.grid_w
    host = make_inputs(shape, dtype, seed=replica_seed(0, ri.rank))
    g = torch.Generator().manual_seed(replica_seed(7, ri.rank))
    hdo = torch.randn(host[2].shape, generator=g).to(host[2].dtype)
    hdsf = torch.randn(B, H, 64, 64, generator=g)
    units = B * H * gh * gw
    call_bytes = 1536 * units + B * H * 64 * 64 * 4
    R = max(2, math.ceil(2 * L2_BYTES / call_bytes))
    sets = [[t.to(dev) for t in (*host, hdo, hdsf)] for _ in range(R)]
    ws = torch.empty(gla.gtr_gla_bwd_workspace_size(B, H, gh, gw), dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def step(i, ev=None):
        q, k, v, la, do, dsf = sets[i % R]
        if ev is not None:
            ev[0].record(stream)
        gla.gtr_gla_bwd(q, k, v, la, do, i % 4, d_final_state=dsf, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    assert gla.gtr_gla_status(stream) == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
    launches0 = gla.gtr_gla_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            step(i, evs[i])
    launches = gla.gtr_gla_launch_count() - launches0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(ri.local_rank))
    sampler.start()
    time.sleep(0.2)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist_barrier(dist)
    clocks = sampler.stop(t0, t1)
    assert gla.gtr_gla_status(stream) == 0
    elapsed = max_over_ranks(start.elapsed_time(end), device=dev)
    call_ms = [e[0].elapsed_time(e[1]) for e in evs]
    del graph
    mean_s = statistics.mean(call_ms) / 1000.0
    peak, kind = measured_peaks()
    src = "measured copy bandwidth (burst)" if kind == "measured" else "fallback (6.65 TB/s)"
    achieved = call_bytes / mean_s / 1e9
    line = {
        "metric": "GLA backward image tokens/s and us per call; % of HBM roofline", "value":
            aggregate_rate(ri.world, K, B * gh * gw, elapsed), "unit": "tokens/s", "n_gpus": ri.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": f"bwd_{args.config}", "B": B, "H": H, "grid": [gh, gw], "d": 64, "chunk": 64,
                   "directions": 4, "l2": f"inputs rotate over {R} sets", "cuda_graph": True},
        "kernel_us_per_call": {"mean": 1e6 * mean_s, "median": 1e3 * statistics.median(call_ms),
                               "min": 1e3 * min(call_ms)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": src, "bytes_per_call": call_bytes,
                     "timed_unit": "one gtr_gla_bwd call (its seven kernels)"},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if ri.rank == 0 and ri.world == 1 and not args.no_cpu_baseline:
        import oracle.backward as ob

        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 10.0 and reps < 100:
            ob.backward(*host, hdo, reps % 4, d_final_state=hdsf)
            reps += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * B * gh * gw / el, "unit": "tokens/s", "cores": host_threads(),
                                "kind": "oracle", "sample": f"{reps} full backward calls (fp64) in {el:.1f} s"}
    if ri.rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def run_tail(args):
    """Output-tail leg (not the headline): token-heads/s of the tail on the
    workload's attention output (B, H, grid, d_v), its HBM roofline fraction
    (6 d_v bytes per token-head: o and z read, y written), the fp64 oracle on
    the host."""
    import torch
    from recurrent_vision_backbone_chunkwise_b200 import gla, output_tail
    from recurrent_vision_backbone_chunkwise_b200.inputs import make_tail_inputs

    ri = rank_info()
    torch.cuda.set_device(ri.local_rank)
    dev = torch.device("cuda", ri.local_rank)
    dist = dist_setup(ri, dev)
    shape, dtype = CONFIGS[args.config]
    dtype = "f16" if dtype == "f32" else dtype
    B, H, gh, gw, dv = shape.B, shape.H, shape.grid_h, shape.grid_w, shape.d_v
    units = B * H * gh * gw  # token-heads per call
    ins = make_tail_inputs(B, H, gh, gw, dv, dtype, seed=replica_seed(0, ri.rank))
    call_bytes = 6 * dv * units + H * dv * 4
    set_bytes = call_bytes
    R = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    sets = [([t.to(dev) for t in ins], torch.empty((B, gh, gw, H * dv), dtype=ins[0].dtype, device=dev))
            for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)

    def step(i, ev=None):
        (o, z, w), y = sets[i % R]
        if ev is not None:
            ev[0].record(stream)
        output_tail.gtr_output_tail_fwd(o, z, w, out=y, stream=stream)
        if ev is not None:
            ev[1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    stream.synchronize()
    assert gla.gtr_gla_status(stream) == 0
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(K)]
    launches0 = gla.gtr_gla_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(K):
            step(i, evs[i])
    launches = gla.gtr_gla_launch_count() - launches0
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(smi_index(ri.local_rank))
    sampler.start()
    time.sleep(0.2)
    dist_barrier(dist)
    torch.cuda.synchronize()
    t0 = time.time()
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    dist_barrier(dist)
    clocks = sampler.stop(t0, t1)
    assert gla.gtr_gla_status(stream) == 0
    elapsed = max_over_ranks(start.elapsed_time(end), device=dev)
    call_ms = [e[0].elapsed_time(e[1]) for e in evs]
    del graph
    # end to end: o and z in from pinned host memory, y back, every step
    ho, hz = ins[0].pin_memory(), ins[1].pin_memory()
    hy = torch.empty((B, gh, gw, H * dv), dtype=ins[0].dtype).pin_memory()
    K2 = min(K, 200)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist_barrier(dist)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(K2):
            (o, z, w), y = sets[i % R]
            o.copy_(ho, non_blocking=True)
            z.copy_(hz, non_blocking=True)
            output_tail.gtr_output_tail_fwd(o, z, w, out=y, stream=stream)
            hy.copy_(y, non_blocking=True)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)
    mean_s = statistics.mean(call_ms) / 1000.0
    peak, peak_kind = measured_peaks()
    achieved = call_bytes / mean_s / 1e9
    line = {
        "metric": "GLA output tail token-heads/s; % of HBM roofline", "value":
            aggregate_rate(ri.world, K, units, elapsed), "unit": "token-heads/s", "n_gpus": ri.world,
        "steps": K, "warmup": args.warmup, "ms_per_step": elapsed / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": f"tail_{args.config}", "B": B, "H": H, "grid": [gh, gw], "d_v": dv,
                   "l2": f"inputs rotate over {R} sets ({R * set_bytes / 2**20:.0f} MiB > 126 MiB L2)",
                   "cuda_graph": True},
        "kernel_us_per_call": {"mean": 1e6 * mean_s, "median": 1e3 * statistics.median(call_ms),
                               "min": 1e3 * min(call_ms)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(args.config, "output_tail_kernel_1024_b4.md", TAIL_FILES),
                     "peak_source": peak_kind, "bytes_per_call": call_bytes,
                     "timed_unit": "one call of output_tail_kernel"},
        "gpu_launches": int(launches),
        "e2e": {"value": aggregate_rate(ri.world, K2, units, e2e_ms), "unit": "token-heads/s",
                "h2d_bytes_per_step": 4 * dv * units, "d2h_bytes_per_step": 2 * dv * units, "steps": K2},
        "clocks": clocks,
    }
    if ri.rank == 0 and ri.world == 1 and not args.no_cpu_baseline:
        import oracle.output_tail as otail

        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 10.0 and reps < 1000:
            otail.forward(*ins)
            reps += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * units / el, "unit": "token-heads/s", "cores": os.cpu_count(),
                                "kind": "oracle",
                                "sample": f"{reps} calls of the full tail (numpy fp64) in {el:.1f} s"}
    if ri.rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.gpu = gpu_index
        self.period = period_ms
        self.samples = []
        self.proc = None
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", f"-lms={self.period}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self, t0: float, t1: float):
        if self.proc is None:
            return None
        time.sleep(self.period / 1000.0 * 2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        window = [r for r in rows if t0 <= r[0] <= t1]
        scope = "timed"
        if not window:
            window, scope = rows, "warmup+timed"
        if not window:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in window:
            for name, flag in zip(names, r[3][1:]):
                if flag.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in window),
                "sm_max_mhz": max(r[2] for r in window), "reasons": sorted(reasons),
                "samples": len(window), "window": scope}


def image_tokens(shape) -> int:
    """Image tokens of one call: B * grid_h * grid_w (every head of a token is
    in the same call, so heads are not counted again)."""
    return shape.B * shape.tokens


_HOST_THREADS = []


def host_threads() -> int:
    """OpenMP threads of the host (all cores), read once: a call with an
    explicit thread count changes what OpenMP reports afterwards."""
    if not _HOST_THREADS:
        import oracle

        _HOST_THREADS.append(int(oracle.max_threads()))
    return _HOST_THREADS[0]


def oracle_sample(shape, dtype, seconds: float):
    """Inputs of a bounded CPU sample of `shape`: the grid is cut to its first
    rows so that one direction of every plane takes about `seconds` / 4 on
    all host cores (the whole grid when that fits)."""
    import numpy as np

    import oracle

    q, k, v, la = (t.double().numpy() for t in make_inputs(shape, dtype, seed=0))
    cores = host_threads()
    rows = shape.grid_h
    probe = max(1, min(rows, 8))
    t0 = time.perf_counter()
    oracle.forward(*(np.ascontiguousarray(a[:, :, :probe]) for a in (q, k, v, la)), 0,
                   n_threads=cores)
    per_row = (time.perf_counter() - t0) / probe
    rows = max(1, min(rows, int(seconds / 4.0 / max(per_row, 1e-9))))
    return tuple(np.ascontiguousarray(a[:, :, :rows]) for a in (q, k, v, la)), rows


def cpu_oracle_rate(shape, dtype, seconds: float = 10.0, threads=None, max_reps: int = 100000):
    """The fp64 oracle, as it stands, on this host: image tokens/s over the four
    directions of a bounded sample of the workload (its first grid rows, all
    planes), repeated until ~`seconds` of CPU work.  `threads` = OpenMP
    threads (all host cores by default); the oracle runs one (b,h) plane per
    thread, so at most B*H of them do work."""
    import oracle

    (q, k, v, la), rows = oracle_sample(shape, dtype, seconds if threads != 1 else seconds / 8)
    cores = host_threads() if threads is None else int(threads)
    used = min(cores, shape.B * shape.H)
    reps = 0
    t0 = time.perf_counter()
    while True:
        for d in DIRECTIONS:
            oracle.forward(q, k, v, la, d, n_threads=cores)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds or reps >= max_reps:
            break
    tokens = reps * len(DIRECTIONS) * shape.B * rows * shape.grid_w
    sample = (f"{reps} steps x 4 directions of all {shape.B * shape.H} planes on the first "
              f"{rows} of {shape.grid_h} grid rows in {el:.1f} s, {cores} OpenMP threads "
              f"({used} busy: one plane per thread)")
    return {"value": tokens / el, "unit": "tokens/s", "cores": used, "threads": cores,
            "kind": "oracle", "sample": sample}


def workload_config(name: str, world: int, chunk: int = 64) -> dict:
    """The `config` object of a bench line; both arms print the same one."""
    shape, dtype = CONFIGS[name]
    in_bytes = shape.B * shape.H * shape.tokens * (
        (2 * shape.d_k + shape.d_v) * ESIZE[dtype] + 4 * shape.d_k)
    set_bytes = in_bytes + len(DIRECTIONS) * shape.B * shape.H * shape.tokens * shape.d_v * ESIZE[dtype]
    R = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    return {"workload": name, "B": shape.B, "H": shape.H, "grid": [shape.grid_h, shape.grid_w],
            "tokens": shape.tokens, "d_k": shape.d_k, "d_v": shape.d_v, "io_dtype": dtype,
            "chunk": chunk, "directions": 4,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": f"inputs rotate over {R} buffer sets "
                  f"({R * set_bytes / 2**20:.0f} MiB > 126 MiB L2)"}


def run_reference(args):
    """The oracle as the reference arm: exactly `--steps` timed steps after
    `--warmup` untimed ones, each step one scan direction (cycling) of every
    (b,h) plane of the workload's grid cut to its first rows, so that the whole
    run takes about a minute of host time; tokens/s counts the image tokens
    the sample holds."""
    if rank_info().rank != 0:
        return
    import oracle

    shape, dtype = CONFIGS[args.config]
    budget = 60.0 / (args.steps + args.warmup)  # seconds of host time per step
    (qs, ks, vs, las), rows = oracle_sample(shape, dtype, 4.0 * budget)
    cores = host_threads()
    for i in range(args.warmup):
        oracle.forward(qs, ks, vs, las, DIRECTIONS[i % 4], n_threads=cores)
    t0 = time.perf_counter()
    for i in range(args.steps):
        oracle.forward(qs, ks, vs, las, DIRECTIONS[i % 4], n_threads=cores)
    el = time.perf_counter() - t0
    tokens = shape.B * rows * shape.grid_w
    rate = args.steps * tokens / el
    used = min(cores, shape.B * shape.H)
    sample = (f"{args.steps} steps, each one direction of all {shape.B * shape.H} planes "
              f"on the first {rows} of {shape.grid_h} grid rows ({tokens} image tokens), "
              f"{el:.1f} s, {cores} OpenMP threads ({used} busy: one plane per thread)")
    line = {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args.config, args.gpus),
        "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": used, "threads": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def gla_sets(shape, dtype, dev, rank):
    """Device buffer sets of one workload, enough of them that consecutive
    steps never find their inputs in L2."""
    import torch

    q0, k0, v0, la0 = make_inputs(shape, dtype, seed=replica_seed(0, rank))
    in_bytes = sum(t.numel() * t.element_size() for t in (q0, k0, v0, la0))
    out_bytes = shape.B * shape.H * shape.tokens * shape.d_v * ESIZE[dtype]
    set_bytes = in_bytes + len(DIRECTIONS) * out_bytes
    R = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    sets = []
    for _ in range(R):
        ins = [t.to(dev) for t in (q0, k0, v0, la0)]
        outs = [torch.empty((shape.B, shape.H, shape.grid_h, shape.grid_w, shape.d_v),
                            dtype=q0.dtype, device=dev) for _ in DIRECTIONS]
        fss = [torch.empty((shape.B, shape.H, shape.d_k, shape.d_v), dtype=torch.float32,
                           device=dev) for _ in DIRECTIONS]
        sets.append((ins, outs, fss))
    return (q0, k0, v0, la0), sets, in_bytes, out_bytes


def time_gla(name, K, W, dev, stream, rank, use_graph=True, chunk=64, with_eager=True):
    """Time K steps (the four directions, one call each) of workload `name`
    after W warm-up steps: the whole timed region and every call, with CUDA
    events on the launching stream.  Returns the measurements as a dict."""
    import torch
    from recurrent_vision_backbone_chunkwise_b200 import gla

    shape, dtype = CONFIGS[name]
    host, sets, in_bytes, out_bytes = gla_sets(shape, dtype, dev, rank)
    R = len(sets)
    ws = torch.zeros(max(1, gla.gtr_gla_workspace_size(shape.B, shape.H, shape.grid_h,
                                                         shape.grid_w, shape.d_k, shape.d_v,
                                                         gla._DTYPE_CODE[host[0].dtype], chunk)),
                     dtype=torch.uint8, device=dev)

    def step(i, ev=None):
        (q, k, v, la), outs, fss = sets[i % R]
        for j, d in enumerate(DIRECTIONS):
            if ev is not None:
                ev[2 * j].record(stream)
            gla.gtr_gla_fwd_ex(q, k, v, la, d, chunk=chunk, workspace=ws, out=outs[j],
                               final_state=fss[j], stream=stream)
            if ev is not None:
                ev[2 * j + 1].record(stream)

    with torch.cuda.stream(stream):
        for i in range(W):
            step(i)
    stream.synchronize()
    assert gla.gtr_gla_status(stream) == 0
    call_events = [[torch.cuda.Event(enable_timing=True, external=use_graph) for _ in range(8)]
                   for _ in range(K)]
    graph = None
    launches0 = gla.gtr_gla_launch_count()
    if use_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(K):
                step(i, call_events[i])
        launches = gla.gtr_gla_launch_count() - launches0
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0 = time.time()
    launches_before = gla.gtr_gla_launch_count()
    with torch.cuda.stream(stream):  # the graph replays on the current stream
        start.record(stream)
        if use_graph:
            graph.replay()
        else:
            for i in range(K):
                step(i, call_events[i])
        end.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    if not use_graph:
        launches = gla.gtr_gla_launch_count() - launches_before
    assert gla.gtr_gla_status(stream) == 0
    call_ms = [call_events[i][2 * j].elapsed_time(call_events[i][2 * j + 1])
               for i in range(K) for j in range(len(DIRECTIONS))]
    res = {"elapsed_ms": start.elapsed_time(end), "call_ms": call_ms, "eager_ms": call_ms,
           "launches": int(launches), "wall": (t0, t1), "host": host, "sets": sets, "ws": ws,
           "in_bytes": in_bytes, "out_bytes": out_bytes, "R": R, "step": step}
    if graph is not None:
        del graph
        if with_eager:  # the same calls without graph capture (not the headline)
            Ke = min(K, 200)
            ev = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(Ke)]
            with torch.cuda.stream(stream):
                for i in range(Ke):
                    step(i, ev[i])
            stream.synchronize()
            res["eager_ms"] = [ev[i][2 * j].elapsed_time(ev[i][2 * j + 1])
                               for i in range(Ke) for j in range(len(DIRECTIONS))]
    return res


def roofline_entry(name, call_ms, chunk=64):
    """The HBM roofline object of one workload from its per-call times."""
    shape, dtype = CONFIGS[name]
    call_bytes = workload_bytes(shape, dtype)
    mean_s = statistics.mean(call_ms) / 1000.0
    peak, peak_kind = measured_peaks()
    achieved = call_bytes / mean_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak,
            "traffic": profiled_traffic(name) if chunk == 64 else None,
            "frac_vs_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "peak_source": f"{peak_kind} copy bandwidth (burst)",
            "bytes_per_call": call_bytes,
            "timed_unit": "one library call (all kernels of one direction)"}


def us_entry(call_ms, eager_ms):
    return {"mean": 1e3 * statistics.mean(call_ms), "median": 1e3 * statistics.median(call_ms),
            "min": 1e3 * min(call_ms), "eager_median": 1e3 * statistics.median(eager_ms),
            "eager_min": 1e3 * min(eager_ms)}


# The metric is quoted at 1600, 4096 and 16384 tokens: the default run times
# these workloads too, after the headline one, and reports them under
# "per_config" (same K and W, same timing method).
PER_CONFIG = ("1024_b4", "16k_d64", "16k_d128")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="640_b1", choices=sorted(CONFIGS))
    ap.add_argument("--chunk", type=int, default=64, choices=[32, 64, 128])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only --config (skip the other token counts of the metric)")
    ap.add_argument("--op", default="gla", choices=["gla", "swiglu", "tail", "backbone", "bwd"],
                    help="gla: the headline (chunkwise GLA); swiglu: the Spatial SwiGLU block; "
                         "tail: the attention's output tail; backbone: the 12-layer stack; "
                         "bwd: the attention's backward pass")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.op == "swiglu" and args.impl == "ours":
        run_swiglu(args)
        return
    if args.op == "tail" and args.impl == "ours":
        run_tail(args)
        return
    if args.op == "backbone" and args.impl == "ours":
        run_backbone(args)
        return
    if args.op == "bwd" and args.impl == "ours":
        run_bwd(args)
        return

    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist
    from recurrent_vision_backbone_chunkwise_b200 import gla

    ri = rank_info()
    world, rank, local = ri.world, ri.rank, ri.local_rank
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    shape, dtype = CONFIGS[args.config]
    chunk = args.chunk
    stream = torch.cuda.Stream(device=dev)
    use_graph = not args.no_graph
    K = args.steps

    # warm-up and graph capture happen inside time_gla; the clock sampler runs
    # from before the timed region to after it
    sampler = ClockSampler(smi_index(local))
    sampler.start()
    time.sleep(0.2)
    if world > 1:
        dist.barrier()
    res = time_gla(args.config, K, args.warmup, dev, stream, rank, use_graph, chunk)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop(*res["wall"])
    elapsed_ms = max_over_ranks(res["elapsed_ms"], device=dev)
    call_ms, eager_ms = res["call_ms"], res["eager_ms"]

    # end-to-end through the public API: inputs copied in from pinned host
    # memory and every output and final state copied back, each step
    sets, R, step = res["sets"], res["R"], res["step"]
    q0, k0, v0, la0 = res["host"]
    in_bytes, out_bytes = res["in_bytes"], res["out_bytes"]
    fs_bytes = shape.B * shape.H * shape.d_k * shape.d_v * 4
    K_e2e = min(K, 200)
    host_in = [t.pin_memory() for t in (q0, k0, v0, la0)]
    host_out = [torch.empty(sets[0][1][0].shape, dtype=q0.dtype).pin_memory()
                for _ in DIRECTIONS]
    host_fs = [torch.empty(sets[0][2][0].shape, dtype=torch.float32).pin_memory()
               for _ in DIRECTIONS]
    # The copies are pipelined as a caller would: step i's inputs go in on a
    # copy stream while step i - 1 computes, and its results come back on a
    # third stream while step i + 1 computes (the device sets rotate, so a set
    # is refilled only after its step's results have been read back).  Every
    # step's copies and calls lie inside the timed region.
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(K_e2e)]
    ev_done = [torch.cuda.Event() for _ in range(K_e2e)]
    ev_back = [torch.cuda.Event() for _ in range(K_e2e)]
    with torch.cuda.stream(stream):
        for i in range(3):
            step(i)
        stream.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(stream)
        s_in.wait_event(e0)
        for i in range(K_e2e):
            (q, k, v, la), outs, fss = sets[i % R]
            with torch.cuda.stream(s_in):
                if i >= R:
                    s_in.wait_event(ev_back[i - R])  # the set's previous results are home
                for dst, src in zip((q, k, v, la), host_in):
                    dst.copy_(src, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            for j, d in enumerate(DIRECTIONS):
                if chunk == 64 and dtype == "f16":
                    gla.gtr_gla_fwd(q, k, v, la, d, out=outs[j], final_state=fss[j], stream=stream)
                else:
                    gla.gtr_gla_fwd_ex(q, k, v, la, d, chunk=chunk, workspace=res["ws"],
                                       out=outs[j], final_state=fss[j], stream=stream)
            ev_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                for j in range(len(DIRECTIONS)):
                    host_out[j].copy_(outs[j], non_blocking=True)
                    host_fs[j].copy_(fss[j], non_blocking=True)
                ev_back[i].record(s_out)
        stream.wait_event(ev_back[K_e2e - 1])
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device=dev)

    tokens_per_step = len(DIRECTIONS) * image_tokens(shape)
    value = aggregate_rate(world, K, tokens_per_step, elapsed_ms)
    e2e_value = aggregate_rate(world, K_e2e, tokens_per_step, e2e_ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": workload_config(args.config, world, chunk),
        "timing": {"cuda_graph": use_graph, "per_call": "CUDA events around every call"},
        "kernel_us_per_call": us_entry(call_ms, eager_ms),
        "token_heads_per_s": value * shape.H,
        "roofline": roofline_entry(args.config, call_ms, chunk),
        "gpu_launches": res["launches"],
        "e2e": {"value": e2e_value, "unit": "tokens/s",
                "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": len(DIRECTIONS) * (out_bytes + fs_bytes), "steps": K_e2e,
                "copies": "pinned host buffers, inputs on a copy stream one step ahead, results back on a third"},
        "clocks": clocks,
    }
    del res, sets, step
    torch.cuda.empty_cache()

    if not args.no_per_config and chunk == 64:
        per = {}
        for name in PER_CONFIG:
            if name == args.config:
                continue
            sampler = ClockSampler(smi_index(local))
            sampler.start()
            time.sleep(0.2)
            if world > 1:
                dist.barrier()
            r = time_gla(name, K, args.warmup, dev, stream, rank, use_graph, chunk)
            if world > 1:
                dist.barrier()
            ck = sampler.stop(*r["wall"])
            el = max_over_ranks(r["elapsed_ms"], device=dev)
            s2, _ = CONFIGS[name]
            per[name] = {"tokens": s2.tokens, "config": workload_config(name, world, chunk),
                         "value": aggregate_rate(world, K, len(DIRECTIONS) * image_tokens(s2), el),
                         "unit": "tokens/s", "ms_per_step": el / K,
                         "kernel_us_per_call": us_entry(r["call_ms"], r["eager_ms"]),
                         "roofline": roofline_entry(name, r["call_ms"], chunk),
                         "gpu_launches": r["launches"], "clocks": ck}
            del r
            torch.cuda.empty_cache()
        line["per_config"] = per

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_oracle_rate(shape, dtype, seconds=10.0)
        base["single_thread"] = cpu_oracle_rate(shape, dtype, seconds=4.0, threads=1)
        line["cpu_baseline"] = base
        for name, entry in line.get("per_config", {}).items():
            s2, d2 = CONFIGS[name]
            b2 = cpu_oracle_rate(s2, d2, seconds=3.0)
            b2["single_thread"] = cpu_oracle_rate(s2, d2, seconds=1.5, threads=1)
            entry["cpu_baseline"] = b2
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

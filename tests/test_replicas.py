"""Multi-process host logic (CPU, gloo, world size 2).

Runs on several GPUs are independent replicas: each rank draws its own
seeded inputs, runs the whole workload, and the only cross-rank steps are the
barriers and the max-over-ranks reduction of the measured times.  These tests
exercise exactly those steps with two gloo ranks on the CPU, plus the
reference arm's rule that ranks other than 0 exit without work.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from recurrent_vision_backbone_chunkwise_b200.inputs import Shape, make_inputs
from recurrent_vision_backbone_chunkwise_b200.replicas import (
    aggregate_rate, max_over_ranks, rank_info, replica_seed)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    try:
        from datetime import timedelta

        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
        ri = rank_info()
        shape = Shape(1, 2, 4, 5, 8, 8)
        qq, kk, vv, la = make_inputs(shape, "f32", seed=replica_seed(0, ri.rank))
        checksum = float(qq.double().sum() + la.double().sum())
        sums = [None] * world
        dist.all_gather_object(sums, checksum)
        # per-rank "device times": rank r measured 10 + 7 r ms
        dist.barrier()
        t = max_over_ranks(10.0 + 7.0 * ri.rank)
        t2 = max_over_ranks(-1.0 - ri.rank)  # the max, not the sum or rank 0's value
        rate = aggregate_rate(ri.world, 5, 1000, t)
        q.put((ri.rank, ri.world, ri.local_rank, sums, t, t2, rate))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # pragma: no cover - reported to the parent
        q.put(("error", rank, repr(e)))


def test_two_gloo_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert not any(r[0] == "error" for r in results), results
    results.sort()
    sums = results[0][3]
    assert sums == results[1][3]
    assert sums[0] != sums[1], "replicas must draw different inputs"
    for rank, (r, w, local, _, t, t2, rate) in enumerate(results):
        assert (r, w, local) == (rank, world, rank)
        assert t == 17.0 and t2 == -1.0
        assert rate == pytest.approx(2 * 5 * 1000 / 0.017)


def test_rank_info_and_rate():
    assert rank_info({}) == rank_info({"WORLD_SIZE": "1", "RANK": "0"})
    ri = rank_info({"WORLD_SIZE": "4", "RANK": "3", "LOCAL_RANK": "3"})
    assert (ri.rank, ri.world, ri.local_rank) == (3, 4, 3)
    with pytest.raises(ValueError):
        rank_info({"WORLD_SIZE": "2", "RANK": "2"})
    with pytest.raises(ValueError):
        aggregate_rate(1, 1, 1, 0.0)
    assert max_over_ranks(3.5) == 3.5  # no process group: the value itself
    assert replica_seed(0, 0) != replica_seed(0, 1)
    # weak scaling: doubling the ranks at the same per-rank time doubles the rate
    assert aggregate_rate(2, 10, 100, 4.0) == 2 * aggregate_rate(1, 10, 100, 4.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""

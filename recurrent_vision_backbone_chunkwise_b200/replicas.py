"""Host-side bookkeeping for runs on several GPUs of one node.

Every (batch, head) plane of the forward pass is an independent scan, so a
run on N GPUs is N independent replicas of one workload, one process per GPU:
no collective touches the data path.  The only cross-rank steps are the
barriers around a timed region and the max-over-ranks reduction of the times
measured on each device; throughput is then the units all ranks processed
divided by that maximum.
"""
from __future__ import annotations

import os
from dataclasses import dataclass
from typing import Mapping


@dataclass(frozen=True)
class RankInfo:
    rank: int
    local_rank: int
    world: int


def rank_info(env: Mapping[str, str] | None = None) -> RankInfo:
    """Rank, local rank and world size as torchrun exports them (1 process
    when none is set)."""
    env = os.environ if env is None else env
    world = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if world < 1 or not 0 <= rank < world or local < 0:
        raise ValueError(f"inconsistent rank environment: rank {rank}, world {world}, "
                         f"local rank {local}")
    return RankInfo(rank, local, world)


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic inputs: distinct replicas, reproducible."""
    return base_seed + rank


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks of the default process group (the
    value itself without one).  Every rank must call it, in the same order."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, steps: int, units_per_step: int, elapsed_ms: float) -> float:
    """Whole-job throughput: units processed by all `world` replicas over
    `steps` steps, divided by the slowest rank's time."""
    if elapsed_ms <= 0.0:
        raise ValueError("elapsed time must be positive")
    return world * steps * units_per_step / (elapsed_ms / 1000.0)

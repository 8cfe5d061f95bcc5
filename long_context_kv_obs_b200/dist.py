"""Process-group plumbing of the multi-GPU run: one process per GPU, each compressing
its own sequence.

The compression path has no exchange step: every sequence is scored, selected and
compacted on its own GPU, so N GPUs run N independent problems (weak scaling) and the
only collectives are for measurement - the max over ranks of each device-timed region,
and agreement on whether an optional measurement runs at all (a rank that skipped it
while another waits in its barrier would hang the job).
"""
from __future__ import annotations

import os
from typing import Mapping, Tuple


def rank_env(env: Mapping[str, str] = os.environ) -> Tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment (1 process if unset)."""
    rank = int(env.get("RANK", "0"))
    world = int(env.get("WORLD_SIZE", "1"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if not (0 <= rank < world) or local < 0:
        raise ValueError(f"inconsistent rank environment: RANK={rank} WORLD_SIZE={world} LOCAL_RANK={local}")
    return rank, world, local


def sequence_seed(base: int, rank: int) -> int:
    """Seed of the synthetic sequence rank `rank` compresses (distinct per rank)."""
    return base + rank


def max_over_ranks(x: float, dist, device) -> float:
    """The largest x over all ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_agree(flag: bool, dist, device) -> bool:
    """True only if every rank passes True; every rank gets the same answer."""
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return bool(flag)
    import torch
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def weak_throughput(world: int, units_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job units per second: every rank processes units_per_rank per step, and the
    job takes `ms` (max over ranks) for `steps` steps."""
    if ms <= 0:
        raise ValueError("elapsed time must be positive")
    return world * units_per_rank * steps / (ms * 1e-3)

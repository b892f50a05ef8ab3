"""Host logic of running the path as independent replicas, one per GPU.

The rows of a batch (sequence, layer, KV head) never exchange data, so N
GPUs run N independent batches and the only cross-rank traffic is the
timing reduction: every rank times its own steps, the job's step time is the
maximum over ranks, and the job's throughput counts the units of all ranks.
"""
from __future__ import annotations

import os
from dataclasses import dataclass
from datetime import timedelta


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    """Rank, world size and local rank from the launcher's environment (1 process when unset)."""
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                    int(os.environ.get("LOCAL_RANK", 0)))


def replica_seed(base_seed: int, rank: int) -> int:
    """Each replica draws its own synthetic batch; rank 0 keeps the base seed."""
    return base_seed + rank


def init_group(backend: str, world: int, device=None, timeout_s: float = 180.0) -> bool:
    """Joins the process group when there is more than one rank; returns whether it did."""
    if world <= 1:
        return False
    import torch.distributed as dist

    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return True


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of a per-rank scalar (a step time) over all ranks."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, ms_max: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("step time must be positive")
    return world * units_per_rank / (ms_max * 1e-3)

"""Process-group plumbing for data-parallel runs (one process per GPU).

The hybrid linear shards by tokens with no exchange inside the layer: every
rank multiplies its own rows of X by a replicated packed weight. The only
cross-rank steps are timing ones: a barrier before the timed region and the
maximum of the per-rank durations after it.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as td


def env_ranks() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str, timeout_s: float = 120.0) -> bool:
    """Join the process group when the launcher started more than one rank.
    Returns True when a group is active."""
    _, _, world = env_ranks()
    if world <= 1:
        return False
    td.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return True


def barrier(active: bool) -> None:
    if active:
        td.barrier()


def max_over_ranks(value: float, active: bool, device="cpu") -> float:
    """Largest `value` over all ranks (the job is as slow as its slowest rank)."""
    if not active:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the work every rank did, over the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("duration must be positive")
    return world * work_per_rank / (ms_max / 1e3)


def shutdown(active: bool) -> None:
    if active:
        td.destroy_process_group()

"""Rank plumbing for running the decode step as independent replicas on the GPUs of one node.

At batch-1 decode the rotated linear stack has no step that exchanges data between GPUs.
Each linear reads its own packed weights and a single activation vector. So N GPUs run N
independent replicas, one process per GPU, over their own token streams:

* throughput is the units every rank processed divided by the slowest rank's time;
* the per-step time is the maximum over ranks, reduced on the device (NCCL) or on the
  host (gloo);
* barriers bracket the timed region.

No collective runs on the data path.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class Ranks:
    rank: int
    world: int
    local_rank: int


def from_env() -> Ranks:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (defaults: one rank)."""
    return Ranks(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                 int(os.environ.get("LOCAL_RANK", "0")))


def init(r: Ranks, backend: str, timeout_s: float = 300.0) -> None:
    """Joins the process group when there is more than one rank. A short timeout makes a
    rank that never arrives end the others' next collective with an error."""
    if r.world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, rank=r.rank, world_size=r.world,
                                timeout=datetime.timedelta(seconds=timeout_s))


def barrier(r: Ranks) -> None:
    if r.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(r: Ranks, value: float, device=None) -> float:
    """The maximum of `value` over all ranks (every rank gets it). `device` is where the
    reduction runs: a CUDA device for NCCL, None (CPU) for gloo."""
    if r.world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(r: Ranks, units_per_rank: int, ms_max: float) -> float:
    """Units per second over the whole job: every rank processed `units_per_rank` units
    within `ms_max` milliseconds, the slowest rank's time."""
    if ms_max <= 0:
        raise ValueError("elapsed time must be positive")
    return r.world * units_per_rank / (ms_max / 1e3)


def finish(r: Ranks) -> None:
    """Last barrier, then leaves the process group."""
    if r.world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()

"""Replica bookkeeping for running the verify step on several GPUs of a node.

Sequences are independent, so N GPUs run N replicas of the verify step with
no data-path collective; the only cross-rank traffic is the timing reduction:
the job's time is the slowest rank's, and the job's work is the sum over
ranks. These helpers run on any torch.distributed backend (NCCL on the GPUs,
gloo in the CPU tests).
"""
from __future__ import annotations

import datetime
import os

import torch


def env_ranks():
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0, device=None):
    import torch.distributed as dist
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def _reduce(x: float, op, world: int, device) -> float:
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.MAX if world > 1 else None, world, device)


def sum_over_ranks(x: float, world: int, device="cpu") -> float:
    import torch.distributed as dist
    return _reduce(x, dist.ReduceOp.SUM if world > 1 else None, world, device)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def job_throughput(units_this_rank: float, seconds_this_rank: float, world: int, device="cpu") -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    total = sum_over_ranks(units_this_rank, world, device)
    slowest = max_over_ranks(seconds_this_rank, world, device)
    return total / slowest

"""Replica execution on the GPUs of one node.

The layer shards by sequence and by head with no exchange, so running it on N GPUs means
N independent copies of a workload, one process per GPU.  This module holds the host-side
rank logic of that mode: rank discovery from the launcher's environment (torchrun sets
RANK, WORLD_SIZE and LOCAL_RANK), process-group set-up and teardown, the slowest rank's
time (device times are compared as a MAX over ranks, never by wall clock) and the job's
throughput (all ranks' units over the slowest rank's time).  It moves no layer data.
"""

from __future__ import annotations

import datetime
import os


def rank_info(env=None):
    """(rank, world, local_rank) from the launcher's environment; (0, 1, 0) without one."""
    env = os.environ if env is None else env
    return int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")), int(env.get("LOCAL_RANK", "0"))


def init(world: int, local_rank: int, backend: str = "nccl", timeout_s: float = 120.0) -> None:
    """Joins the process group for world > 1 (NCCL on GPUs; gloo for CPU-only runs).  The
    short timeout turns a rank that never arrives into an error instead of a hang."""
    if world <= 1:
        return
    import torch
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl":
        torch.cuda.set_device(local_rank)
        kw["device_id"] = torch.device("cuda", local_rank)
    dist.init_process_group(backend, **kw)


def finish(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's `value` (e.g. the slowest rank's step time)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job rate: every rank processes `units_per_rank` in at most `slowest_seconds`."""
    return world * units_per_rank / slowest_seconds

"""Replica plumbing for the decode on N GPUs of one node, one process per GPU (torch.distributed).

A batch-1 decode step has no exchange between GPUs: every rank runs an identical, independent replica
(weak scaling, fixed work per rank).  The only collectives are the barriers around the timed region and
the maximum of the per-rank device times, so the reported rate is the work of all ranks over the slowest
rank's time.  The functions take the world size explicitly and work with any process-group backend
(NCCL on GPUs, gloo on the CPU).
"""

import torch
import torch.distributed as dist


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks (every rank gets the same value)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Units processed by all ranks per second of the slowest rank."""
    return world * units_per_rank / seconds_max

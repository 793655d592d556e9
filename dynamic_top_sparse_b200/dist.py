"""Host-side helpers for running the decode step on several GPUs.

The decode step partitions into independent units (sequence b, KV head g)
with no exchange between them, so the bench's N GPUs run N independent
replicas (one process per GPU, torch.distributed for the barrier and the
timing reduction only).  One long sequence over several GPUs is the
context-sharded step of shard.py.
"""
from __future__ import annotations

import torch


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(x: float, world: int, device=None) -> float:
    """Maximum of a host float over ranks (time of the slowest rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def allreduce_sum(x: float, world: int, device=None) -> float:
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own synthetic sequences (independent replicas)."""
    return int(base) * 1000003 + int(rank)

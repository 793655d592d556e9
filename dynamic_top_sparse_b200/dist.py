"""Host-side helpers for running the decode step on several GPUs.

The step partitions into independent units (sequence b, KV head g) with no
exchange between them, so N GPUs run N independent shards (one process per
GPU, torch.distributed for the barrier and the timing reduction only).
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


def shard_units(B: int, H_kv: int, world: int, rank: int) -> list[tuple[int, int]]:
    """(sequence, KV head) units owned by `rank`: whole sequences are dealt
    round-robin first; when there are fewer sequences than ranks, KV heads
    of each sequence are dealt across the ranks that share it."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    units = [(b, g) for b in range(B) for g in range(H_kv)]
    if B >= world:
        return [(b, g) for (b, g) in units if b % world == rank]
    return [u for i, u in enumerate(units) if i % world == rank]


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own synthetic sequences (independent replicas)."""
    return int(base) * 1000003 + int(rank)

"""The multi-GPU host logic on world_size-2 gloo ranks on CPU: barrier and
max-over-ranks timing of the replicated bench, per-rank seeds, and the
exchanges of the context-sharded step."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dynamic_top_sparse_b200 import dist as rdist


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rdist.barrier(world)
        t = rdist.allreduce_max(1.5 + rank, world)
        s = rdist.allreduce_sum(10.0, world)
        q.put((rank, t, s))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, s in res:
        assert t == 2.5          # slowest rank
        assert s == 20.0


def test_rank_seeds_are_distinct_and_rank0_keeps_the_base():
    seeds = [rdist.rank_seed(0, r) for r in range(8)]
    assert seeds[0] == 0                      # rank 0 serves the single-GPU workload
    assert len(set(seeds)) == 8
    assert not set(seeds) & {rdist.rank_seed(1, r) for r in range(8)}


def _shard_worker(rank, world, port, q):
    """The context-shard exchanges on gloo ranks: histogram sum, candidate
    gather (different counts per rank and head), partial gather."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from dynamic_top_sparse_b200.shard import TorchComm
        comm = TorchComm()
        hist = torch.full((6, 640), float(rank + 1), dtype=torch.float64)
        comm.allreduce_sum_(hist)
        nh, width = 3, 10
        keys = torch.arange(nh * width, dtype=torch.int64).view(nh, width) + 1000 * rank
        counts = torch.tensor([rank + 1, 0, 2 * rank], dtype=torch.int32)
        all_keys, all_counts = comm.gather_candidates(keys, counts)
        part = torch.full((nh, 132), float(rank))
        parts = comm.allgather(part)
        q.put((rank, hist[0, 0].item(), all_keys.tolist(), all_counts.tolist(), parts[:, 0, 0].tolist()))
    finally:
        dist.destroy_process_group()


def test_shard_exchanges_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, h, keys, counts, parts in res:
        assert h == 3.0                                   # 1 + 2
        assert counts == [1 + 2, 0, 0 + 2]                # per head, summed over ranks
        # head 0: rank 0's first key, then rank 1's first two; head 2: rank 1's first two
        assert keys[0][:3] == [0, 1000, 1001]
        assert keys[2][:2] == [1020, 1021]
        assert parts == [0.0, 1.0]


def test_gather_candidates_local():
    """The same placement in one process: shard p's first counts[p][h]
    candidates of head h follow those of shards 0 .. p-1."""
    from dynamic_top_sparse_b200.shard import gather_candidates
    k0 = torch.tensor([[1, 2, 3], [4, 5, 6]])
    k1 = torch.tensor([[7, 8, 9], [10, 11, 12]])
    keys, counts = gather_candidates([k0, k1], [torch.tensor([2, 0], dtype=torch.int32),
                                                torch.tensor([1, 3], dtype=torch.int32)])
    assert counts.tolist() == [3, 3]
    assert keys[0].tolist() == [1, 2, 7]
    assert keys[1].tolist() == [10, 11, 12]

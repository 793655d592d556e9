"""Context-sharded decode step: one long sequence split over P GPUs.

Each rank holds a contiguous range of every sequence's tokens (its own K/V
and index-key caches, shard_off[b] = the global position of its token 0) and
runs the C-ABI shard calls of librtp.so; between them the ranks exchange

  1. the per-head level-1 mass histograms (an all-reduce sum, fp64,
     B * H_q * 640 values),
  2. the boundary-bin candidates of every head (an all-gather of counts,
     then of the keys padded to the largest count), and
  3. the per-head attention partials (an all-gather of B * H_q records of
     132 floats),

and every rank ends with the output of the whole sequence.  The GPU work is
all in the library; this module only moves the exchanged buffers.  The
exchanges go through a `comm` object: `TorchComm` wraps torch.distributed
(NCCL over NVLink between GPUs, or gloo), and `run_local_shards` runs P
shards in one process on one device, exchanging by plain tensor operations
(the single-GPU check of the same arithmetic).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import ops


@dataclass
class Shard:
    """One rank's part of a step: its caches and workspace.  seq_lens in
    dims are the shard's own token counts; glob_len the sequences' lengths."""
    dims: ops.Dims
    q: torch.Tensor          # [B, H_q, d] fp32 pre-RoPE
    q_rope: torch.Tensor     # [B, H_q, d] fp32 post-RoPE
    k: torch.Tensor          # this shard's caches [B, H_kv, N_shard, d] bf16
    v: torch.Tensor
    kidx: torch.Tensor       # [B, H_kv, N_shard, r] bf16
    Wq: torch.Tensor         # [H_q, r, d] fp32
    head_class: object
    shard_off: torch.Tensor  # [B] int32, device
    glob_len: torch.Tensor   # [B] int32, device
    ws: ops.Workspace
    opts: ops.Opts | None = None


def gather_candidates(keys: list, counts: list):
    """Every shard's boundary candidates of each head side by side:
    keys[p] [n_heads, W_p] int64, counts[p] [n_heads] int32 ->
    (all_keys [n_heads, stride] int64, all_counts [n_heads] int32)."""
    cnt = torch.stack([c.to(torch.int64) for c in counts])          # [P, n_heads]
    total = cnt.sum(0)
    nh = cnt.shape[1]
    stride = max(1, int(total.max()))
    out = torch.zeros((nh, stride), dtype=torch.int64, device=cnt.device)
    start = torch.cumsum(cnt, 0) - cnt                                # exclusive, per shard
    rows = torch.arange(nh, device=cnt.device)[:, None]
    for p, k in enumerate(keys):
        w = min(k.shape[1], int(cnt[p].max()) if cnt.shape[1] else 0)
        if w == 0:
            continue
        j = torch.arange(w, device=cnt.device)[None, :]
        valid = j < cnt[p][:, None]
        dest = start[p][:, None] + j
        out[rows.expand(-1, w)[valid], dest[valid]] = k[:, :w][valid]
    return out, total.to(torch.int32)


def phase_scan(s: Shard, p: float) -> torch.Tensor:
    ops.shard_scan(s.dims, s.q, s.kidx, s.Wq, s.head_class, p, s.ws, s.opts)
    return ops.shard_hist(s.dims, s.ws)


def phase_collect(s: Shard, p: float):
    ops.shard_collect(s.dims, s.kidx, s.head_class, p, s.shard_off, s.ws, s.opts)
    return ops.shard_cands(s.dims, s.ws)


def phase_finish(s: Shard, p: float, window: int, n_sink: int, all_keys, all_counts) -> torch.Tensor:
    nh = s.dims.B * s.dims.H_q
    part = torch.empty((nh, ops.PART_STRIDE), dtype=torch.float32, device=s.q.device)
    ops.shard_finish(s.dims, s.q_rope, s.k, s.v, s.kidx, s.head_class, p, window, n_sink, s.shard_off,
                     s.glob_len, all_keys, all_counts, part, s.ws, s.opts)
    return part


def run_local_shards(shards: list, p: float, window: int, n_sink: int, out: torch.Tensor) -> list:
    """All shards of a step in one process on one device, in lockstep; the
    exchanges are tensor operations.  Returns each shard's partials."""
    all_keys = all_counts = None
    if p < 1.0:          # p >= 1 keeps every token: no threshold, no exchanges before the partials
        hists = [phase_scan(s, p) for s in shards]
        total = torch.stack(hists).sum(0)
        for h in hists:
            h.copy_(total)
        cands = [phase_collect(s, p) for s in shards]
        all_keys, all_counts = gather_candidates([c[0] for c in cands], [c[1] for c in cands])
    parts = [phase_finish(s, p, window, n_sink, all_keys, all_counts) for s in shards]
    ops.merge_shards(torch.stack(parts).contiguous(), out)
    return parts


class TorchComm:
    """Exchanges over torch.distributed (every rank calls every method, in
    the same order)."""

    def __init__(self, group=None):
        self.group = group
        self.world = torch.distributed.get_world_size(group)

    def allreduce_sum_(self, t: torch.Tensor):
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM, group=self.group)

    def allgather(self, t: torch.Tensor) -> torch.Tensor:
        out = [torch.empty_like(t) for _ in range(self.world)]
        torch.distributed.all_gather(out, t.contiguous(), group=self.group)
        return torch.stack(out)

    def gather_candidates(self, keys: torch.Tensor, counts: torch.Tensor):
        cnt_all = self.allgather(counts.to(torch.int32).contiguous())             # [P, n_heads]
        width = max(1, int(cnt_all.max()))
        padded = torch.zeros((keys.shape[0], width), dtype=torch.int64, device=keys.device)
        w = min(width, keys.shape[1])
        padded[:, :w] = keys[:, :w]
        keys_all = self.allgather(padded)                                          # [P, n_heads, width]
        return gather_candidates(list(keys_all), list(cnt_all))


def sharded_decode_step(comm, s: Shard, p: float, window: int, n_sink: int, out: torch.Tensor) -> torch.Tensor:
    """This rank's part of a context-sharded step; every rank ends with the
    whole step's output in `out`.  Returns this rank's partials."""
    all_keys = all_counts = None
    if p < 1.0:          # p >= 1 keeps every token: no threshold, no exchanges before the partials
        hist = phase_scan(s, p)
        comm.allreduce_sum_(hist)
        keys, counts = phase_collect(s, p)
        all_keys, all_counts = comm.gather_candidates(keys, counts)
    part = phase_finish(s, p, window, n_sink, all_keys, all_counts)
    parts = comm.allgather(part)
    ops.merge_shards(parts.contiguous(), out)
    return part

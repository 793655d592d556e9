"""Seeded synthetic inputs for the sparse decode step.

This module only draws random numbers and arranges them into the shapes,
dtypes and needle structure of the workloads the decode step is measured
on.  It performs none of the step's arithmetic (no projection of a query or
key through an indexer, no score, no softmax, no selection, no attention):
where a needle must stand out for a query head, the generator first draws
the head's low-dimensional query direction ``qi`` and then builds a
pre-RoPE query that projects onto it (a least-squares solve), so it never
multiplies a query by a projector.  Both the CUDA path and the CPU oracle
consume exactly these tensors.

Workloads (32 query / 4 KV heads, head dim 128, 16-dim indexer, the
attention shape of Qwen3-30B-A3B; contexts and sparsity levels of the
"Full Attention Strikes Back" experiments):

  1  parity case: B=1, 4 q / 1 KV head, N=4096, fp32, all retrieval,
     8 needle keys k = 3*q_dir + N(0, 0.3^2), p=0.9, no RoPE.
  2  64K context, B=1, KV0 retrieval, KV1-3 local (window 4096 + 4 sinks),
     4 needles per retrieval q head at scale 3, p=0.9, bf16, RoPE base 1e6.
  3  512K context, KV0 and KV2 retrieval; the 16 retrieval q heads are
     ranked j=0..15 with round(4*1024^(j/15)) needles at scale
     4*0.3^(j/15) (very peaked to broad), p=0.9.
  4  48 layers, B=8, 128K per sequence, one retrieval KV head per layer
     (seeded pick), 4 needles per retrieval q head per sequence at scale 3.
  5  1M context, B=1, all 4 KV heads retrieval, needle mix over j=0..31
     (round(4*1024^(j/31)) needles, scale 4*0.3^(j/31)), p swept over
     {0.8, 0.9, 0.95, 1.0}.

A needle at "scale s" lifts the head's index logit by s*ln(N)/2 nats
(plus N(0, 0.25^2) jitter) above its N(0, ~0.35^2) background, and lifts
its full-attention logit by the same amount, so the indexer and the full
attention agree on where the needles are.
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field

import numpy as np
import torch

HEAD_LOCAL = 0
HEAD_RETRIEVAL = 1

D = 128
R = 16
ROPE_BASE = 1.0e6
NEEDLE_JITTER = 0.25


@dataclass
class Spec:
    name: str
    B: int
    H_q: int
    H_kv: int
    N: int
    kv_dtype: str = "bf16"
    idx_dtype: str = "bf16"
    d: int = D
    r: int = R
    p: float = 0.9
    window: int = 4096
    n_sink: int = 4
    layers: int = 1
    rope: bool = True
    # head_class per layer: list of lists of length H_kv
    head_class: list = field(default_factory=list)
    # needle recipe: "direction", "uniform", "ranked" or "none"
    needles: str = "uniform"
    needles_per_head: int = 4
    needle_scale: float = 3.0
    seq_lens: list | None = None    # ragged lengths (default: all N)
    N_max: int | None = None


# The workloads, by key: the shapes of the pages' 64K-1M decode settings plus
# a small fp32 case that the oracle finishes in seconds.
WORKLOADS = ("ctx4k-fp32", "ctx64k", "ctx512k", "ctx128k-b8-48layer", "ctx1m")


def spec_for(key: str) -> Spec:
    if key == "ctx4k-fp32":
        return Spec("4K ctx, B1, 4q/1kv, fp32, all retrieval, 8 planted needles, p=0.9",
                    B=1, H_q=4, H_kv=1, N=4096, kv_dtype="f32", idx_dtype="f32",
                    rope=False, head_class=[[1]], needles="direction", window=4096, n_sink=4)
    if key == "ctx64k":
        return Spec("64K ctx, B1, 32q/4kv, bf16, KV0 retrieval + 3 local (w4096+4 sinks), p=0.9",
                    B=1, H_q=32, H_kv=4, N=65536, head_class=[[1, 0, 0, 0]],
                    needles="uniform", needles_per_head=4, needle_scale=3.0)
    if key == "ctx512k":
        return Spec("512K ctx, B1, 32q/4kv, bf16, KV0+KV2 retrieval, ranked needles, p=0.9",
                    B=1, H_q=32, H_kv=4, N=524288, head_class=[[1, 0, 1, 0]],
                    needles="ranked")
    if key == "ctx128k-b8-48layer":
        return Spec("48 layers, B8, 128K ctx, 32q/4kv, bf16, 1 retrieval KV head/layer, p=0.9",
                    B=8, H_q=32, H_kv=4, N=131072, layers=48, head_class=[],
                    needles="uniform", needles_per_head=4, needle_scale=3.0)
    if key == "ctx1m":
        return Spec("1M ctx, B1, 32q/4kv, bf16, all retrieval, ranked needles",
                    B=1, H_q=32, H_kv=4, N=1048576, head_class=[[1, 1, 1, 1]],
                    needles="ranked")
    raise ValueError(f"unknown workload {key!r}; one of {WORKLOADS}")


def layer_head_class(spec: Spec, layer: int, seed: int) -> np.ndarray:
    """Head classes of one layer; the 48-layer workload picks its one
    retrieval KV head per layer with a seeded uniform draw."""
    if spec.head_class:
        hc = spec.head_class[layer % len(spec.head_class)]
        return np.asarray(hc, dtype=np.uint8)
    g = torch.Generator().manual_seed(_sub(seed, 4, layer, 99))
    pick = int(torch.randint(0, spec.H_kv, (1,), generator=g))
    hc = np.zeros(spec.H_kv, np.uint8)
    hc[pick] = HEAD_RETRIEVAL
    return hc


def _sub(*xs) -> int:
    """Derive a sub-seed from integers (splitmix-style, deterministic)."""
    h = 0x9E3779B97F4A7C15
    for x in xs:
        h ^= (int(x) + 0x9E3779B97F4A7C15 + (h << 6) + (h >> 2)) & 0xFFFFFFFFFFFFFFFF
        h = (h * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    return h & 0x7FFFFFFFFFFFFFFF


def _tdtype(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


@dataclass
class Case:
    spec: Spec
    layer: int
    q: torch.Tensor              # [B, H_q, d] fp32, pre-RoPE
    q_rope: torch.Tensor | None  # [B, H_q, d] fp32, post-RoPE (None: no RoPE)
    k_cache: torch.Tensor        # [B, H_kv, N_max, d] kv dtype (post-RoPE)
    v_cache: torch.Tensor        # [B, H_kv, N_max, d] kv dtype
    kidx_cache: torch.Tensor     # [B, H_kv, N_max, r] idx dtype
    W_q_idx: torch.Tensor        # [H_q, r, d] fp32
    W_k_idx: torch.Tensor        # [H_kv, r, d] fp32
    k_pre_new: torch.Tensor      # [B, H_kv, 1, d] kv dtype: pre-RoPE key of the current token
    head_class: np.ndarray       # [H_kv] uint8
    seq_lens: torch.Tensor       # [B] int32
    p: float
    window: int
    n_sink: int
    needles: dict                # (b, h) -> np.ndarray of needle positions
    k_pre_all: torch.Tensor | None = None  # ctx4k-fp32: pre-RoPE keys of every row (index keys come from the append step)

    @property
    def B(self):
        return self.spec.B

    @property
    def N_max(self):
        return self.k_cache.shape[2]


def rope_neox(x: torch.Tensor, pos: torch.Tensor, base: float = ROPE_BASE) -> torch.Tensor:
    """Half-split (NeoX / Qwen) rotary embedding of x [..., d] at positions
    pos (broadcast over leading dims), computed in fp64.  Input plumbing
    only: the library applies no RoPE itself."""
    d = x.shape[-1]
    half = d // 2
    inv = base ** (-torch.arange(half, dtype=torch.float64, device=x.device) * 2.0 / d)
    ang = pos.to(torch.float64)[..., None] * inv
    c, s = torch.cos(ang), torch.sin(ang)
    x = x.to(torch.float64)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def _randn(shape, gen, device, std=1.0, dtype=torch.float32):
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _needle_plan(spec: Spec, head_class: np.ndarray, N: int):
    """(h -> (count, scale)) for every retrieval query head."""
    G = spec.H_q // spec.H_kv
    ret_heads = [h for h in range(spec.H_q) if head_class[h // G] == HEAD_RETRIEVAL]
    plan = {}
    if spec.needles in ("uniform",):
        for h in ret_heads:
            plan[h] = (spec.needles_per_head, spec.needle_scale)
    elif spec.needles == "ranked":
        J = len(ret_heads)
        for j, h in enumerate(ret_heads):
            f = j / max(J - 1, 1)
            plan[h] = (int(round(4 * 1024 ** f)), 4.0 * 0.3 ** f)
    return plan


def make_case(spec: Spec | str, device="cpu", seed: int = 0, layer: int = 0) -> Case:
    """Build one layer of synthetic decode-step inputs, seeded by
    (seed, workload name, layer).  Large cases should be built with
    device='cuda' (torch's CUDA generator is deterministic for a seed)."""
    if isinstance(spec, str):
        spec = spec_for(spec)
    dev = torch.device(device)
    B, H_q, H_kv, d, r, N = spec.B, spec.H_q, spec.H_kv, spec.d, spec.r, spec.N
    N_max = spec.N_max or N
    G = H_q // H_kv
    head_class = layer_head_class(spec, layer, seed)
    base = _sub(seed, zlib.crc32(spec.name.encode()), layer)
    gen = torch.Generator(device=dev).manual_seed(base)
    cpu_gen = torch.Generator().manual_seed(_sub(base, 1))
    kvdt, idt = _tdtype(spec.kv_dtype), _tdtype(spec.idx_dtype)
    if spec.seq_lens is not None:
        seq_lens = torch.tensor(spec.seq_lens, dtype=torch.int32)
    else:
        seq_lens = torch.full((B,), N, dtype=torch.int32)
    lens = seq_lens.tolist()
    tau = 1.0 / math.sqrt(d)

    W_k_idx = _randn((H_kv, r, d), cpu_gen, "cpu", std=1.0 / math.sqrt(d))
    k_pre_new = _randn((B, H_kv, 1, d), cpu_gen, "cpu").to(kvdt)
    needles: dict = {}

    if spec.needles == "direction":
        # q, k, v ~ N(0,1); one 16x128 query projector shared by the group's
        # heads; 8 needle keys k = 3*q_dir + N(0, 0.3^2), needle i for head i mod G.
        W1 = _randn((r, d), cpu_gen, "cpu", std=1.0 / math.sqrt(d))
        W_q_idx = W1.expand(H_q, r, d).contiguous()
        q = _randn((B, H_q, d), cpu_gen, "cpu")
        k_pre = _randn((B, H_kv, N_max, d), cpu_gen, "cpu")
        v = _randn((B, H_kv, N_max, d), cpu_gen, "cpu")
        for b in range(B):
            pos = torch.randperm(lens[b] - 1, generator=cpu_gen)[:8]
            for i in range(8):
                h = i % H_q
                g = h // G
                qdir = q[b, h] / q[b, h].norm()
                t = int(pos[i])
                k_pre[b, g, t] = 3.0 * qdir + 0.3 * _randn((d,), cpu_gen, "cpu")
                needles.setdefault((b, h), []).append(t)
        case = Case(spec, layer, q.to(dev), None, k_pre.to(kvdt).to(dev), v.to(kvdt).to(dev),
                    torch.zeros((B, H_kv, N_max, r), dtype=idt, device=dev),
                    W_q_idx.to(dev), W_k_idx.to(dev), k_pre_new.to(dev), head_class,
                    seq_lens.to(dev), spec.p, spec.window, spec.n_sink,
                    {k: np.asarray(sorted(v_)) for k, v_ in needles.items()},
                    k_pre_all=k_pre.to(kvdt).to(dev))
        return case

    # --- the bf16 workloads and generic cases: needles planted in index space
    W_q_idx = _randn((H_q, r, d), cpu_gen, "cpu", std=1.0 / math.sqrt(d)).to(torch.float64)
    qi = torch.randn((B, H_q, r), generator=cpu_gen, dtype=torch.float64)
    noise = torch.randn((B, H_q, d), generator=cpu_gen, dtype=torch.float64)
    # q_pre = W^+ qi + (I - W^+ W) n: a pre-RoPE query whose projection is qi.
    Wp = torch.linalg.pinv(W_q_idx)                       # [H_q, d, r]
    null = torch.eye(d, dtype=torch.float64) - Wp @ W_q_idx  # [H_q, d, d]
    q64 = torch.einsum("hdr,bhr->bhd", Wp, qi) + torch.einsum("hde,bhe->bhd", null, noise)
    q = q64.to(torch.float32)
    if spec.rope:
        pos_q = (seq_lens.to(torch.float64) - 1.0)[:, None]
        q_rope = rope_neox(q.to(torch.float64), pos_q).to(torch.float32)
    else:
        q_rope = None
    W_q_idx = W_q_idx.to(torch.float32)

    kidx = _randn((B, H_kv, N_max, r), gen, dev)
    k_cache = _randn((B, H_kv, N_max, d), gen, dev)
    v_cache = _randn((B, H_kv, N_max, d), gen, dev, dtype=kvdt)

    plan = _needle_plan(spec, head_class, N)
    qa = (q_rope if q_rope is not None else q)
    for b in range(B):
        Nb = lens[b]
        if Nb < 2:
            continue
        for h, (cnt, scale) in plan.items():
            g = h // G
            cnt = min(cnt, Nb - 1)
            if cnt <= 0:
                continue
            pos = torch.randperm(Nb - 1, generator=cpu_gen)[:cnt]
            lift = scale * math.log(Nb) / 2.0 + NEEDLE_JITTER * torch.randn(cnt, generator=cpu_gen, dtype=torch.float64)
            qd = qi[b, h] / (qi[b, h] @ qi[b, h])              # qi / |qi|^2
            add_idx = (lift[:, None] / tau) * qd[None, :]       # [cnt, r]
            qa_h = qa[b, h].to(torch.float64)
            add_k = (lift[:, None] / tau) * (qa_h / (qa_h @ qa_h))[None, :]
            pd = pos.to(dev)
            kidx[b, g].index_add_(0, pd, add_idx.to(torch.float32).to(dev))
            k_cache[b, g].index_add_(0, pd, add_k.to(torch.float32).to(dev))
            needles[(b, h)] = np.sort(pos.numpy())
    c = lambda t: t.contiguous()
    return Case(spec, layer, c(q.to(dev)), None if q_rope is None else c(q_rope.to(dev)),
                c(k_cache.to(kvdt)), c(v_cache), c(kidx.to(idt)), c(W_q_idx.to(dev)), c(W_k_idx.to(dev)),
                c(k_pre_new.to(dev)), head_class, seq_lens.to(dev), spec.p, spec.window,
                spec.n_sink, needles)


def small_spec(B=2, H_q=8, H_kv=2, N=1000, kv_dtype="bf16", idx_dtype="bf16",
               head_class=(1, 0), p=0.9, window=64, n_sink=4, seq_lens=None,
               needles="uniform", needles_per_head=3, needle_scale=2.0, rope=True,
               N_max=None, name="small") -> Spec:
    """A small generic case for parity tests (ragged lengths allowed)."""
    return Spec(name, B=B, H_q=H_q, H_kv=H_kv, N=N, kv_dtype=kv_dtype, idx_dtype=idx_dtype,
                p=p, window=window, n_sink=n_sink, rope=rope, head_class=[list(head_class)],
                needles=needles, needles_per_head=needles_per_head, needle_scale=needle_scale,
                seq_lens=seq_lens, N_max=N_max)


def random_logits(n_heads: int, N: int, kind: str, seed: int = 0) -> np.ndarray:
    """Index logits z [n_heads, N] (fp32 values) for exercising the top-p
    threshold alone: 'normal' (N(0, 0.35^2)), 'peaked' (a few tokens
    10-20 nats up), 'ties' (values on a coarse grid, many exact ties),
    'uniform' (all equal), 'wide' (N(0, 8^2))."""
    g = np.random.default_rng(_sub(seed, N, n_heads, zlib.crc32(kind.encode())))
    if kind == "normal":
        z = g.normal(0.0, 0.35, (n_heads, N))
    elif kind == "peaked":
        z = g.normal(0.0, 0.35, (n_heads, N))
        for h in range(n_heads):
            k = max(1, min(N, int(g.integers(1, 9))))
            pos = g.choice(N, size=k, replace=False)
            z[h, pos] += g.uniform(10.0, 20.0, size=k)
    elif kind == "ties":
        z = g.integers(-8, 8, (n_heads, N)).astype(np.float64) * 0.25
    elif kind == "uniform":
        z = np.full((n_heads, N), 0.75)
    elif kind == "wide":
        z = g.normal(0.0, 8.0, (n_heads, N))
    else:
        raise ValueError(kind)
    return z.astype(np.float32)

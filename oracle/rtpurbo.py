"""Plain CPU oracle for the RTPurbo per-head sparse decode step.

TEST INFRASTRUCTURE ONLY. This module is imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline / reference leg of
``bench.py``; nothing in the product path (the CUDA library and its Python
binding) may import or call it.  It shares no code with the CUDA path.

It restates, as slowly and plainly as possible, what the method computes,
following these descriptions of "Full Attention Strikes Back: Transferring
Full Attention into Sparse within Hundred Training Steps" (arXiv 2605.16928):

* the gist.science technical summary (Japanese and Italian versions),
  Method section 1 "head specialisation and offline calibration"
  (retrieval heads vs local heads; local heads use a sliding window with
  attention sinks, retrieval heads switch to dynamic sparse selection at
  decode);
* same summary, Method section 2 "low-dimensional token indexing"
  (a 16-dimensional projection of query and key, applied before RoPE);
* same summary, Method section 3 "dynamic top-p vs static top-k"
  (accumulate attention mass in the low-dimensional space until it reaches
  p, e.g. 0.9);
* same summary, Method section 4 "two-stage training", stage 1 (the
  low-dimensional distribution is trained to imitate the full-attention
  softmax: it is a softmax over all cached tokens);
* same summary, Method section 5 "hardware-aware kernels" (sparse decode:
  attention over the selected tokens only);
* the arXiv abstract (retrieval heads keep the full KV cache; a
  16-dimensional indexer).

Numbers: inputs are fp32 or bf16 values (bf16 widens exactly to fp32); all
arithmetic is fp64 and results are returned in fp64.  The selection rule is
the plain definition (a full stable sort by descending score, then a
cumulative sum), not the histogram method the GPU uses.

Readings where those descriptions are silent (each one is a parameter or a stated
rule below): index and attention softmax scale 1/sqrt(d); ties in the
descending order go to the lower token index; p >= 1 keeps every token and
p <= 0 keeps the single top token; retrieval heads choose among all N cached
tokens (no forced sinks or window); selection is per query head; the
softmax is renormalised over the kept set; the local set is the union of
the first ``n_sink`` positions and the last ``window`` positions.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, brute force, hand-derived fixtures in ``tests/golden/`` or
independent formulations.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

HEAD_LOCAL = 0
HEAD_RETRIEVAL = 1


def default_scale(d: int) -> float:
    """Softmax temperature 1/sqrt(d) (standard attention scale; the method's
    descriptions state none, and stage-1 training makes the index softmax imitate the
    full-attention one, so the same scale serves both)."""
    return 1.0 / math.sqrt(d)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def round_to_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits and fp32's exponent range.  Written
    from the format's definition: x = m * 2**e with 0.5 <= |m| < 1, so
    x * 2**(8 - e) has 8 integer bits; ``np.rint`` rounds half to even.
    Below the smallest normal (2**-126) the spacing is fixed at 2**-133.
    Magnitudes that round past the largest finite value become inf.
    """
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, -125)
    r = np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)
    big = np.abs(r) >= 2.0 ** 128
    if np.any(big):
        r = np.where(big, np.copysign(np.inf, x), r)
    return r


def round_to_f32(x) -> np.ndarray:
    """Round fp64 values to the nearest fp32 value (numpy's cast is
    round-to-nearest-even), returned as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(x, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return round_to_f32(x)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# a0 / a1: the low-dimensional indexer (Method section 2)
# ---------------------------------------------------------------------------

def project_index_key(k_pre: np.ndarray, W_k_idx: np.ndarray) -> np.ndarray:
    """k_idx = W_k_idx . k, with k the pre-RoPE key ([..., d]) and W_k_idx
    the [r, d] projector of its KV head.  fp64, unrounded."""
    return np.asarray(k_pre, np.float64) @ np.asarray(W_k_idx, np.float64).T


def append_index_keys(kidx_cache: np.ndarray, k_pre: np.ndarray,
                      W_k_idx: np.ndarray, pos, idx_dtype: str,
                      head_class=None) -> np.ndarray:
    """Write the index keys of T new tokens into a copy of the cache.

    kidx_cache: [B, H_kv, N_max, r]; k_pre: [B, H_kv, T, d] (pre-RoPE);
    W_k_idx: [H_kv, r, d]; pos: [B] first row to write.  Rows
    [pos_b, pos_b + T) of every retrieval KV head get W_k_idx[g] . k,
    computed in fp64 and rounded once to the cache dtype.  Only retrieval
    heads keep index keys (the arXiv abstract: only retrieval heads keep the
    whole KV cache); rows of local heads are left as they were.
    """
    out = np.array(kidx_cache, dtype=np.float64, copy=True)
    B, H_kv, T, _ = k_pre.shape
    for b in range(B):
        p0 = int(pos[b])
        for g in range(H_kv):
            if head_class is not None and head_class[g] != HEAD_RETRIEVAL:
                continue
            out[b, g, p0:p0 + T, :] = round_to(
                project_index_key(k_pre[b, g], W_k_idx[g]), idx_dtype)
    return out


def query_index(q_pre: np.ndarray, W_q_idx_h: np.ndarray) -> np.ndarray:
    """q_idx = W_q_idx[h] . q_h (pre-RoPE query of head h, [d]) -> [r]."""
    return np.asarray(W_q_idx_h, np.float64) @ np.asarray(q_pre, np.float64)


def index_logits(q_idx: np.ndarray, kidx_rows: np.ndarray, scale: float) -> np.ndarray:
    """z_t = scale * (q_idx . k_idx_t) for each cached row t ([N, r]).

    Each row's dot product is summed the same way (an elementwise product
    reduced along the row), so equal keys give exactly equal scores and the
    tie rule decides between them; a blocked matrix-vector product may round
    rows of different blocks differently."""
    k = np.asarray(kidx_rows, np.float64)
    q = np.asarray(q_idx, np.float64)
    return scale * np.sum(k * q[None, :], axis=1)


# ---------------------------------------------------------------------------
# a3 / a4 / a5: softmax mass and the top-p rule (Method section 3)
# ---------------------------------------------------------------------------

def softmax_mass(z: np.ndarray) -> np.ndarray:
    """pi_t = exp(z_t - max z) / sum_u exp(z_u - max z)."""
    z = np.asarray(z, np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def descending_order(z: np.ndarray) -> np.ndarray:
    """Token indices by descending score; equal scores by ascending index."""
    z = np.asarray(z, np.float64)
    return np.lexsort((np.arange(z.shape[0]), -z))


@dataclass
class Selection:
    kept: np.ndarray      # kept token indices, in descending-score order
    order: np.ndarray     # all token indices in descending-score order
    excl: np.ndarray      # excl[i] = mass of order[:i] (mass strictly before)
    pi: np.ndarray        # softmax mass per token (token order)

    @property
    def mass(self) -> float:
        return float(self.pi[self.kept].sum())

    def ambiguous(self, p: float, tol: float) -> np.ndarray:
        """Tokens whose cumulative mass before them lies within tol of p:
        the only ones whose membership may differ under rounding."""
        return self.order[np.abs(self.excl - p) <= tol]


def topp_select(z: np.ndarray, p: float) -> Selection:
    """The smallest set of tokens, taken by descending score, whose softmax
    mass reaches p.

    With the tokens in descending order and excl_i the mass strictly before
    the i-th one, the kept set is {order[i] : excl_i < p}: accumulation stops
    at the first token whose inclusion reaches p.  excl is non-decreasing,
    so this is a prefix, and it always holds order[0].  p >= 1 keeps every
    token and p <= 0 keeps order[0] alone (the summary gives p = 0.9 only as
    an example, so the ends are fixed here).
    """
    if isinstance(p, float) and math.isnan(p):
        raise ValueError("p is NaN")
    z = np.asarray(z, np.float64)
    n = z.shape[0]
    if n == 0:
        raise ValueError("no tokens")
    order = descending_order(z)
    pi = softmax_mass(z)
    excl = np.concatenate(([0.0], np.cumsum(pi[order])[:-1]))
    if p >= 1.0:
        keep = n
    elif p <= 0.0:
        keep = 1
    else:
        keep = max(1, int(np.count_nonzero(excl < p)))
    return Selection(kept=order[:keep], order=order, excl=excl, pi=pi)


def topk_select(z: np.ndarray, k: int) -> Selection:
    """The k tokens with the largest scores: the fixed-budget selection that
    the summary's Method section 3 ("dynamic top-p vs static top-k") sets
    the top-p rule against.  The first min(k, N) tokens of the same
    descending order as topp_select (equal scores by ascending index); a
    budget below one token is an error (attention over no rows is
    undefined).
    """
    k = int(k)
    if k < 1:
        raise ValueError("k < 1")
    z = np.asarray(z, np.float64)
    n = z.shape[0]
    if n == 0:
        raise ValueError("no tokens")
    order = descending_order(z)
    pi = softmax_mass(z)
    excl = np.concatenate(([0.0], np.cumsum(pi[order])[:-1]))
    return Selection(kept=order[:min(k, n)], order=order, excl=excl, pi=pi)


# ---------------------------------------------------------------------------
# a6 / a7: attention over a set of rows
# ---------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, rows, scale: float) -> np.ndarray:
    """Exact softmax attention of one query over the given cache rows only:
    o = sum_t w_t v_t, w = softmax over the rows of scale * (q . k_t)."""
    rows = np.asarray(rows, dtype=np.int64)
    if rows.size == 0:
        raise ValueError("empty row set")
    Kr = np.asarray(K)[rows].astype(np.float64)
    Vr = np.asarray(V)[rows].astype(np.float64)
    s = scale * (Kr @ np.asarray(q, np.float64))
    w = np.exp(s - s.max())
    w /= w.sum()
    return w @ Vr


def local_rows(N: int, window: int, n_sink: int) -> np.ndarray:
    """Rows a local head reads: the first n_sink positions (attention sinks)
    and the last `window` positions (current token included), as a set."""
    if window < 1 or n_sink < 0:
        raise ValueError("window >= 1 and n_sink >= 0 required")
    sinks = np.arange(0, min(n_sink, N))
    recent = np.arange(max(0, N - window), N)
    return np.union1d(sinks, recent)


# ---------------------------------------------------------------------------
# the whole decode step
# ---------------------------------------------------------------------------

@dataclass
class StepResult:
    out: np.ndarray                                   # [B, H_q, d] fp64
    selections: dict = field(default_factory=dict)    # (b, h) -> Selection
    z: dict = field(default_factory=dict)             # (b, h) -> index logits


def decode_step(q, q_rope, k_cache, v_cache, kidx_cache, W_q_idx, head_class,
                seq_lens, p: float, window: int, n_sink: int,
                idx_scale: float | None = None, attn_scale: float | None = None,
                heads=None, topk: int | None = None, force_local: bool = False) -> StepResult:
    """One decode step of one layer.

    q: [B, H_q, d] pre-RoPE query (indexer input); q_rope: [B, H_q, d]
    post-RoPE query for attention (None: q serves both); k_cache, v_cache:
    [B, H_kv, N_max, d]; kidx_cache: [B, H_kv, N_max, r]; W_q_idx:
    [H_q, r, d]; head_class: [H_kv] (per KV head); seq_lens: [B].

    Query head h belongs to KV head h // (H_q // H_kv).  Local heads attend
    over local_rows(); retrieval heads score every cached token with the
    indexer, keep the top-p set (or, with ``topk``, the top-k set; p is then
    unused), and attend exactly over those rows.  With ``force_local`` a
    retrieval head attends over its kept set united with the local heads'
    rows (a serving option beside the method: sinks and window kept for every
    head).
    ``heads`` optionally restricts the computation to a list of (b, h).
    """
    q = np.asarray(q, np.float64)
    q_rope = q if q_rope is None else np.asarray(q_rope, np.float64)
    B, H_q, d = q.shape
    H_kv = k_cache.shape[1]
    G = H_q // H_kv
    isc = default_scale(d) if idx_scale is None else idx_scale
    asc = default_scale(d) if attn_scale is None else attn_scale
    out = np.full((B, H_q, d), np.nan)
    res = StepResult(out=out)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H_q)]
    for b, h in todo:
        N = int(seq_lens[b])
        g = h // G
        K = k_cache[b, g, :N]
        V = v_cache[b, g, :N]
        if head_class[g] == HEAD_RETRIEVAL:
            z = index_logits(query_index(q[b, h], W_q_idx[h]), kidx_cache[b, g, :N], isc)
            sel = topp_select(z, p) if topk is None else topk_select(z, topk)
            res.selections[(b, h)] = sel
            res.z[(b, h)] = z
            rows = sel.kept
            if force_local:
                rows = np.union1d(rows, local_rows(N, window, n_sink))
        else:
            rows = local_rows(N, window, n_sink)
        out[b, h] = attend(q_rope[b, h], K, V, rows, asc)
    return res


def dense_decode(q_rope, k_cache, v_cache, seq_lens, attn_scale: float | None = None,
                 heads=None) -> np.ndarray:
    """Full attention of every query head over all N cached rows (the
    comparison the sparse step is measured against)."""
    q_rope = np.asarray(q_rope, np.float64)
    B, H_q, d = q_rope.shape
    H_kv = k_cache.shape[1]
    G = H_q // H_kv
    asc = default_scale(d) if attn_scale is None else attn_scale
    out = np.full((B, H_q, d), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H_q)]
    for b, h in todo:
        N = int(seq_lens[b])
        g = h // G
        out[b, h] = attend(q_rope[b, h], k_cache[b, g, :N], v_cache[b, g, :N], np.arange(N), asc)
    return out


# ---------------------------------------------------------------------------
# prefill
# ---------------------------------------------------------------------------

def prefill_attention(q, k_cache, v_cache, head_class, pos0, window: int, n_sink: int,
                      attn_scale: float | None = None, rows_of=None) -> np.ndarray:
    """Attention of a prompt's query tokens during prefill (summary, Method
    section 1: local heads keep a sliding window with attention sinks at
    every step, retrieval heads keep the full KV cache).

    q: [B, H_q, T, d] post-RoPE queries of T consecutive prompt tokens; query
    i of sequence b sits at position P = pos0[b] + i.  It sees the cached
    tokens 0..P (its own key included: causal), so it is the decode step's
    attention with N = P + 1 tokens: a local head attends over
    local_rows(P + 1, window, n_sink), a retrieval head over all P + 1
    tokens.  ``rows_of`` optionally restricts the work to a list of
    (b, h, i); the other outputs stay NaN.  Returns [B, H_q, T, d] fp64.
    """
    q = np.asarray(q, np.float64)
    B, H_q, T, d = q.shape
    H_kv = k_cache.shape[1]
    G = H_q // H_kv
    asc = default_scale(d) if attn_scale is None else attn_scale
    out = np.full((B, H_q, T, d), np.nan)
    todo = rows_of if rows_of is not None else [(b, h, i) for b in range(B) for h in range(H_q)
                                                for i in range(T)]
    for b, h, i in todo:
        g = h // G
        n = int(pos0[b]) + i + 1
        if head_class[g] == HEAD_RETRIEVAL:
            rows = np.arange(n)
        else:
            rows = local_rows(n, window, n_sink)
        out[b, h, i] = attend(q[b, h, i], k_cache[b, g, :n], v_cache[b, g, :n], rows, asc)
    return out

"""GPU parity of static top-k selection (the fixed budget that the summary's
Method section 3 sets the dynamic top-p rule against) with the CPU oracle:
rtp_topk_select on given logits (exact sets, ties included) and
rtp_decode_step with the topk option (sets exact except where the GPU's
fp32 logits and the oracle's fp64 logits can order two tokens differently;
attention over the kept rows)."""
import math

import numpy as np
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import OUT_TOL, OUT_TOL_SAME_SET, GpuCase, np32, np64, oracle_kidx, within

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def _dims(B, H_q, H_kv, N_max, seq):
    return ops.make_dims(B, H_q, H_kv, N_max, seq, ops.RTP_BF16, ops.RTP_BF16)


@pytest.mark.parametrize("kind", ["normal", "ties", "uniform", "wide"])
@pytest.mark.parametrize("N", [1, 17, 4097, 40000])
@pytest.mark.parametrize("k", [1, 3, 100, 4097, 10 ** 6])
def test_topk_select(kind, N, k):
    """Counts are exact integers on both sides and the logits are the same
    fp32 values, so the kept set equals the oracle's exactly, ties
    included."""
    H = 8
    z = synth.random_logits(H, N, kind, seed=N + k)
    seq = torch.tensor([N], dtype=torch.int32).cuda()
    dims = _dims(1, H, 1, N, seq)
    ws = ops.Workspace(dims)
    idx = torch.full((1, H, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, H), dtype=torch.int32, device="cuda")
    ops.topk_select(dims, torch.from_numpy(z).cuda().view(1, H, N), [1], k, idx, cnt, ws)
    assert ws.check() == 0
    for h in range(H):
        ref = oracle.topk_select(z[h].astype(np.float64), k).kept
        n = int(cnt[0, h])
        assert n == min(k, N), (kind, N, k, h, n)
        got = idx[0, h, :n].cpu().numpy()
        assert np.array_equal(np.sort(got), np.sort(ref)), (kind, N, k, h)


def test_topk_select_ragged_batch_and_reuse():
    B, H_q, H_kv, N_max, k = 3, 16, 2, 9000, 700
    lens = [9000, 1, 4500]
    g = np.random.default_rng(5)
    z = np.round(g.normal(0, 1.0, (B, H_q, N_max)), 2).astype(np.float32)   # many ties
    z[1, :, 1:] = np.nan      # beyond N_b: must not be read
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    dims = _dims(B, H_q, H_kv, N_max, seq)
    ws = ops.Workspace(dims)
    for _ in range(2):
        idx = torch.full((B, H_q, N_max), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((B, H_q), dtype=torch.int32, device="cuda")
        ops.topk_select(dims, torch.from_numpy(z).cuda(), [1, 1], k, idx, cnt, ws)
        assert ws.check() == 0
        for b in range(B):
            for h in range(H_q):
                ref = oracle.topk_select(z[b, h, : lens[b]].astype(np.float64), k).kept
                n = int(cnt[b, h])
                assert n == min(k, lens[b])
                assert np.array_equal(np.sort(idx[b, h, :n].cpu().numpy()), np.sort(ref)), (b, h)


def _check_step_topk(gc: GpuCase, k: int, out, si, sc, heads=None):
    """Every retrieval head: |S| = min(k, N), the set equals the oracle's
    except tokens whose fp64 logit lies within the GPU logits' forward
    error of the k-th largest (where fp32 rounding can swap two tokens);
    output within 2e-3 of the oracle over its own set and within 1e-4 over
    the GPU's set.  Local heads against their window."""
    c = gc.c
    kidx = oracle_kidx(gc, c.spec.idx_dtype, True)
    q = np64(c.q)
    qr = q if c.q_rope is None else np64(c.q_rope)
    K, V, Wq = np32(c.k_cache), np32(c.v_cache), np64(c.W_q_idx)
    tau = 1 / math.sqrt(128)
    u = 2.0 ** -24
    G = gc.H_q // gc.H_kv
    o = out.cpu().numpy()
    todo = heads if heads is not None else [(b, h) for b in range(gc.B) for h in range(gc.H_q)]
    for b, h in todo:
        N = int(c.seq_lens[b])
        g = h // G
        if c.head_class[g] != oracle.HEAD_RETRIEVAL:
            rows = oracle.local_rows(N, c.window, c.n_sink)
            within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], rows, tau), OUT_TOL, f"local {b},{h}")
            continue
        qi = oracle.query_index(q[b, h], Wq[h])
        z = oracle.index_logits(qi, kidx[b, g, :N], tau)
        sel = oracle.topk_select(z, k)
        n = int(sc[b, h])
        assert n == min(k, N), (b, h, n)
        ids = si[b, h, :n].cpu().numpy()
        assert np.unique(ids).size == n and ids.min() >= 0 and ids.max() < N
        qabs = np.abs(Wq[h]) @ np.abs(q[b, h])
        bound = tau * (np.abs(kidx[b, g, :N]) @ (qabs * 130 * u + np.abs(qi) * 20 * u))
        zk = z[sel.order[min(k, N) - 1]]
        amb = set(np.nonzero(np.abs(z - zk) <= 2 * bound.max() + 1e-30)[0].tolist())
        diff = set(sel.kept.tolist()) ^ set(ids.tolist())
        assert diff <= amb, f"b={b} h={h}: {len(diff - amb)} ids differ outside the rounding window"
        within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], sel.kept, tau), OUT_TOL, f"{b},{h}")
        within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], ids, tau), OUT_TOL_SAME_SET,
               f"{b},{h} (same set)")


STEP = [
    (dict(B=2, H_q=16, H_kv=2, N=5000, head_class=(1, 0), seq_lens=[5000, 1777]), 64),
    (dict(B=1, H_q=32, H_kv=4, N=9000, head_class=(0, 1, 1, 0), window=256, n_sink=0), 1),
    (dict(B=2, H_q=8, H_kv=1, N=3000, head_class=(1,), seq_lens=[3000, 40]), 500),
    (dict(B=1, H_q=8, H_kv=2, N=2000, head_class=(1, 1), needles="none"), 2500),     # k > N: every token
    # k > N with more rows than finalize attends itself: the list pass takes them
    (dict(B=2, H_q=8, H_kv=1, N=6000, head_class=(1,), needles="none", seq_lens=[6000, 3000]), 10 ** 6),
    (dict(B=1, H_q=8, H_kv=1, N=20000, head_class=(1,), needles="none"), 9000),
    # every token of a 262K-token sequence: the list pass over every SM takes them
    (dict(B=1, H_q=8, H_kv=1, N=262200, head_class=(1,), needles="none"), 10 ** 6),
    (dict(B=2, H_q=4, H_kv=4, N=3000, head_class=(1, 0, 1, 0), kv_dtype="f32", idx_dtype="f32"), 300),
    (dict(B=2, H_q=16, H_kv=2, N=6000, head_class=(1, 0), kv_dtype="f32", idx_dtype="bf16"), 2048),
]


@pytest.mark.parametrize("i", range(len(STEP)))
def test_step_topk_small(i):
    kw, k = STEP[i]
    gc = GpuCase(synth.make_case(synth.small_spec(**kw, name=f"topk{i}")))
    gc.append_current()
    out, si, sc, _ = gc.step(0.9, topk=k)
    _check_step_topk(gc, k, out, si, sc)


@pytest.mark.slow
def test_step_topk_ctx512k():
    gc = GpuCase(synth.make_case("ctx512k", device="cuda"))
    gc.append_current()
    for k in (2048, 16):
        out, si, sc, _ = gc.step(0.9, topk=k)
        _check_step_topk(gc, k, out, si, sc)

"""GPU parity of each C-ABI call against the CPU oracle (small and ragged
sizes that still span several tiles and a ragged tail)."""
import math

import numpy as np
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import (OUT_TOL_SAME_SET, GpuCase, check_selection, np64,
                           within)

pytestmark = pytest.mark.gpu

DT = {"bf16": torch.bfloat16, "f32": torch.float32}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def _dims(B, H_q, H_kv, N_max, seq, kvdt="bf16", idt="bf16"):
    return ops.make_dims(B, H_q, H_kv, N_max, seq, ops.RTP_BF16 if kvdt == "bf16" else ops.RTP_F32,
                         ops.RTP_BF16 if idt == "bf16" else ops.RTP_F32)


# ------------------------------------------------------------------- a0

@pytest.mark.parametrize("kvdt,idt,T", [("bf16", "bf16", 1), ("bf16", "bf16", 37), ("f32", "f32", 5),
                                        ("f32", "bf16", 300), ("bf16", "f32", 2)])
def test_append_index_keys(kvdt, idt, T):
    g = torch.Generator().manual_seed(T)
    B, H_q, H_kv, N_max = 3, 8, 4, 700
    seq = torch.tensor([700, 400, 350], dtype=torch.int32).cuda()
    k = torch.randn(B, H_kv, T, 128, generator=g).to(DT[kvdt])
    W = (torch.randn(H_kv, 16, 128, generator=g) / math.sqrt(128)).float()
    cache = torch.randn(B, H_kv, N_max, 16, generator=g).to(DT[idt])
    pos = torch.tensor([0, 17, N_max - T], dtype=torch.int32)
    hc = np.array([1, 0, 1, 1], np.uint8)
    dims = _dims(B, H_q, H_kv, N_max, seq, kvdt, idt)
    ws = ops.Workspace(dims)
    out = cache.cuda()
    ops.append_index_keys(dims, k.cuda(), W.cuda(), pos.cuda(), hc, out, ws)
    assert ws.check() == 0
    ref = oracle.append_index_keys(np64(cache), np64(k), np64(W), pos.numpy(), idt, head_class=hc)
    got = np64(out)
    # Rows not written must be untouched.  Written rows differ from the fp64
    # reference by the fp32 accumulation error (128 products: at most
    # 130 u sum|W k|, u = 2^-24) plus at most one unit in the last place of
    # the cache type when that error moves the sum across a rounding
    # boundary.
    mask = np.zeros(ref.shape, bool)
    for b in range(B):
        for g in range(H_kv):
            if hc[g]:
                mask[b, g, int(pos[b]):int(pos[b]) + T] = True
    assert np.array_equal(ref[~mask], got[~mask])
    absdot = np.zeros(ref.shape)
    for b in range(B):
        for g in range(H_kv):
            absdot[b, g, int(pos[b]):int(pos[b]) + T] = np.abs(np64(k)[b, g]) @ np.abs(np64(W)[g]).T
    ulp = np.abs(ref) * (2.0 ** -7 if idt == "bf16" else 2.0 ** -23)
    bound = 130 * 2.0 ** -24 * absdot + ulp + 1e-30
    assert np.all(np.abs(ref - got) <= bound)
    if idt == "bf16":
        assert (ref == got)[mask].mean() > 0.999


# ---------------------------------------------------------------- a1 + a2

@pytest.mark.parametrize("idt", ["bf16", "f32"])
def test_index_scores(idt):
    spec = synth.small_spec(B=2, H_q=16, H_kv=2, N=5000, head_class=(1, 1), seq_lens=[5000, 4097],
                            idx_dtype=idt)
    c = synth.make_case(spec)
    gc = GpuCase(c)
    z = torch.full((2, 16, gc.N_max), float("nan"), device="cuda")
    ops.index_scores(gc.dims, gc.q, gc.Wq, gc.kidx, gc.hc, z, gc.ws)
    assert gc.ws.check() == 0
    q, Wq, kidx = np64(c.q), np64(c.W_q_idx), np64(c.kidx_cache)
    zg = z.cpu().numpy().astype(np.float64)
    tau = 1 / math.sqrt(128)
    u = 2.0 ** -24
    for b in range(2):
        N = int(c.seq_lens[b])
        for h in range(16):
            qi = oracle.query_index(q[b, h], Wq[h])
            ref = oracle.index_logits(qi, kidx[b, h // 8, :N], tau)
            # forward error bound: fp32 projection (128 terms) then fp32 dot (16 terms)
            qabs = np.abs(Wq[h]) @ np.abs(q[b, h])
            bound = tau * (np.abs(kidx[b, h // 8, :N]) @ (qabs * 130 * u + np.abs(qi) * 20 * u)) + 1e-30
            assert np.all(np.abs(zg[b, h, :N] - ref) <= bound), (b, h)
            assert np.all(np.isnan(zg[b, h, N:]))


# ------------------------------------------------------------- a3-a5

@pytest.mark.parametrize("kind", ["normal", "peaked", "ties", "uniform", "wide"])
@pytest.mark.parametrize("N", [1, 2, 15, 16, 17, 255, 4097])
@pytest.mark.parametrize("p", [1e-9, 0.5, 0.9, 1.0])
def test_topp_select(kind, N, p):
    H = 8
    z = synth.random_logits(H, N, kind, seed=N)
    seq = torch.tensor([N], dtype=torch.int32).cuda()
    dims = _dims(1, H, 1, N, seq)
    ws = ops.Workspace(dims)
    idx = torch.full((1, H, N), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, H), dtype=torch.int32, device="cuda")
    mass = torch.zeros((1, H), dtype=torch.float32, device="cuda")
    ops.topp_select(dims, torch.from_numpy(z).cuda().view(1, H, N), [1], p, idx, cnt, mass, ws)
    assert ws.check() == 0
    for h in range(H):
        sel = oracle.topp_select(z[h].astype(np.float64), p)
        ids = idx[0, h, : int(cnt[0, h])].cpu().numpy()
        if kind in ("ties", "uniform"):
            # identical fp32 logits on both sides: the tie-break decides
            # exactly, so sets agree except within the mass window
            pass
        check_selection(ids, sel, p, f"{kind} N={N} p={p} h={h}")
        assert abs(float(mass[0, h]) - float(sel.pi[ids].sum())) < 1e-5


@pytest.mark.parametrize("lift", [40.0, 100.0, 200.0])
@pytest.mark.parametrize("p", [0.5, 0.9, 0.99])
def test_topp_select_large_logits(lift, p):
    """Logits far from 0, where a level-1 bin spans several nats: peaked
    heads shifted up by `lift` nats (the softmax is unchanged, the bins are
    not) and a wide N(0, 40^2) spread.  The set rule and the mass within
    1e-5 hold over the whole accepted range |z| < 256."""
    H, N = 8, 4097
    zs = [synth.random_logits(H, N, "peaked", seed=int(lift)) + lift,
          np.clip(synth.random_logits(H, N, "wide", seed=int(lift)) * 5.0, -250.0, 250.0)]
    for z in zs:
        z = z.astype(np.float32)
        seq = torch.tensor([N], dtype=torch.int32).cuda()
        dims = _dims(1, H, 1, N, seq)
        ws = ops.Workspace(dims)
        idx = torch.full((1, H, N), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((1, H), dtype=torch.int32, device="cuda")
        mass = torch.zeros((1, H), dtype=torch.float32, device="cuda")
        ops.topp_select(dims, torch.from_numpy(z).cuda().view(1, H, N), [1], p, idx, cnt, mass, ws)
        assert ws.check() == 0
        for h in range(H):
            sel = oracle.topp_select(z[h].astype(np.float64), p)
            ids = idx[0, h, : int(cnt[0, h])].cpu().numpy()
            check_selection(ids, sel, p, f"lift={lift} p={p} h={h}")
            assert abs(float(mass[0, h]) - float(sel.pi[ids].sum())) < 1e-5


def test_topp_select_ragged_batch_and_reuse():
    """Ragged lengths across a batch, several heads per group, two calls on
    the same workspace give the same sets."""
    B, H_q, H_kv, N_max = 3, 16, 2, 9000
    lens = [9000, 1, 4500]
    g = np.random.default_rng(1)
    z = g.normal(0, 1.0, (B, H_q, N_max)).astype(np.float32)
    z[1, :, 1:] = np.nan      # beyond N_b: must not be read
    seq = torch.tensor(lens, dtype=torch.int32).cuda()
    dims = _dims(B, H_q, H_kv, N_max, seq)
    ws = ops.Workspace(dims)
    zt = torch.from_numpy(z).cuda()
    res = []
    for _ in range(2):
        idx = torch.full((B, H_q, N_max), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((B, H_q), dtype=torch.int32, device="cuda")
        ops.topp_select(dims, zt, [1, 1], 0.8, idx, cnt, None, ws)
        assert ws.check() == 0
        res.append((idx.cpu(), cnt.cpu()))
    for b in range(B):
        for h in range(H_q):
            n0, n1 = int(res[0][1][b, h]), int(res[1][1][b, h])
            s0 = set(res[0][0][b, h, :n0].tolist())
            assert s0 == set(res[1][0][b, h, :n1].tolist())
            sel = oracle.topp_select(z[b, h, : lens[b]].astype(np.float64), 0.8)
            check_selection(np.array(sorted(s0)), sel, 0.8, f"b={b} h={h}")


# ------------------------------------------------------------------ a6

@pytest.mark.parametrize("kvdt", ["bf16", "f32"])
def test_sparse_decode(kvdt):
    spec = synth.small_spec(B=2, H_q=8, H_kv=2, N=3000, head_class=(1, 0), kv_dtype=kvdt,
                            seq_lens=[3000, 1234])
    c = synth.make_case(spec)
    gc = GpuCase(c)
    g = np.random.default_rng(0)
    idx = torch.full((2, 8, gc.N_max), -1, dtype=torch.int32)
    cnt = torch.zeros((2, 8), dtype=torch.int32)
    sets = {}
    for b in range(2):
        N = int(c.seq_lens[b])
        for h in range(4):
            n = int(g.choice([1, 3, 255, 256, 257, N]))
            ids = g.choice(N, size=min(n, N), replace=False).astype(np.int32)
            sets[(b, h)] = ids
            idx[b, h, : ids.size] = torch.from_numpy(ids)
            cnt[b, h] = ids.size
    out = torch.full((2, 8, 128), 7.0, device="cuda")
    ops.sparse_decode(gc.dims, gc.q_rope, gc.k, gc.v, idx.cuda(), cnt.cuda(), gc.hc, out, gc.ws)
    assert gc.ws.check() == 0
    o = out.cpu().numpy()
    K, V, qr = np64(c.k_cache), np64(c.v_cache), np64(c.q_rope)
    for (b, h), ids in sets.items():
        ref = oracle.attend(qr[b, h], K[b, 0], V[b, 0], ids, 1 / math.sqrt(128))
        within(o[b, h], ref, OUT_TOL_SAME_SET, f"b={b} h={h}")
    assert np.all(o[:, 4:] == 7.0)    # local heads untouched


@pytest.mark.parametrize("kvdt", ["bf16", "f32"])
def test_sparse_decode_list_sizes(kvdt):
    """List lengths around the list kernel's row groups (bf16: a half-warp
    per row, 16 rows per warp and pass, so one half may have no row; f32: 8
    rows per warp and pass) and its per-head slices of 64 rows."""
    counts = [1, 2, 15, 16, 17, 33, 1023, 4999]
    spec = synth.small_spec(B=1, H_q=8, H_kv=1, N=5000, head_class=(1,), kv_dtype=kvdt, name=f"lists_{kvdt}")
    c = synth.make_case(spec)
    gc = GpuCase(c)
    g = np.random.default_rng(3)
    idx = torch.full((1, 8, gc.N_max), -1, dtype=torch.int32)
    cnt = torch.tensor([counts], dtype=torch.int32)
    sets = []
    for h, n in enumerate(counts):
        ids = g.choice(5000, size=n, replace=False).astype(np.int32)
        sets.append(ids)
        idx[0, h, :n] = torch.from_numpy(ids)
    out = torch.full((1, 8, 128), float("nan"), device="cuda")
    ops.sparse_decode(gc.dims, gc.q_rope, gc.k, gc.v, idx.cuda(), cnt.cuda(), gc.hc, out, gc.ws)
    assert gc.ws.check() == 0
    o = out.cpu().numpy()
    K, V, qr = np64(c.k_cache), np64(c.v_cache), np64(c.q_rope)
    for h, ids in enumerate(sets):
        ref = oracle.attend(qr[0, h], K[0, 0], V[0, 0], ids, 1 / math.sqrt(128))
        within(o[0, h], ref, OUT_TOL_SAME_SET, f"h={h} n={len(ids)}")


# ------------------------------------------------------------------ a7 / dense

@pytest.mark.parametrize("kvdt", ["bf16", "f32"])
@pytest.mark.parametrize("window,n_sink", [(64, 4), (1, 0), (5000, 4), (300, 400), (256, 0), (257, 1)])
def test_local_decode(kvdt, window, n_sink):
    spec = synth.small_spec(B=3, H_q=12, H_kv=3, N=2500, head_class=(0, 1, 0), kv_dtype=kvdt,
                            seq_lens=[2500, 700, 1])
    c = synth.make_case(spec)
    gc = GpuCase(c)
    out = torch.full((3, 12, 128), 7.0, device="cuda")
    ops.local_decode(gc.dims, gc.q_rope, gc.k, gc.v, gc.hc, window, n_sink, out, gc.ws)
    assert gc.ws.check() == 0
    o = out.cpu().numpy()
    K, V, qr = np64(c.k_cache), np64(c.v_cache), np64(c.q_rope)
    for b in range(3):
        N = int(c.seq_lens[b])
        rows = oracle.local_rows(N, window, n_sink)
        for h in list(range(0, 4)) + list(range(8, 12)):
            ref = oracle.attend(qr[b, h], K[b, h // 4], V[b, h // 4], rows, 1 / math.sqrt(128))
            within(o[b, h], ref, OUT_TOL_SAME_SET, f"b={b} h={h}")
        assert np.all(o[b, 4:8] == 7.0)


@pytest.mark.parametrize("kvdt", ["bf16", "f32"])
def test_dense_decode(kvdt):
    spec = synth.small_spec(B=2, H_q=16, H_kv=2, N=20000, head_class=(1, 0), kv_dtype=kvdt,
                            seq_lens=[20000, 333])
    c = synth.make_case(spec)
    gc = GpuCase(c)
    out = torch.zeros((2, 16, 128), device="cuda")
    ops.dense_decode(gc.dims, gc.q_rope, gc.k, gc.v, out, gc.ws)
    assert gc.ws.check() == 0
    ref = oracle.dense_decode(np64(c.q_rope), np64(c.k_cache), np64(c.v_cache), c.seq_lens.numpy())
    within(out.cpu().numpy(), ref, OUT_TOL_SAME_SET, "dense")

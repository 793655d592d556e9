"""Paged K/V caches: the same caches scattered into shuffled pages of a
pool, addressed through a block table.  Every entry point that reads K/V
rows must give the results of the contiguous layout (which the other GPU
tests check against the oracle): bit for bit where the kernels' arithmetic
order is fixed, within fp32 summation-order noise where kept rows are
appended by atomics (the fused step's lists)."""
import math

import numpy as np
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import OUT_TOL, GpuCase, np32, np64, within

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def page_caches(k, v, page, seed, spare=5):
    """Pools [num_pages, H_kv, page, d] holding k and v in shuffled pages,
    and the block table [B, pages per sequence]."""
    B, H_kv, N_max, d = k.shape
    npg = (N_max + page - 1) // page
    num = B * npg + spare
    g = torch.Generator().manual_seed(seed)
    table = torch.randperm(num, generator=g)[: B * npg].view(B, npg).to(torch.int32)
    pools = []
    for x in (k, v):
        xp = torch.zeros(B, H_kv, npg * page, d, dtype=x.dtype, device=x.device)
        xp[:, :, :N_max] = x
        blocks = xp.view(B, H_kv, npg, page, d).permute(0, 2, 1, 3, 4).reshape(B * npg, H_kv, page, d)
        pool = torch.full((num, H_kv, page, d), float("nan"), dtype=x.dtype, device=x.device)
        pool[table.flatten().long().to(x.device)] = blocks
        pools.append(pool.contiguous())
    return pools[0], pools[1], table.to(k.device), num


def test_page_caches_layout():
    """The helper itself: row t of (b, g) is at pool[table[b, t // P], g, t % P]."""
    k = torch.randn(2, 3, 100, 128)
    kp, _, table, _ = page_caches(k, k, 16, 1)
    for b, g, t in [(0, 0, 0), (1, 2, 99), (0, 1, 37), (1, 0, 64)]:
        assert torch.equal(kp[int(table[b, t // 16]), g, t % 16], k[b, g, t])


CASES = [
    (dict(B=2, H_q=16, H_kv=2, N=5000, head_class=(1, 0), seq_lens=[5000, 1777], window=256, n_sink=4), 16),
    (dict(B=1, H_q=32, H_kv=4, N=9000, head_class=(0, 1, 1, 0), window=1000, n_sink=4), 256),
    (dict(B=2, H_q=8, H_kv=2, N=3000, head_class=(1, 1), kv_dtype="f32", idx_dtype="f32", window=64,
          n_sink=2), 64),
]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_paged_decode_calls_match_contiguous(i):
    kw, page = CASES[i]
    gc = GpuCase(synth.make_case(synth.small_spec(**kw, name=f"paged{i}")))
    gc.append_current()
    kp, vp, table, num = page_caches(gc.k, gc.v, page, seed=i)
    pg = ops.kv_pages(table, page, num)
    popt = ops.make_opts(kv_pages=pg)
    c = gc.c
    B, H_q = gc.B, gc.H_q
    qr = gc.q_rope if gc.q_rope is not None else gc.q

    def run(fn):
        out = torch.full((B, H_q, 128), float("nan"), device="cuda")
        fn(out)
        st = gc.ws.check()
        assert st == 0, ops.error_string(st)
        return out

    # dense and local decode: bf16 caches take the same arithmetic in the
    # same order (bit-exact); the fp32-cache kernel sums its warps'
    # accumulators with shared-memory atomics, in no fixed order
    exact = gc.k.dtype == torch.bfloat16

    def same(x, y, what):
        if x.numel() == 0:
            return
        if exact:
            assert torch.equal(x, y), what
        else:
            within(x.cpu().numpy(), y.cpu().numpy(), 1e-6, what)

    a = run(lambda o: ops.dense_decode(gc.dims, qr, gc.k, gc.v, o, gc.ws))
    b = run(lambda o: ops.dense_decode(gc.dims, qr, kp, vp, o, gc.ws, popt))
    same(a, b, "dense")
    a = run(lambda o: ops.local_decode(gc.dims, qr, gc.k, gc.v, gc.hc, c.window, c.n_sink, o, gc.ws))
    b = run(lambda o: ops.local_decode(gc.dims, qr, kp, vp, gc.hc, c.window, c.n_sink, o, gc.ws, popt))
    G = H_q // gc.H_kv
    loc = [h for h in range(H_q) if c.head_class[h // G] == 0]
    same(a[:, loc], b[:, loc], "local")
    # the decode step (kept sets too), top-p and static top-k, plain and with forced local rows
    for extra in (dict(), dict(topk=200), dict(force_local=True)):
        outs = []
        for kv in (None, pg):
            sel_idx = torch.full((B, H_q, gc.N_max), -1, dtype=torch.int32, device="cuda")
            sel_cnt = torch.zeros((B, H_q), dtype=torch.int32, device="cuda")
            opts = ops.make_opts(sel_idx=sel_idx, sel_count=sel_cnt, kv_pages=kv, **extra)
            kk, vv = (gc.k, gc.v) if kv is None else (kp, vp)
            out = run(lambda o: ops.decode_step(gc.dims, gc.q, gc.q_rope, kk, vv, gc.kidx, gc.Wq, gc.hc, 0.9,
                                                c.window, c.n_sink, o, gc.ws, opts))
            outs.append((out, sel_idx, sel_cnt))
        (o0, i0, c0), (o1, i1, c1) = outs
        assert torch.equal(c0, c1), extra
        for bb in range(B):
            for h in range(H_q):
                n = int(c0[bb, h])
                assert set(i0[bb, h, :n].tolist()) == set(i1[bb, h, :n].tolist()), (extra, bb, h)
        within(o0.cpu().numpy(), o1.cpu().numpy(), 1e-5, f"step {extra}")
    # a given list (rtp_sparse_decode) over the step's kept sets
    a = run(lambda o: ops.sparse_decode(gc.dims, qr, gc.k, gc.v, i0, c0, gc.hc, o, gc.ws))
    b = run(lambda o: ops.sparse_decode(gc.dims, qr, kp, vp, i0, c0, gc.hc, o, gc.ws, popt))
    ret = [h for h in range(H_q) if c.head_class[h // G] == 1]
    same(a[:, ret], b[:, ret], "sparse")


def test_paged_prefill_matches_contiguous_and_oracle():
    B, H_q, H_kv, N, T = 2, 16, 2, 2000, 300
    g = torch.Generator(device="cuda").manual_seed(4)
    q = torch.randn(B, H_q, T, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, H_kv, N, 128, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, H_kv, N, 128, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor([2000, 1500], dtype=torch.int32, device="cuda")
    pos0 = (seq - T).to(torch.int32)
    kp, vp, table, num = page_caches(k, v, 32, seed=9)
    dims = ops.make_dims(B, H_q, H_kv, N, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims, ops.OP_PREFILL)
    hc = (1, 0)
    a = torch.empty(B, H_q, T, 128, device="cuda")
    b = torch.empty_like(a)
    ops.prefill_attention(dims, q, pos0, k, v, hc, 128, 4, a, ws)
    ops.prefill_attention(dims, q, pos0, kp, vp, hc, 128, 4, b, ws, ops.make_opts(kv_pages=ops.kv_pages(table, 32, num)))
    assert ws.check() == 0
    assert torch.equal(a, b)
    rows = [(bb, h, i) for bb in range(B) for h in (0, 5, 8, 15) for i in (0, 150, T - 1)]
    ref = oracle.prefill_attention(np64(q), np64(k), np64(v), np.array(hc, np.uint8), pos0.cpu().numpy(), 128, 4,
                                   rows_of=rows)
    o = b.cpu().numpy()
    for bb, h, i in rows:
        within(o[bb, h, i], ref[bb, h, i], 1e-4, f"{bb},{h},{i}")


def test_paged_bad_page_reported():
    """A block-table entry outside the pool is reported, not read."""
    spec = synth.small_spec(B=1, H_q=8, H_kv=1, N=600, head_class=(0,), window=64, n_sink=4)
    gc = GpuCase(synth.make_case(spec))
    kp, vp, table, num = page_caches(gc.k, gc.v, 16, seed=2)
    table[0, 5] = num + 7
    out = torch.zeros(1, 8, 128, device="cuda")
    ops.dense_decode(gc.dims, gc.q_rope, kp, vp, out, gc.ws, ops.make_opts(kv_pages=ops.kv_pages(table, 16, num)))
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG


@pytest.mark.slow
def test_paged_ctx512k_step_against_oracle():
    """The 512K workload from a paged pool (page 256): every head against
    the oracle, as in the contiguous workload test."""
    gc = GpuCase(synth.make_case("ctx512k", device="cuda"))
    gc.append_current()
    kp, vp, table, num = page_caches(gc.k, gc.v, 256, seed=3)
    gc.k, gc.v = kp, vp
    c = gc.c
    B, H_q = gc.B, gc.H_q
    sel_idx = torch.full((B, H_q, gc.N_max), -1, dtype=torch.int32, device="cuda")
    sel_cnt = torch.zeros((B, H_q), dtype=torch.int32, device="cuda")
    sel_mass = torch.zeros((B, H_q), device="cuda")
    opts = ops.make_opts(sel_idx=sel_idx, sel_count=sel_cnt, sel_mass=sel_mass,
                         kv_pages=ops.kv_pages(table, 256, num))
    out = torch.full((B, H_q, 128), float("nan"), device="cuda")
    ops.decode_step(gc.dims, gc.q, gc.q_rope, kp, vp, gc.kidx, gc.Wq, gc.hc, 0.9, c.window, c.n_sink, out, gc.ws,
                    opts)
    assert gc.ws.check() == 0
    from tests.test_gpu_step import _compare
    _compare(gc, out, sel_idx, sel_cnt, sel_mass, 0.9)

"""Context-sharded decode step on one GPU: P shards of each sequence run in
lockstep in one process (the exchanges are tensor operations; on several
GPUs they are NCCL collectives, with the same arithmetic on each rank).
The merged output and the union of the shards' kept lists are the step of
the whole sequence: checked against the oracle (set rule, output) and
against the unsharded rtp_decode_step."""
import math

import numpy as np
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, shard, synth
from tests.helpers import OUT_TOL, OUT_TOL_SAME_SET, GpuCase, check_selection, np32, np64, oracle_kidx, within

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def make_shards(gc: GpuCase, cuts):
    """Shards of every sequence at the fractions `cuts` of its length (each
    shard gets at least one token of each sequence)."""
    lens = gc.seq.cpu().tolist()
    B = gc.B
    P = len(cuts) + 1
    bounds = []
    for n in lens:
        pts = [0] + [max(1, min(n - 1, int(round(c * n)))) for c in cuts] + [n]
        for i in range(1, len(pts)):
            pts[i] = max(pts[i], pts[i - 1] + 1)        # non-empty shards
        assert pts[-1] == n, "sequence too short for the shard count"
        bounds.append(pts)
    shards = []
    for pi in range(P):
        off = [bounds[b][pi] for b in range(B)]
        cnt = [bounds[b][pi + 1] - bounds[b][pi] for b in range(B)]
        nmax = max(cnt)

        def cut(x):
            y = torch.zeros((B, x.shape[1], nmax, x.shape[3]), dtype=x.dtype, device=x.device)
            for b in range(B):
                y[b, :, :cnt[b]] = x[b, :, off[b]:off[b] + cnt[b]]
            return y.contiguous()

        seq = torch.tensor(cnt, dtype=torch.int32, device="cuda")
        k, v, kidx = cut(gc.k), cut(gc.v), cut(gc.kidx)
        dims = ops.make_dims(B, gc.H_q, gc.H_kv, nmax, seq, ops.RTP_BF16, ops.RTP_BF16)
        sel_idx = torch.full((B, gc.H_q, nmax), -1, dtype=torch.int32, device="cuda")
        sel_cnt = torch.zeros((B, gc.H_q), dtype=torch.int32, device="cuda")
        sel_mass = torch.zeros((B, gc.H_q), device="cuda")
        s = shard.Shard(dims, gc.q, gc.q_rope, k, v, kidx, gc.Wq, gc.hc,
                        torch.tensor(off, dtype=torch.int32, device="cuda"), gc.seq.clone(), ops.Workspace(dims),
                        ops.make_opts(sel_idx=sel_idx, sel_count=sel_cnt, sel_mass=sel_mass))
        s.sel = (sel_idx, sel_cnt, sel_mass, seq)
        shards.append(s)
    return shards


def run_sharded(gc, cuts, p):
    shards = make_shards(gc, cuts)
    out = torch.full((gc.B, gc.H_q, 128), float("nan"), device="cuda")
    shard.run_local_shards(shards, p, gc.c.window, gc.c.n_sink, out)
    for s in shards:
        st = s.ws.check()
        assert st == 0, ops.error_string(st)
    return out, shards


def check_against_oracle(gc, out, shards, p):
    c = gc.c
    kidx = oracle_kidx(gc, "bf16", True)
    q, qr = np64(c.q), np64(c.q_rope)
    K, V, Wq = np32(c.k_cache), np32(c.v_cache), np64(c.W_q_idx)
    tau = 1 / math.sqrt(128)
    G = gc.H_q // gc.H_kv
    o = out.cpu().numpy()
    for b in range(gc.B):
        N = int(c.seq_lens[b])
        for h in range(gc.H_q):
            g = h // G
            if c.head_class[g] != oracle.HEAD_RETRIEVAL:
                rows = oracle.local_rows(N, c.window, c.n_sink)
                within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], rows, tau), OUT_TOL, f"{b},{h}")
                continue
            z = oracle.index_logits(oracle.query_index(q[b, h], Wq[h]), kidx[b, g, :N], tau)
            sel = oracle.topp_select(z, p)
            if p < 1.0:
                ids = np.concatenate([s.sel[0][b, h, :int(s.sel[1][b, h])].cpu().numpy() for s in shards])
                _, mass = check_selection(ids, sel, p, f"b={b} h={h}")
                for s in shards:          # every shard reports the mass of the whole kept set
                    assert abs(float(s.sel[2][b, h]) - mass) < 1e-5
                # each shard lists only its own tokens
                for s in shards:
                    own = s.sel[0][b, h, :int(s.sel[1][b, h])].cpu().numpy()
                    lo = int(s.shard_off[b])
                    assert np.all((own >= lo) & (own < lo + int(s.sel[3][b])))
                within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], ids, tau), OUT_TOL_SAME_SET,
                       f"b={b} h={h} (same set)")
            within(o[b, h], oracle.attend(qr[b, h], K[b, g, :N], V[b, g, :N], sel.kept, tau), OUT_TOL, f"{b},{h}")


CASES = [
    (dict(B=2, H_q=16, H_kv=2, N=20000, head_class=(1, 0), seq_lens=[20000, 9000], window=3000, n_sink=4),
     [0.5], 0.9),
    (dict(B=1, H_q=32, H_kv=4, N=30000, head_class=(0, 1, 1, 0), window=4096, n_sink=4), [0.3, 0.55, 0.9], 0.9),
    (dict(B=2, H_q=8, H_kv=1, N=12000, head_class=(1,), seq_lens=[12000, 5000], needles_per_head=6,
          needle_scale=3.0), [0.2, 0.7], 0.5),
    (dict(B=1, H_q=16, H_kv=2, N=8000, head_class=(1, 0), window=512, n_sink=2), [0.4], 1.0),
]


@pytest.mark.parametrize("i", range(len(CASES)))
def test_sharded_step_matches_oracle_and_whole_step(i):
    kw, cuts, p = CASES[i]
    gc = GpuCase(synth.make_case(synth.small_spec(**kw, name=f"shard{i}")))
    gc.append_current()
    out, shards = run_sharded(gc, cuts, p)
    check_against_oracle(gc, out, shards, p)
    whole, _, _, _ = gc.step(p, want_sel=False)
    within(out.cpu().numpy(), whole.cpu().numpy(), OUT_TOL_SAME_SET, "sharded vs whole-sequence step")


def test_sharded_step_repeats_on_the_same_workspaces():
    kw, cuts, p = CASES[0]
    gc = GpuCase(synth.make_case(synth.small_spec(**kw, name="shard_rep")))
    gc.append_current()
    shards = make_shards(gc, cuts)
    outs = []
    for _ in range(3):
        out = torch.full((gc.B, gc.H_q, 128), float("nan"), device="cuda")
        shard.run_local_shards(shards, p, gc.c.window, gc.c.n_sink, out)
        outs.append(out)
    for s in shards:
        assert s.ws.check() == 0
    # kept ids are listed in atomic order, which sets the fp32 summation order
    within(outs[0].cpu().numpy(), outs[2].cpu().numpy(), 1e-5, "repeat")


@pytest.mark.slow
def test_sharded_ctx1m_four_shards():
    """The 1M workload split over 4 shards against the whole-sequence step
    (the smaller cases above check the sharded path against the oracle)."""
    gc = GpuCase(synth.make_case("ctx1m", device="cuda"))
    gc.append_current()
    out, shards = run_sharded(gc, [0.25, 0.5, 0.75], 0.9)
    whole, _, _, _ = gc.step(0.9, want_sel=False)
    within(out.cpu().numpy(), whole.cpu().numpy(), OUT_TOL_SAME_SET, "sharded vs whole-sequence step")

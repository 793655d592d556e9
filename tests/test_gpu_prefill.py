"""GPU parity of the prefill side against the CPU oracle: the index keys of a
whole prompt (rtp_append_index_keys with T = the prompt length) and the
causal prefill attention (rtp_prefill_attention: local heads over sinks and
window, retrieval heads over every earlier token)."""
import math

import numpy as np
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import OUT_TOL_SAME_SET, np64

pytestmark = pytest.mark.gpu

# Prefill output vs the oracle: the products q.k are exact (bf16 inputs,
# fp32 accumulation over 128 terms) and the softmax weights enter P.V as a
# two-term bf16 split (relative error <= 2^-18), so only fp32 accumulation
# error remains: the same bound as the decode kernels over a given set.
PREFILL_TOL = OUT_TOL_SAME_SET


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def _prefill_case(B, H_q, H_kv, N_max, T, lens, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn(B, H_q, T, 128, generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn(B, H_kv, N_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn(B, H_kv, N_max, 128, generator=g, device="cuda").to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
    pos0 = (seq - T).to(torch.int32)            # the prompt's last T tokens
    return q, k, v, seq, pos0


def _run(q, k, v, seq, pos0, hc, window, n_sink):
    B, H_q, T, _ = q.shape
    H_kv, N_max = k.shape[1], k.shape[2]
    dims = ops.make_dims(B, H_q, H_kv, N_max, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims, ops.OP_PREFILL)
    out = torch.full((B, H_q, T, 128), float("nan"), device="cuda")
    ops.prefill_attention(dims, q, pos0, k, v, hc, window, n_sink, out, ws)
    st = ws.check()
    assert st == 0, ops.error_string(st)
    return out


SMALL = [
    # (B, H_q, H_kv, N_max, T, lens, head_class, window, n_sink)
    (2, 16, 2, 3000, 600, [3000, 1777], (1, 0), 256, 4),
    (1, 16, 2, 1500, 1500, [1500], (0, 1), 100, 0),          # the whole prompt from position 0
    (2, 8, 2, 900, 300, [900, 450], (0, 0), 64, 70),         # sinks reach past the window start
    (1, 3, 1, 700, 333, [700], (0,), 50, 2),                 # G = 3: 6 of 8 warps hold rows
    (1, 4, 4, 500, 129, [500], (1, 0, 1, 0), 10000, 4),      # G = 1; window wider than the cache
    (3, 16, 2, 400, 1, [400, 3, 1], (1, 0), 16, 1),          # one prompt token: the decode step
]


@pytest.mark.parametrize("k_", range(len(SMALL)))
def test_prefill_small(k_):
    B, H_q, H_kv, N_max, T, lens, hc, window, n_sink = SMALL[k_]
    q, k, v, seq, pos0 = _prefill_case(B, H_q, H_kv, N_max, T, lens, seed=k_)
    out = _run(q, k, v, seq, pos0, hc, window, n_sink)
    ref = oracle.prefill_attention(np64(q), np64(k), np64(v), np.asarray(hc, np.uint8),
                                   pos0.cpu().numpy(), window, n_sink)
    err = float(np.max(np.abs(out.cpu().numpy() - ref)))
    assert err <= PREFILL_TOL, f"max abs err {err:.3e}"


def test_prefill_last_token_equals_decode_step_kernels():
    """The prompt's last token against the library's own decode kernels over
    the same cache (dense for a retrieval head, local for a local head)."""
    B, H_q, H_kv, N = 2, 16, 2, 5000
    q, k, v, seq, pos0 = _prefill_case(B, H_q, H_kv, N, 64, [5000, 2100], seed=11)
    hc = (1, 0)
    out = _run(q, k, v, seq, pos0, hc, 512, 4)
    dims = ops.make_dims(B, H_q, H_kv, N, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims)
    ql = q[:, :, -1].float().contiguous()
    dense = torch.zeros(B, H_q, 128, device="cuda")
    local = torch.zeros(B, H_q, 128, device="cuda")
    ops.dense_decode(dims, ql, k, v, dense, ws)
    ops.local_decode(dims, ql, k, v, hc, 512, 4, local, ws)
    assert ws.check() == 0
    last = out[:, :, -1]
    assert float((last[:, :8] - dense[:, :8]).abs().max()) <= 2 * PREFILL_TOL
    assert float((last[:, 8:] - local[:, 8:]).abs().max()) <= 2 * PREFILL_TOL


def test_prefill_device_arg_checked():
    """A prompt that does not fit its sequence is reported, and its outputs
    are zeros; the other sequence is still computed."""
    q, k, v, seq, pos0 = _prefill_case(2, 8, 1, 300, 50, [300, 200], seed=3)
    pos0[1] = 160                                 # 160 + 50 > 200
    B, H_q, T, _ = q.shape
    dims = ops.make_dims(B, H_q, 1, 300, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims, ops.OP_PREFILL)
    out = torch.full((B, H_q, T, 128), float("nan"), device="cuda")
    ops.prefill_attention(dims, q, pos0, k, v, (0,), 32, 4, out, ws)
    assert ws.check() == ops.RTP_ERR_DEVICE_ARG
    assert bool((out[1] == 0).all())
    ref = oracle.prefill_attention(np64(q[:1]), np64(k[:1]), np64(v[:1]), np.array([0], np.uint8),
                                   pos0[:1].cpu().numpy(), 32, 4)
    assert float(np.max(np.abs(out[:1].cpu().numpy() - ref))) <= PREFILL_TOL


def test_prompt_index_keys():
    """Index keys of a whole 64K-token prompt in one call (T = N): the
    fp64 oracle's keys up to fp32 accumulation and one unit in the last
    place, and >= 99.9 % bit-exact."""
    B, H_kv, N = 1, 4, 65536
    g = torch.Generator(device="cuda").manual_seed(5)
    k_pre = torch.randn(B, H_kv, N, 128, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(H_kv, 16, 128, generator=g, device="cuda") / math.sqrt(128)).float()
    cache = torch.zeros(B, H_kv, N, 16, dtype=torch.bfloat16, device="cuda")
    seq = torch.tensor([N], dtype=torch.int32, device="cuda")
    dims = ops.make_dims(B, 32, H_kv, N, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims, ops.OP_APPEND_INDEX_KEYS)
    hc = np.array([1, 0, 1, 1], np.uint8)
    ops.append_index_keys(dims, k_pre, W, torch.zeros(B, dtype=torch.int32, device="cuda"), hc, cache, ws)
    assert ws.check() == 0
    ref = oracle.append_index_keys(np.zeros((B, H_kv, N, 16)), np64(k_pre), np64(W), np.zeros(B, np.int64),
                                   "bf16", head_class=hc)
    got = np64(cache)
    assert np.all(got[:, 1] == 0)                 # the local head's rows are not written
    sel = hc.astype(bool)
    absdot = np.abs(np64(k_pre)[0, sel]) @ np.abs(np64(W)[sel]).transpose(0, 2, 1)
    bound = 130 * 2.0 ** -24 * absdot + np.abs(ref[0, sel]) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(ref[0, sel] - got[0, sel]) <= bound)
    assert (ref[0, sel] == got[0, sel]).mean() > 0.999


@pytest.mark.slow
def test_prefill_64k_prompt_sampled():
    """A 16K-token prompt tail at 64K context in the 64K workload's shape
    (32 q / 4 KV heads, KV0 retrieval, window 4096 + 4 sinks): rows the
    oracle computes one by one -- the first, the last, and a seeded sample
    of tokens in every head."""
    spec = synth.spec_for("ctx64k")
    B, H_q, H_kv, N, T = 1, spec.H_q, spec.H_kv, spec.N, 16384
    q, k, v, seq, pos0 = _prefill_case(B, H_q, H_kv, N, T, [N], seed=21)
    hc = (1, 0, 0, 0)
    out = _run(q, k, v, seq, pos0, hc, spec.window, spec.n_sink).cpu().numpy()
    rng = np.random.default_rng(0)
    rows = [(0, h, i) for h in range(H_q) for i in [0, T - 1, *rng.integers(0, T, 6).tolist()]]
    ref = oracle.prefill_attention(np64(q), np64(k), np64(v), np.asarray(hc, np.uint8), pos0.cpu().numpy(),
                                   spec.window, spec.n_sink, rows_of=rows)
    for b, h, i in rows:
        err = float(np.max(np.abs(out[b, h, i] - ref[b, h, i])))
        assert err <= PREFILL_TOL, f"h={h} i={i}: {err:.3e}"

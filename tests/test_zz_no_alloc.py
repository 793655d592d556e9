"""rtp_dense_decode_noalloc: dense decode whose scratch lives in a fixed
device array inside the library instead of a caller workspace.  It must give
the same outputs as rtp_dense_decode, call after call, whatever ran before it
in the process (this file is collected last on purpose)."""
import pytest
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import OUT_TOL, OUT_TOL_SAME_SET, GpuCase, np32, np64, within

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def _case(kvdt):
    spec = synth.small_spec(B=2, H_q=16, H_kv=2, N=20000, head_class=(1, 0), kv_dtype=kvdt,
                            seq_lens=[20000, 333])
    return GpuCase(synth.make_case(spec))


def _max_abs(a, b):
    return float((a - b).abs().max())


@pytest.mark.parametrize("kvdt", ["bf16", "f32"])
def test_noalloc_matches_dense_two_calls(kvdt):
    gc = _case(kvdt)
    ref = torch.zeros((2, 16, 128), device="cuda")
    ops.dense_decode(gc.dims, gc.q_rope, gc.k, gc.v, ref, gc.ws)
    assert gc.ws.check() == 0
    c = gc.c
    exact = oracle.dense_decode(np64(c.q_rope), np32(c.k_cache), np32(c.v_cache), c.seq_lens.cpu().numpy())
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full((2, 16, 128), float("nan"), device="cuda")
        ops.dense_decode_noalloc(gc.dims, gc.q_rope, gc.k, gc.v, out, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0, f"call {call}"
        assert torch.isfinite(out).all(), f"call {call}"
        err = _max_abs(out, ref)
        assert err <= OUT_TOL_SAME_SET, f"call {call}: max abs diff {err}"
        # and the oracle's dense attention over the same caches
        within(out.cpu().numpy(), exact, OUT_TOL, f"call {call} vs oracle")


def test_noalloc_status_is_per_call():
    gc = _case("bf16")
    st = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = torch.zeros((2, 16, 128), device="cuda")
    gc.seq[1] = gc.N_max + 5          # out of range on the device only
    ops.dense_decode_noalloc(gc.dims, gc.q_rope, gc.k, gc.v, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == ops.RTP_ERR_DEVICE_ARG
    # the next call starts from a cleared status word and clean counters
    gc.seq[1] = 333
    ref = torch.zeros((2, 16, 128), device="cuda")
    ops.dense_decode(gc.dims, gc.q_rope, gc.k, gc.v, ref, gc.ws)
    assert gc.ws.check() == 0
    ops.dense_decode_noalloc(gc.dims, gc.q_rope, gc.k, gc.v, out, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert _max_abs(out, ref) <= OUT_TOL_SAME_SET


def test_noalloc_rejects_too_many_groups():
    B, H_kv = ops.NOALLOC_MAX_GROUPS // 8 + 1, 8
    seq = torch.ones(B, dtype=torch.int32, device="cuda")
    dims = ops.make_dims(B, H_kv, H_kv, 256, seq, ops.RTP_BF16, ops.RTP_BF16)
    t = torch.zeros(64, device="cuda")
    with pytest.raises(ops.RtpError) as e:
        ops.dense_decode_noalloc(dims, t, t, t, t)
    assert e.value.code == ops.RTP_ERR_WORKSPACE

"""Device-side error reporting: bad device-resident arguments and logits out
of the binned range are recorded in the workspace status word and returned
by rtp_check(); the kernels skip the offending work (no fault, no hang)."""

import pytest
import torch

from dynamic_top_sparse_b200 import ops, synth
from tests.helpers import GpuCase

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    ops.lib()


def _case(**kw):
    spec = synth.small_spec(B=2, H_q=8, H_kv=2, N=2000, head_class=(1, 0), **kw)
    return GpuCase(synth.make_case(spec))


def test_bad_seq_len_reports_and_zeroes():
    gc = _case()
    gc.seq[1] = gc.N_max + 5          # out of range on the device only
    out = torch.full((2, 8, 128), 7.0, device="cuda")
    ops.decode_step(gc.dims, gc.q, gc.q_rope, gc.k, gc.v, gc.kidx, gc.Wq, gc.hc, 0.9, 64, 4, out, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG
    assert torch.all(out[1] == 0)
    assert torch.isfinite(out[0]).all()
    assert gc.ws.check() == 0          # cleared
    gc.seq[1] = 0
    ops.decode_step(gc.dims, gc.q, gc.q_rope, gc.k, gc.v, gc.kidx, gc.Wq, gc.hc, 0.9, 64, 4, out, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG
    # the workspace stays usable
    gc.seq[1] = 2000
    ops.decode_step(gc.dims, gc.q, gc.q_rope, gc.k, gc.v, gc.kidx, gc.Wq, gc.hc, 0.9, 64, 4, out, gc.ws)
    assert gc.ws.check() == 0


def test_nonfinite_logit_reports_range():
    gc = _case()
    gc.kidx[0, 0, 123, 3] = float("nan")
    gc.kidx[1, 0, 77, 0] = float("inf")
    out = torch.zeros((2, 8, 128), device="cuda")
    ops.decode_step(gc.dims, gc.q, gc.q_rope, gc.k, gc.v, gc.kidx, gc.Wq, gc.hc, 0.9, 64, 4, out, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_RANGE
    assert torch.isfinite(out).all()


def test_sparse_decode_bad_ids_report():
    gc = _case()
    idx = torch.zeros((2, 8, gc.N_max), dtype=torch.int32, device="cuda")
    idx[0, 0, :3] = torch.tensor([5, 2000, 7], dtype=torch.int32)      # 2000 >= N
    cnt = torch.ones((2, 8), dtype=torch.int32, device="cuda")
    cnt[0, 0] = 3
    out = torch.zeros((2, 8, 128), device="cuda")
    ops.sparse_decode(gc.dims, gc.q_rope, gc.k, gc.v, idx, cnt, gc.hc, out, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG
    cnt[0, 1] = 5000                    # count > N
    ops.sparse_decode(gc.dims, gc.q_rope, gc.k, gc.v, idx, cnt, gc.hc, out, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG
    assert torch.all(out[0, 1] == 0)


def test_append_bad_position_reports():
    gc = _case()
    pos = torch.tensor([0, gc.N_max], dtype=torch.int32, device="cuda")   # second one past the end
    before = gc.kidx.clone()
    ops.append_index_keys(gc.dims, gc.k_new, gc.Wk, pos, gc.hc, gc.kidx, gc.ws)
    assert gc.ws.check() == ops.RTP_ERR_DEVICE_ARG
    assert torch.equal(gc.kidx[1], before[1])


def test_bounded_wait_runs_out_and_context_stays_usable():
    """A device-side wait that nothing ends gives up after its bound and
    reports RTP_ERR_TIMEOUT; the next step on the same context is correct."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.selftest_wait_timeout(st)
    torch.cuda.synchronize()
    assert int(st.item()) == ops.RTP_ERR_TIMEOUT
    gc = _case()
    out = torch.zeros((2, 8, 128), device="cuda")
    ops.decode_step(gc.dims, gc.q, gc.q_rope, gc.k, gc.v, gc.kidx, gc.Wq, gc.hc, 0.9, 64, 4, out, gc.ws)
    assert gc.ws.check() == 0
    assert torch.isfinite(out).all()

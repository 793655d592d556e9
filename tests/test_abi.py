"""The C-ABI library loads, exports every symbol include/rtp.h declares, and
rejects bad arguments on the host before any launch (no GPU needed: every
call here fails validation, so nothing reaches the device)."""
import ctypes
import math
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from dynamic_top_sparse_b200 import build, ops
    build.build()
    return ops.lib()


def _declared():
    with open(os.path.join(ROOT, "include", "rtp.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"RTP_API[^;(]*?\b(rtp_\w+)\s*\(", src)))


def test_header_declares_the_step_calls():
    names = set(_declared())
    for n in ("rtp_append_index_keys", "rtp_index_scores", "rtp_topp_select", "rtp_sparse_decode",
              "rtp_local_decode", "rtp_decode_step", "rtp_dense_decode", "rtp_workspace_size",
              "rtp_check", "rtp_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from dynamic_top_sparse_b200 import ops
    for name in _declared():
        assert hasattr(L, name), name
    assert set(_declared()) == set(ops.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", ops.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(_declared())


def test_library_needs_no_cuda_shared_libraries():
    from dynamic_top_sparse_b200 import ops
    out = subprocess.run(["ldd", ops.LIB_PATH], capture_output=True, text=True).stdout
    assert "libtorch" not in out and "libc10" not in out


def test_error_strings(L):
    from dynamic_top_sparse_b200 import ops
    for code in range(8):
        assert len(ops.error_string(code)) > 0
    assert L.rtp_version() >= 100


def _dims(ops, **kw):
    base = dict(B=1, H_q=32, H_kv=4, d=128, r=16, kv_dtype=ops.RTP_BF16, idx_dtype=ops.RTP_BF16,
                reserved=0, N_max=65536, seq_lens=0x10000)
    base.update(kw)
    return ops.Dims(**base)


def test_workspace_size_monotone_and_invalid(L):
    from dynamic_top_sparse_b200 import ops
    d = _dims(ops)
    sizes = [ops.workspace_size(d, op) for op in range(7)]
    assert all(s > 0 for s in sizes)
    assert sizes[ops.OP_DECODE_STEP] == max(sizes)
    bigger = _dims(ops, N_max=131072)
    assert ops.workspace_size(bigger) > ops.workspace_size(d)
    assert ops.workspace_size(_dims(ops, d=64)) == 0
    assert ops.workspace_size(_dims(ops, H_q=30)) == 0
    assert L.rtp_workspace_size(None, 6) == 0


FAKE = 0x7f0000000000   # never dereferenced: validation fails first


def _step(L, ops, dims, p=0.9, window=4096, n_sink=4, ws=FAKE, ws_bytes=None, hc=(1, 0, 0, 0),
          q=FAKE, out=FAKE):
    if ws_bytes is None:
        ws_bytes = ops.workspace_size(dims) if ops.workspace_size(dims) else 1 << 40
    arr = (ctypes.c_uint8 * len(hc))(*hc)
    return L.rtp_decode_step(ctypes.byref(dims), None, q, q, FAKE, FAKE, FAKE, FAKE, arr, p, window,
                             n_sink, out, ws, ws_bytes, None)


def test_decode_step_rejects_bad_arguments(L):
    from dynamic_top_sparse_b200 import ops
    d = _dims(ops)
    assert _step(L, ops, _dims(ops, d=64)) == ops.RTP_ERR_UNSUPPORTED
    assert _step(L, ops, _dims(ops, r=32)) == ops.RTP_ERR_UNSUPPORTED
    assert _step(L, ops, _dims(ops, H_q=64, H_kv=4)) == ops.RTP_ERR_UNSUPPORTED   # G = 16 > 8
    assert _step(L, ops, _dims(ops, H_q=30)) == ops.RTP_ERR_INVALID_ARG           # H_q % H_kv
    assert _step(L, ops, _dims(ops, kv_dtype=7)) == ops.RTP_ERR_UNSUPPORTED
    assert _step(L, ops, _dims(ops, B=0)) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, _dims(ops, seq_lens=0)) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, p=math.nan) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, window=0) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, n_sink=-1) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, hc=(1, 0, 2, 0)) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, q=FAKE + 4) == ops.RTP_ERR_INVALID_ARG              # misaligned
    assert _step(L, ops, d, q=0) == ops.RTP_ERR_INVALID_ARG
    assert _step(L, ops, d, ws=0) == ops.RTP_ERR_WORKSPACE
    assert _step(L, ops, d, ws=FAKE + 128) == ops.RTP_ERR_WORKSPACE
    assert _step(L, ops, d, ws_bytes=1024) == ops.RTP_ERR_WORKSPACE
    # options: a negative top-k budget; forced local rows beyond the bitmap's reach
    opts = ops.Opts(0.0, 0.0, None, None, None, None, -1, 0)
    arr = (ctypes.c_uint8 * 4)(1, 0, 0, 0)
    ws_b = ops.workspace_size(d) or (1 << 40)
    assert L.rtp_decode_step(ctypes.byref(d), ctypes.byref(opts), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, arr, 0.9,
                             4096, 4, FAKE, FAKE, ws_b, None) == ops.RTP_ERR_INVALID_ARG
    big = _dims(ops, N_max=1 << 20)
    opts = ops.Opts(0.0, 0.0, None, None, None, None, 0, 1)
    assert L.rtp_decode_step(ctypes.byref(big), ctypes.byref(opts), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, arr, 0.9,
                             500000, 4, FAKE, FAKE, 1 << 40, None) == ops.RTP_ERR_UNSUPPORTED
    assert L.rtp_decode_step(None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0.9, 1, 0, FAKE, FAKE,
                             1 << 40, None) == ops.RTP_ERR_INVALID_ARG


def test_other_calls_reject_bad_arguments(L):
    from dynamic_top_sparse_b200 import ops
    d = _dims(ops)
    hc = (ctypes.c_uint8 * 4)(1, 0, 0, 0)
    big = 1 << 40
    assert L.rtp_topp_select(ctypes.byref(d), FAKE, hc, math.nan, FAKE, FAKE, None, FAKE, big,
                             None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_topp_select(ctypes.byref(d), FAKE, hc, 0.9, None, FAKE, None, FAKE, big,
                             None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_topp_select(ctypes.byref(d), FAKE, hc, 0.9, FAKE, FAKE, None, FAKE, 100,
                             None) == ops.RTP_ERR_WORKSPACE
    assert L.rtp_local_decode(ctypes.byref(d), None, FAKE, FAKE, FAKE, hc, 0, 4, FAKE, FAKE, big,
                              None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_local_decode(ctypes.byref(d), None, FAKE, FAKE, FAKE, None, 16, 4, FAKE, FAKE, big,
                              None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_sparse_decode(ctypes.byref(d), None, FAKE, FAKE, FAKE, None, FAKE, hc, FAKE, FAKE, big,
                               None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_dense_decode(ctypes.byref(_dims(ops, d=96)), None, FAKE, FAKE, FAKE, FAKE, FAKE, big,
                              None) == ops.RTP_ERR_UNSUPPORTED
    assert L.rtp_index_scores(ctypes.byref(d), None, FAKE, FAKE, FAKE, hc, FAKE + 8, FAKE, big,
                              None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_append_index_keys(ctypes.byref(d), FAKE, 0, FAKE, FAKE, hc, FAKE, FAKE, big,
                                   None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_append_index_keys(ctypes.byref(d), FAKE, 70000, FAKE, FAKE, hc, FAKE, FAKE, big,
                                   None) == ops.RTP_ERR_INVALID_ARG
    for kk in (0, -5):
        assert L.rtp_topk_select(ctypes.byref(d), FAKE, hc, kk, FAKE, FAKE, FAKE, big,
                                 None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_topk_select(ctypes.byref(d), None, hc, 8, FAKE, FAKE, FAKE, big, None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_topk_select(ctypes.byref(d), FAKE + 4, hc, 8, FAKE, FAKE, FAKE, big,
                             None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_topk_select(ctypes.byref(d), FAKE, hc, 8, FAKE, FAKE, FAKE, 100, None) == ops.RTP_ERR_WORKSPACE
    # paged K/V: page size a power of two >= 16, a table, enough pages per sequence
    for ps, mp, npg, tab in ((24, 4096, 10, FAKE), (8, 8192, 10, FAKE), (16, 10, 10, FAKE), (16, 4096, 0, FAKE),
                             (16, 4096, 10, 0), (16, 4096, 10, FAKE + 2)):
        pg = ops.KvPages(tab, ps, mp, npg, 0)
        o = ops.Opts(0.0, 0.0, None, None, None, None, 0, 0, ctypes.pointer(pg))
        assert L.rtp_dense_decode(ctypes.byref(d), ctypes.byref(o), FAKE, FAKE, FAKE, FAKE, FAKE, big,
                                  None) == ops.RTP_ERR_INVALID_ARG, (ps, mp, npg)
    # prefill: prompt length, window, cache type, workspace
    pf = L.rtp_prefill_attention
    assert pf(ctypes.byref(d), None, FAKE, 0, FAKE, FAKE, FAKE, hc, 16, 4, FAKE, FAKE, big,
              None) == ops.RTP_ERR_INVALID_ARG
    assert pf(ctypes.byref(d), None, FAKE, 70000, FAKE, FAKE, FAKE, hc, 16, 4, FAKE, FAKE, big,
              None) == ops.RTP_ERR_INVALID_ARG
    assert pf(ctypes.byref(d), None, FAKE, 8, FAKE, FAKE, FAKE, hc, 0, 4, FAKE, FAKE, big,
              None) == ops.RTP_ERR_INVALID_ARG
    assert pf(ctypes.byref(d), None, None, 8, FAKE, FAKE, FAKE, hc, 16, 4, FAKE, FAKE, big,
              None) == ops.RTP_ERR_INVALID_ARG
    assert pf(ctypes.byref(_dims(ops, kv_dtype=ops.RTP_F32)), None, FAKE, 8, FAKE, FAKE, FAKE, hc, 16, 4,
              FAKE, FAKE, big, None) == ops.RTP_ERR_UNSUPPORTED
    assert pf(ctypes.byref(d), None, FAKE, 8, FAKE, FAKE, FAKE, hc, 16, 4, FAKE, FAKE, 100,
              None) == ops.RTP_ERR_WORKSPACE
    assert L.rtp_workspace_size(ctypes.byref(d), ops.OP_PREFILL) == 256
    assert L.rtp_workspace_init(None, 100, None) == ops.RTP_ERR_WORKSPACE
    assert L.rtp_check(None, None) == ops.RTP_ERR_WORKSPACE
    assert L.rtp_selftest_wait_timeout(None, None) == ops.RTP_ERR_INVALID_ARG
    assert L.rtp_selftest_wait_timeout(FAKE + 2, None) == ops.RTP_ERR_INVALID_ARG     # misaligned


def test_prepared_call_raises_the_library_error(L):
    """ops.Prepared re-issues one call and raises what the library returns
    (a null dims pointer is rejected before anything touches the GPU)."""
    from dynamic_top_sparse_b200 import ops
    call = ops.Prepared("rtp_decode_step", (None,) * 9 + (0.9, 0, 0) + (None, None, 0, None))
    with pytest.raises(ops.RtpError) as e:
        call()
    assert e.value.code == ops.RTP_ERR_INVALID_ARG and "rtp_decode_step" in str(e.value)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    """No CPU fallback: with the library missing every call raises."""
    from dynamic_top_sparse_b200 import ops
    monkeypatch.setattr(ops, "_lib", None)
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "librtp.so"))
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()
    with pytest.raises(RuntimeError, match="missing"):
        ops.error_string(0)

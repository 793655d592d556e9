"""Python binding of librtp.so (ctypes).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of librtp.so.  Tensors are torch CUDA tensors; each call is queued
on torch's current stream.  There is no fallback: if the library is missing
or a call returns an error, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librtp.so")

RTP_OK = 0
RTP_ERR_INVALID_ARG = 1
RTP_ERR_UNSUPPORTED = 2
RTP_ERR_WORKSPACE = 3
RTP_ERR_CUDA = 4
RTP_ERR_TIMEOUT = 5
RTP_ERR_DEVICE_ARG = 6
RTP_ERR_RANGE = 7

RTP_F32 = 0
RTP_BF16 = 1
HEAD_LOCAL = 0
HEAD_RETRIEVAL = 1

OP_APPEND_INDEX_KEYS = 0
OP_INDEX_SCORES = 1
OP_TOPP_SELECT = 2
OP_SPARSE_DECODE = 3
OP_LOCAL_DECODE = 4
OP_DENSE_DECODE = 5
OP_DECODE_STEP = 6
OP_PREFILL = 7
PART_STRIDE = 132          # floats per partial record: m, l, 2 unused, o[128]

EXPORTS = ("rtp_workspace_size", "rtp_workspace_init", "rtp_check", "rtp_error_string",
           "rtp_version", "rtp_append_index_keys", "rtp_index_scores", "rtp_topp_select", "rtp_topk_select",
           "rtp_sparse_decode", "rtp_local_decode", "rtp_dense_decode", "rtp_decode_step",
           "rtp_prof_init", "rtp_prof_elapsed", "rtp_prof_destroy", "rtp_dense_decode_noalloc",
           "rtp_selftest_wait_timeout", "rtp_prefill_attention", "rtp_shard_scan", "rtp_shard_hist",
           "rtp_shard_collect", "rtp_shard_cands", "rtp_shard_finish", "rtp_merge_shards")

NOALLOC_SCRATCH_BYTES = 8 << 20
NOALLOC_MAX_GROUPS = 1024


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H_q", ctypes.c_int32), ("H_kv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("r", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("idx_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("N_max", ctypes.c_int64), ("seq_lens", ctypes.c_void_p)]


class Prof(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("count", ctypes.c_int32),
                ("ev_start", ctypes.POINTER(ctypes.c_void_p)),
                ("ev_stop", ctypes.POINTER(ctypes.c_void_p)),
                ("name", ctypes.POINTER(ctypes.c_char_p)), ("filter", ctypes.c_char_p)]


class KvPages(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("page_size", ctypes.c_int32), ("max_pages", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class Opts(ctypes.Structure):
    _fields_ = [("idx_scale", ctypes.c_float), ("attn_scale", ctypes.c_float),
                ("sel_idx", ctypes.c_void_p), ("sel_count", ctypes.c_void_p),
                ("sel_mass", ctypes.c_void_p), ("prof", ctypes.POINTER(Prof)), ("topk", ctypes.c_int32),
                ("force_local", ctypes.c_int32), ("kv_pages", ctypes.POINTER(KvPages))]


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "rtp_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(Dims), ctypes.c_int]),
    "rtp_workspace_init": (ctypes.c_int, [_P, ctypes.c_size_t, _P]),
    "rtp_check": (ctypes.c_int, [_P, _P]),
    "rtp_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "rtp_version": (ctypes.c_int, []),
    "rtp_append_index_keys": (ctypes.c_int, [ctypes.POINTER(Dims), _P, ctypes.c_int32, _P, _P, _P, _P,
                                             _P, ctypes.c_size_t, _P]),
    "rtp_index_scores": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P,
                                        _P, ctypes.c_size_t, _P]),
    "rtp_topp_select": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, ctypes.c_float, _P, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
    "rtp_topk_select": (ctypes.c_int, [ctypes.POINTER(Dims), _P, _P, ctypes.c_int32, _P, _P, _P,
                                       ctypes.c_size_t, _P]),
    "rtp_sparse_decode": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P,
                                         _P, _P, _P, ctypes.c_size_t, _P]),
    "rtp_local_decode": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P,
                                        ctypes.c_int32, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]),
    "rtp_dense_decode": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "rtp_decode_step": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P, _P,
                                       _P, ctypes.c_float, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                       ctypes.c_size_t, _P]),
    "rtp_prof_init": (ctypes.c_int, [ctypes.POINTER(Prof), ctypes.c_int32]),
    "rtp_prof_elapsed": (ctypes.c_int, [ctypes.POINTER(Prof), ctypes.c_int32,
                                        ctypes.POINTER(ctypes.c_float)]),
    "rtp_prof_destroy": (ctypes.c_int, [ctypes.POINTER(Prof)]),
    "rtp_dense_decode_noalloc": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P,
                                                _P]),
    "rtp_selftest_wait_timeout": (ctypes.c_int, [_P, _P]),
    "rtp_shard_scan": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, ctypes.c_float,
                                      _P, ctypes.c_size_t, _P]),
    "rtp_shard_hist": (ctypes.c_int, [ctypes.POINTER(Dims), _P, ctypes.POINTER(ctypes.c_void_p),
                                      ctypes.POINTER(ctypes.c_int64)]),
    "rtp_shard_collect": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, ctypes.c_float, _P,
                                         _P, ctypes.c_size_t, _P]),
    "rtp_shard_cands": (ctypes.c_int, [ctypes.POINTER(Dims), _P, ctypes.POINTER(ctypes.c_void_p),
                                       ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int64),
                                       ctypes.POINTER(ctypes.c_int64)]),
    "rtp_shard_finish": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, _P, _P, _P, _P,
                                        ctypes.c_float, ctypes.c_int32, ctypes.c_int32, _P, _P, _P, _P,
                                        ctypes.c_int64, _P, _P, ctypes.c_size_t, _P]),
    "rtp_merge_shards": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, _P, _P]),
    "rtp_prefill_attention": (ctypes.c_int, [ctypes.POINTER(Dims), ctypes.POINTER(Opts), _P, ctypes.c_int32, _P,
                                             _P, _P, _P, ctypes.c_int32, ctypes.c_int32, _P, _P,
                                             ctypes.c_size_t, _P]),
}


class RtpError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {error_string(code)} (code {code})")


def lib() -> ctypes.CDLL:
    """Load librtp.so (built in-tree by dynamic_top_sparse_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m dynamic_top_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().rtp_error_string(code).decode()


def _ck(code: int, where: str):
    if code != RTP_OK:
        raise RtpError(code, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return RTP_BF16
    if t.dtype == torch.float32:
        return RTP_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _hc(head_class) -> ctypes.Array:
    arr = np.ascontiguousarray(np.asarray(head_class, dtype=np.uint8))
    return (ctypes.c_uint8 * len(arr)).from_buffer_copy(arr.tobytes())


def make_dims(B, H_q, H_kv, N_max, seq_lens: torch.Tensor, kv_dtype, idx_dtype, d=128, r=16) -> Dims:
    """The dims struct of a call; it holds the device address of seq_lens and
    keeps the tensor alive with it (a freed tensor's memory would be reused)."""
    if seq_lens.dtype != torch.int32:
        raise ValueError("seq_lens must be int32")
    dm = Dims(B, H_q, H_kv, d, r, kv_dtype, idx_dtype, 0, N_max, _ptr(seq_lens))
    dm._seq_lens = seq_lens
    return dm


def dims_for(k_cache: torch.Tensor, kidx_cache: torch.Tensor | None, H_q: int,
             seq_lens: torch.Tensor) -> Dims:
    B, H_kv, N_max, d = k_cache.shape
    r = kidx_cache.shape[-1] if kidx_cache is not None else 16
    idt = _dt(kidx_cache) if kidx_cache is not None else RTP_BF16
    return make_dims(B, H_q, H_kv, N_max, seq_lens, _dt(k_cache), idt, d=d, r=r)


def workspace_size(dims: Dims, op: int = OP_DECODE_STEP) -> int:
    return lib().rtp_workspace_size(ctypes.byref(dims), op)


class Workspace:
    """A device workspace for the library, zeroed once on creation."""

    def __init__(self, dims: Dims, op: int = OP_DECODE_STEP, device=None):
        n = workspace_size(dims, op)
        if n == 0:
            raise RtpError(RTP_ERR_INVALID_ARG, "rtp_workspace_size")
        self.nbytes = n
        self.buf = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256
        _ck(lib().rtp_workspace_init(self.ptr, self.nbytes, _stream()), "rtp_workspace_init")

    def check(self) -> int:
        """Synchronise and return the device status word (and clear it)."""
        return lib().rtp_check(self.ptr, _stream())


class Profiler:
    """Event slots for per-kernel device times (rtp_prof)."""

    def __init__(self, capacity: int, filter: str | None = None):
        self.p = Prof()
        _ck(lib().rtp_prof_init(ctypes.byref(self.p), capacity), "rtp_prof_init")
        self._filter = filter.encode() if filter else None
        self.p.filter = self._filter

    def reset(self):
        self.p.count = 0

    def times(self):
        out = []
        for i in range(self.p.count):
            ms = ctypes.c_float()
            _ck(lib().rtp_prof_elapsed(ctypes.byref(self.p), i, ctypes.byref(ms)), "rtp_prof_elapsed")
            out.append((self.p.name[i].decode(), ms.value))
        return out

    def close(self):
        if self.p.ev_start:
            lib().rtp_prof_destroy(ctypes.byref(self.p))


def make_opts(idx_scale=0.0, attn_scale=0.0, sel_idx=None, sel_count=None, sel_mass=None,
              prof: Profiler | None = None, topk: int = 0, force_local: bool = False,
              kv_pages: KvPages | None = None) -> Opts:
    o = Opts(idx_scale, attn_scale, _ptr(sel_idx), _ptr(sel_count), _ptr(sel_mass), None, int(topk),
             1 if force_local else 0, None)
    if kv_pages is not None:
        o.kv_pages = ctypes.pointer(kv_pages)
        o._keep = kv_pages                     # the struct must outlive the options
    if prof is not None:
        o.prof = ctypes.pointer(prof.p)
    return o


# ---------------------------------------------------------------- entry points

def kv_pages(block_table, page_size: int, num_pages: int) -> KvPages:
    """Paged K/V description: block_table [B, max_pages] int32 on the device."""
    if block_table.dtype != torch.int32 or block_table.dim() != 2:
        raise ValueError("block_table must be a 2-D int32 tensor")
    pg = KvPages(_ptr(block_table), int(page_size), int(block_table.shape[1]), int(num_pages), 0)
    pg._table = block_table                    # keep the table alive with the struct
    return pg


def append_index_keys(dims: Dims, k_pre, W_k_idx, pos, head_class, kidx_cache, ws: Workspace):
    T = k_pre.shape[2]
    hc = _hc(head_class) if head_class is not None else None
    _ck(lib().rtp_append_index_keys(ctypes.byref(dims), _ptr(k_pre), T, _ptr(W_k_idx), _ptr(pos), hc,
                                    _ptr(kidx_cache), ws.ptr, ws.nbytes, _stream()),
        "rtp_append_index_keys")


def index_scores(dims: Dims, q, W_q_idx, kidx_cache, head_class, z_out, ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_index_scores(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q),
                               _ptr(W_q_idx), _ptr(kidx_cache), _hc(head_class), _ptr(z_out), ws.ptr,
                               ws.nbytes, _stream()), "rtp_index_scores")


def topp_select(dims: Dims, z, head_class, p: float, idx_out, count_out, mass_out, ws: Workspace):
    _ck(lib().rtp_topp_select(ctypes.byref(dims), _ptr(z), _hc(head_class), float(p), _ptr(idx_out),
                              _ptr(count_out), _ptr(mass_out), ws.ptr, ws.nbytes, _stream()),
        "rtp_topp_select")


def topk_select(dims: Dims, z, head_class, k: int, idx_out, count_out, ws: Workspace):
    _ck(lib().rtp_topk_select(ctypes.byref(dims), _ptr(z), _hc(head_class), int(k), _ptr(idx_out),
                              _ptr(count_out), ws.ptr, ws.nbytes, _stream()), "rtp_topk_select")


def sparse_decode(dims: Dims, q_rope, k_cache, v_cache, idx, count, head_class, out, ws: Workspace,
                  opts: Opts | None = None):
    _ck(lib().rtp_sparse_decode(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q_rope),
                                _ptr(k_cache), _ptr(v_cache), _ptr(idx), _ptr(count), _hc(head_class),
                                _ptr(out), ws.ptr, ws.nbytes, _stream()), "rtp_sparse_decode")


def local_decode(dims: Dims, q_rope, k_cache, v_cache, head_class, window: int, n_sink: int, out,
                 ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_local_decode(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q_rope),
                               _ptr(k_cache), _ptr(v_cache), _hc(head_class), int(window), int(n_sink),
                               _ptr(out), ws.ptr, ws.nbytes, _stream()), "rtp_local_decode")


def dense_decode(dims: Dims, q_rope, k_cache, v_cache, out, ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_dense_decode(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q_rope),
                               _ptr(k_cache), _ptr(v_cache), _ptr(out), ws.ptr, ws.nbytes, _stream()),
        "rtp_dense_decode")


class Prepared:
    """One C-ABI call with every argument marshalled once (pointers, sizes,
    head classes, stream): calling the object re-issues the same call, so the
    tensors it names may change contents between calls but not storage.  For
    decode loops in which converting the arguments on every call would cost
    more host time than the GPU spends on the step."""

    __slots__ = ("_fn", "_args", "_name", "_keep")

    def __init__(self, name: str, args, keep=()):
        self._fn = getattr(lib(), name)
        self._args = tuple(args)
        self._name = name
        self._keep = keep           # objects the marshalled pointers refer to

    def __call__(self):
        code = self._fn(*self._args)
        if code != RTP_OK:
            raise RtpError(code, self._name)


def _vp(t) -> ctypes.c_void_p:
    return ctypes.c_void_p(_ptr(t))


def prepare_append_index_keys(dims: Dims, k_pre, W_k_idx, pos, head_class, kidx_cache,
                              ws: Workspace) -> Prepared:
    """append_index_keys with its arguments marshalled once, on the current stream."""
    hc = _hc(head_class) if head_class is not None else None
    return Prepared("rtp_append_index_keys",
                    (ctypes.byref(dims), _vp(k_pre), k_pre.shape[2], _vp(W_k_idx), _vp(pos), hc,
                     _vp(kidx_cache), ctypes.c_void_p(ws.ptr), ws.nbytes, _stream()), keep=(dims, hc, ws))


def prepare_decode_step(dims: Dims, q, q_rope, k_cache, v_cache, kidx_cache, W_q_idx, head_class, p: float,
                        window: int, n_sink: int, out, ws: Workspace, opts: Opts | None = None) -> Prepared:
    """decode_step with its arguments marshalled once, on the current stream."""
    hc = _hc(head_class)
    return Prepared("rtp_decode_step",
                    (ctypes.byref(dims), ctypes.byref(opts) if opts else None, _vp(q),
                     _vp(q_rope) if q_rope is not None else None, _vp(k_cache), _vp(v_cache),
                     _vp(kidx_cache), _vp(W_q_idx), hc, float(p), int(window), int(n_sink), _vp(out),
                     ctypes.c_void_p(ws.ptr), ws.nbytes, _stream()), keep=(dims, opts, hc, ws))


def decode_step(dims: Dims, q, q_rope, k_cache, v_cache, kidx_cache, W_q_idx, head_class, p: float,
                window: int, n_sink: int, out, ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_decode_step(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q),
                              _ptr(q_rope), _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache), _ptr(W_q_idx),
                              _hc(head_class), float(p), int(window), int(n_sink), _ptr(out), ws.ptr,
                              ws.nbytes, _stream()), "rtp_decode_step")


def prefill_attention(dims: Dims, q, pos0, k_cache, v_cache, head_class, window: int, n_sink: int, out,
                      ws: Workspace, opts: Opts | None = None):
    """Causal prefill attention of T prompt tokens per sequence (q [B, H_q, T, d]
    bf16, pos0 [B] int32 device positions of token 0, out [B, H_q, T, d] fp32)."""
    T = q.shape[2]
    _ck(lib().rtp_prefill_attention(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q), int(T),
                                    _ptr(pos0), _ptr(k_cache), _ptr(v_cache), _hc(head_class), int(window),
                                    int(n_sink), _ptr(out), ws.ptr, ws.nbytes, _stream()),
        "rtp_prefill_attention")


# ------------------------------------------------- context-sharded decode step

def shard_scan(dims: Dims, q, kidx_cache, W_q_idx, head_class, p: float, ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_shard_scan(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q), _ptr(kidx_cache),
                             _ptr(W_q_idx), _hc(head_class), float(p), ws.ptr, ws.nbytes, _stream()),
        "rtp_shard_scan")


def _dev_view(ptr: int, count: int, dtype, like: torch.Tensor) -> torch.Tensor:
    """A torch view of `count` elements of device memory at `ptr` inside the
    workspace buffer `like` (no copy)."""
    esize = torch.empty(0, dtype=dtype).element_size()
    off = ptr - like.data_ptr()
    if off < 0 or off % esize or off + count * esize > like.numel() * like.element_size():
        raise ValueError("region outside the workspace")
    return like.view(torch.uint8)[off:off + count * esize].view(dtype)


def shard_hist(dims: Dims, ws: Workspace) -> torch.Tensor:
    """The workspace's per-head level-1 histograms (fp64) that exchange 1
    sums over the shards, as a view."""
    p, n = ctypes.c_void_p(), ctypes.c_int64()
    _ck(lib().rtp_shard_hist(ctypes.byref(dims), ws.ptr, ctypes.byref(p), ctypes.byref(n)), "rtp_shard_hist")
    return _dev_view(p.value, n.value, torch.float64, ws.buf)


def shard_collect(dims: Dims, kidx_cache, head_class, p: float, shard_off, ws: Workspace, opts: Opts | None = None):
    _ck(lib().rtp_shard_collect(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(kidx_cache),
                                _hc(head_class), float(p), _ptr(shard_off), ws.ptr, ws.nbytes, _stream()),
        "rtp_shard_collect")


def shard_cands(dims: Dims, ws: Workspace):
    """This shard's boundary candidates (views): keys [B*H_q, N_max] int64
    (the bits of the 64-bit keys) and their counts [B*H_q] int32."""
    c, n, st, cst = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_int64(), ctypes.c_int64()
    _ck(lib().rtp_shard_cands(ctypes.byref(dims), ws.ptr, ctypes.byref(c), ctypes.byref(n), ctypes.byref(st),
                              ctypes.byref(cst)), "rtp_shard_cands")
    nh = dims.B * dims.H_q
    keys = _dev_view(c.value, nh * st.value, torch.int64, ws.buf).view(nh, st.value)
    cnts = _dev_view(n.value, nh * cst.value, torch.int32, ws.buf).view(nh, cst.value)[:, 0]
    return keys, cnts


def shard_finish(dims: Dims, q_rope, k_cache, v_cache, kidx_cache, head_class, p: float, window: int, n_sink: int,
                 shard_off, glob_len, all_cands, all_counts, part_out, ws: Workspace, opts: Opts | None = None):
    stride = all_cands.shape[1] if all_cands is not None else 0
    _ck(lib().rtp_shard_finish(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q_rope),
                               _ptr(k_cache), _ptr(v_cache), _ptr(kidx_cache), _hc(head_class), float(p), int(window),
                               int(n_sink), _ptr(shard_off), _ptr(glob_len), _ptr(all_cands), _ptr(all_counts),
                               int(stride), _ptr(part_out), ws.ptr, ws.nbytes, _stream()), "rtp_shard_finish")


def merge_shards(parts, out):
    """parts [P, B*H_q, 132] fp32 -> out [B*H_q, 128] (or [B, H_q, 128])."""
    P, nh = parts.shape[0], parts.shape[1]
    _ck(lib().rtp_merge_shards(_ptr(parts), int(P), int(nh), _ptr(out), _stream()), "rtp_merge_shards")


def selftest_wait_timeout(dev_status):
    """Launch the bounded-wait self-test: its one waiting thread gives up
    after 0.2 s and writes RTP_ERR_TIMEOUT into the zeroed device int32."""
    _ck(lib().rtp_selftest_wait_timeout(_ptr(dev_status), _stream()), "rtp_selftest_wait_timeout")


def dense_decode_noalloc(dims: Dims, q_rope, k_cache, v_cache, out, dev_status=None, opts: Opts | None = None):
    """Dense decode with no workspace argument: the library keeps the scratch
    in a fixed device array (for callers that cannot allocate device memory).
    Calls on one device share that array, so order them on one stream."""
    _ck(lib().rtp_dense_decode_noalloc(ctypes.byref(dims), ctypes.byref(opts) if opts else None, _ptr(q_rope),
                                       _ptr(k_cache), _ptr(v_cache), _ptr(out), _ptr(dev_status), _stream()),
        "rtp_dense_decode_noalloc")

"""Benchmark of the sparse decode step (one layer's append + decode per
step; 48 layers per step for the 48-layer workload) on synthetic caches.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ctx512k] [--p P]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) give every rank
sequences of its own, seeded per rank, of the same workload shape (the step
shards by sequence and KV head with no data exchange): value = steps of all
ranks / max rank time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import itertools
import math
import os
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_top_sparse_b200 import ops, synth  # noqa: E402
from dynamic_top_sparse_b200.dist import allreduce_max, barrier, rank_seed  # noqa: E402

METRIC = "sparse decode attention steps/s and achieved HBM GB/s (% peak) at 64K-1M ctx"
L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM = 6650.0


# --------------------------------------------------------------------- utils

def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM, "fallback"


# the sources of the scan kernel (its code and the helpers it inlines): a
# recorded DRAM-traffic figure stays valid while these hash the same
SCAN_SOURCES = ("rtp_common.cuh", "rtp_select.cuh")


def csrc_hash():
    h = hashlib.sha256()
    for name in SCAN_SOURCES:
        with open(os.path.join(ROOT, "dynamic_top_sparse_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken
    on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    for r in rec.get("records", []):
        if r.get("kernel") == kernel and r.get("workload") == workload and r.get("csrc") == csrc_hash():
            return r.get("bytes_per_launch")
    return None


class Clocks:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, dev: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                bus = torch.cuda.get_device_properties(dev).pci_bus_id
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(
                    f"{torch.cuda.get_device_properties(dev).pci_domain_id:08x}:{bus:02x}:"
                    f"{torch.cuda.get_device_properties(dev).pci_device_id:02x}.0")
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(dev)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)
        self._stop = threading.Event()

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h) if hasattr(
            nv, "nvmlDeviceGetCurrentClocksEventReasons") else nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit and name != "gpu_idle":
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def ctypes_elapsed(prof, slot):
    import ctypes
    ms = ctypes.c_float()
    rc = ops.lib().rtp_prof_elapsed(ctypes.byref(prof.p), slot, ctypes.byref(ms))
    if rc != 0:
        raise ops.RtpError(rc, "rtp_prof_elapsed")
    return ms.value


# ------------------------------------------------------------------ workload

class Layer:
    """Device tensors of one layer of the workload, plus the library state."""

    def __init__(self, case: synth.Case):
        self.case = case
        self.q, self.q_rope = case.q.cuda(), (case.q_rope.cuda() if case.q_rope is not None else None)
        self.k, self.v, self.kidx = case.k_cache, case.v_cache, case.kidx_cache
        self.Wq, self.Wk = case.W_q_idx.cuda(), case.W_k_idx.cuda()
        self.k_new = case.k_pre_new.cuda()
        self.seq = case.seq_lens.cuda()
        self.pos = (self.seq - 1).to(torch.int32)
        self.hc = case.head_class
        self.H_q = self.q.shape[1]
        self.dims = ops.dims_for(self.k, self.kidx, self.H_q, self.seq)

    def clone_caches(self):
        other = object.__new__(Layer)
        other.__dict__.update(self.__dict__)
        other.k, other.v, other.kidx = self.k.clone(), self.v.clone(), self.kidx.clone()
        other.dims = ops.dims_for(other.k, other.kidx, other.H_q, other.seq)
        return other


def build_workload(key: str, seed: int = 0):
    spec = synth.spec_for(key)
    layers = []
    for l in range(spec.layers):
        c = synth.make_case(spec, device="cuda", seed=seed, layer=l)
        if c.k_pre_all is not None:
            c.kidx_cache = c.kidx_cache.cuda()
        layers.append(Layer(c))
    return spec, layers


def required_bytes(spec, layers, sel, p=None, topk=0):
    """Algorithmic bytes a step must read: index keys of retrieval heads
    (only when a threshold is computed: p < 1 or static top-k), the union of kept K/V rows
    per KV group (every row at p >= 1), window+sink rows of local heads, and
    the query projector of retrieval heads (only when selecting)."""
    p = spec.p if p is None else p
    selecting = topk > 0 or p < 1.0
    total = 0
    kv_el = 2 if spec.kv_dtype == "bf16" else 4
    ix_el = 2 if spec.idx_dtype == "bf16" else 4
    for li, L in enumerate(layers):
        G = L.H_q // L.hc.shape[0]
        lens = L.case.seq_lens.tolist()
        for b in range(spec.B):
            N = lens[b]
            for g in range(L.hc.shape[0]):
                if L.hc[g] == synth.HEAD_RETRIEVAL:
                    if not selecting or sel is None:
                        total += N * 2 * spec.d * kv_el
                        if selecting:
                            total += N * spec.r * ix_el
                    else:
                        total += N * spec.r * ix_el
                        idx, cnt = sel[li]
                        u = set()
                        for h in range(g * G, (g + 1) * G):
                            u.update(idx[b, h, : int(cnt[b, h])].tolist())
                        total += len(u) * 2 * spec.d * kv_el
                else:
                    rows = min(N, spec.n_sink) + (N - max(min(N, spec.n_sink), N - spec.window))
                    total += rows * 2 * spec.d * kv_el
        if selecting:
            n_rq = sum(G for g in range(L.hc.shape[0]) if L.hc[g] == synth.HEAD_RETRIEVAL)
            total += n_rq * spec.r * spec.d * 4
    return total


def index_bytes(spec, layers):
    """Index keys the scan reads per step (every layer's retrieval groups)."""
    ix_el = 2 if spec.idx_dtype == "bf16" else 4
    tot = 0
    for L in layers:
        n_ret = int((L.hc == synth.HEAD_RETRIEVAL).sum())
        tot += n_ret * int(L.case.seq_lens.sum()) * spec.r * ix_el
    return tot


def replicas_for(spec, req, max_replicas):
    """Rotating cache replicas so that K steps in a row read >= 3 x L2 of
    distinct required bytes (one replica when a step alone exceeds that)."""
    if spec.layers > 1:
        return 1
    return max(1, min(max_replicas, math.ceil(3 * L2_BYTES / max(req, 1))))


# ------------------------------------------------------------------ our arm

class Bench:
    """One workload on this rank: its layers, rotating replicas, a workspace
    and the step through the C ABI."""

    def __init__(self, key, seed, dev):
        self.key = key
        self.spec, self.layers0 = build_workload(key, seed=seed)
        self.dev = dev
        self.out = torch.empty((self.spec.B, self.spec.H_q, self.spec.d), device=dev)
        self.ws = ops.Workspace(self.layers0[0].dims)
        self.reps = [self.layers0]
        self.stream = torch.cuda.Stream()

    def set_replicas(self, n):
        while len(self.reps) < n:
            self.reps.append([L.clone_caches() for L in self.layers0])
        self.reps = self.reps[:n]

    def step(self, layers, p, prof=None, sel=None, topk=0):
        """One step of every layer: top-p with p, or static top-k when topk > 0."""
        spec = self.spec
        for li, L in enumerate(layers):
            ops.append_index_keys(L.dims, L.k_new, L.Wk, L.pos, L.hc, L.kidx, self.ws)
            opts = None
            if prof is not None or sel is not None or topk:
                kw = {}
                if sel is not None:
                    kw = dict(sel_idx=sel[li][0], sel_count=sel[li][1])
                opts = ops.make_opts(prof=prof, topk=topk, **kw)
            ops.decode_step(L.dims, L.q, L.q_rope, L.k, L.v, L.kidx, L.Wq, L.hc, p, spec.window,
                            spec.n_sink, self.out, self.ws, opts)

    def dense_step(self, layers, out):
        for L in layers:
            ops.dense_decode(L.dims, L.q_rope if L.q_rope is not None else L.q, L.k, L.v, out, self.ws)

    def check(self):
        st = self.ws.check()
        if st:
            raise RuntimeError(f"device status {st}: {ops.error_string(st)}")

    def selection(self, p, topk=0):
        """Kept sets of one step -> (required bytes, kept counts per layer)."""
        spec = self.spec
        if p >= 1.0 and not topk:
            self.step(self.layers0, p)
            self.check()
            return required_bytes(spec, self.layers0, None, p), []
        sel = [(torch.full((spec.B, spec.H_q, L.k.shape[2]), -1, dtype=torch.int32, device=self.dev),
                torch.zeros((spec.B, spec.H_q), dtype=torch.int32, device=self.dev)) for L in self.layers0]
        self.step(self.layers0, p, sel=sel, topk=topk)
        self.check()
        req = required_bytes(spec, self.layers0, [(a.cpu().numpy(), b.cpu().numpy()) for a, b in sel], p,
                             topk)
        kept = [[int(x) for x in b.cpu().numpy().ravel() if x > 0] for _, b in sel]
        return req, kept

    def capture(self, fn):
        """One CUDA graph per replica of fn(replica)."""
        with torch.cuda.stream(self.stream):
            self.stream.wait_stream(torch.cuda.current_stream())
            for R in self.reps:
                fn(R)
        torch.cuda.current_stream().wait_stream(self.stream)
        torch.cuda.synchronize()
        graphs = []
        for R in self.reps:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(R)
            graphs.append(g)
        torch.cuda.synchronize()
        return graphs

    def time_graphs(self, graphs, steps, warmup, world, clocks=None):
        """Device ms per step over `steps` replays (max over ranks)."""
        n = len(graphs)
        for i in range(warmup):
            graphs[i % n].replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx = clocks if clocks is not None else _Null()
        with ctx:
            e0.record()
            for i in range(steps):
                graphs[i % n].replay()
            e1.record()
            torch.cuda.synchronize()
        barrier(world)
        return allreduce_max(e0.elapsed_time(e1), world, self.dev) / steps

    def launches_per_step(self, p, topk=0):
        pr = ops.Profiler(1024)
        self.step(self.reps[0], p, prof=pr, topk=topk)
        torch.cuda.synchronize()
        # rtp_append_index_keys takes no options, so its one launch per layer
        # is not in the profiler's count
        n = pr.p.count + len(self.layers0)
        pr.close()
        return n

    def breakdown(self, p, n_prof, per_step_slots, topk=0):
        """Per-kernel device times: the step captured with event-record nodes
        around every kernel (one graph per replica, distinct event slots),
        replayed with a sync after each replay to read the slots."""
        n_rep = len(self.reps)
        pr = ops.Profiler(per_step_slots * n_rep)
        pgraphs = []
        for R in self.reps:
            g = torch.cuda.CUDAGraph()
            first = pr.p.count
            with torch.cuda.graph(g):
                self.step(R, p, prof=pr, topk=topk)
            pgraphs.append((g, first, pr.p.count))
        torch.cuda.synchronize()
        times = {}
        for i in range(n_prof + n_rep):
            g, lo, hi = pgraphs[i % n_rep]
            g.replay()
            torch.cuda.synchronize()
            if i < n_rep:
                continue          # first pass over each graph: warm-up
            for slot in range(lo, hi):
                times.setdefault(pr.p.name[slot].decode(), []).append(ctypes_elapsed(pr, slot))
        pr.close()
        del pgraphs
        return times

    def dense_ms(self, steps, world):
        dense_out = torch.empty_like(self.out)
        graphs = self.capture(lambda R: self.dense_step(R, dense_out))
        ms = self.time_graphs(graphs, steps, 3, world)
        del graphs
        return ms

    def free(self):
        self.reps = []
        self.layers0 = []
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def kept_stats(kept):
    flat = [x for k in kept for x in k]
    if not flat:
        return {"min": 0, "max": 0, "mean": 0.0}
    return {"min": min(flat), "max": max(flat), "mean": float(np.mean(flat))}


def measure_point(bn, p, steps, warmup, world, hbm_peak, max_replicas, n_prof, clocks=None, topk=0):
    """One (workload, p) point -- or static top-k with topk > 0: step time,
    required bytes and their rate, the scan kernel's rate and the per-kernel
    times."""
    spec = bn.spec
    req, kept = bn.selection(p, topk)
    bn.set_replicas(replicas_for(spec, req, max_replicas))
    lps = bn.launches_per_step(p, topk)
    graphs = bn.capture(lambda R: bn.step(R, p, topk=topk))
    ms = bn.time_graphs(graphs, steps, warmup, world, clocks)
    del graphs
    times = bn.breakdown(p, n_prof, lps + 4, topk)
    hist = times.get("hist", [])
    # one scan launch per layer: its time per launch, and the index keys of
    # one layer's retrieval groups per launch
    hist_ms = float(np.mean(hist)) if hist else None
    idx_b = index_bytes(spec, bn.layers0) // max(1, len(bn.layers0)) if (p < 1.0 or topk) else 0
    scan_gbs = idx_b / (hist_ms * 1e-3) / 1e9 if hist_ms else None
    gbs = req / (ms * 1e-3) / 1e9
    n_rep = len(bn.reps)
    return {
        "p": None if topk else p, "topk": topk or None, "ms_per_step": ms, "steps_per_s": 1e3 / ms, "required_bytes_per_step": int(req),
        "achieved_gbs": gbs, "pct_peak": gbs / hbm_peak, "pct_of_8tbs": gbs / 8000.0,
        "scan": {"gbs": scan_gbs, "frac": scan_gbs / hbm_peak if scan_gbs else None,
                 "avg_launch_ms": hist_ms, "bytes_per_launch": idx_b},
        "kernels": {k: {"avg_ms": float(np.mean(v)), "launches_per_step": len(v) / n_prof}
                    for k, v in times.items()},
        "kept_rows_per_retrieval_head": kept_stats(kept),
        "launches_per_step": lps,
        "replicas": n_rep,
        "l2": f"rotating {n_rep} cache replicas ({n_rep} x {req / 1e6:.1f} MB >= 3 x L2)" if n_rep > 1
        else f"{spec.layers} layer(s) per step ({req / 1e6:.0f} MB > L2)" if req > 3 * L2_BYTES
        else f"1 replica ({req / 1e6:.1f} MB per step)",
    }


def e2e_measure(bn, p, graphs, steps, world):
    """End to end through the C ABI from pinned host memory: every step
    copies its q, q_rope and new key from the host, runs the C-ABI calls
    (rtp_append_index_keys + rtp_decode_step per layer) and copies the
    output back.  The headline form keeps each replica's step inputs in one
    device buffer (one pinned host buffer per double-buffer slot), so a step
    moves them with one copy, issues the calls through `ops.Prepared` (their
    arguments marshalled once) into an output buffer of the replica's own,
    runs the two copies on copy streams ordered by events (a step's copies
    overlap its neighbours' kernels) and waits on the host once per `depth`
    steps.  Also measured: the same with the copies in the compute stream;
    the binding's per-call marshalling with one copy per tensor; a host wait
    after every step; and the per-step-wait form with the calls replayed
    from a CUDA graph."""
    n_rep = len(bn.reps)
    L0 = bn.reps[0]
    has_rope = L0[0].q_rope is not None
    spec = bn.spec

    def pinned_like(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)

    # packed step inputs of each replica: (layer, q / q_rope / k_new) pieces at
    # 256-byte offsets of one buffer
    def pieces(R):
        out = []
        for L in R:
            out.append(L.q)
            if has_rope:
                out.append(L.q_rope)
            out.append(L.k_new)
        return out

    def layout(ts):
        offs, o = [], 0
        for t in ts:
            offs.append(o)
            o += (t.numel() * t.element_size() + 255) // 256 * 256
        return offs, o

    offs, total = layout(pieces(L0))
    packed, prepared, prepared_own, outs = [], [], [], []
    for R in bn.reps:
        dev = torch.empty(total, dtype=torch.uint8, device=bn.dev)
        views = []
        for t, o in zip(pieces(R), offs):
            v = dev[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
            v.copy_(t)
            views.append(v)
        own = torch.empty_like(bn.out)
        calls, calls_own, it = [], [], iter(views)
        for L in R:
            q = next(it)
            qr = next(it) if has_rope else None
            kn = next(it)
            a = ops.prepare_append_index_keys(L.dims, kn, L.Wk, L.pos, L.hc, L.kidx, bn.ws)
            calls.append(a)
            calls.append(ops.prepare_decode_step(L.dims, q, qr, L.k, L.v, L.kidx, L.Wq, L.hc, p, spec.window,
                                                 spec.n_sink, bn.out, bn.ws))
            calls_own.append(a)
            calls_own.append(ops.prepare_decode_step(L.dims, q, qr, L.k, L.v, L.kidx, L.Wq, L.hc, p,
                                                     spec.window, spec.n_sink, own, bn.ws))
        packed.append((dev, views))
        prepared.append(calls)
        prepared_own.append(calls_own)
        outs.append(own)
    hpk = []
    for _ in range(2):
        h = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        h.copy_(packed[0][0].cpu())
        hpk.append(h)
    hout = [pinned_like(bn.out) for _ in range(2)]
    # the per-call form's host buffers (one per tensor)
    bufs = []
    for _ in range(2):
        hq = [pinned_like(L.q) for L in L0]
        hqr = [pinned_like(L.q) for L in L0]
        hk = [pinned_like(L.k_new) for L in L0]
        for i, L in enumerate(L0):
            hq[i].copy_(L.q)
            hqr[i].copy_(L.q_rope if L.q_rope is not None else L.q)
            hk[i].copy_(L.k_new)
        bufs.append((hq, hqr, hk))
    h2d = sum(t.numel() * t.element_size() for t in pieces(L0))
    d2h = bn.out.numel() * bn.out.element_size()

    def one_prepared(i, wait):
        packed[i % n_rep][0].copy_(hpk[i % 2], non_blocking=True)
        for c in prepared[i % n_rep]:
            c()
        hout[i % 2].copy_(bn.out, non_blocking=True)
        if wait:
            torch.cuda.current_stream().synchronize()

    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(n_rep)]
    ev_done = [torch.cuda.Event() for _ in range(n_rep)]
    ev_out = [torch.cuda.Event() for _ in range(n_rep)]

    def one_overlapped(i, wait):
        r = i % n_rep
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[r])          # the replica's previous step has read its inputs
            packed[r][0].copy_(hpk[i % 2], non_blocking=True)
            ev_in[r].record(s_in)
        main.wait_event(ev_in[r])
        main.wait_event(ev_out[r])               # its previous output has been copied out
        for c in prepared_own[r]:
            c()
        ev_done[r].record(main)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[r])
            hout[i % 2].copy_(outs[r], non_blocking=True)
            ev_out[r].record(s_out)
        if wait:
            torch.cuda.synchronize()

    def one_per_call(i, use_graph, wait):
        hq, hqr, hk = bufs[i % 2]
        R = bn.reps[i % n_rep]
        for j, L in enumerate(R):
            L.q.copy_(hq[j], non_blocking=True)
            if has_rope:
                L.q_rope.copy_(hqr[j], non_blocking=True)
            L.k_new.copy_(hk[j], non_blocking=True)
        if use_graph:
            graphs[i % n_rep].replay()
        else:
            bn.step(R, p)
        hout[i % 2].copy_(bn.out, non_blocking=True)
        if wait:
            torch.cuda.current_stream().synchronize()

    def run(one, depth):
        for i in range(3):
            one(i, True)
        barrier(world)
        x0, x1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        x0.record()
        s_in.wait_stream(main)                   # the first input copy is inside the timed region
        for i in range(steps):
            one(i, (i + 1) % depth == 0)
        main.wait_stream(s_out)                  # the last output copy is inside the timed region
        x1.record()
        torch.cuda.synchronize()
        return world * steps / (allreduce_max(x0.elapsed_time(x1), world, bn.dev) / 1e3)

    depth = 64
    overlapped = run(one_overlapped, depth)
    pipelined = run(one_prepared, depth)
    per_call = run(lambda i, w: one_per_call(i, False, w), depth)
    per_step = run(one_prepared, 1)
    graph_step = run(lambda i, w: one_per_call(i, True, w), 1)
    return {"value": overlapped, "unit": "steps/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "note": f"per step: the step's q/q_rope/k_new of every layer, packed in one pinned host buffer "
                    f"(double-buffered), -> device in one copy on a copy stream; the C-ABI calls "
                    f"(rtp_append_index_keys + rtp_decode_step per layer) through ops.Prepared into the "
                    f"replica's output buffer; out -> pinned host on a second copy stream; streams ordered "
                    f"by events; one host wait per {depth} steps",
            "inorder_value": pipelined,
            "inorder_note": "the same with both copies in the compute stream and one output buffer",
            "per_call_value": per_call,
            "per_call_note": "the same with the binding's per-call argument marshalling and one host-to-device "
                             "copy per tensor",
            "sync_value": per_step,
            "sync_note": "the headline form with a host wait after every step",
            "graph_value": graph_step,
            "graph_note": "one copy per tensor, the step's C-ABI calls captured once in a CUDA graph and "
                          "replayed, a host wait after every step"}


# static top-k budget measured beside the headline's top-p (tokens per head)
TOPK_BUDGET = 2048

# workloads measured beside the headline line, in the same run
SWEEP = (("ctx64k", (0.9,)), ("ctx1m", (0.8, 0.9, 0.95, 1.0)), ("ctx128k-b8-48layer", (0.9,)))


def measure_workload(key, ps, args, rank, world, dev, hbm_peak):
    bn = Bench(key, rank_seed(0, rank), dev)
    try:
        pts = {}
        for p in ps:
            pts[str(p)] = measure_point(bn, p, args.sweep_steps, args.warmup, world, hbm_peak,
                                        args.max_replicas, min(args.prof_steps, 50))
        dense = bn.dense_ms(max(3, min(args.sweep_steps, args.dense_steps)), world)
        spec = bn.spec
        for v in pts.values():
            v["dense_ms_per_step"] = dense
            v["speedup_sparse_vs_dense"] = dense / v["ms_per_step"]
        return {"workload": spec.name, "B": spec.B, "ctx": spec.N, "layers": spec.layers,
                "dense_bytes_per_step": int(sum(2 * L.k.numel() * L.k.element_size() for L in bn.layers0)),
                "points": pts}
    finally:
        bn.free()
        del bn
        torch.cuda.empty_cache()


def local_pairs(n: int, window: int, n_sink: int) -> int:
    """Rows a local head attends over at a step with n cached tokens."""
    s = min(n_sink, n)
    return s + (n - max(s, n - window))


def prefill_pairs(pos0: int, T: int, window: int, n_sink: int, local: bool) -> int:
    """(query, key) pairs of one head's causal prefill attention over prompt
    tokens at positions pos0 .. pos0 + T - 1."""
    if not local:
        a, b = pos0 + 1, pos0 + T
        return (a + b) * T // 2
    return sum(local_pairs(P + 1, window, n_sink) for P in range(pos0, pos0 + T))


def measure_sharded(args, world, dev, Ps=(2, 4)):
    """The context-sharded step on the 1M-token workload, its P shards run
    one after another on this one GPU (the exchanges as tensor operations):
    each phase's device time per shard (CUDA events, L2 flushed before each
    repetition) and the bytes each exchange moves.  On P GPUs the shards'
    phases would run side by side with NCCL exchanges between them; that
    time is not measured here (every run of this bench has its own GPU)."""
    from dynamic_top_sparse_b200 import shard as rshard
    spec = synth.spec_for("ctx1m")
    p = 0.9
    c = synth.make_case(spec, device="cuda", seed=rank_seed(0, 0), layer=0)
    L = Layer(c)
    ops.append_index_keys(L.dims, L.k_new, L.Wk, L.pos, L.hc, L.kidx, ops.Workspace(L.dims))
    N = int(c.seq_lens[0])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    whole = torch.empty((1, spec.H_q, spec.d), device=dev)
    ws = ops.Workspace(L.dims)
    ops.decode_step(L.dims, L.q, L.q_rope, L.k, L.v, L.kidx, L.Wq, L.hc, p, spec.window, spec.n_sink, whole, ws)
    res = {"workload": "1M ctx, B1, 32q/4kv, bf16, all retrieval, ranked needles, p=0.9, split into P "
                       "contiguous token ranges", "p": p, "points": {}}
    for P in Ps:
        bounds = [round(i * N / P) for i in range(P + 1)]
        shards, seqs = [], []          # dims hold the device address of seq_lens: keep them alive
        for i in range(P):
            lo, n = bounds[i], bounds[i + 1] - bounds[i]
            seqs.append(torch.tensor([n], dtype=torch.int32, device=dev))
            dims = ops.make_dims(1, spec.H_q, spec.H_kv, n, seqs[-1], ops.RTP_BF16, ops.RTP_BF16)
            shards.append(rshard.Shard(dims, L.q, L.q_rope, L.k[:, :, lo:lo + n].contiguous(),
                                       L.v[:, :, lo:lo + n].contiguous(), L.kidx[:, :, lo:lo + n].contiguous(),
                                       L.Wq, L.hc, torch.tensor([lo], dtype=torch.int32, device=dev),
                                       c.seq_lens.clone(), ops.Workspace(dims)))
        out = torch.empty_like(whole)
        ev = lambda: torch.cuda.Event(enable_timing=True)
        times = {"scan": [], "collect": [], "finish": []}
        ncand = 0
        for rep in range(4):
            flush.fill_(rep)
            marks = {k: [] for k in times}
            hists = []
            for sh in shards:
                e0, e1 = ev(), ev()
                e0.record(); hists.append(rshard.phase_scan(sh, p)); e1.record()
                marks["scan"].append((e0, e1))
            total = torch.stack(hists).sum(0)
            for h in hists:
                h.copy_(total)
            cands = []
            for sh in shards:
                e0, e1 = ev(), ev()
                e0.record(); cands.append(rshard.phase_collect(sh, p)); e1.record()
                marks["collect"].append((e0, e1))
            all_keys, all_counts = rshard.gather_candidates([k for k, _ in cands], [n for _, n in cands])
            parts = []
            for sh in shards:
                e0, e1 = ev(), ev()
                e0.record()
                parts.append(rshard.phase_finish(sh, p, spec.window, spec.n_sink, all_keys, all_counts))
                e1.record()
                marks["finish"].append((e0, e1))
            ops.merge_shards(torch.stack(parts).contiguous(), out)
            torch.cuda.synchronize()
            if rep > 0:                                   # the first repetition warms up
                for k in times:
                    times[k].append([a.elapsed_time(b) for a, b in marks[k]])
            ncand = int(all_counts.sum())
        for sh in shards:
            st = sh.ws.check()
            if st:
                raise RuntimeError(f"sharded step: device status {st}: {ops.error_string(st)}")
        per = {k: [float(np.median([r[i] for r in v])) for i in range(P)] for k, v in times.items()}
        nh = spec.H_q
        res["points"][str(P)] = {
            "P": P,
            "ms_per_shard": per,
            "ms_sum_of_phase_maxima": sum(max(v) for v in per.values()),
            "exchange_bytes": {"histograms_allreduce": nh * 640 * 8,
                               "candidates_allgather": ncand * 8 + P * nh * 4,
                               "partials_allgather": P * nh * ops.PART_STRIDE * 4},
            "max_abs_diff_vs_whole_step": float((out - whole).abs().max()),
        }
        del shards, seqs
    res["whole_step_ms_note"] = "the unsharded 1M step at p = 0.9 is the ctx1m point of `workloads`"
    return res


def measure_prefill(args, world, dev):
    """Prefill of a whole 64K-token prompt in the 64K workload's shape (32 q /
    4 KV heads, KV0 retrieval, window 4096 + 4 sinks): the prompt's index
    keys (rtp_append_index_keys, T = N) and its causal attention
    (rtp_prefill_attention), against the same attention with every head
    keeping the full cache.  Tensor-bound: FLOPs = 4 d per (query, key)
    pair (q.k and p.v)."""
    spec = synth.spec_for("ctx64k")
    B, H_q, H_kv, N, d = 1, spec.H_q, spec.H_kv, spec.N, spec.d
    G = H_q // H_kv
    hc = np.array([1, 0, 0, 0], np.uint8)
    g = torch.Generator(device=dev).manual_seed(rank_seed(17, 0))
    q = torch.randn(B, H_q, N, d, generator=g, device=dev).to(torch.bfloat16)
    k = torch.randn(B, H_kv, N, d, generator=g, device=dev).to(torch.bfloat16)
    v = torch.randn(B, H_kv, N, d, generator=g, device=dev).to(torch.bfloat16)
    W = torch.randn(H_kv, spec.r, d, generator=g, device=dev) / math.sqrt(d)
    kidx = torch.zeros(B, H_kv, N, spec.r, dtype=torch.bfloat16, device=dev)
    seq = torch.full((B,), N, dtype=torch.int32, device=dev)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    dims = ops.make_dims(B, H_q, H_kv, N, seq, ops.RTP_BF16, ops.RTP_BF16)
    ws = ops.Workspace(dims)
    out = torch.empty(B, H_q, N, d, device=dev)

    def timed(fn, n):
        fn()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return allreduce_max(e0.elapsed_time(e1), world, dev) / n

    n = max(2, args.prefill_steps)
    ms_rtp = timed(lambda: ops.prefill_attention(dims, q, pos0, k, v, hc, spec.window, spec.n_sink, out, ws), n)
    ms_full = timed(lambda: ops.prefill_attention(dims, q, pos0, k, v, np.ones(H_kv, np.uint8), spec.window,
                                                  spec.n_sink, out, ws), n)
    ms_keys = timed(lambda: ops.append_index_keys(dims, k, W, pos0, hc, kidx, ws), max(n, 20))
    if ws.check():
        raise RuntimeError("prefill: device status set")
    pairs = sum(G * prefill_pairs(0, N, spec.window, spec.n_sink, hc[gi] == 0) for gi in range(H_kv))
    pairs_full = H_q * prefill_pairs(0, N, spec.window, spec.n_sink, False)
    fl, fl_full = 4 * d * pairs, 4 * d * pairs_full
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tf_peak, tf_src = float(json.load(f)["bf16_tflops"]), "measured bf16_tflops (cuBLAS burst)"
    except Exception:
        tf_peak, tf_src = 1590.0, "fallback 1590 TFLOP/s"
    ret = int(hc.sum())
    key_bytes = B * ret * N * (d * 2 + spec.r * 2)
    res = {
        "workload": f"prefill of a {N}-token prompt, B1, 32q/4kv, KV0 retrieval (full causal), "
                    f"KV1-3 local (window {spec.window} + {spec.n_sink} sinks), bf16",
        "attention_ms": ms_rtp, "flops": fl, "tflops": fl / (ms_rtp * 1e-3) / 1e12,
        "full_attention_ms": ms_full, "full_flops": fl_full,
        "full_tflops": fl_full / (ms_full * 1e-3) / 1e12,
        "speedup_vs_full": ms_full / ms_rtp,
        "roofline": {"bound": "tensor", "achieved": fl / (ms_rtp * 1e-3) / 1e12, "peak": tf_peak,
                     "unit": "TFLOP/s", "frac": fl / (ms_rtp * 1e-3) / 1e12 / tf_peak,
                     "peak_source": tf_src},
        "index_keys_ms": ms_keys, "index_keys_gbs": key_bytes / (ms_keys * 1e-3) / 1e9,
        "index_keys_bytes": key_bytes,
        "steps": n,
    }
    del q, k, v, kidx, out
    torch.cuda.empty_cache()
    return res


def run_ours(args, rank, world, dev):
    # each rank serves sequences of its own (rank 0's are the single-GPU workload)
    hbm_peak, peak_src = peaks()
    bn = Bench(args.workload, rank_seed(0, rank), dev)
    spec = bn.spec
    if args.p is not None:
        spec.p = args.p
    p = spec.p
    clocks = Clocks(dev.index)
    pt = measure_point(bn, p, args.steps, args.warmup, world, hbm_peak, args.max_replicas,
                       max(1, min(args.steps, args.prof_steps)), clocks)
    ms_per_step = pt["ms_per_step"]
    value = world / (ms_per_step * 1e-3)
    dense_ms = bn.dense_ms(max(3, min(args.steps, args.dense_steps)), world)
    # static top-k on the same caches, beside top-p: the fixed budget of
    # TOPK_BUDGET tokens per head
    topk_pt = measure_point(bn, p, args.sweep_steps, args.warmup, world, hbm_peak, args.max_replicas,
                            min(args.prof_steps, 50), topk=TOPK_BUDGET)
    topk_pt["dense_ms_per_step"] = dense_ms
    topk_pt["speedup_sparse_vs_dense"] = dense_ms / topk_pt["ms_per_step"]
    bn.set_replicas(pt["replicas"])

    e2e = None
    if not args.no_e2e:
        graphs = bn.capture(lambda R: bn.step(R, p))
        e2e = e2e_measure(bn, p, graphs, max(3, min(args.steps, args.e2e_steps)), world)
        del graphs
    dense_bytes = int(sum(2 * L.k.numel() * L.k.element_size() for L in bn.layers0))
    n_rep = pt["replicas"]
    workload = spec.name
    bn.free()
    del bn

    sweep = {}
    if not args.no_sweep:
        for key, ps in SWEEP:
            if key == args.workload:
                continue
            sweep[key] = measure_workload(key, ps, args, rank, world, dev, hbm_peak)

    prefill = None if args.no_prefill else measure_prefill(args, world, dev)
    sharded = None if args.no_sharded or world > 1 else measure_sharded(args, world, dev)

    sc = pt["scan"]
    res = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload, "key": args.workload, "B": spec.B, "ctx": spec.N, "H_q": spec.H_q,
                   "H_kv": spec.H_kv, "d": spec.d, "r": spec.r, "layers": spec.layers, "p": p,
                   "window": spec.window, "n_sink": spec.n_sink, "cache_dtype": spec.kv_dtype,
                   "index_dtype": spec.idx_dtype, "accumulate": "f32", "l2": pt["l2"],
                   "timing": "CUDA graph replays, CUDA events, max over ranks",
                   "parallelism": f"replicas x{world} (independent sequences per rank)"},
        "required_bytes_per_step": pt["required_bytes_per_step"],
        "achieved_gbs": pt["achieved_gbs"],
        "pct_peak": pt["pct_peak"],
        "pct_of_8tbs": pt["pct_of_8tbs"],
        "kept_rows_per_retrieval_head": pt["kept_rows_per_retrieval_head"],
        "roofline": {"bound": "hbm", "kernel": "hist (index-key scan + mass histogram)",
                     "achieved": sc["gbs"], "peak": hbm_peak, "unit": "GB/s",
                     "frac": sc["frac"],
                     "traffic": traffic_for("hist", workload),
                     "bytes_per_launch": sc["bytes_per_launch"], "avg_launch_ms": sc["avg_launch_ms"],
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback 6650 GB/s"},
        "dense": {"ms_per_step": dense_ms, "speedup_sparse_vs_dense": dense_ms / ms_per_step,
                  "bytes_per_step": dense_bytes},
        "kernels": pt["kernels"],
        "gpu_launches": int(pt["launches_per_step"] * args.steps),
        "launches_per_step": pt["launches_per_step"],
        "replicas": n_rep,
        "clocks": clocks.report(),
        "e2e": e2e,
        "topk": topk_pt,
        "workloads": sweep,
        "prefill": prefill,
        "sharded": sharded,
        "pages_context": {"decode_speedup_1M_H20": 2.01, "prefill_speedup_1M_H20": 9.36},
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(args.workload, spec, args.cpu_seconds)
    return res


# ------------------------------------------------------------------ oracle arm

def cpu_baseline(key, spec=None, budget_s=15.0):
    """The oracle, as it stands, on host cores over a bounded sample of the
    workload (whole layers of one replica); steps/s scaled to full steps."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(limits=1)
    except Exception:
        lim = None
    spec = spec or synth.spec_for(key)
    layers_done, t_tot = 0, 0.0
    seqs = list(range(spec.B))
    # layers are taken in turn (again from the first when the step has fewer
    # layers than the budget covers) until about budget_s of oracle time
    last = None
    for l in itertools.cycle(range(spec.layers)):
        if last is None or last[0] != l:
            last = None
            c = synth.make_case(spec, device="cuda" if torch.cuda.is_available() else "cpu", layer=l)
            q = c.q.cpu().numpy()
            qr = None if c.q_rope is None else c.q_rope.cpu().numpy()
            K, V = c.k_cache.float().cpu().numpy(), c.v_cache.float().cpu().numpy()
            if c.k_pre_all is not None:
                kidx0 = oracle.append_index_keys(np.zeros(tuple(c.kidx_cache.shape)),
                                                 c.k_pre_all.float().cpu().numpy(), c.W_k_idx.cpu().numpy(),
                                                 np.zeros(spec.B, np.int64), spec.idx_dtype)
            else:
                kidx0 = c.kidx_cache.float().cpu().numpy()
            last = (l, c, q, qr, K, V, kidx0)
        _, c, q, qr, K, V, kidx = last
        heads = [(b, h) for b in seqs for h in range(spec.H_q)]
        t0 = time.perf_counter()
        kidx = oracle.append_index_keys(kidx, c.k_pre_new.float().cpu().numpy(), c.W_k_idx.cpu().numpy(),
                                        c.seq_lens.cpu().numpy() - 1, spec.idx_dtype, head_class=c.head_class)
        oracle.decode_step(q, qr, K, V, kidx, c.W_q_idx.cpu().numpy(), c.head_class, c.seq_lens.cpu().numpy(),
                           spec.p, spec.window, spec.n_sink, heads=heads)
        t_tot += time.perf_counter() - t0
        layers_done += 1
        del kidx
        if t_tot >= budget_s:
            break
    if lim is not None:
        lim.unregister() if hasattr(lim, "unregister") else None
    per_layer = t_tot / layers_done
    step_s = per_layer * spec.layers
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{layers_done} layer pass(es) over a step of {spec.layers} layer(s), all {spec.B} "
                      f"sequence(s) x {spec.H_q} heads each, {t_tot:.1f} s of single-threaded numpy fp64; "
                      f"steps/s = 1 / (mean per-layer time x layers)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    spec = synth.spec_for(args.workload)
    if args.p is not None:
        spec.p = args.p
    cb = cpu_baseline(args.workload, spec, args.cpu_seconds)
    v = cb["value"]
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / v, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name, "key": args.workload, "B": spec.B, "ctx": spec.N, "p": spec.p},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "note": "the CPU oracle (numpy fp64), timed on host cores over a bounded sample"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default="ctx512k", choices=list(synth.WORKLOADS))
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--prof-steps", type=int, default=200)
    ap.add_argument("--dense-steps", type=int, default=200)
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--max-replicas", type=int, default=64)
    ap.add_argument("--no-sweep", action="store_true",
                    help="measure only --workload (no other workloads in the same run)")
    ap.add_argument("--sweep-steps", type=int, default=400)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-sharded", action="store_true")
    ap.add_argument("--prefill-steps", type=int, default=5)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        sys.exit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; launch N > 1 ranks with "
                 f"torch.distributed.run --nproc-per-node N")
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res))
        return
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    try:
        res = run_ours(args, rank, world, dev)
        if rank == 0:
            print(json.dumps(res))
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

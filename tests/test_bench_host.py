"""Host-side arithmetic of bench.py (CPU): the step's required bytes, the
numerator of its roofline."""
import types

import numpy as np
import pytest
import torch

import bench
from dynamic_top_sparse_b200 import synth


def _layer(lens, hc, H_q):
    case = types.SimpleNamespace(seq_lens=torch.tensor(lens, dtype=torch.int32))
    return types.SimpleNamespace(case=case, hc=np.asarray(hc, np.uint8), H_q=H_q)


def _spec(B, N, p=0.9, kv="bf16", idx="bf16"):
    return synth.Spec("t", B=B, H_q=8, H_kv=2, N=N, kv_dtype=kv, idx_dtype=idx, p=p, window=16, n_sink=4)


def test_required_bytes_counts_the_group_union_once():
    """Group 0 retrieval (query heads 0-3), group 1 local; two sequences.
    Kept rows of the group's heads overlap: their union is read once."""
    spec = _spec(B=2, N=100)
    L = _layer([100, 60], [1, 0], 8)
    idx = np.full((2, 8, 100), -1, np.int32)
    cnt = np.zeros((2, 8), np.int32)
    kept = {(0, 0): [5, 6, 7], (0, 1): [6, 7, 8], (0, 2): [99], (0, 3): [5],
            (1, 0): [0], (1, 1): [0], (1, 2): [0], (1, 3): [59, 58]}
    for (b, h), ids in kept.items():
        idx[b, h, :len(ids)] = ids
        cnt[b, h] = len(ids)
    got = bench.required_bytes(spec, [L], [(idx, cnt)])
    kidx = (100 + 60) * 16 * 2                      # index keys of the retrieval group, bf16
    rows = (5 + 3) * 2 * 128 * 2                    # unions {5,6,7,8,99} and {0,58,59}: K and V rows
    local = (4 + 16) * 2 * 128 * 2 * 2              # 4 sinks + 16 window rows, both sequences
    wq = 4 * 16 * 128 * 4                           # W_q_idx of the 4 retrieval query heads, fp32
    assert got == kidx + rows + local + wq


def test_required_bytes_short_sequence_reads_each_local_row_once():
    """N below window + sinks: every row once, not sinks and window twice."""
    spec = _spec(B=1, N=10)
    L = _layer([10], [0, 0], 8)
    got = bench.required_bytes(spec, [L], [(np.zeros((1, 8, 10), np.int32), np.zeros((1, 8), np.int32))])
    assert got == 2 * 10 * 2 * 128 * 2


@pytest.mark.parametrize("p", [1.0, 1.5])
def test_required_bytes_keep_all_reads_every_row(p):
    """p >= 1 keeps every token without a threshold: the step reads every
    K/V row of the retrieval groups and neither index keys nor W_q_idx."""
    spec = _spec(B=1, N=50, p=p, kv="f32", idx="f32")
    L = _layer([50], [1, 1], 8)
    got = bench.required_bytes(spec, [L], None)
    assert got == 2 * 50 * 2 * 128 * 4
    # the p argument overrides the workload's own
    assert bench.required_bytes(_spec(B=1, N=50, p=0.5, kv="f32", idx="f32"), [L], None, p) == got


def test_index_bytes_per_layer_and_sequence_lengths():
    """Index keys the scan reads: retrieval groups x the sequences' own
    lengths, summed over layers."""
    spec = _spec(B=2, N=100)
    la = _layer([100, 60], [1, 0], 8)
    lb = _layer([100, 60], [1, 1], 8)
    assert bench.index_bytes(spec, [la, lb]) == (1 + 2) * 160 * 16 * 2


def test_replicas_cover_three_l2():
    spec = _spec(B=1, N=100)
    assert bench.replicas_for(spec, 8_500_000, 64) == 47      # 3 x 126 MiB / 8.5 MB
    assert bench.replicas_for(spec, 8_500_000, 16) == 16
    assert bench.replicas_for(spec, 2_000_000_000, 64) == 1
    spec.layers = 48
    assert bench.replicas_for(spec, 1000, 64) == 1


def test_gpus_must_match_world_size(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr("sys.argv", ["bench.py", "--gpus", "8"])
    with pytest.raises(SystemExit) as e:
        bench.main()
    assert "WORLD_SIZE=1" in str(e.value)


class _FakeNvml:
    """Reads only: clocks and clock-event reason words from fixed lists."""
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, reasons, fail_init=False):
        self._c, self._r, self._fail = iter(clocks), iter(reasons), fail_init

    def nvmlInit(self):
        if self._fail:
            raise RuntimeError("no driver")

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        raise RuntimeError("by index instead")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        return next(self._c)

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return next(self._r)


def test_clock_report_decodes_reasons_and_takes_the_median(monkeypatch):
    import sys
    fake = _FakeNvml([1965, 1965, 1800, 1965, 1300], [0x1, 0x4, 0x0, 0x4 | 0x20, 0x8])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    c = bench.Clocks(0)
    for _ in range(5):
        c._sample()
    rep = c.report()
    assert rep["sm_mhz"] == 1965 and rep["sm_max_mhz"] == 1965 and rep["samples"] == 5
    # gpu_idle is not a slowdown; the others are named as NVML defines the bits
    assert rep["reasons"] == ["hw_slowdown", "sw_power_cap", "sw_thermal_slowdown"]


def test_clock_report_without_nvml(monkeypatch):
    import sys
    monkeypatch.setitem(sys.modules, "pynvml", _FakeNvml([], [], fail_init=True))
    rep = bench.Clocks(0).report()
    assert rep["sm_mhz"] is None and rep["reasons"] == [] and "NVML" in rep["note"]


def test_recorded_traffic_is_used_only_while_the_scan_sources_are_unchanged(tmp_path, monkeypatch):
    import json
    import shutil
    src = tmp_path / "dynamic_top_sparse_b200" / "csrc"
    src.mkdir(parents=True)
    for name in bench.SCAN_SOURCES:
        shutil.copy(f"{bench.ROOT}/dynamic_top_sparse_b200/csrc/{name}", src / name)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"records": [{"kernel": "hist", "workload": "w", "csrc": bench.csrc_hash(), "bytes_per_launch": 123}]}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_for("hist", "w") == 123
    assert bench.traffic_for("hist", "other workload") is None
    with open(src / bench.SCAN_SOURCES[-1], "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_for("hist", "w") is None


def test_reference_arm_under_two_ranks_prints_one_line_from_rank0():
    """The reference arm (the oracle on host cores) launched like the
    multi-GPU bench: rank 0 prints one JSON line, the other rank exits 0
    without output."""
    import json
    import os
    import socket
    import subprocess
    import sys
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "3", "--warmup", "3", "--workload", "ctx4k-fp32", "--cpu-seconds", "1"]
    r = subprocess.run(cmd, cwd=bench.ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["n_gpus"] == 2 and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


def test_prefill_pairs_closed_forms():
    """Causal pairs: T tokens from position 0 see 1 + 2 + ... + T keys; a
    local head's tokens see min(P + 1, window + sinks) keys once the
    window has passed the sinks."""
    assert bench.prefill_pairs(0, 10, 4, 1, False) == 55
    assert bench.prefill_pairs(5, 3, 4, 1, False) == 6 + 7 + 8
    # window 4, 1 sink: positions 0..9 see 1, 2, 3, 4, 5, then 5 each
    assert bench.prefill_pairs(0, 10, 4, 1, True) == 1 + 2 + 3 + 4 + 5 * 6
    assert bench.local_pairs(3, 100, 4) == 3
    assert bench.local_pairs(1000, 4096, 4) == 1000
    assert bench.local_pairs(65536, 4096, 4) == 4100

"""Comparison helpers shared by the GPU parity tests (test infrastructure)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from dynamic_top_sparse_b200 import ops, synth

# Tolerances.  Sets: bit-exact except tokens whose oracle cumulative mass
# (strictly before them, descending order) lies within MASS_TOL of p; the
# kept set's oracle mass must reach p - MASS_TOL.
MASS_TOL = 1e-5
# Attention output vs the oracle over its own kept set (bf16 caches, fp32
# accumulation).
OUT_TOL = 2e-3
# Attention output vs the oracle over the GPU's kept set: only fp32
# accumulation error remains (fp32 products and sums over <= 1M rows of
# unit-scale values, exp2 of fp32 logits).
OUT_TOL_SAME_SET = 1e-4


def np64(t: torch.Tensor) -> np.ndarray:
    """Exact widening to fp64 (bf16 -> fp32 is exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def np32(t: torch.Tensor) -> np.ndarray:
    """Exact fp32 host copy (bf16 -> fp32 is exact); the oracle widens the
    rows it uses to fp64."""
    return t.detach().float().cpu().numpy()


def gpu_set(sel_idx: torch.Tensor, sel_count: torch.Tensor, b: int, h: int) -> np.ndarray:
    n = int(sel_count[b, h])
    ids = sel_idx[b, h, :n].cpu().numpy()
    return ids


def check_selection(ids: np.ndarray, sel: oracle.Selection, p: float, where: str = ""):
    """The set rule (bit-exact except tokens within MASS_TOL of the p
    boundary) plus the mass floor.  Returns (n_diff, mass)."""
    assert ids.size >= 1, f"{where}: empty kept set"
    assert np.unique(ids).size == ids.size, f"{where}: duplicate ids"
    n = sel.pi.shape[0]
    assert ids.min() >= 0 and ids.max() < n, f"{where}: id out of range"
    ref = set(sel.kept.tolist())
    got = set(ids.tolist())
    diff = ref ^ got
    if diff:
        amb = set(sel.ambiguous(p, MASS_TOL).tolist())
        bad = diff - amb
        assert not bad, (f"{where}: {len(bad)} ids differ outside the {MASS_TOL} mass window "
                         f"(|S_gpu|={len(got)}, |S*|={len(ref)}), e.g. {sorted(bad)[:8]}")
    mass = float(sel.pi[ids].sum())
    if p < 1.0:
        assert mass >= min(p, 1.0) - MASS_TOL, f"{where}: kept mass {mass} < p - tol"
    return len(diff), mass


def within(a: np.ndarray, b: np.ndarray, tol: float, where: str = ""):
    err = float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))
    assert err <= tol, f"{where}: max abs err {err:.3e} > {tol:.1e}"
    return err


class GpuCase:
    """A synth.Case moved to the GPU plus everything the library needs."""

    def __init__(self, case: synth.Case):
        self.c = case
        dev = torch.device("cuda")
        # fresh device copies: the library writes index keys into its own
        # copy, never into the tensors the oracle reads
        mv = lambda t: None if t is None else t.to(dev).clone().contiguous()
        self.q = mv(case.q)
        self.q_rope = mv(case.q_rope)
        self.k = mv(case.k_cache)
        self.v = mv(case.v_cache)
        self.kidx = mv(case.kidx_cache)
        self.Wq = mv(case.W_q_idx)
        self.Wk = mv(case.W_k_idx)
        self.k_new = mv(case.k_pre_new)
        self.seq = mv(case.seq_lens)
        self.hc = case.head_class
        B, H_kv, N_max, d = self.k.shape
        self.B, self.H_kv, self.N_max = B, H_kv, N_max
        self.H_q = self.q.shape[1]
        self.dims = ops.dims_for(self.k, self.kidx, self.H_q, self.seq)
        self.ws = ops.Workspace(self.dims)
        if case.k_pre_all is not None:
            # index keys of every row come from the append step
            pos = torch.zeros(B, dtype=torch.int32, device=dev)
            ops.append_index_keys(self.dims, mv(case.k_pre_all), self.Wk, pos, self.hc, self.kidx, self.ws)

    def append_current(self):
        """Append the current token's index key (row N_b - 1)."""
        pos = (self.seq - 1).to(torch.int32)
        ops.append_index_keys(self.dims, self.k_new, self.Wk, pos, self.hc, self.kidx, self.ws)

    def step(self, p, window=None, n_sink=None, want_sel=True, out=None, topk=0, idx_scale=0.0,
             force_local=False):
        window = self.c.window if window is None else window
        n_sink = self.c.n_sink if n_sink is None else n_sink
        dev = self.q.device
        out = torch.full((self.B, self.H_q, 128), float("nan"), device=dev) if out is None else out
        sel_idx = sel_cnt = sel_mass = None
        if want_sel:
            sel_idx = torch.full((self.B, self.H_q, self.N_max), -1, dtype=torch.int32, device=dev)
            sel_cnt = torch.zeros((self.B, self.H_q), dtype=torch.int32, device=dev)
            sel_mass = torch.zeros((self.B, self.H_q), dtype=torch.float32, device=dev)
        opts = ops.make_opts(idx_scale=idx_scale, sel_idx=sel_idx, sel_count=sel_cnt, sel_mass=sel_mass, topk=topk,
                             force_local=force_local)
        ops.decode_step(self.dims, self.q, self.q_rope, self.k, self.v, self.kidx, self.Wq, self.hc, p,
                        window, n_sink, out, self.ws, opts)
        st = self.ws.check()
        assert st == 0, f"device status {st}: {ops.error_string(st)}"
        return out, sel_idx, sel_cnt, sel_mass


def oracle_kidx(gc: GpuCase, idx_dtype: str, with_current: bool):
    """The oracle's own index-key cache: the 4K fp32 workload builds every row with its
    append; with_current appends the current token's key at N_b - 1."""
    c = gc.c
    if c.k_pre_all is not None:
        B, H_kv, N_max, _ = c.k_pre_all.shape
        kidx = oracle.append_index_keys(np.zeros((B, H_kv, N_max, 16)), np64(c.k_pre_all), np64(c.W_k_idx),
                                        np.zeros(B, np.int64), idx_dtype, head_class=c.head_class)
    else:
        kidx = np64(c.kidx_cache)
    if with_current:
        pos = c.seq_lens.cpu().numpy() - 1
        kidx = oracle.append_index_keys(kidx, np64(c.k_pre_new), np64(c.W_k_idx), pos, idx_dtype,
                                        head_class=c.head_class)
    return kidx

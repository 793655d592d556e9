"""Pins for the CPU oracle: each test checks the oracle against something
other than itself -- hand-derived fixtures, brute force, closed forms,
special cases that reduce to plain dense attention, and invariants -- so
that a dropped term, a wrong sign or index, or a transposed operand fails.
CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from dynamic_top_sparse_b200 import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- fixtures

def test_golden_topp_rational(golden_dir):
    fx = _load(golden_dir, "topp_rational.json")
    for c in fx["cases"]:
        z = np.log(np.asarray(c["w"], dtype=np.float64))
        sel = oracle.topp_select(z, c["p"])
        assert sel.kept.tolist() == c["kept"], c
        assert abs(sel.mass - c["mass"]) < 1e-12


def test_golden_attend_rational(golden_dir):
    fx = _load(golden_dir, "attend_rational.json")
    a = np.asarray(fx["a"], dtype=np.float64)
    K = np.stack([np.log(a), np.zeros_like(a)], axis=1)
    V = np.asarray(fx["V"], dtype=np.float64)
    q = np.array([1.0, 0.0])
    for c in fx["cases"]:
        o = oracle.attend(q, K, V, c["rows"], 1.0)
        np.testing.assert_allclose(o, c["out"], rtol=0, atol=1e-12)


def test_golden_local_rows(golden_dir):
    fx = _load(golden_dir, "local_rows.json")
    for c in fx["cases"]:
        assert oracle.local_rows(c["N"], c["window"], c["n_sink"]).tolist() == c["rows"], c


def test_golden_bf16_rounding(golden_dir):
    fx = _load(golden_dir, "bf16_rounding.json")
    for c in fx["cases"]:
        y = float(oracle.round_to_bf16(np.array([float(c["x"])]))[0])
        assert y == float(c["y"]), c


def test_golden_f32_rounding(golden_dir):
    fx = _load(golden_dir, "f32_rounding.json")
    for c in fx["cases"]:
        y = float(oracle.round_to(np.array([float(c["x"])]), "f32")[0])
        assert y == float(c["y"]), c


def test_bf16_rounding_matches_torch_cast():
    """fp32 -> bf16 rounding of torch's cast (round to nearest even) agrees
    with the oracle on fp32 inputs (single rounding from fp32)."""
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(7)
    x = np.concatenate([g.normal(0, 1, 20000), g.normal(0, 1e-30, 2000),
                        g.normal(0, 1e30, 2000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    ours = oracle.round_to_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(ours, ref)


# ------------------------------------------------------- top-p, brute force

def _brute_min_set(pi, p):
    """Smallest subset size reaching mass p, and the largest mass among
    subsets of that size (enumeration of all subsets)."""
    n = len(pi)
    for k in range(1, n + 1):
        best = max(math.fsum(pi[list(c)]) for c in itertools.combinations(range(n), k))
        if best >= p:
            return k, best
    return n, math.fsum(pi)


@pytest.mark.parametrize("seed", range(40))
def test_topp_bruteforce(seed):
    g = np.random.default_rng(seed)
    n = int(g.integers(1, 12))
    if seed % 3 == 0:
        z = g.integers(-2, 3, n).astype(np.float64) * 0.7     # many ties
    else:
        z = g.normal(0, 1.5, n)
    p = float(g.uniform(0.05, 0.99))
    # independent softmax (math.fsum)
    ez = np.array([math.exp(v - max(z)) for v in z])
    pi = ez / math.fsum(ez)
    k_min, best = _brute_min_set(pi, p)
    sel = oracle.topp_select(z, p)
    # a set whose mass lies within rounding of p makes the minimal size
    # ambiguous; skip those draws rather than widening the check.
    masses = sorted(pi, reverse=True)
    if any(abs(math.fsum(masses[:k]) - p) < 1e-12 for k in range(1, n + 1)):
        pytest.skip("p on a rounding boundary")
    assert len(sel.kept) == k_min
    assert abs(sel.mass - best) < 1e-12
    # the kept set is the top-|S| by score, ties by lower index
    zs = [(-z[i], i) for i in range(n)]
    assert sorted(sel.kept.tolist()) == sorted(i for _, i in sorted(zs)[:k_min])


def test_topp_tiny_p_is_argmax_with_lowest_index():
    z = np.array([0.1, 3.0, -1.0, 3.0, 2.9])
    for p in (1e-9, 0.0, -1.0):
        assert oracle.topp_select(z, p).kept.tolist() == [1]


def test_topp_p_at_least_one_keeps_all():
    z = np.array([50.0, -50.0, 0.0, -800.0])   # -800: mass underflows to 0
    for p in (1.0, 1.5):
        assert sorted(oracle.topp_select(z, p).kept.tolist()) == [0, 1, 2, 3]


def test_topp_nan_rejected():
    with pytest.raises(ValueError):
        oracle.topp_select(np.zeros(3), float("nan"))


@pytest.mark.parametrize("N,p", [(1000, 0.9005), (4096, 0.3), (777, 0.5001), (10, 0.95)])
def test_topp_uniform_closed_form(N, p):
    """All scores equal: mass 1/N each, so the kept set is the first
    ceil(p*N) tokens by index."""
    assert abs(p * N - round(p * N)) > 1e-6
    sel = oracle.topp_select(np.full(N, 0.75), p)
    assert sel.kept.tolist() == list(range(math.ceil(p * N)))


def test_topp_permutation_equivariant():
    g = np.random.default_rng(3)
    z = g.normal(0, 1, 500)
    perm = g.permutation(500)
    a = set(oracle.topp_select(z, 0.8).kept.tolist())
    b = set(perm[oracle.topp_select(z[perm], 0.8).kept].tolist())
    assert a == b


# ---------------------------------------------------------- attention pins

def _masked_dense_attention(q, K, V, mask, scale):
    """Independent formulation: logits with -inf outside the mask, then a
    two-pass softmax written with explicit loops."""
    n = K.shape[0]
    logits = [(scale * sum(float(q[j]) * float(K[t, j]) for j in range(K.shape[1]))
               if mask[t] else -math.inf) for t in range(n)]
    m = max(logits)
    w = [math.exp(l - m) if l != -math.inf else 0.0 for l in logits]
    s = math.fsum(w)
    return np.array([math.fsum(w[t] * float(V[t, j]) for t in range(n)) / s
                     for j in range(V.shape[1])])


def test_identity_indexer_p1_reproduces_dense_attention():
    """r = d, W_q_idx = I, index keys = keys, no RoPE, p = 1: the step's
    output is plain dense softmax attention."""
    g = np.random.default_rng(11)
    B, H_q, H_kv, d, N = 1, 4, 2, 8, 37
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    W = np.broadcast_to(np.eye(d), (H_q, d, d))
    hc = np.array([1, 1], np.uint8)
    res = oracle.decode_step(q, None, K, V, K, W, hc, [N], p=1.0, window=4, n_sink=1)
    for h in range(H_q):
        ref = _masked_dense_attention(q[0, h], K[0, h // 2], V[0, h // 2], np.ones(N, bool),
                                      1 / math.sqrt(d))
        np.testing.assert_allclose(res.out[0, h], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("p", [0.2, 0.5, 0.9, 0.99])
def test_identity_indexer_mass_of_kept_set(p):
    """With the identity indexer the index softmax is the true attention
    distribution, so the kept set carries at least p of the true mass, and
    dropping its last token would fall below p (minimality)."""
    g = np.random.default_rng(int(p * 100))
    d, N = 16, 300
    q = g.normal(0, 2, d)
    K = g.normal(0, 1, (N, d))
    z = oracle.index_logits(oracle.query_index(q, np.eye(d)), K, 1 / math.sqrt(d))
    logits = np.array([sum(q[j] * K[t, j] for j in range(d)) for t in range(N)]) / math.sqrt(d)
    w = np.exp(logits - logits.max())
    w /= w.sum()
    sel = oracle.topp_select(z, p)
    assert w[sel.kept].sum() >= p - 1e-12
    assert w[sel.kept[:-1]].sum() < p + 1e-12


def test_local_heads_equal_masked_dense():
    g = np.random.default_rng(5)
    B, H_q, H_kv, d, N = 1, 2, 1, 8, 50
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    for window, n_sink in [(7, 3), (1, 0), (60, 2), (10, 45)]:
        res = oracle.decode_step(q, None, K, V, np.zeros((B, H_kv, N, 4)), np.zeros((H_q, 4, d)),
                                 np.array([0], np.uint8), [N], 0.9, window, n_sink)
        mask = np.zeros(N, bool)
        mask[:n_sink] = True
        mask[max(0, N - window):] = True
        for h in range(H_q):
            ref = _masked_dense_attention(q[0, h], K[0, 0], V[0, 0], mask, 1 / math.sqrt(d))
            np.testing.assert_allclose(res.out[0, h], ref, rtol=0, atol=1e-12)


def test_singletons():
    g = np.random.default_rng(9)
    d = 8
    K = g.normal(0, 1, (1, 1, 1, d))
    V = g.normal(0, 1, (1, 1, 1, d))
    q = g.normal(0, 1, (1, 1, d))
    res = oracle.decode_step(q, None, K, V, g.normal(0, 1, (1, 1, 1, 4)), g.normal(0, 1, (1, 4, d)),
                             np.array([1], np.uint8), [1], 0.9, 4, 1)
    np.testing.assert_array_equal(res.out[0, 0], V[0, 0, 0])
    # a single kept row returns that row's value exactly
    N = 20
    K = g.normal(0, 1, (1, 1, N, d))
    V = g.normal(0, 1, (1, 1, N, d))
    kidx = g.normal(0, 1, (1, 1, N, 4))
    W = g.normal(0, 1, (1, 4, d))
    res = oracle.decode_step(q, None, K, V, kidx, W, np.array([1], np.uint8), [N], 1e-9, 4, 1)
    t = res.selections[(0, 0)].kept
    assert len(t) == 1
    z = kidx[0, 0] @ (W[0] @ q[0, 0])
    assert t[0] == int(np.argmax(z))
    np.testing.assert_array_equal(res.out[0, 0], V[0, 0, t[0]])


def test_step_permutation_invariance():
    """Permuting cache rows (distinct scores) permutes the kept set and
    leaves the output unchanged."""
    g = np.random.default_rng(21)
    B, H_q, H_kv, d, r, N = 1, 4, 1, 16, 4, 200
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    kidx = g.normal(0, 3, (B, H_kv, N, r))
    W = g.normal(0, 1, (H_q, r, d))
    hc = np.array([1], np.uint8)
    a = oracle.decode_step(q, None, K, V, kidx, W, hc, [N], 0.7, 8, 2)
    perm = g.permutation(N)
    b = oracle.decode_step(q, None, K[:, :, perm], V[:, :, perm], kidx[:, :, perm], W, hc, [N], 0.7, 8, 2)
    np.testing.assert_allclose(a.out, b.out, rtol=0, atol=1e-12)
    for h in range(H_q):
        assert set(a.selections[(0, h)].kept.tolist()) == set(perm[b.selections[(0, h)].kept].tolist())


def test_gqa_head_to_kv_mapping():
    """Query head h reads KV head h // G: swapping the two KV heads' caches
    and the two query groups swaps the outputs."""
    g = np.random.default_rng(2)
    B, H_q, H_kv, d, r, N = 1, 4, 2, 8, 4, 30
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    kidx = g.normal(0, 1, (B, H_kv, N, r))
    W = g.normal(0, 1, (H_q, r, d))
    hc = np.array([1, 0], np.uint8)
    a = oracle.decode_step(q, None, K, V, kidx, W, hc, [N], 0.8, 5, 1)
    sw = [2, 3, 0, 1]
    b = oracle.decode_step(q[:, sw], None, K[:, ::-1], V[:, ::-1], kidx[:, ::-1], W[sw], hc[::-1].copy(),
                           [N], 0.8, 5, 1)
    np.testing.assert_allclose(a.out[:, sw], b.out, rtol=0, atol=1e-12)


def test_q_rope_used_for_attention_and_q_for_index():
    """The indexer reads the pre-RoPE query and attention the post-RoPE one:
    with p = 1 the output depends only on q_rope, and the kept set only on q."""
    g = np.random.default_rng(4)
    B, H_q, H_kv, d, r, N = 1, 2, 1, 8, 4, 40
    q = g.normal(0, 1, (B, H_q, d))
    q2 = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    kidx = g.normal(0, 1, (B, H_kv, N, r))
    W = g.normal(0, 1, (H_q, r, d))
    hc = np.array([1], np.uint8)
    a = oracle.decode_step(q, q2, K, V, kidx, W, hc, [N], 1.0, 5, 1)
    ref = oracle.dense_decode(q2, K, V, [N])
    np.testing.assert_allclose(a.out, ref, rtol=0, atol=1e-12)
    b = oracle.decode_step(q, q2, K, V, kidx, W, hc, [N], 0.5, 5, 1)
    c = oracle.decode_step(q, -q2, K, V, kidx, W, hc, [N], 0.5, 5, 1)
    for h in range(H_q):
        assert b.selections[(0, h)].kept.tolist() == c.selections[(0, h)].kept.tolist()


# ----------------------------------------------------------- indexer pins

def test_index_projection_selector():
    """A projector whose rows pick coordinates returns those coordinates
    (transposition or index mistakes fail this)."""
    d, r = 8, 3
    W = np.zeros((r, d))
    sel = [5, 0, 2]
    for j, c in enumerate(sel):
        W[j, c] = 1.0
    q = np.arange(1.0, d + 1)
    assert oracle.query_index(q, W).tolist() == [6.0, 1.0, 3.0]
    k = np.arange(10.0, 10.0 + d)
    assert oracle.project_index_key(k, W).tolist() == [15.0, 10.0, 12.0]
    rows = np.array([[1.0, 0.0, 0.0], [0.0, 2.0, 0.0], [1.0, 1.0, 1.0]])
    np.testing.assert_allclose(oracle.index_logits(np.array([6.0, 1.0, 3.0]), rows, 0.5),
                               [3.0, 1.0, 5.0], rtol=0, atol=0)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_append_index_keys_rows_and_rounding(dtype, golden_dir):
    g = np.random.default_rng(8)
    B, H_kv, N_max, d, r, T = 2, 2, 10, 8, 3, 2
    W = np.zeros((H_kv, r, d))
    W[:, 0, 1] = 1.0
    W[:, 1, 3] = 1.0
    W[:, 2, 7] = 0.5
    k = g.normal(0, 1, (B, H_kv, T, d))
    cache = np.full((B, H_kv, N_max, r), -7.0)
    # one key of the f32 cache carries a hand-worked rounding case: 1 + 3*2^-24
    # is halfway between two fp32 values and goes to the even one, 1 + 2^-22
    k[0, 0, 0, 1] = 1 + 3 * 2.0 ** -24
    out = oracle.append_index_keys(cache, k, W, [3, 8], dtype, head_class=[1, 0])
    rnd = oracle.round_to_bf16 if dtype == "bf16" else oracle.round_to_f32
    for b, p0 in enumerate([3, 8]):
        exp = rnd(np.stack([k[b, 0, :, 1], k[b, 0, :, 3], 0.5 * k[b, 0, :, 7]], -1))
        np.testing.assert_array_equal(out[b, 0, p0:p0 + T], exp)
        mask = np.ones(N_max, bool)
        mask[p0:p0 + T] = False
        assert np.all(out[b, 0, mask] == -7.0)
        assert np.all(out[b, 1] == -7.0)      # local head untouched
    # bf16: 1 + 3*2^-24 is far below the halfway point 1 + 2^-8, so it is 1
    assert out[0, 0, 3, 0] == (1 + 2.0 ** -22 if dtype == "f32" else 1.0)


# ------------------------------------------------------ synthetic workloads

def test_planted_needles_are_selected():
    """With needles far above the background and carrying more than p of
    the mass, every kept token is a needle."""
    spec = synth.small_spec(B=1, H_q=4, H_kv=1, N=3000, head_class=(1,), p=0.9,
                            needles_per_head=5, needle_scale=4.0)
    c = synth.make_case(spec)
    B, H_q = 1, 4
    res = oracle.decode_step(c.q.numpy(), c.q_rope.numpy(), c.k_cache.float().numpy(),
                             c.v_cache.float().numpy(), c.kidx_cache.float().numpy(),
                             c.W_q_idx.numpy(), c.head_class, c.seq_lens.numpy(), 0.9,
                             c.window, c.n_sink)
    for h in range(H_q):
        kept = set(res.selections[(0, h)].kept.tolist())
        assert kept <= set(c.needles[(0, h)].tolist()), (h, kept)
        assert len(kept) >= 1


def test_needle_margin_in_index_space():
    """The generator lifts each needle's index logit by about
    scale*ln(N)/2 over the background."""
    spec = synth.small_spec(B=1, H_q=2, H_kv=1, N=5000, head_class=(1,), needles_per_head=6,
                            needle_scale=3.0)
    c = synth.make_case(spec)
    for h in range(2):
        qi = oracle.query_index(c.q[0, h].numpy(), c.W_q_idx[h].numpy())
        z = oracle.index_logits(qi, c.kidx_cache[0, 0].float().numpy(), 1 / math.sqrt(128))
        nd = c.needles[(0, h)]
        bg = np.delete(z, nd)
        lift = 3.0 * math.log(5000) / 2
        assert abs(np.median(z[nd]) - lift) < 1.5
        # background keys ~ N(0, I_r): logit std is |q_idx| / sqrt(d)
        assert abs(bg.std() / (np.linalg.norm(qi) / math.sqrt(128)) - 1.0) < 0.1


# ------------------------------------------- static top-k (the fixed budget)

@pytest.mark.parametrize("seed", range(30))
def test_topk_bruteforce(seed):
    """Among all k-subsets the kept set has the largest mass; every kept
    score is >= every dropped one; at the k-th score the lowest indices
    are the ones kept."""
    g = np.random.default_rng(100 + seed)
    n = int(g.integers(1, 11))
    z = (g.integers(-2, 3, n) * 0.7) if seed % 2 == 0 else g.normal(0, 1.5, n)
    z = np.asarray(z, np.float64)
    k = int(g.integers(1, n + 2))
    ez = np.array([math.exp(v - max(z)) for v in z])
    pi = ez / math.fsum(ez)
    sel = oracle.topk_select(z, k)
    kept = sel.kept.tolist()
    assert len(kept) == min(k, n) and len(set(kept)) == len(kept)
    best = max(math.fsum(pi[list(c)]) for c in itertools.combinations(range(n), min(k, n)))
    assert abs(math.fsum(pi[kept]) - best) < 1e-12
    dropped = [i for i in range(n) if i not in kept]
    if dropped:
        assert min(z[kept]) >= max(z[dropped])
        edge = min(z[kept])
        tied_kept = sorted(i for i in kept if z[i] == edge)
        tied_all = sorted(i for i in range(n) if z[i] == edge)
        assert tied_kept == tied_all[:len(tied_kept)]


def test_topk_closed_forms():
    z = np.array([0.1, 3.0, -1.0, 3.0, 2.9])
    assert oracle.topk_select(z, 1).kept.tolist() == [1]            # argmax, lowest index
    assert sorted(oracle.topk_select(z, 5).kept.tolist()) == [0, 1, 2, 3, 4]
    assert sorted(oracle.topk_select(z, 99).kept.tolist()) == [0, 1, 2, 3, 4]
    assert oracle.topk_select(np.full(50, -0.3), 7).kept.tolist() == list(range(7))
    for bad in (0, -3):
        with pytest.raises(ValueError):
            oracle.topk_select(z, bad)


@pytest.mark.parametrize("seed", range(8))
def test_topk_with_the_topp_size_is_the_topp_set(seed):
    """The top-p set is a prefix of the descending order, so the top-k set
    of its size is the same set."""
    g = np.random.default_rng(200 + seed)
    z = g.normal(0, 2.0, 3000)
    p = float(g.uniform(0.1, 0.99))
    a = oracle.topp_select(z, p).kept
    b = oracle.topk_select(z, len(a)).kept
    assert set(a.tolist()) == set(b.tolist())


def test_step_with_topk_attends_the_k_best_index_scores():
    """The step with a budget k equals masked dense attention over the k
    tokens of largest index score (ranked here with Python's sort), and
    with k >= N equals dense attention."""
    g = np.random.default_rng(21)
    B, H_q, H_kv, d, r, N = 1, 4, 2, 16, 4, 29
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    kidx = g.normal(0, 1, (B, H_kv, N, r))
    W = g.normal(0, 0.3, (H_q, r, d))
    hc = np.array([1, 1], np.uint8)
    sc = 1 / math.sqrt(d)
    for k in (1, 5, N, N + 3):
        res = oracle.decode_step(q, None, K, V, kidx, W, hc, [N], p=0.5, window=4, n_sink=1, topk=k)
        for h in range(H_q):
            gq = h // 2
            qi = [sum(W[h, j, i] * q[0, h, i] for i in range(d)) for j in range(r)]
            zs = [sc * sum(qi[j] * kidx[0, gq, t, j] for j in range(r)) for t in range(N)]
            best = sorted(range(N), key=lambda t: (-zs[t], t))[:min(k, N)]
            mask = np.zeros(N, bool)
            mask[best] = True
            ref = _masked_dense_attention(q[0, h], K[0, gq], V[0, gq], mask, sc)
            np.testing.assert_allclose(res.out[0, h], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------ prefill pins

def _prefill_case(seed, B=2, H_q=4, H_kv=2, T=6, d=8, pos0=(3, 0)):
    g = np.random.default_rng(seed)
    N_max = max(pos0) + T
    q = g.normal(0, 1, (B, H_q, T, d))
    K = g.normal(0, 1, (B, H_kv, N_max, d))
    V = g.normal(0, 1, (B, H_kv, N_max, d))
    return q, K, V, np.asarray(pos0)


@pytest.mark.parametrize("window,n_sink", [(3, 1), (1, 0), (2, 2), (100, 0)])
def test_prefill_matches_explicit_causal_window_mask(window, n_sink):
    """Each query against the explicit mask: key position j is visible to
    the query at position P when j <= P and, for a local head, j < n_sink
    or P - j < window (loops, no shared helper)."""
    q, K, V, pos0 = _prefill_case(5)
    hc = np.array([0, 1], np.uint8)
    out = oracle.prefill_attention(q, K, V, hc, pos0, window, n_sink)
    B, H_q, T, d = q.shape
    for b in range(B):
        for h in range(H_q):
            g = h // 2
            for i in range(T):
                P = int(pos0[b]) + i
                mask = np.array([j <= P and (hc[g] == 1 or j < n_sink or P - j < window)
                                 for j in range(K.shape[2])])
                ref = _masked_dense_attention(q[b, h, i], K[b, g], V[b, g], mask, 1 / math.sqrt(d))
                np.testing.assert_allclose(out[b, h, i], ref, rtol=0, atol=1e-12)


def test_prefill_last_query_is_the_decode_step():
    """The last prompt token's attention is the decode step's attention over
    the same cache (p = 1 keeps every token of a retrieval head)."""
    q, K, V, pos0 = _prefill_case(6, T=5, pos0=(7, 2))
    B, H_q, T, d = q.shape
    hc = np.array([1, 0], np.uint8)
    out = oracle.prefill_attention(q, K, V, hc, pos0, 3, 1)
    lens = pos0 + T
    kidx = np.random.default_rng(1).normal(0, 1, (B, 2, K.shape[2], 4))
    W = np.random.default_rng(2).normal(0, 1, (H_q, 4, d))
    dec = oracle.decode_step(q[:, :, T - 1], None, K, V, kidx, W, hc, lens, 1.0, 3, 1)
    np.testing.assert_allclose(out[:, :, T - 1], dec.out, rtol=0, atol=1e-12)


def test_prefill_first_position_returns_v0_and_wide_window_is_causal():
    q, K, V, pos0 = _prefill_case(7, pos0=(0, 4))
    loc = oracle.prefill_attention(q, K, V, np.array([0, 0], np.uint8), pos0, 10**6, 0)
    ret = oracle.prefill_attention(q, K, V, np.array([1, 1], np.uint8), pos0, 3, 1)
    full = oracle.prefill_attention(q, K, V, np.array([1, 1], np.uint8), pos0, 1, 0)
    np.testing.assert_allclose(loc, full, rtol=0, atol=1e-12)      # a window past position 0 is all causal rows
    np.testing.assert_allclose(ret, full, rtol=0, atol=1e-12)      # retrieval heads ignore window and sinks
    for h in range(q.shape[1]):
        np.testing.assert_array_equal(loc[0, h, 0], K[0, h // 2, 0] * 0 + V[0, h // 2, 0])


def test_force_local_unites_kept_set_with_sinks_and_window():
    """force_local: a retrieval head attends over its top-p set plus the
    sink and window rows, each row once (checked against the explicit union
    and an explicit mask)."""
    g = np.random.default_rng(21)
    B, H_q, H_kv, d, r, N = 1, 2, 1, 8, 4, 40
    q = g.normal(0, 1, (B, H_q, d))
    K = g.normal(0, 1, (B, H_kv, N, d))
    V = g.normal(0, 1, (B, H_kv, N, d))
    kidx = g.normal(0, 1, (B, H_kv, N, r))
    W = g.normal(0, 1, (H_q, r, d))
    hc = np.array([1], np.uint8)
    for p in (1e-9, 0.5):
        plain = oracle.decode_step(q, None, K, V, kidx, W, hc, [N], p, 5, 2)
        forced = oracle.decode_step(q, None, K, V, kidx, W, hc, [N], p, 5, 2, force_local=True)
        for h in range(H_q):
            kept = set(plain.selections[(0, h)].kept.tolist())
            rows = kept | {0, 1} | set(range(N - 5, N))
            mask = np.array([t in rows for t in range(N)])
            ref = _masked_dense_attention(q[0, h], K[0, 0], V[0, 0], mask, 1 / math.sqrt(d))
            np.testing.assert_allclose(forced.out[0, h], ref, rtol=0, atol=1e-12)
            if p == 1e-9:
                assert len(kept) == 1


@pytest.mark.parametrize("N,p", [(19999, 0.3), (7001, 0.9), (40000, 0.50001)])
def test_equal_index_keys_tie_and_keep_the_first_tokens(N, p):
    """Every index key equal: the scores tie exactly (not merely to
    rounding), so the kept set is the first ceil(p N) tokens by index."""
    g = np.random.default_rng(N)
    kidx = np.broadcast_to(g.normal(0, 1, 16), (N, 16)).copy()
    q = g.normal(0, 1, 16)
    z = oracle.index_logits(q, kidx, 1 / math.sqrt(128))
    assert np.unique(z).size == 1
    assert oracle.topp_select(z, p).kept.tolist() == list(range(math.ceil(p * N)))

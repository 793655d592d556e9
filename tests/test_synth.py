"""The seeded workloads against the recipe they are documented with (CPU):
shapes, dtypes and head classes of each workload, the ranked needle plan,
and the 48-layer workload's one retrieval KV head per layer."""
import math

import numpy as np
import pytest

from dynamic_top_sparse_b200 import synth


@pytest.mark.parametrize("key,B,H_q,H_kv,N,layers,kv,idx,hc", [
    ("ctx4k-fp32", 1, 4, 1, 4096, 1, "f32", "f32", [[1]]),
    ("ctx64k", 1, 32, 4, 65536, 1, "bf16", "bf16", [[1, 0, 0, 0]]),
    ("ctx512k", 1, 32, 4, 524288, 1, "bf16", "bf16", [[1, 0, 1, 0]]),
    ("ctx128k-b8-48layer", 8, 32, 4, 131072, 48, "bf16", "bf16", []),
    ("ctx1m", 1, 32, 4, 1048576, 1, "bf16", "bf16", [[1, 1, 1, 1]]),
])
def test_workload_shapes(key, B, H_q, H_kv, N, layers, kv, idx, hc):
    s = synth.spec_for(key)
    assert (s.B, s.H_q, s.H_kv, s.N, s.layers) == (B, H_q, H_kv, N, layers)
    assert (s.kv_dtype, s.idx_dtype, s.d, s.r) == (kv, idx, 128, 16)
    assert s.head_class == hc
    assert (s.p, s.window, s.n_sink) == (0.9, 4096, 4)
    assert s.rope == (key != "ctx4k-fp32")
    assert key in synth.WORKLOADS


@pytest.mark.parametrize("key,heads", [("ctx512k", list(range(0, 8)) + list(range(16, 24))),
                                       ("ctx1m", list(range(32)))])
def test_ranked_needle_plan(key, heads):
    """Retrieval query heads ranked j = 0..J-1 in head order: round(4 *
    1024^(j/(J-1))) needles at scale 4 * 0.3^(j/(J-1)), from 4 needles at
    scale 4 to 4096 needles at scale 1.2."""
    s = synth.spec_for(key)
    hc = synth.layer_head_class(s, 0, 0)
    plan = synth._needle_plan(s, hc, s.N)
    assert sorted(plan) == heads
    J = len(heads)
    for j, h in enumerate(heads):
        n, sc = plan[h]
        assert n == round(4 * 1024 ** (j / (J - 1)))
        assert math.isclose(sc, 4 * 0.3 ** (j / (J - 1)), rel_tol=1e-12)
    assert plan[heads[0]] == (4, 4.0) and plan[heads[-1]][0] == 4096
    assert math.isclose(plan[heads[-1]][1], 1.2, rel_tol=1e-12)


def test_uniform_needle_plan_covers_the_retrieval_heads_only():
    s = synth.spec_for("ctx64k")
    plan = synth._needle_plan(s, synth.layer_head_class(s, 0, 0), s.N)
    assert sorted(plan) == list(range(8))                 # KV head 0's query heads
    assert all(v == (4, 3.0) for v in plan.values())


def test_48_layer_workload_has_one_seeded_retrieval_head_per_layer():
    s = synth.spec_for("ctx128k-b8-48layer")
    picks = []
    for layer in range(s.layers):
        hc = synth.layer_head_class(s, layer, 0)
        assert hc.shape == (4,) and int(hc.sum()) == 1
        picks.append(int(np.argmax(hc)))
        assert np.array_equal(hc, synth.layer_head_class(s, layer, 0))      # deterministic
    assert set(picks) == {0, 1, 2, 3}                     # every KV head is drawn somewhere
    other = [int(np.argmax(synth.layer_head_class(s, layer, 1))) for layer in range(s.layers)]
    assert other != picks                                 # the draw follows the seed


def test_small_case_needles_are_distinct_positions_in_range():
    spec = synth.small_spec(B=2, H_q=8, H_kv=2, N=1500, head_class=(1, 0), seq_lens=[1500, 700],
                            needles_per_head=5)
    c = synth.make_case(spec, seed=3)
    for (b, h), pos in c.needles.items():
        assert h < 4                                      # retrieval KV head 0's query heads
        assert pos.size == 5 and np.unique(pos).size == 5
        assert pos.min() >= 0 and pos.max() < int(c.seq_lens[b])

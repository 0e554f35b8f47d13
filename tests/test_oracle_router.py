"""Oracle pins for the router ("DeepSeek-V3.2-Exp · Router").

Every check here is fixed by something other than the oracle's own code:
hand-worked examples, brute-force enumeration, closed-form invariants from
the "All 4 steps" equations, and special cases that reduce to plain top-k.
"""
import itertools
import math

import numpy as np
import pytest

from conftest import read_golden
from oracle.moe_oracle import MoEShape, router

TINY = MoEShape(dim=8, n_routed_experts=16, n_expert_groups=4, n_limited_groups=2,
                n_activated_experts=4, moe_inter_dim=8)
V3 = MoEShape(dim=64, n_routed_experts=256, n_expert_groups=8, n_limited_groups=4,
              n_activated_experts=8, moe_inter_dim=8)


def _rand(shape: MoEShape, T: int, seed: int, bias_scale=0.1):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, shape.dim)).astype(np.float32)
    w = (rng.standard_normal((shape.n_routed_experts, shape.dim)) / math.sqrt(shape.dim)).astype(np.float32)
    b = rng.uniform(-bias_scale, bias_scale, shape.n_routed_experts).astype(np.float32)
    return x, w, b


def test_hand_worked_bias_only():
    g = read_golden("router_bias_only.txt")
    b = np.array([int(v) for v in g["bias_64ths"]], dtype=np.float32) / 64
    x = np.zeros((3, TINY.dim), dtype=np.float32)
    w = np.random.default_rng(0).standard_normal((16, TINY.dim)).astype(np.float32)
    r = router(x, w, b, TINY)
    for t in range(3):
        assert r.indices[t].tolist() == [int(v) for v in g["indices"]]
        assert r.kept_groups[t].tolist() == [int(v) for v in g["kept_groups"]]
        assert np.all(r.weights[t] == [float(v) for v in g["weights"]])
        assert r.gap_set[t] == int(g["gap_set_64ths"][0]) / 64
        assert r.gap_order[t] == int(g["gap_order_64ths"][0]) / 64
    all_groups = MoEShape(**{**TINY.__dict__, "n_limited_groups": 4})
    r2 = router(x, w, b, all_groups)
    assert r2.indices[0].tolist() == [int(v) for v in g["indices_all_groups"]]


def test_hand_worked_bias_selects_score_weighs():
    g = read_golden("router_bias_weights.txt")
    odds = np.array([float(v) for v in g["odds"]])
    shape = MoEShape(dim=1, n_routed_experts=8, n_expert_groups=1, n_limited_groups=1,
                     n_activated_experts=2, moe_inter_dim=1)
    w_r = np.log(odds).astype(np.float32)[:, None]
    b = np.array([float(v) for v in g["bias"]], dtype=np.float32)
    r = router(np.ones((1, 1), dtype=np.float32), w_r, b, shape)
    assert r.indices[0].tolist() == [int(v) for v in g["indices"]]
    want = np.array([float(v) for v in g["weights"]])
    # fp32 scores: s carries ~1e-7 relative error from fp32 ln(odds) and fp32 s
    assert np.allclose(r.weights[0], want, rtol=1e-6, atol=0)


def test_zero_input_selects_by_bias_and_weights_are_uniform():
    x = np.zeros((5, V3.dim), dtype=np.float32)
    _, w, b = _rand(V3, 1, 3)
    r = router(x, w, b, V3)
    assert np.all(r.scores == 0.5)
    assert np.all(r.weights == 2.5 / 8)            # exactly 0.3125
    # selection by the bias alone: best 4 groups by their top-2 bias sum, then
    # the top 8 biases inside them
    c = (np.float32(0.5) + b).astype(np.float32)
    gs = [sorted(c[32 * q:32 * q + 32])[-1] + sorted(c[32 * q:32 * q + 32])[-2] for q in range(8)]
    keep = sorted(range(8), key=lambda q: (-gs[q], q))[:4]
    cand = [e for e in range(256) if e // 32 in keep]
    want = sorted(cand, key=lambda e: (-c[e], e))[:8]
    assert r.indices[0].tolist() == want


def _brute_force(c: np.ndarray, G: int, Gk: int, k: int):
    """Exhaustive search: best group subset by total group score, then best
    k-subset of the experts in those groups by total biased score."""
    E = c.size
    per = E // G
    gscore = []
    for q in range(G):
        vals = [float(c[e]) for e in range(q * per, (q + 1) * per)]
        gscore.append(max(vals[a] + vals[b] for a, b in itertools.combinations(range(per), 2)))
    best_groups = max(itertools.combinations(range(G), Gk), key=lambda s: sum(gscore[q] for q in s))
    allowed = [e for e in range(E) if e // per in best_groups]
    best_set = max(itertools.combinations(allowed, k), key=lambda s: sum(float(c[e]) for e in s))
    # the 1820-subset search over all experts, filtered by the group constraint
    best_any = max((s for s in itertools.combinations(range(E), k)
                    if all(e // per in best_groups for e in s)),
                   key=lambda s: sum(float(c[e]) for e in s))
    assert set(best_any) == set(best_set)
    return set(best_groups), set(best_set)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    x, w, b = _rand(TINY, 40, seed)
    r = router(x, w, b, TINY)
    checked = 0
    for t in range(40):
        if r.gap_set[t] < 1e-6:
            continue
        groups, experts = _brute_force(r.biased[t], 4, 2, 4)
        assert set(r.kept_groups[t].tolist()) == groups
        assert set(r.indices[t].tolist()) == experts
        checked += 1
    assert checked >= 35


@pytest.mark.parametrize("seed", [0, 1])
def test_invariants_v3_shape(seed):
    x, w, b = _rand(V3, 300, seed)
    r = router(x, w, b, V3)
    # sum of gates is route_scale (the G_i equation sums to 2.5)
    assert np.allclose(r.weights.sum(-1), 2.5, rtol=1e-12, atol=0)
    # at most n_limited_groups groups are used
    assert max(len(set((r.indices[t] // 32).tolist())) for t in range(300)) <= 4
    # bias never enters the weights: recompute from the unbiased s alone
    s_sel = np.take_along_axis(r.scores.astype(np.float64), r.indices, -1)
    assert np.allclose(r.weights, 2.5 * s_sel / s_sel.sum(-1, keepdims=True), rtol=1e-15)
    for t in range(300):
        chosen = set(r.indices[t].tolist())
        kept = set(r.kept_groups[t].tolist())
        # every chosen biased score >= every unchosen one in the kept groups
        rest = [r.biased[t, e] for e in range(256) if e // 32 in kept and e not in chosen]
        assert min(r.biased[t, list(chosen)]) >= max(rest)
        # every kept group scores >= every dropped group
        dropped = [q for q in range(8) if q not in kept]
        assert min(r.group_scores[t, list(kept)]) >= max(r.group_scores[t, dropped])
        # chosen experts are listed in descending biased score
        cs = r.biased[t, r.indices[t]]
        assert np.all(cs[:-1] >= cs[1:])


def test_sigmoid_closed_form():
    # s = sigma(z) at z = ln(r) is r / (1 + r)
    odds = np.array([1.0, 3.0, 1 / 3, 9.0, 0.1, 20.0])
    shape = MoEShape(dim=1, n_routed_experts=6, n_expert_groups=1, n_limited_groups=1,
                     n_activated_experts=6, moe_inter_dim=1)
    r = router(np.ones((1, 1), np.float32), np.log(odds).astype(np.float32)[:, None], None, shape)
    assert np.allclose(r.scores[0], odds / (1 + odds), rtol=3e-7)


def test_single_group_is_plain_topk():
    x, w, b = _rand(TINY, 50, 7)
    one = MoEShape(**{**TINY.__dict__, "n_expert_groups": 1, "n_limited_groups": 1})
    allg = MoEShape(**{**TINY.__dict__, "n_limited_groups": 4})
    r1, r2 = router(x, w, b, one), router(x, w, b, allg)
    for t in range(50):
        c = r1.biased[t]
        want = sorted(range(16), key=lambda e: (-c[e], e))[:4]
        assert r1.indices[t].tolist() == want
        assert r2.indices[t].tolist() == want


def test_uniform_bias_shift_is_invisible():
    x, w, b = _rand(V3, 200, 11)
    r1 = router(x, w, b, V3)
    r2 = router(x, w, (b + np.float32(0.25)).astype(np.float32), V3)
    ok = (r1.gap_set > 1e-6) & (r1.gap_order > 1e-6)
    assert ok.sum() > 190
    assert np.array_equal(r1.indices[ok], r2.indices[ok])
    assert np.array_equal(r1.weights[ok], r2.weights[ok])


def test_no_bias_uses_group_max():
    # without a bias the group score is the group maximum (amax)
    shape = MoEShape(dim=1, n_routed_experts=8, n_expert_groups=2, n_limited_groups=1,
                     n_activated_experts=2, moe_inter_dim=1, has_bias=False)
    # group 0 scores (odds) 9, 1/9, 1/9, 1/9 (top-2 sum small, max large);
    # group 1 scores 4, 4, 1, 1 (top-2 sum large, max smaller)
    odds = np.array([9, 1 / 9, 1 / 9, 1 / 9, 4, 4, 1, 1])
    r = router(np.ones((1, 1), np.float32), np.log(odds).astype(np.float32)[:, None], None, shape)
    assert r.kept_groups[0].tolist() == [0]
    assert sorted(r.indices[0].tolist()) == [0, 1]   # 0.9, then 0.1 ties -> lowest index
    # the top-2-sum rule (with a zero bias) picks the other group
    r2 = router(np.ones((1, 1), np.float32), np.log(odds).astype(np.float32)[:, None],
                np.zeros(8, np.float32), MoEShape(**{**shape.__dict__, "has_bias": True}))
    assert r2.kept_groups[0].tolist() == [1]
    assert r2.indices[0].tolist() == [4, 5]


def test_softmax_scores_not_renormalised():
    shape = MoEShape(dim=1, n_routed_experts=4, n_expert_groups=1, n_limited_groups=1,
                     n_activated_experts=2, moe_inter_dim=1, score_func="softmax",
                     route_scale=1.0, has_bias=False)
    # z = ln(3), 0, 0, 0 -> softmax = 3/6, 1/6, 1/6, 1/6
    w_r = np.array([[math.log(3)], [0], [0], [0]], dtype=np.float32)
    r = router(np.ones((1, 1), np.float32), w_r, None, shape)
    assert r.indices[0].tolist() == [0, 1]
    assert np.allclose(r.weights[0], [0.5, 1 / 6], rtol=1e-6)   # no division by their sum
    full = MoEShape(**{**shape.__dict__, "n_activated_experts": 4})
    assert math.isclose(router(np.ones((1, 1), np.float32), w_r, None, full).weights.sum(), 1.0,
                        rel_tol=1e-6)

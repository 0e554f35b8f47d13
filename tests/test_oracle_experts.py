"""Oracle pins for the expert FFN and the block output.

Closed forms on one-element shapes, exact identities (zero and doubled
matrices, E = k = 1), and row independence.
"""
import math

import numpy as np

from oracle.moe_oracle import MoEShape, expert_ffn, moe_forward, router, silu


def test_silu_special_values():
    assert silu(np.array([0.0]))[0] == 0.0
    # sigma(ln 3) = 3/4
    assert math.isclose(silu(np.array([math.log(3)]))[0], 0.75 * math.log(3), rel_tol=1e-15)
    assert math.isclose(silu(np.array([-math.log(3)]))[0], -0.25 * math.log(3), rel_tol=1e-15)
    assert silu(np.array([-800.0]))[0] == 0.0 or abs(silu(np.array([-800.0]))[0]) < 1e-300
    assert silu(np.array([50.0]))[0] == 50.0


def test_scalar_ffn_closed_form():
    # D = I = 1: w1 x = ln 3, w3 x = 2, w2 = 4 -> 4 * (0.75 ln 3) * 2 = 6 ln 3
    x = np.array([[1.0]])
    w1 = np.array([[math.log(3)]])
    w3 = np.array([[2.0]])
    w2 = np.array([[4.0]])
    y = expert_ffn(x, w1, w3, w2, "f32")[0, 0]
    assert math.isclose(y, 6 * math.log(3), rel_tol=1e-7)      # h rounded to fp32
    # bf16: h = 1.5 ln 3 = 1.64792 -> 1.6484375 (211 steps of 2^-7 above 0)
    assert expert_ffn(x, w1, w3, w2, "bf16")[0, 0] == 4 * 1.6484375


def _tiny_weights(rng, D, I):
    return ((rng.standard_normal((I, D)) / math.sqrt(D)).astype(np.float32),
            (rng.standard_normal((I, D)) / math.sqrt(D)).astype(np.float32),
            (rng.standard_normal((D, I)) / math.sqrt(I)).astype(np.float32))


def test_zero_and_doubled_w2():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((5, 16)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, 16, 8)
    y = expert_ffn(x, w1, w3, w2, "f32")
    assert np.all(expert_ffn(x, w1, w3, np.zeros_like(w2), "f32") == 0)
    assert np.array_equal(expert_ffn(x, w1, w3, 2 * w2, "f32"), 2 * y)
    assert np.all(expert_ffn(np.zeros_like(x), w1, w3, w2, "f32") == 0)


def test_single_expert_block():
    # E = k = 1: the gate is s / s * 2.5 = 2.5, so y = 2.5 FFN(x) + shared(x)
    rng = np.random.default_rng(1)
    shape = MoEShape(dim=16, n_routed_experts=1, n_expert_groups=1, n_limited_groups=1,
                     n_activated_experts=1, moe_inter_dim=8)
    x = rng.standard_normal((7, 16)).astype(np.float32)
    w_r = rng.standard_normal((1, 16)).astype(np.float32)
    ex, sh = _tiny_weights(rng, 16, 8), _tiny_weights(rng, 16, 8)
    r = router(x, w_r, np.zeros(1, np.float32), shape)
    assert np.all(r.weights == 2.5)
    y = moe_forward(x, r, lambda e: ex, lambda: sh, 1, "f32")
    want = 2.5 * expert_ffn(x, *ex, "f32") + expert_ffn(x, *sh, "f32")
    assert np.allclose(y, want, rtol=1e-14, atol=1e-14)


def _block(seed, T=24):
    rng = np.random.default_rng(seed)
    shape = MoEShape(dim=32, n_routed_experts=16, n_expert_groups=4, n_limited_groups=2,
                     n_activated_experts=4, moe_inter_dim=16)
    x = rng.standard_normal((T, 32)).astype(np.float32)
    w_r = (rng.standard_normal((16, 32)) / math.sqrt(32)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, 16).astype(np.float32)
    experts = [_tiny_weights(rng, 32, 16) for _ in range(16)]
    shared = _tiny_weights(rng, 32, 16)
    return shape, x, router(x, w_r, b, shape), experts, shared


def test_removing_shared_or_one_expert():
    shape, x, r, experts, shared = _block(2)
    y = moe_forward(x, r, lambda e: experts[e], lambda: shared, 16, "bf16")
    y_no_shared = moe_forward(x, r, lambda e: experts[e], None, 16, "bf16")
    assert np.allclose(y - y_no_shared, expert_ffn(x, *shared, "bf16"), rtol=1e-12, atol=1e-12)
    # zero the W2 of one used expert: exactly its weighted term disappears
    e0 = int(r.indices[0, 0])
    zeroed = list(experts)
    zeroed[e0] = (experts[e0][0], experts[e0][1], np.zeros_like(experts[e0][2]))
    y0 = moe_forward(x, r, lambda e: zeroed[e], lambda: shared, 16, "bf16")
    term = np.zeros_like(y)
    for t in range(x.shape[0]):
        for j in range(4):
            if r.indices[t, j] == e0:
                term[t] += r.weights[t, j] * expert_ffn(x[t:t + 1], *experts[e0], "bf16")[0]
    assert np.allclose(y - y0, term, rtol=1e-12, atol=1e-12)


def test_rows_are_independent():
    shape, x, r, experts, shared = _block(3)
    full = moe_forward(x, r, lambda e: experts[e], lambda: shared, 16, "bf16")
    rows = np.array([5, 0, 17])
    part = moe_forward(x, r, lambda e: experts[e], lambda: shared, 16, "bf16", tokens=rows)
    assert np.allclose(part, full[rows], rtol=1e-14, atol=1e-14)


def test_weighted_sum_definition_per_token():
    # y[t] = sum_j w[t, j] FFN_{idx[t, j]}(x[t]) + shared(x[t]) token by token
    shape, x, r, experts, shared = _block(4, T=6)
    y = moe_forward(x, r, lambda e: experts[e], lambda: shared, 16, "f32")
    for t in range(6):
        acc = expert_ffn(x[t:t + 1], *shared, "f32")[0].copy()
        for j in range(4):
            acc += r.weights[t, j] * expert_ffn(x[t:t + 1], *experts[r.indices[t, j]], "f32")[0]
        assert np.allclose(y[t], acc, rtol=1e-12, atol=1e-12)

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


def _two_unit_expert():
    # D = I = 128 (one quantisation block each).  x = 3.5 at column 0, so its
    # block scale is 3.5 / 448 = 2^-7 and x survives the quantisation
    # exactly.  a_0 = ln 3, u_0 = 2 -> h_0 = 1.5 ln 3 = 1.64792 -> bf16
    # 1.6484375; a_1 = ln 3, u_1 = 0.6 -> h_1 = 0.49438 -> bf16 0.494140625.
    # Output row 0 sums h_0 + h_1 (w2 row 0 = 1 at columns 0 and 1).
    D = I = 128
    x = np.zeros((1, D), np.float32)
    x[0, 0] = 3.5
    w1 = np.zeros((I, D))
    w3 = np.zeros((I, D))
    w2 = np.zeros((D, I))
    w1[0, 0] = w1[1, 0] = math.log(3) / 3.5
    w3[0, 0] = 2.0 / 3.5
    w3[1, 0] = 0.6 / 3.5
    w2[0, 0] = w2[0, 1] = 1.0
    return x, w1, w3, w2


def test_two_unit_chain_bf16_and_e4m3():
    x, w1, w3, w2 = _two_unit_expert()
    assert expert_ffn(x, w1, w3, w2, "bf16")[0, 0] == 1.6484375 + 0.494140625
    # e4m3: h's block amax 1.6484375 sets scale = fp32(1.6484375 / 448); h_0
    # becomes 448 steps of it, h_1 = 0.494140625 / scale = 134.29 -> the
    # e4m3 binade [128, 256) has step 16 -> 128 steps
    scale = float(np.float32(1.6484375) / np.float32(448.0))
    assert expert_ffn(x, w1, w3, w2, "e4m3")[0, 0] == (448 + 128) * scale
    assert np.all(expert_ffn(x, w1, w3, w2, "e4m3")[0, 1:] == 0)


def test_two_unit_chain_f16():
    # fp16 keeps 10 fraction bits: h_0 = 1.5 ln 3 in [1, 2) rounds to a
    # multiple of 2^-10, h_1 = 0.45 ln 3 in [0.25, 0.5) to a multiple of 2^-12
    x, w1, w3, w2 = _two_unit_expert()
    h0 = float(np.float32(0.75 * math.log(3) * 2.0))
    h1 = float(np.float32(0.75 * math.log(3) * 0.6))
    want = round(h0 / 2.0 ** -10) * 2.0 ** -10 + round(h1 / 2.0 ** -12) * 2.0 ** -12
    assert want == 1.6474609375 + 0.494384765625
    assert expert_ffn(x, w1, w3, w2, "f16")[0, 0] == want


def test_e4m3_activation_error_is_a_few_percent():
    # the quantisation error of x and h (3 fraction bits, half-step 2^-4
    # relative) shows as a few percent rms on random data; zero or tens of
    # percent would mean a skipped or mis-scaled step
    rng = np.random.default_rng(9)
    x = rng.standard_normal((32, 256)).astype(np.float32)
    w1, w3, w2 = _tiny_weights(rng, 256, 256)
    ref = expert_ffn(x, w1, w3, w2, "f32")
    got = expert_ffn(x, w1, w3, w2, "e4m3")
    rel = np.sqrt(np.mean((got - ref) ** 2) / np.mean(ref ** 2))
    assert 0.01 < rel < 0.1, rel
    f16 = expert_ffn(x, w1, w3, w2, "f16")
    rel16 = np.sqrt(np.mean((f16 - ref) ** 2) / np.mean(ref ** 2))
    assert 1e-5 < rel16 < 1e-3, rel16

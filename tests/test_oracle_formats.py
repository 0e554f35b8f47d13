"""Oracle pins for the number-format helpers (bf16 rounding, e4m3 decoding)."""
import math

import numpy as np
import torch

from oracle.moe_oracle import (bf16_bits_to_f32, dequant_e4m3_block, e4m3_table,
                               round_f32_to_bf16)


def test_bf16_round_special_values():
    one = 1.0
    ulp = 2.0 ** -7                      # spacing of bf16 in [1, 2)
    cases = {
        one + 2.0 ** -8: one,            # halfway, even neighbour is 1
        one + 3 * 2.0 ** -8: one + 2 * ulp,  # halfway, even neighbour is 1 + 2^-6
        one + 2.0 ** -8 + 2.0 ** -20: one + ulp,  # just above halfway
        -(one + 2.0 ** -8): -one,
        0.0: 0.0,
        1.6479184330021645: 1.6484375,   # 210.93 ulps -> 211 ulps
    }
    for v, want in cases.items():
        got = float(round_f32_to_bf16(np.array([v], dtype=np.float32))[0])
        assert got == want, (v, got, want)


def test_bf16_round_matches_torch():
    g = torch.Generator().manual_seed(5)
    v = torch.randn(100000, generator=g) * torch.exp(torch.randn(100000, generator=g) * 4)
    ours = round_f32_to_bf16(v.numpy())
    theirs = v.to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), theirs.view(np.uint32))


def test_bf16_bits_roundtrip():
    x = torch.randn(4096).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits_to_f32(bits), x.float().numpy())


def test_e4m3_known_codes():
    t = e4m3_table()
    assert t[0x00] == 0.0 and t[0x80] == 0.0
    assert t[0x38] == 1.0                 # exponent field 7 = bias
    assert t[0x7E] == 448.0               # largest finite
    assert t[0xFE] == -448.0
    assert t[0x01] == 2.0 ** -9           # smallest subnormal
    assert t[0x08] == 2.0 ** -6           # smallest normal
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert np.isfinite(t).sum() == 254


def test_e4m3_matches_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])


def test_dequant_block_scale_layout():
    # 256 x 384 codes, 2 x 3 scale blocks; code 0x38 (= 1.0) everywhere, so the
    # dequantised matrix shows which scale block covers each element
    q = np.full((256, 384), 0x38, dtype=np.uint8)
    s = np.array([[1, 2, 3], [4, 5, 6]], dtype=np.float32)
    w = dequant_e4m3_block(q, s)
    assert w[0, 0] == 1 and w[127, 127] == 1 and w[0, 128] == 2 and w[0, 383] == 3
    assert w[128, 0] == 4 and w[255, 255] == 5 and w[255, 256] == 6


# ------------------------------------------------------------ fp16, e4m3 encode

from conftest import read_golden  # noqa: E402
from oracle.moe_oracle import (dequant_e4m3_rows, e4m3_code, quantize_e4m3_rows,  # noqa: E402
                               round_f32_to_f16, round_to_e4m3)


def test_f16_round_special_values():
    cases = {
        1.0 + 2.0 ** -11: 1.0,                     # halfway, even neighbour 1
        1.0 + 3 * 2.0 ** -11: 1.0 + 2.0 ** -9,     # halfway, even neighbour 1 + 2^-9
        65504.0: 65504.0,                          # largest finite
        2.0 ** -24: 2.0 ** -24,                    # smallest subnormal
        2.0 ** -25: 0.0,                           # half of it: ties to even (0)
        3 * 2.0 ** -25: 2.0 ** -23,                # 1.5 subnormal steps -> 2
        -(2.0 ** -14 + 2.0 ** -25): -(2.0 ** -14),  # below the normal spacing, rounds down
        0.1: 0.0999755859375,
    }
    for v, want in cases.items():
        got = float(round_f32_to_f16(np.array([v], dtype=np.float32))[0])
        assert got == want, (v, got, want)


def test_f16_round_matches_torch():
    g = torch.Generator().manual_seed(6)
    v = torch.randn(100000, generator=g) * torch.exp(torch.randn(100000, generator=g) * 3)
    v = v.clamp(-60000, 60000)
    assert np.array_equal(round_f32_to_f16(v.numpy()), v.to(torch.float16).double().numpy())


def test_e4m3_round_midpoints_go_to_even_codes():
    # brute force over every pair of neighbouring positive finite codes: the
    # midpoint rounds to the code whose lowest bit is 0, a hair off it to
    # the nearer one
    t = e4m3_table()
    for c in range(0x00, 0x7E):
        lo, hi = t[c], t[c + 1]
        mid = 0.5 * (lo + hi)
        want = lo if c % 2 == 0 else hi
        assert round_to_e4m3(np.array([mid]))[0] == want, (c, mid)
        assert round_to_e4m3(np.array([-mid]))[0] == -want
        assert round_to_e4m3(np.array([mid - 1e-9 * hi]))[0] == lo
        assert round_to_e4m3(np.array([mid + 1e-9 * hi]))[0] == hi


def test_e4m3_round_saturates_and_matches_torch():
    assert round_to_e4m3(np.array([464.0, 1000.0, -1e9]))[0] == 448.0
    assert list(round_to_e4m3(np.array([464.0, 1000.0, -1e9]))) == [448.0, 448.0, -448.0]
    g = torch.Generator().manual_seed(7)
    v = (torch.randn(100000, generator=g) * torch.exp(torch.randn(100000, generator=g) * 3))
    v = v.clamp(-448, 448)
    ref = v.to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(round_to_e4m3(v.double().numpy()), ref)


def test_e4m3_code_inverts_the_table():
    t = e4m3_table()
    codes = np.array([c for c in range(256) if np.isfinite(t[c]) and c != 0x80], dtype=np.uint8)
    assert np.array_equal(e4m3_code(t[codes]), codes)


def test_activation_quantisation_worked_example():
    g = read_golden("e4m3_act_quant.txt")
    v = np.zeros((3, 256), dtype=np.float32)
    v[0, [int(c) for c in g["row0_cols"]]] = [float(x) for x in g["row0_vals"]]
    v[1, [int(c) for c in g["row1_cols"]]] = [float(x) for x in g["row1_vals"]]
    vals, scales = quantize_e4m3_rows(v)
    assert scales.dtype == np.float32 and scales.shape == (3, 1)
    assert list(scales[:, 0]) == [float(x) for x in g["scales"]]
    deq = dequant_e4m3_rows(vals, scales)
    assert list(deq[0, [int(c) for c in g["row0_cols"]]]) == [float(x) for x in g["row0_deq"]]
    assert list(deq[1, [int(c) for c in g["row1_cols"]]]) == [float(x) for x in g["row1_deq"]]
    assert np.count_nonzero(deq) == 8                    # zeros stay zero, row 2 empty


def test_activation_quantisation_blocks_are_independent_rows():
    # with 1 x 128 runs, each run is quantised as a row of its own
    rng = np.random.default_rng(10)
    v = (rng.standard_normal((5, 384)) * np.exp(rng.standard_normal((5, 3)).repeat(128, 1)))
    v = v.astype(np.float32)
    vals, scales = quantize_e4m3_rows(v, block=128)
    assert scales.shape == (5, 3)
    for b in range(3):
        vb, sb = quantize_e4m3_rows(v[:, 128 * b:128 * (b + 1)])
        assert np.array_equal(vals[:, 128 * b:128 * (b + 1)], vb)
        assert np.array_equal(scales[:, b:b + 1], sb)


def test_activation_quantisation_error_bound():
    # every dequantised value is within half an e4m3 step of the value: 2^-4
    # relative above 2^-6 * scale, 2^-10 * scale absolute below
    rng = np.random.default_rng(8)
    v = (rng.standard_normal((64, 512)) * np.exp(rng.standard_normal((64, 1)))).astype(np.float32)
    vals, scales = quantize_e4m3_rows(v)
    deq = dequant_e4m3_rows(vals, scales)
    s = scales.astype(np.float64)
    bound = np.maximum(np.abs(v) * 2.0 ** -4, s * 2.0 ** -10) * (1 + 1e-6)
    assert np.all(np.abs(deq - v) <= bound)
    # the row maximum itself is kept to fp32 rounding of the scale
    assert np.allclose(np.abs(deq).max(-1), np.abs(v).max(-1), rtol=2e-7)

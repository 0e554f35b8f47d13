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

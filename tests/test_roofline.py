"""The roofline arithmetic bench.py reports, pinned to counts written out here.

The block's algorithmic bytes and flops follow from the expert parameter
count of the "DeepSeek-V3.2-Exp · Mixture of experts" page (44,040,192 per
expert = 3 matrices of 7168 x 2048) and the router shapes of the
"DeepSeek-V3.2-Exp · Router" page (a 256 x 7168 fp32 matrix and a 256-entry
bias), so a dropped term or a wrong factor shows up against these sums.
"""
import pytest

from sparse_moe_layer_sum_b200.roofline import (block_work, kernel_work, load_peaks,
                                                 method_bytes, tensor_peak, use_sustained_peak)

D, E, I, K, S = 7168, 256, 2048, 8, 1
PER_EXPERT = 44_040_192  # parameters of one expert, as the page counts them


def test_expert_parameter_count_matches_the_page():
    assert 3 * D * I == PER_EXPERT


@pytest.mark.parametrize("T,n_touched", [(64, 165), (4096, 255), (4096, 256)])
def test_block_work_bf16(T, n_touched):
    w = block_work(D, E, I, K, S, T, n_touched, w_bytes=2, x_bytes=2)
    weights = (n_touched + S) * PER_EXPERT * 2
    router = E * D * 4 + E * 4
    io = T * D * 2 + T * D * 4
    assert w.bytes == weights + router + io
    # every token through k routed experts and the shared one, 3 matmuls of
    # D x I each, plus the router's D x E
    assert w.flops == 2 * T * (K + S) * PER_EXPERT + 2 * T * D * E


def test_block_work_prefill_magnitudes():
    # the figures the configuration discussion works with: about 22.8 GB and
    # 3.25 TFLOP for T = 4096 with every expert touched
    w = block_work(D, E, I, K, S, 4096, 256, w_bytes=2, x_bytes=2)
    assert 22.6e9 < w.bytes < 22.9e9
    assert 3.24e12 < w.flops < 3.27e12


def test_block_work_e4m3_counts_scales():
    scale = 3 * (D // 128) * (I // 128) * 4  # fp32 per 128 x 128 block, three matrices
    w = block_work(D, E, I, K, S, 8192, 256, w_bytes=1, x_bytes=2, scale_bytes_per_expert=scale)
    assert w.bytes == 257 * (PER_EXPERT + scale) + E * D * 4 + E * 4 + 8192 * D * 2 + 8192 * D * 4


def test_kernel_work_splits_the_matmuls():
    T, n = 4096, 255
    kw = kernel_work(D, E, I, K, S, T, n, w_bytes=2, x_bytes=2, scatter=True)
    rows = T * K + T * S
    # first matmul: w1 and w3 of every touched expert and the shared one,
    # the rows in (bf16), h out (bf16)
    assert kw["gemm1"].bytes == (n + 1) * 2 * D * I * 2 + rows * D * 2 + rows * I * 2
    assert kw["gemm1"].flops == rows * 4 * D * I
    # second matmul with the scatter: w2, h in, y (fp32) written once
    assert kw["gemm2"].bytes == (n + 1) * D * I * 2 + rows * I * 2 + T * D * 4
    assert kw["gemm2"].flops == rows * 2 * D * I
    # the two matmuls together carry the block's expert flops
    b = block_work(D, E, I, K, S, T, n, w_bytes=2, x_bytes=2)
    assert kw["gemm1"].flops + kw["gemm2"].flops + kw["router"].flops == b.flops
    # without the scatter, the second matmul writes one fp32 row per slot
    ko = kernel_work(D, E, I, K, S, T, n, w_bytes=2, x_bytes=2, scatter=False)
    assert ko["gemm2"].bytes - kw["gemm2"].bytes == rows * D * 4 - T * D * 4


def test_load_peaks_falls_back_without_a_measurement(tmp_path):
    peaks, src = load_peaks(str(tmp_path))
    assert src == "fallback"
    assert peaks["hbm_gbs"] == 6650.0 and peaks["bf16_tflops"] == 1590.0


def test_method_bytes_are_weights_plus_block_io():
    T, n = 4096, 255
    m = method_bytes(D, I, K, S, T, n, w_bytes=2, x_bytes=2)
    # the first matmul streams w1 and w3 (two thirds of each expert) and x once
    assert m["gemm1"] == (n + 1) * (2 * PER_EXPERT // 3) * 2 + T * D * 2
    # the second streams w2 (one third) and writes y in fp32
    assert m["gemm2"] == (n + 1) * (PER_EXPERT // 3) * 2 + T * D * 4
    # together with the router they are the block's bytes
    b = block_work(D, E, I, K, S, T, n, w_bytes=2, x_bytes=2)
    assert m["gemm1"] + m["gemm2"] + E * D * 4 + E * 4 == b.bytes
    kw = kernel_work(D, E, I, K, S, T, n, w_bytes=2, x_bytes=2, scatter=True)
    assert m["gemm1"] < kw["gemm1"].bytes and m["gemm2"] < kw["gemm2"].bytes


def test_tensor_peak_by_operand_type():
    p = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    assert tensor_peak(p, False, "bf16") == 1600.0
    assert tensor_peak(p, True, "f16") == 1400.0
    assert tensor_peak(p, False, "e4m3") == 3200.0


def test_peak_choice_follows_loop_length_and_power_cap():
    p = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    # a short loop at full clocks: burst
    assert use_sustained_peak(p, 100.0, {"reasons": []}) == (False, False)
    assert use_sustained_peak(p, 100.0, None) == (False, False)
    # a long loop: sustained, with or without a clock record
    assert use_sustained_peak(p, 1000.0, None) == (True, False)
    # a short loop that the clock samples show under the power cap: sustained
    assert use_sustained_peak(p, 100.0, {"reasons": ["sw_power_cap"]}) == (True, True)
    # no sustained figure on record: burst, whatever the loop
    assert use_sustained_peak({"bf16_tflops": 1600.0}, 1000.0,
                              {"reasons": ["sw_power_cap"]}) == (False, True)

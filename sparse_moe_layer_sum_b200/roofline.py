"""Algorithmic work of the MoE block and of each of its kernels.

"Algorithmic" bytes are the bytes any implementation must move from or to
HBM, and flops the multiply-adds it must do, given the routing (which experts
received tokens).  Intermediate buffers an implementation chooses to keep in
HBM (the permuted rows, h, the per-slot expert outputs) are counted only for
the kernel that reads or writes them, never for the block as a whole.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks(root: str) -> tuple[dict, str]:
    """Measured peaks (MEASURED_PEAKS.json at the repo root), else the fallback."""
    path = os.path.join(root, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


@dataclass
class Work:
    bytes: float
    flops: float


def block_work(D, E, I, k, S, T, n_touched, w_bytes, x_bytes, scale_bytes_per_expert=0.0,
               has_bias=True) -> Work:
    """Whole block: weights of the touched experts and the shared expert, the
    fp32 router matrix and bias, x in and fp32 y out; expert and router flops."""
    weights = (n_touched + S) * (3 * D * I * w_bytes + scale_bytes_per_expert)
    router = E * D * 4 + (E * 4 if has_bias else 0)
    io = T * D * x_bytes + T * D * 4
    flops = T * (k + S) * 2 * 3 * D * I + T * 2 * D * E
    return Work(weights + router + io, flops)


def tensor_peak(peaks: dict, sustained: bool, mma: str) -> float:
    """Dense tensor peak (TFLOP/s) for the MMA operand type: the measured bf16
    figure (burst or sustained); fp16 equals it; e4m3 is twice it, the
    nominal fp8 : bf16 ratio of the part (4.5 : 2.25 PFLOP/s dense)."""
    bf16 = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    return {"bf16": 1.0, "f16": 1.0, "e4m3": 2.0, "f32": 1.0}[mma] * bf16


def use_sustained_peak(peaks: dict, ms_timed: float, clocks: dict | None) -> tuple[bool, bool]:
    """Which bf16 tensor peak heads a line: the sustained (power-capped) one
    when the timed loop lasts over half a second, long enough for the clocks
    to settle under the power cap, or when the clock samples taken during it
    show the power cap engaged; else the burst one.  Returns (sustained,
    power cap seen)."""
    capped = "sw_power_cap" in ((clocks or {}).get("reasons") or [])
    return (ms_timed > 500.0 or capped) and "bf16_tflops_sustained" in peaks, capped


def method_bytes(D, I, k, S, T, n_touched, w_bytes, x_bytes, scale_bytes_per_expert=0.0):
    """Bytes of each matmul that the method itself fixes, with no
    implementation buffers: the weights of the touched experts and the
    shared one, plus x read by the first and y (fp32) written by the second.
    The expert-ordered copies of the rows and h are left out."""
    n_w = n_touched + S
    sc = scale_bytes_per_expert / 3.0
    return {"gemm1": n_w * (2 * D * I * w_bytes + 2 * sc) + T * D * x_bytes,
            "gemm2": n_w * (D * I * w_bytes + sc) + T * D * 4}


def kernel_work(D, E, I, k, S, T, n_touched, w_bytes, x_bytes, scale_bytes_per_expert=0.0,
                scatter=False):
    """Per kernel of one forward: the bytes it must move and flops it must do.
    With scatter=True the second matmul adds the gated outputs into y itself
    (y written once, no per-slot outputs) and there is no combine pass."""
    rows = T * k + T * S                       # expert-contiguous rows incl. the shared expert
    n_w = n_touched + S                        # weight matrices actually streamed
    sc = scale_bytes_per_expert / 3.0          # per matrix
    return {
        "router": Work(E * D * 4 + E * 4 + T * D * x_bytes + T * k * 8, T * 2 * D * E),
        "dispatch": Work(T * k * 4 * 3 + (E + 1) * 8, 0.0),
        "gather": Work(T * k * D * x_bytes * 2 + T * D * x_bytes * 2, 0.0),
        # W1 and W3 of each touched expert, the rows in, h out
        "gemm1": Work(n_w * (2 * D * I * w_bytes + 2 * sc) + rows * D * 2 + rows * I * 2,
                      rows * 2 * 2 * D * I),
        # W2 of each touched expert, h in, fp32 expert outputs (or y) out
        "gemm2": Work(n_w * (D * I * w_bytes + sc) + rows * I * 2 +
                      (T * D * 4 if scatter else rows * D * 4), rows * 2 * D * I),
        # k expert rows and the shared row in, y out (all fp32)
        "combine": Work(rows * D * 4 + T * D * 4 + T * k * 8, T * (k + S) * D * 2),
    }

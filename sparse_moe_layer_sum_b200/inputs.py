"""Seeded synthetic inputs for the MoE block (shared by the tests, the bench
and the oracle's callers).

Holds no arithmetic of the method itself -- only random draws and the
storage format of the inputs (bf16 / fp32 casts, and the e4m3 encoding with
one fp32 scale per 128 x 128 weight block for the FP8-weight workload).

Distributions: x ~ N(0, 1); router weight W_r ~ N(0, 1/dim) in fp32; bias ~
U(-0.1, 0.1) in fp32; expert weights ~ N(0, 1/fan_in) (fan_in = dim for
w1/w3 and inter for w2).  Draw order: x, W_r, bias, then for each chunk of
consecutive groups 0..E (E = the shared expert; a chunk holds as many groups
as fit 2^30 elements of one matrix) one draw of w1, one of w3 and one of w2
for all groups of the chunk.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

from .moe import BlockParams, BlockShape

V3 = dict(dim=7168, n_routed=256, n_groups=8, topk_groups=4, topk=8, inter=2048)
TINY = dict(dim=256, n_routed=16, n_groups=4, topk_groups=2, topk=4, inter=128)


@dataclass(frozen=True)
class Workload:
    name: str
    shape: BlockShape
    T: int
    x_dtype: torch.dtype
    w_format: str            # "f32", "bf16" or "e4m3"
    seed: int
    hot_experts: int = 0     # experts given +hot_bias (skewed routing)
    hot_bias: float = 0.0
    note: str = ""
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", BlockShape(**TINY), 64, torch.float32, "f32", 1001,
                         note="dim 256, 16 experts in 4 groups, top-2 groups, top-4, inter 128, "
                              "T=64, fp32 everywhere"),
    "v3_decode_t64": Workload("v3_decode_t64", BlockShape(**V3), 64, torch.bfloat16, "bf16", 1002,
                              note="DeepSeek-V3 block, T=64 decode batch, bf16"),
    "v3_prefill_t4096": Workload("v3_prefill_t4096", BlockShape(**V3), 4096, torch.bfloat16,
                                 "bf16", 1003, note="DeepSeek-V3 block, T=4096 prefill, bf16"),
    "v3_skew_t16384": Workload("v3_skew_t16384", BlockShape(**V3), 16384, torch.bfloat16, "bf16",
                               1004, hot_experts=16, hot_bias=0.5,
                               note="T=16384, +0.5 bias on 16 seeded hot experts, bf16"),
    "v3_fp8_t8192": Workload("v3_fp8_t8192", BlockShape(**V3), 8192, torch.bfloat16, "e4m3", 1005,
                             note="T=8192, e4m3 expert weights with fp32 128x128 block scales, "
                                  "bf16 activations"),
    # profiling-sized stand-in for the T=4096 prefill: same dim/inter and the
    # same ~128 rows per expert, but 32 experts (2.9 GB of weights) so that a
    # multi-pass ncu capture stays small
    "prof_prefill_e32_t512": Workload("prof_prefill_e32_t512",
                                      BlockShape(dim=7168, n_routed=32, n_groups=8, topk_groups=4,
                                                 topk=8, inter=2048), 512, torch.bfloat16,
                                      "bf16", 1006, note="V3 dims, 32 experts, T=512"),
    # the same for the T=64 decode batch: ~2 rows per expert, 32 experts
    "prof_decode_e32_t8": Workload("prof_decode_e32_t8",
                                   BlockShape(dim=7168, n_routed=32, n_groups=8, topk_groups=4,
                                              topk=8, inter=2048), 8, torch.bfloat16,
                                   "bf16", 1007, note="V3 dims, 32 experts, T=8"),
    # the V3 router (dim 7168, 256 experts, T=4096) with narrow experts, so
    # that a capture of the router kernels holds little else on the device
    "prof_router_t4096": Workload("prof_router_t4096",
                                  BlockShape(dim=7168, n_routed=256, n_groups=8, topk_groups=4,
                                             topk=8, inter=128), 4096, torch.bfloat16,
                                  "bf16", 1009, note="V3 router shapes, inter 128, T=4096"),
    # and for the e4m3 T=8192 batch: ~256 rows per expert, 32 experts
    "prof_fp8_e32_t1024": Workload("prof_fp8_e32_t1024",
                                   BlockShape(dim=7168, n_routed=32, n_groups=8, topk_groups=4,
                                              topk=8, inter=2048), 1024, torch.bfloat16,
                                   "e4m3", 1008, note="V3 dims, 32 experts, T=1024, e4m3 weights"),
}


def custom(name: str, T: int, x_dtype=torch.bfloat16, w_format="bf16", seed=7, **shape) -> Workload:
    return Workload(name, BlockShape(**shape), T, x_dtype, w_format, seed)


E4M3_MAX = 448.0


def quantize_e4m3_blocks(w: torch.Tensor, block: int = 128):
    """e4m3 codes (uint8) and fp32 scales [rows/128, cols/128] of a [rows, cols]
    fp32 matrix: scale = block amax / 448, code = e4m3(w / scale)."""
    r, c = w.shape
    wb = w.reshape(r // block, block, c // block, block)
    amax = wb.abs().amax(dim=(1, 3)).clamp_min(1e-30)
    scale = (amax / E4M3_MAX).to(torch.float32)
    q = (wb / scale[:, None, :, None]).clamp(-E4M3_MAX, E4M3_MAX)
    codes = q.reshape(r, c).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


def make_block(w: Workload, device="cuda", x_seed_offset: int = 0):
    """(x [T, dim], BlockParams) for a workload, drawn on `device`."""
    sh = w.shape
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(w.seed)
    D, E, I, S = sh.dim, sh.n_routed, sh.inter, sh.n_shared
    x = torch.randn(w.T, D, generator=g, device=dev, dtype=torch.float32).to(w.x_dtype)
    if x_seed_offset:  # another batch of the same distribution, same weights
        gx = torch.Generator(device=dev).manual_seed(w.seed + 7919 * x_seed_offset)
        x = torch.randn(w.T, D, generator=gx, device=dev, dtype=torch.float32).to(w.x_dtype)
    w_r = torch.randn(E, D, generator=g, device=dev, dtype=torch.float32) / math.sqrt(D)
    bias = None
    if sh.has_bias:
        bias = torch.rand(E, generator=g, device=dev, dtype=torch.float32) * 0.2 - 0.1
        if w.hot_experts:
            hot = torch.randperm(E, generator=torch.Generator().manual_seed(2024))[:w.hot_experts]
            bias[hot.to(dev)] += w.hot_bias
    G = E + S
    if w.w_format == "e4m3":
        w1 = torch.empty(G, I, D, dtype=torch.uint8, device=dev)
        w3 = torch.empty(G, I, D, dtype=torch.uint8, device=dev)
        w2 = torch.empty(G, D, I, dtype=torch.uint8, device=dev)
        s1 = torch.empty(G, I // 128, D // 128, dtype=torch.float32, device=dev)
        s3 = torch.empty_like(s1)
        s2 = torch.empty(G, D // 128, I // 128, dtype=torch.float32, device=dev)
    else:
        wdt = torch.bfloat16 if w.w_format == "bf16" else torch.float32
        w1 = torch.empty(G, I, D, dtype=wdt, device=dev)
        w3 = torch.empty(G, I, D, dtype=wdt, device=dev)
        w2 = torch.empty(G, D, I, dtype=wdt, device=dev)
        s1 = s3 = s2 = None
    # one draw per matrix kind and chunk of groups (a handful of launches in
    # all), chunks bounded so that the fp32 temporaries stay a few GB
    chunk = max(1, min(G, (1 << 30) // (I * D)))
    for e0 in range(0, G, chunk):
        n = min(chunk, G - e0)
        for wt, sc, (r, c), fan in ((w1, s1, (I, D), D), (w3, s3, (I, D), D), (w2, s2, (D, I), I)):
            m = torch.randn(n, r, c, generator=g, device=dev, dtype=torch.float32)
            m.mul_(1.0 / math.sqrt(fan))
            if w.w_format == "e4m3":
                q, s = quantize_e4m3_blocks(m.reshape(n * r, c))
                wt[e0:e0 + n] = q.reshape(n, r, c)
                sc[e0:e0 + n] = s.reshape(n, r // 128, c // 128)
            else:
                wt[e0:e0 + n] = m
            del m
    return x, BlockParams(w_r, bias, w1, w3, w2, s1, s3, s2)


def random_topk_indices(T: int, E: int, k: int, seed: int, device="cpu") -> torch.Tensor:
    """[T, k] int32: k distinct experts per token, uniformly drawn."""
    g = torch.Generator().manual_seed(seed)
    idx = torch.argsort(torch.rand(T, E, generator=g), dim=1)[:, :k].to(torch.int32)
    return idx.to(device)


def sample_tokens(T: int, n: int, seed: int = 7) -> torch.Tensor:
    """A seeded sample of n distinct token rows (all rows when n >= T)."""
    if n >= T:
        return torch.arange(T)
    return torch.randperm(T, generator=torch.Generator().manual_seed(seed))[:n].sort().values


def expert_weights_host(p: BlockParams, e: int, w_format: str):
    """Host copies of expert e's (w1, w3, w2) and scales, exact."""
    out = []
    for wt, sc in ((p.w1, p.s1), (p.w3, p.s3), (p.w2, p.s2)):
        m = wt[e].cpu()
        if w_format == "bf16":
            m = m.to(torch.float32)
        out.append((m.numpy(), None if sc is None else sc[e].cpu().numpy()))
    return out


def to_host_f32(t: torch.Tensor):
    """Exact fp32 host copy of a bf16/fp32 tensor."""
    return t.detach().to("cpu").to(torch.float32).numpy()


__all__ = ["Workload", "WORKLOADS", "make_block", "custom", "random_topk_indices",
           "sample_tokens", "expert_weights_host", "to_host_f32", "quantize_e4m3_blocks"]

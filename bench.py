#!/usr/bin/env python
"""Throughput of the DeepSeek-V3 MoE block forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the CPU oracle on the host cores

One step = one forward of the whole block (router -> dispatch -> experts ->
combine) over one batch of T tokens with inputs already resident in HBM.
Prints one JSON line on rank 0.  Multi-GPU runs (torchrun) are independent
replicas: every rank runs its own batch through its own copy of the weights
(weak scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from datetime import timedelta

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_moe_layer_sum_b200 import moe  # noqa: E402
from sparse_moe_layer_sum_b200.inputs import WORKLOADS, make_block, sample_tokens  # noqa: E402
from sparse_moe_layer_sum_b200.roofline import (block_work, kernel_work, load_peaks,  # noqa: E402
                                                 method_bytes, tensor_peak, use_sustained_peak)

METRIC = "MoE block tokens/s (V3 shape, bf16, T=4096) and % of roofline on 1 B200"
N_X_BATCHES = 4  # rotating input batches: with the 22.6 GB of weights, > L2 per step
# the other configurations timed in short loops after the headline one:
# (workload, FP8 x FP8 activations)
# (workload, variant): "" the default kernels, "fp8act" FP8 x FP8 matmuls,
# "fused" the whole block in one launch (decode)
OTHER_CONFIGS = [("v3_decode_t64", ""), ("v3_decode_t64", "fused"), ("v3_skew_t16384", ""),
                 ("v3_fp8_t8192", ""), ("v3_fp8_t8192", "fp8act")]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v3_prefill_t4096", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-sample", type=int, default=32,
                    help="tokens the oracle pushes through the block for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph replay timing of the same forward")
    ap.add_argument("--other-steps", type=int, default=20,
                    help="timed steps for each other configuration (0: skip them)")
    ap.add_argument("--fp8-act", action="store_true",
                    help="e4m3-weight workloads: quantise the activations to e4m3 too "
                         "(FP8 x FP8 matmuls)")
    ap.add_argument("--fused-decode", action="store_true",
                    help="decode batches: the whole block in one persistent launch")
    ap.add_argument("--parallel", choices=["replicas", "ep"], default="replicas",
                    help="N>1: independent replicas (weak scaling), or expert parallelism: "
                         "one batch, the experts split over the ranks, y all-reduced "
                         "(strong scaling)")
    ap.add_argument("--combine", choices=["scatter", "ordered"], default="scatter",
                    help="weighted sum into y inside the second matmul, or ordered and "
                         "bit-reproducible in a separate pass")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest value of v over all ranks (the job is as slow as its
    slowest replica); v itself when there is one rank."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world: int, T: int, steps: int, ms_total: float) -> float:
    """Whole-job throughput of `world` replicas, each pushing `steps` batches of
    T tokens, when the slowest one took ms_total."""
    return world * T * steps / (ms_total / 1e3)


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples every 200 ms of this process's GPU while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.proc = None
        self.path = None
        try:
            try:
                props = torch.cuda.get_device_properties(device)
                sel = (f"--id={props.pci_domain_id:08X}:{props.pci_bus_id:02X}:"
                       f"{props.pci_device_id:02X}.0")
            except AttributeError:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
                sel = f"--id={vis[device] if device < len(vis) and vis[device] else device}"
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:  # no nvidia-smi: clocks reported as unavailable
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- oracle leg


def cpu_oracle_tokens_per_s(w, x, params, n_tokens: int, seed: int = 7, fp8_act=False,
                            route_all: bool = False):
    """Time the oracle (as it stands) on the workload: the routing of every
    token when route_all (else of the sample only) and the block output of a
    seeded sample of n_tokens tokens.  Returns (tokens/s, cores, seconds):
    the per-token cost is the routing time per routed token plus the expert
    time per sampled token.  Host copies of the expert weights are fetched
    outside the timed part."""
    from oracle import moe_oracle as O
    from threadpoolctl import threadpool_info

    toks = sample_tokens(w.T, n_tokens, seed).numpy()
    xs = x[torch.from_numpy(toks).to(x.device)].float().cpu().numpy()
    x_all = x.float().cpu().numpy() if route_all else xs
    w_r = params.w_r.cpu().numpy()
    bias = None if params.bias is None else params.bias.cpu().numpy()
    b = w.shape
    shape = O.MoEShape(dim=b.dim, n_routed_experts=b.n_routed, n_expert_groups=b.n_groups,
                       n_limited_groups=b.topk_groups, n_activated_experts=b.topk,
                       moe_inter_dim=b.inter, n_shared_experts=b.n_shared,
                       route_scale=b.route_scale, score_func=b.score_func, has_bias=b.has_bias)
    fetch_s = 0.0

    def fetch(e):
        nonlocal fetch_s
        t0 = time.perf_counter()
        mats = []
        for wt, sc in ((params.w1, params.s1), (params.w3, params.s3), (params.w2, params.s2)):
            if w.w_format == "e4m3":
                mats.append(O.dequant_e4m3_block(wt[e].cpu().numpy(), sc[e].cpu().numpy()))
            else:
                mats.append(wt[e].float().cpu().numpy())
        fetch_s += time.perf_counter() - t0
        return mats

    # h rounded as the CUDA path rounds it (the oracle's readings 3 and 6)
    act = ("f32" if w.x_dtype == torch.float32 else
           ("e4m3" if fp8_act else "f16") if w.w_format == "e4m3" else "bf16")
    t0 = time.perf_counter()
    route_all_tok = O.router(x_all, w_r, bias, shape)
    t_route = time.perf_counter() - t0
    route = O.RouterResult(*[a[toks] if route_all and a is not None and not np.isscalar(a)
                             and getattr(a, "shape", (0,))[0] == w.T else a
                             for a in (route_all_tok.weights, route_all_tok.indices,
                                       route_all_tok.scores, route_all_tok.biased,
                                       route_all_tok.group_scores, route_all_tok.kept_groups,
                                       route_all_tok.gap_set, route_all_tok.gap_order)])
    t1 = time.perf_counter()
    O.moe_forward(xs, route, fetch, lambda: fetch(shape.n_routed_experts),
                  shape.n_routed_experts, act)
    t_ffn = time.perf_counter() - t1 - fetch_s
    cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    per_token = t_route / x_all.shape[0] + t_ffn / len(toks)
    return 1.0 / per_token, cores, t_route + t_ffn


# ---------------------------------------------------------------- ours


def traffic_for(kernel_name: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    h = hashlib.sha256()
    for rel in t.get("sources", []):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != t.get("sha256"):
        return None
    entry = t.get("kernels", {}).get(kernel_name)
    if not entry or entry.get("workload") != t.get("bench_workload"):
        return None
    return entry.get("dram_bytes_per_launch")


def make_inputs(w, dev, rank):
    """The block's weights and N_X_BATCHES seeded input batches for this rank."""
    x0, params = make_block(w, dev, x_seed_offset=1 + rank * N_X_BATCHES)
    xs = [x0]
    gx = torch.Generator(device=dev)
    for i in range(1, N_X_BATCHES):
        gx.manual_seed(w.seed + 104729 * (1 + rank * N_X_BATCHES + i))
        xs.append(torch.randn(w.T, w.shape.dim, generator=gx, device=dev).to(w.x_dtype))
    return xs, params


def mma_type(w, fp8_act: bool) -> str:
    """Operand type of the expert matmuls: e4m3 weights are expanded to fp16,
    unless the FP8 x FP8 path quantises the activations too."""
    if w.w_format == "e4m3":
        return "e4m3" if fp8_act else "f16"
    return "bf16" if w.x_dtype == torch.bfloat16 else "f32"


def time_block(w, blk, xs, K, warmup, world, dev, local_rank):
    """Warm up, then time K forwards (max over ranks) with per-kernel events;
    also the routing of each input batch (counts, near-ties)."""
    for i in range(max(warmup, 1)):
        blk.forward(xs[i % N_X_BATCHES])
    torch.cuda.synchronize()
    st = blk.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(10)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    counts, ties = [], []
    for i in range(N_X_BATCHES):   # routing of each input batch, for the byte counts
        blk.forward(xs[i])
        counts.append(blk.counts.cpu())
        # tokens whose smallest routing decision gap (the router's own report)
        # is below 1e-6: their choice may depend on rounding
        ties.append(int((blk.sel_gap < 1e-6).sum()))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    time.sleep(0.25)
    start.record()
    for i in range(K):
        blk.forward_profiled(xs[i % N_X_BATCHES], evs[i])
    end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = max_over_ranks(start.elapsed_time(end), world, dev)
    if blk.device_status() != 0:
        raise RuntimeError(f"device status {blk.device_status()} in the timed region")
    spans = {"router": (0, 1), "dispatch": (1, 2), "gather": (3, 4), "gemm1": (4, 5),
             "gemm2": (6, 7), "combine": (8, 9)}
    dur = {k: statistics.mean(evs[i][a].elapsed_time(evs[i][b]) for i in range(K))
           for k, (a, b) in spans.items()}
    return {"ms_total": ms_total, "ms_step": ms_total / K, "dur": dur, "counts": counts,
            "near_ties": ties, "clocks": clk}


def rooflines(w, blk, K, tm, fp8_act=False, share=1.0):
    """Dominant-kernel and whole-step rooflines from the measured timings.
    share: the part of the block's expert work one GPU does (1/world under
    expert parallelism)."""
    sh = w.shape
    peaks, peak_src = load_peaks(ROOT)
    w_bytes = {"bf16": 2, "f32": 4, "e4m3": 1}[w.w_format]
    x_bytes = 2 if w.x_dtype == torch.bfloat16 else 4
    scale_b = (3 * (sh.dim // 128) * (sh.inter // 128) * 4) if w.w_format == "e4m3" else 0
    touched = [int((c > 0).sum()) for c in tm["counts"]]
    args = (sh.dim, sh.n_routed, sh.inter, sh.topk, sh.n_shared, w.T)
    kw = [kernel_work(*args, n, w_bytes, x_bytes, scale_b, scatter=blk.combine_mode == "scatter")
          for n in touched]
    mb = [method_bytes(sh.dim, sh.inter, sh.topk, sh.n_shared, w.T, n, w_bytes, x_bytes, scale_b)
          for n in touched]
    bw = [block_work(*args, n, w_bytes, x_bytes, scale_b, sh.has_bias) for n in touched]
    steps_per_batch = [sum(1 for i in range(K) if i % N_X_BATCHES == b) for b in range(N_X_BATCHES)]

    def avg(f):
        return sum(f(b) * steps_per_batch[b] for b in range(N_X_BATCHES)) / K

    dur = tm["dur"]
    if getattr(blk, "fused_decode", False):
        # one launch: its span is recorded as the router's; its work is the block's
        dur = {"fused_block": dur["router"], "router": 0.0, "dispatch": 0.0, "gather": 0.0,
               "gemm1": 0.0, "gemm2": 0.0, "combine": 0.0}
        for b in range(len(kw)):
            kw[b]["fused_block"] = bw[b]
            mb[b]["fused_block"] = bw[b].bytes
    dominant = max(("gemm1", "gemm2", "router", "combine", "gather", "dispatch", "fused_block"),
                   key=lambda k: dur.get(k, 0.0))
    bytes_dom = share * avg(lambda b: kw[b][dominant].bytes)
    bytes_meth = (share * avg(lambda b: mb[b][dominant])
                  if dominant in ("gemm1", "gemm2", "fused_block") else bytes_dom)
    flops_dom = share * avg(lambda b: kw[b][dominant].flops)
    # tensor peak: the sustained (power-capped) figure when the timed loop runs
    # long enough for the clocks to settle under the power cap, or when the
    # clock samples show the power cap engaged during it; else the burst one
    sustained, capped = use_sustained_peak(peaks, tm["ms_total"], tm.get("clocks"))
    mma = mma_type(w, fp8_act)
    hbm = peaks["hbm_gbs"]
    tflops = tensor_peak(peaks, sustained, mma)
    dsec = dur[dominant] / 1e3
    gemm = "tc_fp8_gemm" if fp8_act else "tc_expert_gemm"
    kname = {"gemm1": f"{gemm}<1>",
             "gemm2": f"{gemm}<3>" if blk.combine_mode == "scatter" else f"{gemm}<2>",
             "fused_block": "fused::decode_block"}.get(dominant, dominant)
    if bytes_meth / (hbm * 1e9) >= flops_dom / (tflops * 1e12):
        roof = {"bound": "hbm", "achieved": bytes_meth / dsec / 1e9, "peak": hbm, "unit": "GB/s"}
        roof["frac"] = roof["achieved"] / hbm
        roof["frac_method"] = roof["frac"]
        roof["frac_impl"] = bytes_dom / dsec / 1e9 / hbm
    else:
        roof = {"bound": "tensor", "achieved": flops_dom / dsec / 1e12, "peak": tflops,
                "unit": "TFLOP/s"}
        roof["frac"] = roof["frac_method"] = roof["frac_impl"] = roof["achieved"] / tflops
    roof["traffic"] = traffic_for(kname)
    roof["kernel"] = kname
    roof["scope"] = "dominant kernel (the whole step is step_roofline)"
    roof["mma_type"] = mma
    roof["peak_source"] = (f"{peak_src} ({'MEASURED_PEAKS.json' if peak_src == 'measured' else 'recipe fallback'}"
                           f"{(', tensor peak sustained' + (' (power cap seen)' if capped else '')) if sustained else ', tensor peak burst'}"
                           f"{', e4m3 = 2 x bf16 (nominal ratio)' if mma == 'e4m3' else ''})")
    roof["method_bytes_per_launch"] = bytes_meth
    roof["impl_bytes_per_launch"] = bytes_dom
    roof["algorithmic_flops_per_launch"] = flops_dom
    b_alg = share * avg(lambda b: bw[b].bytes)
    f_alg = share * avg(lambda b: bw[b].flops)
    ms_step = tm["ms_step"]
    t_roof = max(b_alg / (hbm * 1e9), f_alg / (tflops * 1e12))
    step_roof = {"bytes": b_alg, "flops": f_alg, "t_roof_ms": t_roof * 1e3,
                 "frac": t_roof * 1e3 / ms_step,
                 "bound": "hbm" if b_alg / (hbm * 1e9) >= f_alg / (tflops * 1e12) else "tensor",
                 "tensor_peak_tflops": tflops,
                 "hbm_frac": b_alg / (ms_step / 1e3) / (hbm * 1e9),
                 "tensor_frac": f_alg / (ms_step / 1e3) / (tflops * 1e12),
                 "hbm_frac_vs_nominal_8TBs": b_alg / (ms_step / 1e3) / 8e12}
    if "bf16_tflops_sustained" in peaks:
        # the tensor fraction against both peaks, whichever one heads the line
        for tag, sus in (("burst", False), ("sustained", True)):
            tp = tensor_peak(peaks, sus, mma)
            step_roof[f"tensor_frac_{tag}"] = f_alg / (ms_step / 1e3) / (tp * 1e12)
            step_roof[f"frac_{tag}"] = max(b_alg / (hbm * 1e9), f_alg / (tp * 1e12)) / (ms_step / 1e3)
            if roof["bound"] == "tensor":
                roof[f"frac_{tag}"] = flops_dom / dsec / 1e12 / tp
    if w.w_format == "e4m3" and mma != "e4m3":
        # the same step against the dense FP8 peak (2 x bf16), which an
        # FP8 x FP8 matmul could reach
        fp8 = tensor_peak(peaks, sustained, "e4m3")
        step_roof["tensor_frac_vs_fp8_peak"] = f_alg / (ms_step / 1e3) / (fp8 * 1e12)
        step_roof["frac_vs_fp8_peak"] = max(b_alg / (hbm * 1e9), f_alg / (fp8 * 1e12)) / (ms_step / 1e3)
    return roof, step_roof, touched


def kernel_times(blk, tm):
    """Per-kernel milliseconds; the fused decode launch is one span."""
    if getattr(blk, "fused_decode", False):
        return {"fused_block": tm["dur"]["router"]}
    return tm["dur"]


def near_tie_report(w, tm):
    n = tm["near_ties"]
    return {"threshold": 1e-6, "tokens_per_batch": n, "fraction": sum(n) / (len(n) * w.T)}


def other_config(name, args, dev, local_rank, variant=""):
    """A short timed loop of another configuration, for the same JSON line."""
    w = WORKLOADS[name]
    xs, params = make_inputs(w, dev, 0)
    fp8_act = variant == "fp8act"
    blk = moe.MoEBlock(w.shape, params, w.T, w.x_dtype, device=dev, combine=args.combine,
                       fp8_act=fp8_act, fused_decode=variant == "fused")
    K = args.other_steps
    tm = time_block(w, blk, xs, K, 3, 1, dev, local_rank)
    roof, step_roof, touched = rooflines(w, blk, K, tm, fp8_act)
    out = {"value": job_tokens_per_s(1, w.T, K, tm["ms_total"]), "unit": "tokens/s",
           "ms_per_step": tm["ms_step"], "steps": K, "warmup": 3, "T": w.T,
           "weights": w.w_format, "mma_type": mma_type(w, fp8_act),
           "step_roofline": step_roof, "roofline": roof, "kernels_ms": kernel_times(blk, tm),
           "gpu_launches_per_step": blk.launches_per_forward,
           "near_ties": near_tie_report(w, tm), "clocks": tm["clocks"],
           "touched_experts": touched}
    if w.hot_experts:
        hot_ids = torch.randperm(w.shape.n_routed, generator=torch.Generator().manual_seed(2024))[:16]
        out["hot_share"] = float(tm["counts"][0][hot_ids].sum() / tm["counts"][0].sum())
    del blk, xs, params
    torch.cuda.empty_cache()
    return out


def run_ours(args, rank, local_rank, world):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    from sparse_moe_layer_sum_b200 import build
    build.build_all()
    w = WORKLOADS[args.workload]
    sh = w.shape
    ep = args.parallel == "ep" and world > 1
    # expert parallelism: every rank holds the same batches and its shard of
    # the experts; replicas: every rank its own batches and all the experts
    xs, params = make_inputs(w, dev, 0 if ep else rank)
    if ep:
        params = moe.shard_params(sh, params, rank, world)
        torch.cuda.empty_cache()
    x0 = xs[0]
    blk = moe.MoEBlock(sh, params, w.T, w.x_dtype, device=dev, combine=args.combine,
                       fp8_act=args.fp8_act, ep=(rank, world) if ep else (0, 1),
                       ep_group=torch.distributed.group.WORLD if ep else None,
                       fused_decode=args.fused_decode)
    K = args.steps
    tm = time_block(w, blk, xs, K, args.warmup, world, dev, local_rank)
    ms_total, ms_step = tm["ms_total"], tm["ms_step"]
    # the job's tokens: one batch per step under expert parallelism, one per
    # replica and step otherwise
    value = job_tokens_per_s(1 if ep else world, w.T, K, ms_total)
    roof, step_roof, touched = rooflines(w, blk, K, tm, args.fp8_act,
                                         share=1.0 / world if ep else 1.0)
    x_bytes = 2 if w.x_dtype == torch.bfloat16 else 4
    w_bytes = {"bf16": 2, "f32": 4, "e4m3": 1}[w.w_format]

    # end to end through the public API from pinned host memory: every step
    # copies its batch in and its y out, overlapped with the neighbouring
    # steps' compute by the block's host pipeline
    x_host = [xx.cpu().pin_memory() for xx in xs]
    y_host = [torch.empty(w.T, sh.dim, dtype=torch.float32).pin_memory() for _ in range(2)]
    pipe = blk.host_pipeline()
    Ke = max(1, min(K, 50))
    for i in range(2):
        pipe.submit(x_host[i % N_X_BATCHES], y_host[i % 2])
    pipe.finish()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(Ke):
        pipe.submit(x_host[i % N_X_BATCHES], y_host[i % 2])
    pipe.finish()
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = {"value": job_tokens_per_s(1 if ep else world, w.T, Ke, ms_e2e), "unit": "tokens/s",
           "h2d_bytes_per_step": w.T * sh.dim * x_bytes, "d2h_bytes_per_step": w.T * sh.dim * 4,
           "steps": Ke}

    # the same forward captured once as a CUDA graph and replayed: what the
    # launch gaps between the kernels cost (each step copies its batch into
    # the graph's input buffer first, inside the timed region)
    graph = None
    if not args.no_graph and not ep:  # (no NCCL call inside a captured graph)
        x_g = xs[0].clone()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            blk.forward(x_g)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            blk.forward(x_g)
        Kg = max(1, min(K, 50))
        for i in range(3):
            x_g.copy_(xs[i % N_X_BATCHES])
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record()
        for i in range(Kg):
            x_g.copy_(xs[i % N_X_BATCHES])
            g.replay()
        g1.record()
        torch.cuda.synchronize()
        ms_g = max_over_ranks(g0.elapsed_time(g1), world, dev)
        if blk.device_status() != 0:
            raise RuntimeError(f"device status {blk.device_status()} in the graph replays")
        graph = {"value": job_tokens_per_s(world, w.T, Kg, ms_g), "unit": "tokens/s",
                 "ms_per_step": ms_g / Kg, "steps": Kg,
                 "gpu_launches_per_step": blk.launches_per_forward}
        del g

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        try:
            tps, cores, wall = cpu_oracle_tokens_per_s(w, x0, params, args.cpu_sample,
                                                       fp8_act=args.fp8_act, route_all=True)
            cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"routing of all {w.T} tokens of the {w.name} batch and the block "
                             f"output of {args.cpu_sample} seeded tokens, fp64 ({wall:.1f} s of "
                             "oracle time; weight copies to the host excluded); tokens/s = 1 / "
                             "(routing time per token + expert time per sampled token)"}
        except Exception as exc:  # reported, never fatal
            cpu = {"value": None, "error": repr(exc)[:200]}

    hot = None
    if w.hot_experts:
        hot_ids = torch.randperm(sh.n_routed, generator=torch.Generator().manual_seed(2024))[:16]
        hot = float(tm["counts"][0][hot_ids].sum() / tm["counts"][0].sum())
    launches = K * blk.launches_per_forward
    kernels_ms = kernel_times(blk, tm)

    # the other configurations, each in a short loop of its own (one GPU only)
    others = None
    if world == 1 and args.other_steps > 0:
        del blk, xs, params, x_host, y_host, pipe
        torch.cuda.empty_cache()
        others = {}
        main_variant = "fp8act" if args.fp8_act else "fused" if args.fused_decode else ""
        for name, variant in OTHER_CONFIGS:
            if name == w.name and variant == main_variant:
                continue
            key = name + ("_" + variant if variant else "")
            try:
                others[key] = other_config(name, args, dev, local_rank, variant)
            except Exception as exc:  # reported, never fatal to the headline
                others[key] = {"error": repr(exc)[:300]}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if ep else "weak", "vs_baseline": None,
        # arithmetic type of the matmuls: e4m3 weights are expanded to f16
        # unless the activations are quantised to e4m3 as well
        "dtype": mma_type(w, args.fp8_act),
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights, U(-0.1,0.1) bias)",
        "config": {"workload": w.name, "T": w.T, "dim": sh.dim, "n_routed": sh.n_routed,
                   "combine": args.combine,
                   "topk": sh.topk, "inter": sh.inter, "weights": w.w_format,
                   "activations": "e4m3 (1x128 blocks)" if args.fp8_act else
                   ("bf16" if w.x_dtype == torch.bfloat16 else "f32"),
                   "parallelism": (f"expert parallel x{world} (NCCL all-reduce of y)" if ep else
                                   f"replicas x{world}" if world > 1 else "single GPU"),
                   "l2": f"inputs larger than L2: {N_X_BATCHES} rotating x batches and "
                         f"{(sh.n_routed + 1) * 3 * sh.dim * sh.inter * w_bytes / 1e9:.1f} GB "
                         "of expert weights per step"},
        "roofline": roof, "step_roofline": step_roof,
        "kernels_ms": kernels_ms, "cpu_baseline": cpu, "e2e": e2e, "graph": graph,
        "gpu_launches": launches,
        "clocks": tm["clocks"], "touched_experts": touched, "hot_share": hot,
        "near_ties": near_tie_report(w, tm),
        "other_configs": others,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- reference


def run_reference(args, rank, world):
    """The oracle, timed on the host cores on the same workload (one seeded
    token per step, routed and pushed through its experts in fp64)."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    x, params = make_block(w, dev, x_seed_offset=1)
    K, W = args.steps, args.warmup
    per_step = 1
    times = []
    cores = 1
    for i in range(W + K):
        _, cores, wall = cpu_oracle_tokens_per_s(w, x, params, per_step, seed=1000 + i)
        if i >= W:
            times.append(wall)
    ms = 1e3 * sum(times) / len(times)
    value = per_step / (ms / 1e3)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "weights": w.w_format},
        "cpu_baseline": {"kind": "oracle", "cores": cores, "value": value, "unit": "tokens/s",
                         "sample": f"{per_step} seeded token per step of the {w.name} batch"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, local_rank, world = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, local_rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()

"""Helpers that run the oracle on host copies of a block's inputs and compare
the CUDA path's results with it.  Test infrastructure only."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from oracle import moe_oracle as O
from sparse_moe_layer_sum_b200.inputs import Workload, to_host_f32

NEAR_TIE = 1e-6  # decision gap below which both outcomes are accepted


def oracle_shape(w: Workload) -> O.MoEShape:
    s = w.shape
    return O.MoEShape(dim=s.dim, n_routed_experts=s.n_routed, n_expert_groups=s.n_groups,
                      n_limited_groups=s.topk_groups, n_activated_experts=s.topk,
                      moe_inter_dim=s.inter, n_shared_experts=s.n_shared,
                      route_scale=s.route_scale, score_func=s.score_func, has_bias=s.has_bias)


def oracle_route(w: Workload, x: torch.Tensor, params) -> O.RouterResult:
    bias = None if params.bias is None else params.bias.cpu().numpy()
    return O.router(to_host_f32(x), params.w_r.cpu().numpy(), bias, oracle_shape(w))


def _expert_getter(params, w_format: str):
    cache = {}

    def get(e):
        if e not in cache:
            mats = []
            for wt, sc in ((params.w1, params.s1), (params.w3, params.s3), (params.w2, params.s2)):
                if w_format == "e4m3":
                    mats.append(O.dequant_e4m3_block(wt[e].cpu().numpy(), sc[e].cpu().numpy()))
                else:
                    mats.append(to_host_f32(wt[e]).astype(np.float64))
            cache.clear()  # keep one expert on the host at a time
            cache[e] = mats
        return cache[e]

    return get


def oracle_act(w: Workload, fp8_act: bool = False) -> str:
    """How the oracle rounds the expert activations for a workload's CUDA path
    (the oracle's readings 3 and 6): fp32 activations stay fp32; bf16 ones
    round h to bf16, except on the e4m3-weight tensor-core path, whose
    second-matmul operand h is fp16; the FP8 x FP8 path quantises x and h
    to e4m3 in 1 x 128 blocks."""
    if w.x_dtype == torch.float32:
        return "f32"
    if w.w_format == "e4m3":
        return "e4m3" if fp8_act else "f16"
    return "bf16"


def oracle_y(w: Workload, x: torch.Tensor, params, route: O.RouterResult, tokens=None,
             fp8_act: bool = False):
    """Oracle block output (fp64) for the rows `tokens` (all when None)."""
    get = _expert_getter(params, w.w_format)
    E = w.shape.n_routed
    act = oracle_act(w, fp8_act)
    xs = to_host_f32(x)
    shared = (lambda: get(E)) if w.shape.n_shared else None
    return O.moe_forward(xs, route, get, shared, E, act, tokens=tokens)


@dataclass
class RoutingReport:
    flagged: int          # tokens whose smallest decision gap is below NEAR_TIE
    set_flips: int        # flagged tokens whose chosen set differs from the oracle's
    order_flips: int      # flagged tokens with the same set in another order
    same_set: np.ndarray  # [T] bool: GPU set == oracle set
    max_w_rel: float      # max relative gate error on same-set tokens


def compare_routing(route: O.RouterResult, gpu_w: np.ndarray, gpu_idx: np.ndarray,
                    group_size: int, w_rtol: float) -> RoutingReport:
    """Indices bit-exact on every token without a near-tie; flagged tokens
    must still make a valid choice; gates within w_rtol where sets agree."""
    T, k = route.indices.shape
    flag = (route.gap_set < NEAR_TIE) | (route.gap_order < NEAR_TIE)
    same_order = np.all(gpu_idx == route.indices, axis=1)
    same_set = np.array([set(gpu_idx[t].tolist()) == set(route.indices[t].tolist())
                         for t in range(T)])
    bad = np.nonzero(~flag & ~same_order)[0]
    assert bad.size == 0, f"{bad.size} unflagged tokens differ, first {bad[:5]}"
    # flagged tokens: the GPU's choice must be within NEAR_TIE of optimal
    for t in np.nonzero(flag & ~same_set)[0]:
        c = route.biased[t].astype(np.float64)
        chosen = gpu_idx[t]
        assert len(set(chosen.tolist())) == k
        if route.kept_groups is not None:
            # the chosen experts may come from a near-tied alternative group
            gs = route.group_scores[t].astype(np.float64)
            used = set((chosen // group_size).tolist())
            kth = np.sort(gs)[::-1][len(route.kept_groups[t]) - 1]
            assert all(gs[q] >= kth - NEAR_TIE for q in used)
            allowed = [e for e in range(c.size) if e // group_size in used]
        else:
            allowed = list(range(c.size))
        rest = [c[e] for e in allowed if e not in set(chosen.tolist())]
        if rest:
            assert c[chosen].min() >= max(rest) - NEAR_TIE
    # gates, slot by slot after aligning the GPU's order to the oracle's
    direct = same_order
    rel = list((np.abs(gpu_w[direct] - route.weights[direct]) /
                np.abs(route.weights[direct])).ravel())
    for t in np.nonzero(same_set & ~same_order)[0]:
        pos = {e: j for j, e in enumerate(gpu_idx[t].tolist())}
        g = gpu_w[t][[pos[e] for e in route.indices[t].tolist()]]
        rel.extend((np.abs(g - route.weights[t]) / np.abs(route.weights[t])).tolist())
    rel = np.asarray(rel)
    max_rel = float(rel.max()) if rel.size else 0.0
    assert max_rel <= w_rtol, f"gate relative error {max_rel} > {w_rtol}"
    return RoutingReport(int(flag.sum()), int((flag & ~same_set).sum()),
                         int((flag & same_set & ~same_order).sum()), same_set, max_rel)


def y_close(y_gpu: np.ndarray, y_orc: np.ndarray, rel_rms: float) -> float:
    """max |dy| / rms(y_oracle); asserts it is within rel_rms."""
    rms = float(np.sqrt(np.mean(y_orc ** 2)))
    err = float(np.max(np.abs(y_gpu.astype(np.float64) - y_orc))) / rms
    assert err <= rel_rms, f"max|dy| = {err:.3e} rms(y) > {rel_rms}"
    return err

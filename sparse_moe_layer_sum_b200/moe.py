"""Python binding for the MoE block libraries.

Argument marshalling only: every step of the block runs in the CUDA kernels
of the four C-ABI libraries; PyTorch provides device memory and the stream.

    block = MoEBlock(shape, params, T, torch.bfloat16)   # weights already on the GPU
    y = block.forward(x)                   # x [T, dim] on the GPU -> y [T, dim] fp32

    pipe = block.host_pipeline()           # end to end from pinned host memory,
    for xh, yh in batches:                 # copies overlapped with compute
        pipe.submit(xh, yh)
    pipe.finish()                          # then synchronise the stream
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import MoECfg, MoEEpShard, MoEExpertWeights, check, fn


@dataclass(frozen=True)
class BlockShape:
    """Block hyper-parameters (names of the gate-init / moe-init excerpts)."""

    dim: int
    n_routed: int
    n_groups: int
    topk_groups: int
    topk: int
    inter: int
    n_shared: int = 1
    route_scale: float = 2.5
    score_func: str = "sigmoid"
    has_bias: bool = True

    def cfg(self) -> MoECfg:
        return MoECfg(self.dim, self.n_routed, self.n_groups, self.topk_groups, self.topk,
                      self.inter, self.n_shared, self.route_scale,
                      _lib.SCORE_FUNCS[self.score_func], int(self.has_bias))


_TORCH_DT = {torch.float32: "f32", torch.bfloat16: "bf16", torch.uint8: "e4m3",
             torch.float8_e4m3fn: "e4m3"}


def _dt(t: torch.Tensor) -> int:
    return _lib.DTYPES[_TORCH_DT[t.dtype]]


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check_cuda(*ts: Optional[torch.Tensor]) -> None:
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _ws(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------- the four


def router_prepare(shape: BlockShape, w_r: torch.Tensor) -> Optional[torch.Tensor]:
    """moe_router_prepare: the three-term bf16 split of w_r (uint8 device
    buffer), or None when the tensor-core scoring cannot apply to the shape."""
    _check_cuda(w_r)
    cfg = shape.cfg()
    n = fn("moe_router", "moe_router_prepare_size")(ctypes.byref(cfg))
    if not n:
        return None
    prep = torch.empty(n, dtype=torch.uint8, device=w_r.device)
    check(fn("moe_router", "moe_router_prepare")(ctypes.byref(cfg), w_r.data_ptr(),
                                                 prep.data_ptr(), n, _stream()),
          "moe_router_prepare")
    return prep


def router_forward(shape: BlockShape, x: torch.Tensor, w_r: torch.Tensor,
                   bias: Optional[torch.Tensor], *, gap: bool = False, ws=None, status=None,
                   prep: Optional[torch.Tensor] = None):
    """moe_router_forward (moe_router_forward_prepared when `prep` from
    router_prepare is given): (weights [T,k] fp32, indices [T,k] int32, gap
    [T] or None)."""
    _check_cuda(x, w_r, bias, prep)
    cfg = shape.cfg()
    T = x.shape[0]
    weights = torch.empty(T, shape.topk, dtype=torch.float32, device=x.device)
    indices = torch.empty(T, shape.topk, dtype=torch.int32, device=x.device)
    sel_gap = torch.empty(T, dtype=torch.float32, device=x.device) if gap else None
    need = fn("moe_router", "moe_router_workspace_size")(ctypes.byref(cfg), T)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    if prep is not None:
        st = fn("moe_router", "moe_router_forward_prepared")(
            ctypes.byref(cfg), T, x.data_ptr(), _dt(x), w_r.data_ptr(), prep.data_ptr(),
            _ptr(bias), weights.data_ptr(), indices.data_ptr(), _ptr(sel_gap), ws.data_ptr(),
            ws.numel(), _ptr(status), _stream())
        check(st, "moe_router_forward_prepared")
        return weights, indices, sel_gap
    st = fn("moe_router", "moe_router_forward")(
        ctypes.byref(cfg), T, x.data_ptr(), _dt(x), w_r.data_ptr(), _ptr(bias),
        weights.data_ptr(), indices.data_ptr(), _ptr(sel_gap), ws.data_ptr(), ws.numel(),
        _ptr(status), _stream())
    check(st, "moe_router_forward")
    return weights, indices, sel_gap


def dispatch_build(shape: BlockShape, indices: torch.Tensor, *, ws=None, status=None):
    """moe_dispatch_build: (counts [E], offsets [E+1], sorted_token [T*k], slot_of [T*k])."""
    _check_cuda(indices)
    cfg = shape.cfg()
    T = indices.shape[0]
    dev = indices.device
    counts = torch.empty(shape.n_routed, dtype=torch.int32, device=dev)
    offsets = torch.empty(shape.n_routed + 1, dtype=torch.int32, device=dev)
    sorted_token = torch.empty(T * shape.topk, dtype=torch.int32, device=dev)
    slot_of = torch.empty(T * shape.topk, dtype=torch.int32, device=dev)
    need = fn("moe_dispatch", "moe_dispatch_workspace_size")(ctypes.byref(cfg), T)
    if ws is None or ws.numel() < need:
        ws = _ws(need, dev)
    st = fn("moe_dispatch", "moe_dispatch_build")(
        ctypes.byref(cfg), T, indices.data_ptr(), counts.data_ptr(), offsets.data_ptr(),
        sorted_token.data_ptr(), slot_of.data_ptr(), ws.data_ptr(), ws.numel(), _ptr(status),
        _stream())
    check(st, "moe_dispatch_build")
    return counts, offsets, sorted_token, slot_of


def expert_weights_struct(w1, w3, w2, s1=None, s3=None, s2=None,
                          fp8_act: bool = False) -> MoEExpertWeights:
    """moe_expert_weights; fp8_act selects the FP8 x FP8 path (e4m3 weights)."""
    _check_cuda(w1, w3, w2, s1, s3, s2)
    return MoEExpertWeights(w1.data_ptr(), w3.data_ptr(), w2.data_ptr(), _dt(w1), _ptr(s1),
                            _ptr(s3), _ptr(s2), int(fp8_act))


def experts_forward(shape: BlockShape, x: torch.Tensor, wstruct: MoEExpertWeights,
                    offsets: torch.Tensor, sorted_token: torch.Tensor, *, out_perm=None,
                    out_shared=None, ws=None, status=None):
    """moe_experts_forward: (out_perm [T*k, dim] fp32, out_shared [T, dim] fp32 or None)."""
    _check_cuda(x, offsets, sorted_token)
    cfg = shape.cfg()
    T = x.shape[0]
    dev = x.device
    if out_perm is None:
        out_perm = torch.empty(T * shape.topk, shape.dim, dtype=torch.float32, device=dev)
    if out_shared is None and shape.n_shared:
        out_shared = torch.empty(T, shape.dim, dtype=torch.float32, device=dev)
    need = fn("moe_experts", "moe_experts_workspace_size")(ctypes.byref(cfg), T, _dt(x),
                                                            wstruct.w_dt)
    if ws is None or ws.numel() < need:
        ws = _ws(need, dev)
    st = fn("moe_experts", "moe_experts_forward")(
        ctypes.byref(cfg), T, x.data_ptr(), _dt(x), ctypes.byref(wstruct), offsets.data_ptr(),
        sorted_token.data_ptr(), out_perm.data_ptr(), _ptr(out_shared), ws.data_ptr(),
        ws.numel(), _ptr(status), _stream())
    check(st, "moe_experts_forward")
    return out_perm, out_shared


def experts_forward_combine(shape: BlockShape, x: torch.Tensor, wstruct: MoEExpertWeights,
                            offsets: torch.Tensor, sorted_token: torch.Tensor,
                            indices: torch.Tensor, weights: torch.Tensor, *, y=None, ws=None,
                            status=None):
    """moe_experts_forward_combine: y [T, dim] fp32 (experts + weighted scatter)."""
    _check_cuda(x, offsets, sorted_token, indices, weights)
    cfg = shape.cfg()
    T = x.shape[0]
    if y is None:
        y = torch.empty(T, shape.dim, dtype=torch.float32, device=x.device)
    need = fn("moe_experts", "moe_experts_workspace_size")(ctypes.byref(cfg), T, _dt(x),
                                                            wstruct.w_dt)
    if ws is None or ws.numel() < need:
        ws = _ws(need, x.device)
    st = fn("moe_experts", "moe_experts_forward_combine")(
        ctypes.byref(cfg), T, x.data_ptr(), _dt(x), ctypes.byref(wstruct), offsets.data_ptr(),
        sorted_token.data_ptr(), indices.data_ptr(), weights.data_ptr(), y.data_ptr(),
        ws.data_ptr(), ws.numel(), _ptr(status), _stream())
    check(st, "moe_experts_forward_combine")
    return y


def combine(shape: BlockShape, weights: torch.Tensor, slot_of: torch.Tensor,
            out_perm: torch.Tensor, out_shared: Optional[torch.Tensor], *, y=None, status=None):
    """moe_combine: y [T, dim] fp32."""
    _check_cuda(weights, slot_of, out_perm, out_shared)
    cfg = shape.cfg()
    T = weights.shape[0]
    if y is None:
        y = torch.empty(T, shape.dim, dtype=torch.float32, device=weights.device)
    st = fn("moe_combine", "moe_combine")(
        ctypes.byref(cfg), T, weights.data_ptr(), slot_of.data_ptr(), out_perm.data_ptr(),
        _ptr(out_shared), y.data_ptr(), _ptr(status), _stream())
    check(st, "moe_combine")
    return y


def quantize_e4m3_rows(src: torch.Tensor):
    """moe_quantize_e4m3_rows: (codes [rows, K] uint8, scales [rows] fp32) of
    a bf16 [rows, K] matrix, one scale per row."""
    _check_cuda(src)
    if src.dtype != torch.bfloat16 or src.dim() != 2:
        raise ValueError("src must be a 2-D bf16 tensor")
    rows, K = src.shape
    q = torch.empty(rows, K, dtype=torch.uint8, device=src.device)
    sc = torch.empty(rows, dtype=torch.float32, device=src.device)
    check(fn("moe_experts", "moe_quantize_e4m3_rows")(src.data_ptr(), rows, K, q.data_ptr(),
                                                      sc.data_ptr(), _stream()),
          "moe_quantize_e4m3_rows")
    return q, sc


def ep_plan(shape: BlockShape, T: int, rank: int, world: int) -> tuple:
    """moe_ep_plan: (first expert, end expert, first token, end token) of the
    shared expert's slice for expert-parallel rank `rank` of `world`."""
    cfg = shape.cfg()
    out = (ctypes.c_int32 * 4)()
    check(fn("moe_experts", "moe_ep_plan")(ctypes.byref(cfg), T,
                                           ctypes.byref(MoEEpShard(rank, world)), out),
          "moe_ep_plan")
    return tuple(out)


def shard_params(shape: BlockShape, params: "BlockParams", rank: int, world: int) -> "BlockParams":
    """The weights expert-parallel rank `rank` holds: its routed experts in
    order, then the shared expert(s); the router weight and bias whole."""
    e0, e1, _, _ = ep_plan(shape, 0, rank, world)
    E = shape.n_routed

    def part(t):
        if t is None:
            return None
        return torch.cat([t[e0:e1], t[E:]]).contiguous()

    p = params
    return BlockParams(p.w_r, p.bias, part(p.w1), part(p.w3), part(p.w2), part(p.s1),
                       part(p.s3), part(p.s2))


def selftest_wait(limit_ns: int, status: torch.Tensor) -> None:
    check(fn("moe_experts", "moe_experts_selftest_wait")(limit_ns, status.data_ptr(), _stream()),
          "moe_experts_selftest_wait")


# ------------------------------------------------------------- the block


@dataclass
class BlockParams:
    """Device tensors of one block.  w1/w3 [E+S, I, D], w2 [E+S, D, I]
    (bf16, fp32, or e4m3 codes as uint8 with s1/s3/s2 block scales)."""

    w_r: torch.Tensor
    bias: Optional[torch.Tensor]
    w1: torch.Tensor
    w3: torch.Tensor
    w2: torch.Tensor
    s1: Optional[torch.Tensor] = None
    s3: Optional[torch.Tensor] = None
    s2: Optional[torch.Tensor] = None


class MoEBlock:
    """One MoE block with its workspaces, for repeated forwards on a fixed T.

    forward() enqueues router -> dispatch -> experts -> combine on the current
    stream with no host synchronisation; all buffers are preallocated, so the
    call can be captured in a CUDA graph.

    combine="scatter" (default) adds the gated expert outputs straight into y
    from the second matmul (moe_experts_forward_combine); "ordered" writes
    the per-slot outputs and sums them in a fixed order (moe_experts_forward
    + moe_combine), bit-reproducible run to run.
    """

    def __init__(self, shape: BlockShape, params: BlockParams, T: int, x_dtype: torch.dtype,
                 device=None, combine: str = "scatter", fp8_act: bool = False,
                 ep: tuple = (0, 1), ep_group=None, fused_decode: bool = False):
        if combine not in ("scatter", "ordered"):
            raise ValueError(combine)
        # expert parallelism: (rank, world); params then hold the rank's
        # shard (shard_params) and y is summed over the ranks of ep_group by
        # an all-reduce (left partial when ep_group is None)
        self.ep_rank, self.ep_world = ep
        self.ep_group = ep_group
        if self.ep_world > 1 and combine != "scatter":
            raise ValueError("expert parallelism uses the scatter combine")
        # the whole block in one launch (moe_block_forward_decode): decode
        # batches, bf16, scatter combine, one GPU
        self.fused_decode = fused_decode
        if fused_decode and (combine != "scatter" or fp8_act or self.ep_world > 1):
            raise ValueError("the fused decode launch uses the scatter combine on one GPU")
        if fp8_act and params.s1 is None:
            raise ValueError("fp8_act needs e4m3 expert weights")
        self.fp8_act = fp8_act
        self.combine_mode = combine
        self.x_dtype = x_dtype
        self.shape, self.p, self.T = shape, params, T
        dev = torch.device(device or params.w1.device)
        self.cfg = shape.cfg()
        k, D = shape.topk, shape.dim
        self.wstruct = expert_weights_struct(params.w1, params.w3, params.w2, params.s1,
                                             params.s3, params.s2, fp8_act)
        cfgp = ctypes.byref(self.cfg)
        x_dt = _lib.DTYPES[_TORCH_DT[x_dtype]]
        self.ws_router = _ws(fn("moe_router", "moe_router_workspace_size")(cfgp, T), dev)
        # the router weight's three-term bf16 split, written once here and
        # read by every forward (tensor-core scoring path only)
        self.router_prep = None
        nprep = fn("moe_router", "moe_router_prepare_size")(cfgp)
        if nprep and x_dtype == torch.bfloat16:
            self.router_prep = torch.empty(nprep, dtype=torch.uint8, device=dev)
            check(fn("moe_router", "moe_router_prepare")(
                cfgp, params.w_r.data_ptr(), self.router_prep.data_ptr(), nprep, _stream()),
                "moe_router_prepare")
        self.ws_dispatch = _ws(fn("moe_dispatch", "moe_dispatch_workspace_size")(cfgp, T), dev)
        self.ws_experts = _ws(fn("moe_experts", "moe_experts_workspace_size")(
            cfgp, T, x_dt, self.wstruct.w_dt), dev)
        f32, i32 = torch.float32, torch.int32
        self.weights = torch.empty(T, k, dtype=f32, device=dev)
        self.indices = torch.empty(T, k, dtype=i32, device=dev)
        self.sel_gap = torch.empty(T, dtype=f32, device=dev)
        self.counts = torch.empty(shape.n_routed, dtype=i32, device=dev)
        self.offsets = torch.empty(shape.n_routed + 1, dtype=i32, device=dev)
        self.sorted_token = torch.empty(T * k, dtype=i32, device=dev)
        self.slot_of = torch.empty(T * k, dtype=i32, device=dev)
        ordered = combine == "ordered"
        self.out_perm = torch.empty(T * k if ordered else 0, D, dtype=f32, device=dev)
        self.out_shared = (torch.empty(T if ordered else 0, D, dtype=f32, device=dev)
                           if shape.n_shared else None)
        self.y = torch.empty(T, D, dtype=f32, device=dev)
        self.status = torch.zeros(1, dtype=i32, device=dev)
        self.ws_fused = (_ws(fn("moe_experts", "moe_block_decode_workspace_size")(cfgp, T), dev)
                         if fused_decode else None)

    # kernels one forward launches: router 2 (scores, selection; the weight
    # split is prepared once), dispatch 3, experts 5 on the
    # tensor-core path, with bf16 or e4m3 weights (two tile tables, row
    # gather, two GEMMs) or 4 on the CUDA-core path, then combine 1 (ordered)
    # or nothing (scatter; y is zeroed by a memset node)
    @property
    def launches_per_forward(self) -> int:
        if self.fused_decode:
            return 1  # (plus a 8-byte memset of its grid barrier)
        sh = self.shape
        tc_router = (self.x_dtype == torch.bfloat16 and sh.n_routed % 128 == 0
                     and sh.dim % 64 == 0 and self.T >= 32)
        tc_experts = (self.x_dtype == torch.bfloat16 and sh.dim % 128 == 0
                      and sh.inter % 128 == 0
                      and self.p.w1.dtype in (torch.bfloat16, torch.uint8, torch.float8_e4m3fn))
        # the FP8 x FP8 path adds the quantisation of h (six expert launches)
        return ((2 if tc_router and self.router_prep is not None else 3 if tc_router else 2)
                + 3 + (6 if self.fp8_act else 5 if tc_experts else 4)
                + (1 if self.combine_mode == "ordered" else 0))

    def _router(self, x, cfgp, s):
        p = self.p
        if self.router_prep is not None:
            check(fn("moe_router", "moe_router_forward_prepared")(
                cfgp, self.T, x.data_ptr(), _dt(x), p.w_r.data_ptr(), self.router_prep.data_ptr(),
                _ptr(p.bias), self.weights.data_ptr(), self.indices.data_ptr(),
                self.sel_gap.data_ptr(), self.ws_router.data_ptr(), self.ws_router.numel(),
                self.status.data_ptr(), s), "moe_router_forward_prepared")
            return
        check(fn("moe_router", "moe_router_forward")(
            cfgp, self.T, x.data_ptr(), _dt(x), p.w_r.data_ptr(), _ptr(p.bias),
            self.weights.data_ptr(), self.indices.data_ptr(), self.sel_gap.data_ptr(),
            self.ws_router.data_ptr(), self.ws_router.numel(), self.status.data_ptr(), s),
            "moe_router_forward")

    def _dispatch(self, cfgp, s):
        check(fn("moe_dispatch", "moe_dispatch_build")(
            cfgp, self.T, self.indices.data_ptr(), self.counts.data_ptr(),
            self.offsets.data_ptr(), self.sorted_token.data_ptr(), self.slot_of.data_ptr(),
            self.ws_dispatch.data_ptr(), self.ws_dispatch.numel(), self.status.data_ptr(), s),
            "moe_dispatch_build")

    def _experts(self, x, cfgp, s, y):
        if self.ep_world > 1:
            shard = MoEEpShard(self.ep_rank, self.ep_world)
            check(fn("moe_experts", "moe_experts_forward_combine_ep")(
                cfgp, self.T, x.data_ptr(), _dt(x), ctypes.byref(self.wstruct),
                ctypes.byref(shard), self.offsets.data_ptr(), self.sorted_token.data_ptr(),
                self.indices.data_ptr(), self.weights.data_ptr(), y.data_ptr(),
                self.ws_experts.data_ptr(), self.ws_experts.numel(), self.status.data_ptr(), s),
                "moe_experts_forward_combine_ep")
            return
        if self.combine_mode == "scatter":
            check(fn("moe_experts", "moe_experts_forward_combine")(
                cfgp, self.T, x.data_ptr(), _dt(x), ctypes.byref(self.wstruct),
                self.offsets.data_ptr(), self.sorted_token.data_ptr(), self.indices.data_ptr(),
                self.weights.data_ptr(), y.data_ptr(), self.ws_experts.data_ptr(),
                self.ws_experts.numel(), self.status.data_ptr(), s),
                "moe_experts_forward_combine")
            return
        check(fn("moe_experts", "moe_experts_forward")(
            cfgp, self.T, x.data_ptr(), _dt(x), ctypes.byref(self.wstruct),
            self.offsets.data_ptr(), self.sorted_token.data_ptr(), self.out_perm.data_ptr(),
            _ptr(self.out_shared), self.ws_experts.data_ptr(), self.ws_experts.numel(),
            self.status.data_ptr(), s), "moe_experts_forward")

    def _combine(self, cfgp, s, y):
        if self.ep_world > 1 and self.ep_group is not None:
            # the ranks' partial sums (the moe-forward excerpt's all_reduce)
            torch.distributed.all_reduce(y, group=self.ep_group)
            return
        if self.combine_mode == "scatter":
            return  # done inside the experts' second matmul
        check(fn("moe_combine", "moe_combine")(
            cfgp, self.T, self.weights.data_ptr(), self.slot_of.data_ptr(),
            self.out_perm.data_ptr(), _ptr(self.out_shared), y.data_ptr(),
            self.status.data_ptr(), s), "moe_combine")

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Enqueue the four libraries for x [T, dim]; returns y (fp32 [T, dim],
        self.y unless another device buffer is given)."""
        assert x.shape == (self.T, self.shape.dim) and x.is_cuda and x.is_contiguous()
        if y is None:
            y = self.y
        assert y.shape == (self.T, self.shape.dim) and y.dtype == torch.float32 and y.is_contiguous()
        cfgp, s = ctypes.byref(self.cfg), _stream()
        if self.fused_decode:
            self._fused(x, cfgp, s, y)
            return y
        self._router(x, cfgp, s)
        self._dispatch(cfgp, s)
        self._experts(x, cfgp, s, y)
        self._combine(cfgp, s, y)
        return y

    def _fused(self, x, cfgp, s, y):
        p = self.p
        check(fn("moe_experts", "moe_block_forward_decode")(
            cfgp, self.T, x.data_ptr(), _dt(x), p.w_r.data_ptr(), _ptr(p.bias),
            ctypes.byref(self.wstruct), self.weights.data_ptr(), self.indices.data_ptr(),
            self.sel_gap.data_ptr(), self.counts.data_ptr(), self.offsets.data_ptr(),
            self.sorted_token.data_ptr(), self.slot_of.data_ptr(), y.data_ptr(),
            self.ws_fused.data_ptr(), self.ws_fused.numel(), self.status.data_ptr(), s),
            "moe_block_forward_decode")

    def forward_profiled(self, x: torch.Tensor, ev) -> torch.Tensor:
        """forward() with 10 CUDA events recorded on the stream: around the
        router [0,1], dispatch [1,2], the row gather [3,4], the two expert
        GEMMs [4,5] and [6,7], and the combine [8,9]."""
        cfgp, s = ctypes.byref(self.cfg), _stream()
        if self.fused_decode:  # one launch: the whole step is the router's span
            ev[0].record()
            self._fused(x, cfgp, s, self.y)
            for e in ev[1:]:
                e.record()
            return self.y
        ev[0].record()
        self._router(x, cfgp, s)
        ev[1].record()
        self._dispatch(cfgp, s)
        ev[2].record()
        for e in ev[3:8]:   # mark them recorded for torch; the library re-records them
            e.record()
        handles = (ctypes.c_void_p * 5)(*[e.cuda_event for e in ev[3:8]])
        check(fn("moe_experts", "moe_experts_set_profile_events")(handles, 5), "profile events")
        try:
            self._experts(x, cfgp, s, self.y)
        finally:
            fn("moe_experts", "moe_experts_set_profile_events")(None, 0)
        ev[8].record()
        self._combine(cfgp, s, self.y)
        ev[9].record()
        return self.y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, x_dev: torch.Tensor):
        """End to end from host memory: copy x (pinned host) to the device,
        run the block, copy y back into y_host (pinned), all on the current
        stream; the caller synchronises."""
        x_dev.copy_(x_host, non_blocking=True)
        self.forward(x_dev)
        y_host.copy_(self.y, non_blocking=True)
        return y_host

    def host_pipeline(self) -> "HostPipeline":
        """A HostPipeline over this block (see there)."""
        return HostPipeline(self)

    def device_status(self) -> int:
        """The first device-side error of the forwards so far (0 = none); syncs."""
        return int(self.status.item())


class HostPipeline:
    """End-to-end forwards from pinned host memory with the copies overlapped.

    submit(x_host, y_host) enqueues one batch: its input copy runs on a
    host-to-device stream, the block on the caller's current stream, and the
    copy of its y into y_host on a device-to-host stream.  Two device input
    and output buffers alternate, so batch i's copies overlap the compute of
    batches i-1 and i+1.  Ordering is kept with CUDA events only (no host
    synchronisation); finish() makes the current stream wait for the last
    output copy.  y_host must stay untouched until then.
    """

    def __init__(self, blk: "MoEBlock"):
        self.blk = blk
        dev = blk.y.device
        T, D = blk.T, blk.shape.dim
        self.x_dev = [torch.empty(T, D, dtype=blk.x_dtype, device=dev) for _ in range(2)]
        self.y_dev = [torch.empty(T, D, dtype=torch.float32, device=dev) for _ in range(2)]
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        ev = lambda: [torch.cuda.Event() for _ in range(2)]  # noqa: E731
        self.x_ready, self.x_free, self.y_ready, self.y_free = ev(), ev(), ev(), ev()
        self.used = [False, False]
        self.i = 0
        self.last = None

    def submit(self, x_host: torch.Tensor, y_host: torch.Tensor) -> None:
        b = self.i % 2
        comp = torch.cuda.current_stream(self.x_dev[b].device)
        if self.i == 0:  # copies start after whatever the caller enqueued so far
            self.h2d.wait_stream(comp)
            self.d2h.wait_stream(comp)
        with torch.cuda.stream(self.h2d):
            if self.used[b]:
                self.h2d.wait_event(self.x_free[b])     # the block two batches back read it
            self.x_dev[b].copy_(x_host, non_blocking=True)
            self.x_ready[b].record(self.h2d)
        comp.wait_event(self.x_ready[b])
        if self.used[b]:
            comp.wait_event(self.y_free[b])             # its output copy has left
        self.blk.forward(self.x_dev[b], self.y_dev[b])
        self.x_free[b].record(comp)
        self.y_ready[b].record(comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(self.y_ready[b])
            y_host.copy_(self.y_dev[b], non_blocking=True)
            self.y_free[b].record(self.d2h)
        self.last = self.y_free[b]
        self.used[b] = True
        self.i += 1

    def finish(self) -> None:
        if self.last is not None:
            torch.cuda.current_stream(self.x_dev[0].device).wait_event(self.last)

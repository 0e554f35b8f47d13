"""ctypes loader for the four C-ABI libraries (moe_router, moe_dispatch,
moe_experts, moe_combine).  Loading fails loudly: there is no fallback."""
from __future__ import annotations

import ctypes
import os

LIBDIR = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib")

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", -1: "MOE_ERR_INVALID", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_WORKSPACE",
    -4: "MOE_ERR_CUDA", -5: "MOE_ERR_TIMEOUT", -6: "MOE_ERR_RANGE",
}
DTYPES = {"f32": 0, "bf16": 1, "e4m3": 2}
SCORE_FUNCS = {"sigmoid": 0, "softmax": 1}


class MoECfg(ctypes.Structure):
    """Mirror of moe_cfg in include/moe_common.h."""

    _fields_ = [
        ("dim", ctypes.c_int32), ("n_routed", ctypes.c_int32), ("n_groups", ctypes.c_int32),
        ("topk_groups", ctypes.c_int32), ("topk", ctypes.c_int32), ("inter", ctypes.c_int32),
        ("n_shared", ctypes.c_int32), ("route_scale", ctypes.c_float),
        ("score_func", ctypes.c_int32), ("has_bias", ctypes.c_int32),
    ]


class MoEExpertWeights(ctypes.Structure):
    """Mirror of moe_expert_weights in include/moe_experts.h."""

    _fields_ = [
        ("w1", ctypes.c_void_p), ("w3", ctypes.c_void_p), ("w2", ctypes.c_void_p),
        ("w_dt", ctypes.c_int32),
        ("s1", ctypes.c_void_p), ("s3", ctypes.c_void_p), ("s2", ctypes.c_void_p),
        ("act_e4m3", ctypes.c_int32),
    ]


class MoEEpShard(ctypes.Structure):
    """Mirror of moe_ep_shard in include/moe_experts.h."""

    _fields_ = [("rank", ctypes.c_int32), ("world", ctypes.c_int32)]


_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_cfgp = ctypes.POINTER(MoECfg)

# (library, symbol) -> (restype, argtypes); this is the full exported C-ABI
SIGNATURES = {
    ("moe_router", "moe_router_workspace_size"): (_sz, [_cfgp, _i64]),
    ("moe_router", "moe_router_forward"): (
        _i32, [_cfgp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    ("moe_router", "moe_router_prepare_size"): (_sz, [_cfgp]),
    ("moe_router", "moe_router_prepare"): (_i32, [_cfgp, _vp, _vp, _sz, _vp]),
    ("moe_router", "moe_router_forward_prepared"): (
        _i32, [_cfgp, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    ("moe_dispatch", "moe_dispatch_workspace_size"): (_sz, [_cfgp, _i64]),
    ("moe_dispatch", "moe_dispatch_build"): (
        _i32, [_cfgp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    ("moe_dispatch", "moe_dispatch_build_noalloc"): (
        _i32, [_cfgp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    ("moe_experts", "moe_experts_workspace_size"): (_sz, [_cfgp, _i64, _i32, _i32]),
    ("moe_experts", "moe_experts_forward"): (
        _i32, [_cfgp, _i64, _vp, _i32, ctypes.POINTER(MoEExpertWeights), _vp, _vp, _vp, _vp,
               _vp, _sz, _vp, _vp]),
    ("moe_experts", "moe_experts_forward_combine"): (
        _i32, [_cfgp, _i64, _vp, _i32, ctypes.POINTER(MoEExpertWeights), _vp, _vp, _vp, _vp, _vp,
               _vp, _sz, _vp, _vp]),
    ("moe_experts", "moe_ep_plan"): (
        _i32, [_cfgp, _i64, ctypes.POINTER(MoEEpShard), ctypes.POINTER(ctypes.c_int32)]),
    ("moe_experts", "moe_experts_forward_combine_ep"): (
        _i32, [_cfgp, _i64, _vp, _i32, ctypes.POINTER(MoEExpertWeights),
               ctypes.POINTER(MoEEpShard), _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    ("moe_experts", "moe_block_decode_workspace_size"): (_sz, [_cfgp, _i64]),
    ("moe_experts", "moe_block_forward_decode"): (
        _i32, [_cfgp, _i64, _vp, _i32, _vp, _vp, ctypes.POINTER(MoEExpertWeights), _vp, _vp, _vp,
               _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]),
    ("moe_experts", "moe_experts_up"): (
        _i32, [_cfgp, _i64, _vp, _i32, ctypes.POINTER(MoEExpertWeights), _vp, _vp, _vp, _sz, _vp,
               _vp]),
    ("moe_experts", "moe_experts_down"): (
        _i32, [_cfgp, _i64, _i32, ctypes.POINTER(MoEExpertWeights), _vp, _vp, _vp, _vp, _sz, _vp,
               _vp]),
    ("moe_experts", "moe_quantize_e4m3_rows"): (_i32, [_vp, _i64, _i32, _vp, _vp, _vp]),
    ("moe_experts", "moe_experts_set_profile_events"): (_i32, [ctypes.POINTER(_vp), _i32]),
    ("moe_experts", "moe_experts_selftest_wait"): (_i32, [_i64, _vp, _vp]),
    ("moe_combine", "moe_combine"): (_i32, [_cfgp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
}

LIBRARIES = ("moe_router", "moe_dispatch", "moe_experts", "moe_combine")

_libs: dict[str, ctypes.CDLL] = {}


def lib_path(name: str) -> str:
    return os.path.join(LIBDIR, f"lib{name}.so")


def load(name: str) -> ctypes.CDLL:
    """Load one library and declare its prototypes.  Raises if it is missing."""
    if name in _libs:
        return _libs[name]
    path = lib_path(name)
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build the CUDA libraries first "
            "(python -m sparse_moe_layer_sum_b200.build)")
    lib = ctypes.CDLL(path)
    for (lname, sym), (res, args) in SIGNATURES.items():
        if lname == name:
            fn = getattr(lib, sym)
            fn.restype = res
            fn.argtypes = args
    _libs[name] = lib
    return lib


def fn(name: str, sym: str):
    return getattr(load(name), sym)


def check(status: int, what: str) -> None:
    if status != MOE_OK:
        raise RuntimeError(f"{what} failed: {STATUS_NAMES.get(status, status)}")

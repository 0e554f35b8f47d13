"""The C-ABI libraries load on a host without a GPU, export every function
their headers declare, and reject bad arguments before launching anything.

No compute call is made here: every call below fails argument validation,
which returns before any CUDA runtime call.
"""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT
from sparse_moe_layer_sum_b200 import _lib
from sparse_moe_layer_sum_b200._lib import MoECfg, MoEExpertWeights, fn

HEADERS = {"moe_router": "moe_router.h", "moe_dispatch": "moe_dispatch.h",
           "moe_experts": "moe_experts.h", "moe_combine": "moe_combine.h"}

INVALID, UNSUPPORTED, WORKSPACE = -1, -2, -3


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()


def declared(header):
    text = open(os.path.join(ROOT, "include", header)).read()
    return re.findall(r"^(?:moe_status|size_t)\s+(\w+)\s*\(", text, flags=re.M)


def test_every_declared_symbol_is_exported():
    for lib, header in HEADERS.items():
        names = declared(header)
        assert names, header
        out = subprocess.run(["nm", "-D", "--defined-only", _lib.lib_path(lib)],
                             capture_output=True, text=True, check=True).stdout
        exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
        for n in names:
            assert n in exported, f"{n} not exported by lib{lib}.so"
            assert (lib, n) in _lib.SIGNATURES, f"{n} has no ctypes prototype"
        # nothing but the declared API is exported
        assert {e for e in exported if e.startswith("moe_")} == set(names)


def v3_cfg(**kw):
    c = dict(dim=7168, n_routed=256, n_groups=8, topk_groups=4, topk=8, inter=2048, n_shared=1,
             route_scale=2.5, score_func=0, has_bias=1)
    c.update(kw)
    return MoECfg(**c)


P = ctypes.c_void_p(0x1000)  # a non-null pointer that is never dereferenced


def router(cfg, T=4, x_dt=1, ws_bytes=1 << 30, bias=P, x=P):
    return fn("moe_router", "moe_router_forward")(
        ctypes.byref(cfg) if cfg is not None else None, T, x, x_dt, P, bias, P, P, None, P,
        ws_bytes, None, None)


def test_router_validation():
    assert router(None) == INVALID
    assert router(v3_cfg(topk=200)) == INVALID                 # k > kept groups' experts
    assert router(v3_cfg(n_groups=7)) == INVALID               # groups must divide experts
    assert router(v3_cfg(topk_groups=9)) == INVALID
    assert router(v3_cfg(score_func=5)) == INVALID
    assert router(v3_cfg(), T=-1) == INVALID
    assert router(v3_cfg(), x=None) == INVALID
    assert router(v3_cfg(), bias=None) == INVALID              # has_bias needs a bias
    assert router(v3_cfg(), x_dt=2) == UNSUPPORTED             # e4m3 activations
    assert router(v3_cfg(topk=40)) == UNSUPPORTED              # more than 32 per token
    assert router(v3_cfg(n_routed=2048, n_groups=8)) == UNSUPPORTED
    assert router(v3_cfg(), ws_bytes=16) == WORKSPACE
    assert router(v3_cfg(), T=0) == 0                          # empty batch: nothing to do


def test_router_prepare_validation():
    size = fn("moe_router", "moe_router_prepare_size")
    prep = fn("moe_router", "moe_router_prepare")
    fwd = fn("moe_router", "moe_router_forward_prepared")
    c = v3_cfg()
    assert size(ctypes.byref(c)) == 3 * 256 * 7168 * 2          # three bf16 terms of W_r
    small = v3_cfg(dim=256, n_routed=16, n_groups=4, topk_groups=2, topk=4, inter=128)
    assert size(ctypes.byref(small)) == 0                      # no tensor-core tiling
    assert size(ctypes.byref(v3_cfg(topk=200))) == 0           # invalid config
    assert size(None) == 0
    assert prep(ctypes.byref(c), None, P, 1 << 30, None) == INVALID
    assert prep(ctypes.byref(c), P, None, 1 << 30, None) == INVALID
    assert prep(ctypes.byref(c), P, P, 1024, None) == WORKSPACE
    assert prep(ctypes.byref(small), P, P, 1 << 30, None) == UNSUPPORTED
    args = lambda pr: (ctypes.byref(c), 4, P, 1, P, pr, P, P, P, None, P, 1 << 30, None, None)
    assert fwd(*args(None)) == INVALID                         # the split is required
    assert fwd(ctypes.byref(c), 0, P, 1, P, P, P, P, P, None, P, 1 << 30, None, None) == 0
    assert fwd(ctypes.byref(c), 4, P, 1, P, P, P, P, P, None, P, 16, None, None) == WORKSPACE


def test_workspace_sizes_grow_with_tokens():
    c = v3_cfg()
    f = fn("moe_router", "moe_router_workspace_size")
    assert f(ctypes.byref(c), 4096) >= 4096 * 256 * 4
    g = fn("moe_experts", "moe_experts_workspace_size")
    assert g(ctypes.byref(c), 4096, 1, 1) > g(ctypes.byref(c), 64, 1, 1) > 0
    assert fn("moe_dispatch", "moe_dispatch_workspace_size")(ctypes.byref(c), 16384) >= 256 * 4
    assert f(ctypes.byref(v3_cfg(topk=200)), 8) == 0            # invalid config -> 0
    # shapes that only the CUDA-core paths take (no tensor-core tiling)
    for E, G in ((16, 4), (24, 4), (64, 8)):
        small = v3_cfg(dim=256, n_routed=E, n_groups=G, topk_groups=2, topk=4, inter=96)
        assert f(ctypes.byref(small), 300) > 0
        assert g(ctypes.byref(small), 300, 0, 0) > 0


def test_dispatch_validation():
    f = fn("moe_dispatch", "moe_dispatch_build")
    c = v3_cfg()
    assert f(None, 4, P, P, P, P, P, P, 1 << 20, None, None) == INVALID
    assert f(ctypes.byref(c), -2, P, P, P, P, P, P, 1 << 20, None, None) == INVALID
    assert f(ctypes.byref(c), 4, None, P, P, P, P, P, 1 << 20, None, None) == INVALID
    assert f(ctypes.byref(c), 4, P, P, P, P, P, P, 4, None, None) == WORKSPACE
    assert f(ctypes.byref(c), 1 << 29, P, P, P, P, P, P, 1 << 40, None, None) == INVALID


def test_experts_validation():
    f = fn("moe_experts", "moe_experts_forward")
    c = v3_cfg()
    w = MoEExpertWeights(0x1000, 0x1000, 0x1000, 1, None, None, None)
    call = lambda cfg=c, x_dt=1, ws=1 << 40, wt=w, sh=P: f(
        ctypes.byref(cfg), 8, P, x_dt, ctypes.byref(wt), P, P, P, sh, P, ws, None, None)
    assert call(ws=8) == WORKSPACE
    assert call(x_dt=2) == UNSUPPORTED
    assert call(cfg=v3_cfg(n_shared=2)) == UNSUPPORTED
    assert call(sh=None) == INVALID                            # shared expert needs out_shared
    fp8 = MoEExpertWeights(0x1000, 0x1000, 0x1000, 2, None, None, None)
    assert call(wt=fp8) == INVALID                             # e4m3 needs block scales
    bad = MoEExpertWeights(0x1000, 0x1000, 0x1000, 7, None, None, None)
    assert call(wt=bad) == UNSUPPORTED
    fc = fn("moe_experts", "moe_experts_forward_combine")
    # missing router outputs or y
    assert fc(ctypes.byref(c), 8, P, 1, ctypes.byref(w), P, P, None, P, P, P, 1 << 40, None,
              None) == INVALID
    assert fc(ctypes.byref(c), 8, P, 1, ctypes.byref(w), P, P, P, P, None, P, 1 << 40, None,
              None) == INVALID
    assert fc(ctypes.byref(c), 8, P, 1, ctypes.byref(w), P, P, P, P, P, P, 8, None,
              None) == WORKSPACE
    # y must be 16-byte aligned (the scatter adds 16-byte vectors)
    assert fc(ctypes.byref(c), 8, P, 1, ctypes.byref(w), P, P, P, P, ctypes.c_void_p(0x1008), P,
              1 << 40, None, None) == INVALID
    # empty batch: validated, then nothing to launch
    assert f(ctypes.byref(c), 0, P, 1, ctypes.byref(w), P, P, P, P, P, 1 << 40, None, None) == 0
    assert fc(ctypes.byref(c), 0, P, 1, ctypes.byref(w), P, P, P, P, P, P, 1 << 40, None,
              None) == 0


def test_fp8_activation_path_validation():
    f = fn("moe_experts", "moe_experts_forward")
    c = v3_cfg()
    call = lambda cfg, wt, x_dt=1: f(ctypes.byref(cfg), 8, P, x_dt, ctypes.byref(wt), P, P, P, P,
                                     P, 1 << 40, None, None)
    fp8 = lambda act: MoEExpertWeights(0x1000, 0x1000, 0x1000, 2, 0x1000, 0x1000, 0x1000, act)
    assert call(c, fp8(2)) == INVALID                          # the flag is 0 or 1
    bf = MoEExpertWeights(0x1000, 0x1000, 0x1000, 1, None, None, None, 1)
    assert call(c, bf) == UNSUPPORTED                          # e4m3 weights only
    assert call(c, fp8(1), x_dt=0) == UNSUPPORTED              # bf16 activations in
    assert call(v3_cfg(dim=7296), fp8(1)) == UNSUPPORTED       # dim % 256 != 0
    # the scatter adds 16-byte vectors into y: a y off that alignment is
    # refused before any launch
    fc = fn("moe_experts", "moe_experts_forward_combine")
    assert fc(ctypes.byref(c), 8, P, 1, ctypes.byref(fp8(1)), P, P, P, P, ctypes.c_void_p(0x1004), P, 1 << 40,
              None, None) == INVALID
    q = fn("moe_experts", "moe_quantize_e4m3_rows")
    assert q(P, 4, 102, P, P, None) == INVALID                 # K % 4 != 0
    assert q(None, 4, 128, P, P, None) == INVALID
    assert q(P, 4, 128, P, None, None) == INVALID
    assert q(P, -1, 128, P, P, None) == INVALID
    assert q(None, 0, 128, None, None, None) == 0              # nothing to do


def test_expert_parallel_plan_and_validation():
    from sparse_moe_layer_sum_b200._lib import MoEEpShard
    plan = fn("moe_experts", "moe_ep_plan")
    c = v3_cfg()
    out = (ctypes.c_int32 * 4)()
    assert plan(ctypes.byref(c), 4096, ctypes.byref(MoEEpShard(3, 8)), out) == 0
    assert list(out) == [96, 128, 1536, 2048]          # experts 96..127, tokens 1536..2047
    assert plan(ctypes.byref(c), 10, ctypes.byref(MoEEpShard(2, 3)), out) == UNSUPPORTED
    assert plan(ctypes.byref(c), 10, ctypes.byref(MoEEpShard(8, 8)), out) == INVALID
    assert plan(ctypes.byref(c), 10, ctypes.byref(MoEEpShard(0, 0)), out) == INVALID
    assert plan(ctypes.byref(c), -1, ctypes.byref(MoEEpShard(0, 1)), out) == INVALID
    assert plan(ctypes.byref(c), 10, None, out) == INVALID
    f = fn("moe_experts", "moe_experts_forward_combine_ep")
    w = MoEExpertWeights(0x1000, 0x1000, 0x1000, 1, None, None, None)
    sh = MoEEpShard(1, 4)
    assert f(ctypes.byref(c), 8, P, 1, ctypes.byref(w), None, P, P, P, P, P, P, 1 << 40, None,
             None) == INVALID                                   # no shard
    assert f(ctypes.byref(c), 8, P, 1, ctypes.byref(w), ctypes.byref(MoEEpShard(1, 3)), P, P, P,
             P, P, P, 1 << 40, None, None) == UNSUPPORTED
    assert f(ctypes.byref(c), 8, P, 1, ctypes.byref(w), ctypes.byref(sh), P, P, None, P, P, P,
             1 << 40, None, None) == INVALID                    # no router indices
    assert f(ctypes.byref(c), 0, P, 1, ctypes.byref(w), ctypes.byref(sh), P, P, P, P, P, P,
             1 << 40, None, None) == 0                          # empty batch


def test_fused_decode_validation():
    size = fn("moe_experts", "moe_block_decode_workspace_size")
    f = fn("moe_experts", "moe_block_forward_decode")
    c = v3_cfg()
    assert size(ctypes.byref(c), 64) > size(ctypes.byref(c), 8) > 0
    assert size(ctypes.byref(v3_cfg(topk=200)), 8) == 0
    w = MoEExpertWeights(0x1000, 0x1000, 0x1000, 1, None, None, None)

    def call(cfg=c, T=64, x_dt=1, wt=w, ws=1 << 40, x=P, y=P):
        return f(ctypes.byref(cfg), T, x, x_dt, P, P, ctypes.byref(wt), P, P, None, P, P, P, P, y,
                 P, ws, None, None)
    assert call(T=4096) == UNSUPPORTED                          # not a decode batch
    assert call(x_dt=0) == UNSUPPORTED                          # bf16 x only
    fp8 = MoEExpertWeights(0x1000, 0x1000, 0x1000, 2, 0x1000, 0x1000, 0x1000)
    assert call(wt=fp8) == UNSUPPORTED                          # bf16 weights only
    assert call(cfg=v3_cfg(n_routed=512, n_groups=8)) == UNSUPPORTED
    assert call(x=None) == INVALID
    assert call(y=ctypes.c_void_p(0x1004)) == INVALID           # y not 16-byte aligned
    assert call(ws=1024) == WORKSPACE
    assert call(T=0) == 0                                       # empty batch
    assert call(T=-1) == INVALID


def test_combine_and_selftest_validation():
    f = fn("moe_combine", "moe_combine")
    c = v3_cfg()
    assert f(ctypes.byref(c), 4, None, P, P, P, P, None, None) == INVALID
    assert f(ctypes.byref(c), 4, P, P, P, None, P, None, None) == INVALID   # n_shared=1
    assert f(ctypes.byref(v3_cfg(dim=7170, inter=2048)), 4, P, P, P, P, P, None, None) == UNSUPPORTED
    assert f(ctypes.byref(c), 0, None, None, None, None, None, None, None) == 0
    g = fn("moe_experts", "moe_experts_selftest_wait")
    assert g(0, P, None) == INVALID
    assert g(3_000_000_000, P, None) == INVALID
    assert g(1000, None, None) == INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIBDIR", str(tmp_path))
    monkeypatch.setattr(_lib, "_libs", {})
    with pytest.raises(RuntimeError, match="missing"):
        _lib.load("moe_router")

"""Parity of the CUDA path with the oracle on small and mid-sized blocks.

Sizes are chosen so the oracle finishes in seconds while the GPU kernels
still run several tiles and ragged tails.  Every call goes through the C-ABI
libraries.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from parity import compare_routing, oracle_act, oracle_route, oracle_shape, oracle_y, y_close
from sparse_moe_layer_sum_b200 import moe
from sparse_moe_layer_sum_b200.moe import BlockShape
from sparse_moe_layer_sum_b200.inputs import (WORKLOADS, Workload, custom, make_block,
                                              random_topk_indices, to_host_f32)

pytestmark = pytest.mark.gpu

TINY_BF16 = custom("tiny_bf16", 300, dim=256, n_routed=16, n_groups=4, topk_groups=2, topk=4,
                   inter=128, seed=11)
MID = custom("mid_bf16", 777, dim=1024, n_routed=64, n_groups=8, topk_groups=4, topk=8,
             inter=256, seed=12)
MID_F32 = custom("mid_f32", 129, x_dtype=torch.float32, w_format="f32", dim=384, n_routed=32,
                 n_groups=4, topk_groups=2, topk=6, inter=160, seed=13)
SOFTMAX_NOBIAS = custom("softmax_nobias", 200, dim=512, n_routed=64, n_groups=8, topk_groups=3,
                        topk=6, inter=128, seed=14, score_func="softmax", has_bias=False,
                        route_scale=1.0)
NOBIAS_SIGMOID = custom("nobias_sigmoid", 160, dim=256, n_routed=32, n_groups=4, topk_groups=2,
                        topk=4, inter=128, seed=15, has_bias=False)
ONE_GROUP = custom("one_group", 90, dim=256, n_routed=16, n_groups=1, topk_groups=1, topk=3,
                   inter=128, seed=16)
DECODE_SMALL = custom("decode_small", 40, dim=1024, n_routed=64, n_groups=8, topk_groups=4,
                      topk=8, inter=256, seed=18)
ONE_TOKEN = custom("one_token", 1, dim=256, n_routed=16, n_groups=4, topk_groups=2, topk=4,
                   inter=128, seed=19)
ROUTER_TC = custom("router_tc", 200, dim=512, n_routed=128, n_groups=8, topk_groups=4, topk=8,
                   inter=128, seed=20)
ROUTER_TC_SPLIT = custom("router_tc_split", 40, dim=2048, n_routed=256, n_groups=8,
                         topk_groups=4, topk=8, inter=128, seed=21)
# dim % 256 != 0: the prefill path falls back to one SM per tile
CG1_PREFILL = custom("cg1_prefill", 230, dim=384, n_routed=16, n_groups=4, topk_groups=2, topk=4,
                     inter=128, seed=22)
# more than 256 experts: the selection's general form (scores in shared
# memory), and 384 experts in groups of 48
ROUTER_E512 = custom("router_e512", 120, dim=512, n_routed=512, n_groups=8, topk_groups=4,
                     topk=8, inter=128, seed=29)
ROUTER_E384 = custom("router_e384", 90, dim=256, n_routed=384, n_groups=8, topk_groups=3,
                     topk=6, inter=128, seed=30, score_func="softmax", has_bias=False,
                     route_scale=1.0)
# dim % 512 == 256: the second matmul's SM pairs keep one weight tile per SM
PAIR_AT1 = custom("pair_at1", 300, dim=768, n_routed=32, n_groups=4, topk_groups=2, topk=8,
                  inter=256, seed=27)
FP8_SMALL = custom("fp8_small", 260, w_format="e4m3", dim=512, n_routed=16, n_groups=4,
                   topk_groups=2, topk=4, inter=256, seed=17)
FP8_DECODE = custom("fp8_decode", 40, w_format="e4m3", dim=1024, n_routed=64, n_groups=8,
                    topk_groups=4, topk=8, inter=256, seed=23)
# skewed routing on the SM-pair path: 8 hot experts get two thirds of the
# 12,000 assignments, so they run as up to six token tiles each (every weight
# tile streamed once per token tile)
MID_SKEW = Workload("mid_skew", BlockShape(dim=1024, n_routed=64, n_groups=8, topk_groups=4,
                                           topk=8, inter=256), 1500, torch.bfloat16, "bf16", 25,
                    hot_experts=8, hot_bias=0.5)
FP8_SKEW = Workload("fp8_skew", BlockShape(dim=1024, n_routed=64, n_groups=8, topk_groups=4,
                                           topk=8, inter=256), 1500, torch.bfloat16, "e4m3", 26,
                    hot_experts=8, hot_bias=0.5)
FP8_CG1 = custom("fp8_cg1", 230, w_format="e4m3", dim=384, n_routed=16, n_groups=4,
                 topk_groups=2, topk=4, inter=128, seed=24)

TOL = {"f32": 1e-4, "bf16": 2e-2, "e4m3": 5e-2}
# mean |error| / rms per expert output, against an oracle that rounds h like
# the kernel (bf16, or fp16 on the e4m3-weight path).  bf16: only rare 1-ulp
# flips of h differ.  e4m3: the tensor-core path also rounds the block scale
# (times 2^8) to fp16 and each dequantised weight q * scale once more to fp16
# (relative errors within +-2^-11, rms 2^-11/sqrt(3) = 2.8e-4 each), in both
# matmuls; the output's relative rms error from these independent roundings
# is about sqrt(4) * 2.8e-4 = 5.6e-4, a mean |error| of about 4.5e-4.  A wrong
# scale block would show errors of tens of percent.
MEAN_TOL = {"f32": 1e-6, "bf16": 2e-4, "e4m3": 1e-3}


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()
    assert torch.cuda.is_available()


def run_block(w, x, params, combine="scatter"):
    blk = moe.MoEBlock(w.shape, params, w.T, x.dtype, combine=combine)
    y = blk.forward(x).clone()
    torch.cuda.synchronize()
    assert blk.device_status() == 0
    return blk, y


@pytest.mark.parametrize("w", [WORKLOADS["tiny_f32"], TINY_BF16, MID, MID_F32, SOFTMAX_NOBIAS,
                               NOBIAS_SIGMOID, ONE_GROUP, ROUTER_TC, ROUTER_TC_SPLIT,
                               ROUTER_E512, ROUTER_E384],
                         ids=lambda w: w.name)
def test_router_matches_oracle(w):
    x, p = make_block(w)
    weights, indices, gap = moe.router_forward(w.shape, x, p.w_r, p.bias, gap=True)
    torch.cuda.synchronize()
    r = oracle_route(w, x, p)
    rep = compare_routing(r, weights.cpu().numpy(), indices.cpu().numpy().astype(np.int64),
                          w.shape.n_routed // w.shape.n_groups, w_rtol=2e-6)
    assert rep.set_flips <= max(1, w.T // 1000)
    # the GPU's own gap report agrees with the oracle's where decisions are clear
    g = gap.cpu().numpy()
    clear = np.minimum(r.gap_set, r.gap_order) > 1e-5
    assert np.allclose(g[clear], np.minimum(r.gap_set, r.gap_order)[clear], rtol=1e-2, atol=1e-5)


@pytest.mark.parametrize("w", [ROUTER_TC, ROUTER_TC_SPLIT, TINY_BF16, MID_F32],
                         ids=lambda w: w.name)
def test_router_prepared_split_gives_identical_results(w):
    """The weight split prepared once gives the same bits as the split each
    forward writes for itself; shapes off the tensor-core path ignore it."""
    x, p = make_block(w)
    prep = moe.router_prepare(w.shape, p.w_r)
    if prep is None:   # dim or experts off the tensor-core tiling
        assert w.shape.n_routed % 128 != 0 or w.shape.dim % 64 != 0
        prep = torch.zeros(16, dtype=torch.uint8, device="cuda")
    a = moe.router_forward(w.shape, x, p.w_r, p.bias, gap=True)
    b = moe.router_forward(w.shape, x, p.w_r, p.bias, gap=True, prep=prep)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (63, 16, 4), (64, 64, 8), (65, 256, 8),
                                   (1000, 256, 8), (16384, 256, 8), (300, 1024, 16)])
def test_dispatch_bit_exact(T, E, k):
    shape = moe.BlockShape(dim=128, n_routed=E, n_groups=1, topk_groups=1, topk=k, inter=128)
    idx = random_topk_indices(T, E, k, seed=T + E)
    counts, offsets, st, so = moe.dispatch_build(shape, idx.cuda())
    d = O.dispatch(idx.numpy().astype(np.int64), E)
    assert np.array_equal(counts.cpu().numpy(), d.counts)
    assert np.array_equal(offsets.cpu().numpy(), d.offsets)
    assert np.array_equal(st.cpu().numpy(), d.sorted_token)
    assert np.array_equal(so.cpu().numpy(), d.slot_of)


def test_dispatch_skewed_and_empty():
    shape = moe.BlockShape(dim=128, n_routed=256, n_groups=1, topk_groups=1, topk=8, inter=128)
    T = 5000
    idx = np.tile(np.arange(8, dtype=np.int32), (T, 1))   # 248 experts get no token
    idx[::7] = np.arange(100, 108)
    counts, offsets, st, so = moe.dispatch_build(shape, torch.from_numpy(idx).cuda())
    d = O.dispatch(idx.astype(np.int64), 256)
    assert np.array_equal(counts.cpu().numpy(), d.counts)
    assert np.array_equal(st.cpu().numpy(), d.sorted_token)
    assert np.array_equal(so.cpu().numpy(), d.slot_of)
    # empty batch: counts and offsets are all zero
    c0, o0, _, _ = moe.dispatch_build(shape, torch.zeros(0, 8, dtype=torch.int32, device="cuda"))
    assert int(c0.abs().sum()) == 0 and int(o0.abs().sum()) == 0


def test_dispatch_reports_out_of_range():
    shape = moe.BlockShape(dim=128, n_routed=16, n_groups=1, topk_groups=1, topk=2, inter=128)
    idx = torch.tensor([[0, 1], [2, 16]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.dispatch_build(shape, idx, status=status)
    assert int(status.item()) == -6  # MOE_ERR_RANGE


@pytest.mark.parametrize("w", [WORKLOADS["tiny_f32"], TINY_BF16, MID, MID_F32, DECODE_SMALL,
                               ONE_TOKEN, CG1_PREFILL, PAIR_AT1, FP8_SMALL, FP8_DECODE, FP8_CG1],
                         ids=lambda w: w.name)
def test_experts_rows_match_oracle(w):
    """Expert outputs row by row, on a seeded index set (routing held fixed)."""
    x, p = make_block(w)
    sh = w.shape
    idx = random_topk_indices(w.T, sh.n_routed, sh.topk, seed=w.seed)
    _, offsets, sorted_token, slot_of = moe.dispatch_build(sh, idx.cuda())
    ws = moe.expert_weights_struct(p.w1, p.w3, p.w2, p.s1, p.s3, p.s2)
    out_perm, out_shared = moe.experts_forward(sh, x, ws, offsets, sorted_token)
    torch.cuda.synchronize()
    d = O.dispatch(idx.numpy().astype(np.int64), sh.n_routed)
    xs = to_host_f32(x)
    act = oracle_act(w)
    from parity import _expert_getter
    get = _expert_getter(p, w.w_format)
    op = out_perm.cpu().numpy()
    worst, mean_sum, n = 0.0, 0.0, 0
    for e in range(sh.n_routed + 1):
        if e < sh.n_routed:
            rows = np.arange(d.offsets[e], d.offsets[e + 1])
            if rows.size == 0:
                continue
            ref = O.expert_ffn(xs[d.sorted_token[rows]], *get(e), act)
            got = op[rows]
        else:
            ref = O.expert_ffn(xs, *get(e), act)
            got = out_shared.cpu().numpy()
        rms = np.sqrt(np.mean(ref ** 2))
        worst = max(worst, float(np.max(np.abs(got - ref)) / rms))
        mean_sum += float(np.mean(np.abs(got - ref)) / rms)
        n += 1
    # the max is dominated by 1-ulp bf16 flips of rare large elements of the
    # heavy-tailed h = silu(a) * u (both sides round h); a systematic error
    # would show in the mean, which stays orders of magnitude lower
    print(f"{w.name}: max |d| {worst:.2e} rms, mean |d| {mean_sum / n:.2e} rms")
    assert worst <= TOL[w.w_format], worst
    assert mean_sum / n <= MEAN_TOL[w.w_format], mean_sum / n


@pytest.mark.parametrize("combine", ["scatter", "ordered"])
@pytest.mark.parametrize("w", [WORKLOADS["tiny_f32"], TINY_BF16, MID, MID_F32, SOFTMAX_NOBIAS,
                               ONE_GROUP, DECODE_SMALL, ONE_TOKEN, CG1_PREFILL, PAIR_AT1,
                               FP8_SMALL, FP8_DECODE, FP8_CG1, MID_SKEW, FP8_SKEW],
                         ids=lambda w: w.name)
def test_block_matches_oracle(w, combine):
    x, p = make_block(w)
    blk, y = run_block(w, x, p, combine)
    r = oracle_route(w, x, p)
    rep = compare_routing(r, blk.weights.cpu().numpy(),
                          blk.indices.cpu().numpy().astype(np.int64),
                          w.shape.n_routed // w.shape.n_groups, w_rtol=2e-6)
    tokens = np.nonzero(rep.same_set)[0]
    y_orc = oracle_y(w, x, p, r, tokens=tokens)
    y_close(y.cpu().numpy()[tokens], y_orc, TOL[w.w_format])
    if w.hot_experts:  # the skew did what it is for
        c = blk.counts.cpu().numpy()
        assert c.max() > 2 * 256
    # counts agree with the oracle's bincount unless a near-tie flipped
    if rep.set_flips == 0:
        d = O.dispatch(r.indices, w.shape.n_routed)
        assert np.array_equal(blk.counts.cpu().numpy(), d.counts)


def test_ordered_combine_is_bit_reproducible():
    x, p = make_block(MID)
    blk = moe.MoEBlock(MID.shape, p, MID.T, x.dtype, combine="ordered")
    y1 = blk.forward(x).clone()
    y2 = blk.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_scatter_and_ordered_combine_agree():
    x, p = make_block(MID)
    ys = moe.MoEBlock(MID.shape, p, MID.T, x.dtype, combine="scatter").forward(x).clone()
    yo = moe.MoEBlock(MID.shape, p, MID.T, x.dtype, combine="ordered").forward(x).clone()
    torch.cuda.synchronize()
    rms = yo.pow(2).mean().sqrt()
    # same fp32 terms, summed in different orders
    assert float((ys - yo).abs().max() / rms) < 1e-5


def test_zero_input_gives_zero_output_and_uniform_gates():
    x, p = make_block(TINY_BF16)
    x = torch.zeros_like(x)
    blk, y = run_block(TINY_BF16, x, p)
    assert torch.all(y == 0)
    assert torch.all(blk.weights == 2.5 / 4)


@pytest.mark.parametrize("combine", ["scatter", "ordered"])
def test_graph_capture_replays(combine):
    w = TINY_BF16
    x, p = make_block(w)
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype, combine=combine)
    ref = blk.forward(x).clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        blk.forward(x)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        blk.forward(x)
    blk.y.zero_()
    g.replay()
    torch.cuda.synchronize()
    if combine == "ordered":
        assert torch.equal(blk.y, ref)
    else:  # fp32 reductions in a run-dependent order
        assert float((blk.y - ref).abs().max() / ref.pow(2).mean().sqrt()) < 1e-5


def test_host_pipeline_matches_forward():
    """Overlapped host-to-host forwards give each batch its own forward's y
    (ordered combine: bit-identical), across several reuses of the two
    device buffers."""
    w = MID
    x, p = make_block(w)
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype, combine="ordered")
    g = torch.Generator(device="cuda").manual_seed(77)
    xs = [x] + [torch.randn(w.T, w.shape.dim, generator=g, device="cuda").to(x.dtype)
                for _ in range(4)]
    refs = [blk.forward(xx).cpu() for xx in xs]
    pipe = blk.host_pipeline()
    xh = [xx.cpu().pin_memory() for xx in xs]
    yh = [torch.full((w.T, w.shape.dim), float("nan")).pin_memory() for _ in xs]
    for a, b in zip(xh, yh):
        pipe.submit(a, b)
    pipe.finish()
    torch.cuda.synchronize()
    for r, b in zip(refs, yh):
        assert torch.equal(r, b)
    assert blk.device_status() == 0


def test_bounded_wait_reports_timeout_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.selftest_wait(20_000_000, status)     # 20 ms, nothing ever arrives
    torch.cuda.synchronize()
    assert int(status.item()) == -5           # MOE_ERR_TIMEOUT
    # the context is still usable
    x, p = make_block(TINY_BF16)
    run_block(TINY_BF16, x, p)

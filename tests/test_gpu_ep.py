"""Expert-parallel shards on one GPU: each rank's kernels run on the rank's
own weight shard (its routed experts, then the shared expert) and write a
partial y; the shards are run one after another (no rank waits on another)
and their sum must be the unsharded block's output, and the oracle's."""
import numpy as np
import pytest
import torch

from parity import compare_routing, oracle_route, oracle_y, y_close
from sparse_moe_layer_sum_b200 import moe
from sparse_moe_layer_sum_b200.inputs import custom, make_block

pytestmark = pytest.mark.gpu

MID = custom("ep_mid", 777, dim=1024, n_routed=64, n_groups=8, topk_groups=4, topk=8,
             inter=256, seed=41)
MID_F8 = custom("ep_mid_f8", 500, w_format="e4m3", dim=1024, n_routed=64, n_groups=8,
                topk_groups=4, topk=8, inter=256, seed=42)
DECODE = custom("ep_decode", 24, dim=1024, n_routed=64, n_groups=8, topk_groups=4, topk=8,
                inter=256, seed=43)


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("w,fp8", [(MID, False), (MID_F8, False), (MID_F8, True), (DECODE, False)],
                         ids=["bf16", "e4m3", "e4m3_fp8act", "decode"])
def test_shards_sum_to_the_block(w, fp8, world):
    x, p = make_block(w)
    full = moe.MoEBlock(w.shape, p, w.T, x.dtype, fp8_act=fp8)
    y_full = full.forward(x).clone()
    y_sum = torch.zeros_like(y_full)
    for r in range(world):
        blk = moe.MoEBlock(w.shape, moe.shard_params(w.shape, p, r, world), w.T, x.dtype,
                           fp8_act=fp8, ep=(r, world))
        y_sum += blk.forward(x)
        torch.cuda.synchronize()
        assert blk.device_status() == 0
        # every rank routes the whole batch identically
        assert torch.equal(blk.indices, full.indices)
    torch.cuda.synchronize()
    rms = y_full.pow(2).mean().sqrt()
    # a shard cuts the shared expert's tokens into other token tiles, whose
    # k-loops start at other k-blocks: h's fp32 sums come out in another
    # order and now and then round to the neighbouring bf16 (or fp16, or
    # e4m3) value.  One such flip moves y[t, d] by 2^-8 |h_i w2[d, i]| (2^-3
    # with e4m3 activations), against rms(y) ~ sqrt(inter) rms(h w2): with
    # h's heavy tail (|h_i| up to ~10 rms) and inter 256 that reaches ~1e-2
    # (measured 3e-4 to 4e-3).  The bound is the path's tolerance; a
    # misplaced expert or token slice would move y by about rms itself.
    assert float((y_sum - y_full).abs().max() / rms) < (5e-2 if fp8 else 2e-2)
    r = oracle_route(w, x, p)
    rep = compare_routing(r, full.weights.cpu().numpy(), full.indices.cpu().numpy().astype(np.int64),
                          w.shape.n_routed // w.shape.n_groups, w_rtol=2e-6)
    tokens = np.nonzero(rep.same_set)[0][:64]
    y_orc = oracle_y(w, x, p, r, tokens=tokens, fp8_act=fp8)
    y_close(y_sum.cpu().numpy()[tokens], y_orc, 5e-2 if w.w_format == "e4m3" else 2e-2)


def test_plan_partitions_experts_and_tokens():
    sh = MID.shape
    plans = [moe.ep_plan(sh, 1001, r, 8) for r in range(8)]
    assert [p[0] for p in plans] == list(range(0, 64, 8))
    assert all(p[1] - p[0] == 8 for p in plans)
    assert plans[0][2] == 0 and plans[-1][3] == 1001
    assert all(plans[i][3] == plans[i + 1][2] for i in range(7))
    with pytest.raises(RuntimeError):
        moe.ep_plan(sh, 10, 0, 3)          # 3 does not divide 64 experts

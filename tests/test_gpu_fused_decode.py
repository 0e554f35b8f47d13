"""The whole block in one launch at decode (moe_block_forward_decode)
against the separate launches and against the oracle.

Both paths run the same expert kernels' code on the same tile tables; the
router scores differ only in how the fp32 sums are formed (FMA tiles here,
the exact three-term tensor-core split there), so the routing agrees on
every token without a near-tie, and the grouping matches moe_dispatch_build
bit for bit on the fused launch's own indices.
"""
import numpy as np
import pytest
import torch

from parity import compare_routing, oracle_route, oracle_y, y_close
from sparse_moe_layer_sum_b200 import moe
from sparse_moe_layer_sum_b200.inputs import WORKLOADS, custom, make_block

pytestmark = pytest.mark.gpu

SMALL = custom("fused_small", 40, dim=1024, n_routed=64, n_groups=8, topk_groups=4, topk=8,
               inter=256, seed=51)
TINY = custom("fused_tiny", 9, dim=256, n_routed=16, n_groups=4, topk_groups=2, topk=4,
              inter=128, seed=52)
ONE = custom("fused_one", 1, dim=512, n_routed=64, n_groups=8, topk_groups=4, topk=6,
             inter=256, seed=53)
NOBIAS = custom("fused_softmax", 24, dim=512, n_routed=64, n_groups=8, topk_groups=3, topk=6,
                inter=128, seed=54, score_func="softmax", has_bias=False, route_scale=1.0)


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()


@pytest.mark.parametrize("w", [SMALL, TINY, ONE, NOBIAS, WORKLOADS["v3_decode_t64"]],
                         ids=lambda w: w.name)
def test_fused_decode_matches_separate_launches_and_oracle(w):
    x, p = make_block(w)
    ref = moe.MoEBlock(w.shape, p, w.T, x.dtype)
    y_ref = ref.forward(x).clone()
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype, fused_decode=True)
    y = blk.forward(x).clone()
    y2 = blk.forward(x).clone()       # a second launch on the same buffers
    torch.cuda.synchronize()
    assert blk.device_status() == 0 and ref.device_status() == 0
    r = oracle_route(w, x, p)
    rep = compare_routing(r, blk.weights.cpu().numpy(), blk.indices.cpu().numpy().astype(np.int64),
                          w.shape.n_routed // w.shape.n_groups,
                          w_rtol=1e-5 if w.shape.dim > 2048 else 2e-6)
    # the grouping equals moe_dispatch_build's on the fused launch's indices
    counts, offsets, st, so = moe.dispatch_build(w.shape, blk.indices)
    torch.cuda.synchronize()
    assert torch.equal(counts, blk.counts) and torch.equal(offsets, blk.offsets)
    assert torch.equal(st, blk.sorted_token) and torch.equal(so, blk.slot_of)
    # the same block output as the separate launches (fp32 sums in another
    # order, gates from scores summed another way)
    same = np.nonzero(rep.same_set)[0]
    rms = float(y_ref.pow(2).mean().sqrt())
    d = (y - y_ref).abs()[torch.from_numpy(same).cuda()].max()
    assert float(d) / rms < 1e-4
    assert float((y2 - y).abs().max()) / rms < 1e-5
    tokens = same[:64]
    y_close(y.cpu().numpy()[tokens], oracle_y(w, x, p, r, tokens=tokens), 2e-2)


def test_fused_decode_graph_capture_replays():
    w = SMALL
    x, p = make_block(w)
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype, fused_decode=True)
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
    assert float((blk.y - ref).abs().max() / ref.pow(2).mean().sqrt()) < 1e-5
    assert blk.device_status() == 0


def test_fused_decode_rejects_prefill_batches():
    w = custom("fused_big", 512, dim=1024, n_routed=64, n_groups=8, topk_groups=4, topk=8,
               inter=256, seed=55)
    x, p = make_block(w)
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype, fused_decode=True)
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        blk.forward(x)

"""Parity at the full DeepSeek-V3 block sizes, in the launch configuration the
benchmark times (MoEBlock.forward on the current stream).

Routing is checked on every token (indices bit-exact away from near-ties,
per-expert counts); the block output on a seeded sample of tokens, which the
oracle computes one by one.
"""
import gc

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from parity import compare_routing, oracle_route, oracle_y, y_close
from sparse_moe_layer_sum_b200 import moe
from sparse_moe_layer_sum_b200.inputs import WORKLOADS, make_block, sample_tokens

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "e4m3": 5e-2}
CASES = [("v3_decode_t64", 64), ("v3_prefill_t4096", 12), ("v3_skew_t16384", 12),
         ("v3_fp8_t8192", 6)]


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()


@pytest.mark.parametrize("name,n_sample", CASES, ids=[c[0] for c in CASES])
def test_v3_block(name, n_sample):
    w = WORKLOADS[name]
    x, p = make_block(w)
    blk = moe.MoEBlock(w.shape, p, w.T, x.dtype)
    y = blk.forward(x)
    torch.cuda.synchronize()
    assert blk.device_status() == 0
    r = oracle_route(w, x, p)
    rep = compare_routing(r, blk.weights.cpu().numpy(), blk.indices.cpu().numpy().astype(np.int64),
                          w.shape.n_routed // w.shape.n_groups, w_rtol=1e-5)
    counts = blk.counts.cpu().numpy()
    assert counts.sum() == w.T * w.shape.topk
    if rep.set_flips == 0:
        assert np.array_equal(counts, O.dispatch(r.indices, w.shape.n_routed).counts)
    # offsets are the exclusive scan of the counts
    assert np.array_equal(blk.offsets.cpu().numpy()[1:], np.cumsum(counts))
    tokens = sample_tokens(w.T, n_sample).numpy()
    tokens = tokens[rep.same_set[tokens]]
    y_orc = oracle_y(w, x, p, r, tokens=tokens)
    err = y_close(y[torch.from_numpy(tokens).cuda()].cpu().numpy(), y_orc, TOL[w.w_format])
    print(f"{name}: near-ties {rep.flagged} set flips {rep.set_flips} order flips "
          f"{rep.order_flips} max gate rel err {rep.max_w_rel:.2e} y err {err:.2e} rms "
          f"touched {(counts > 0).sum()} zero-count {(counts == 0).sum()}")
    if w.hot_experts:
        hot = torch.randperm(256, generator=torch.Generator().manual_seed(2024))[:16].numpy()
        print(f"{name}: hot-expert share {counts[hot].sum() / counts.sum():.3f}")
    del blk, y, x, p
    gc.collect()
    torch.cuda.empty_cache()

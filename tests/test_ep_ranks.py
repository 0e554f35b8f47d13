"""Expert parallelism on CPU: two gloo ranks each take the share moe_ep_plan
(the library's own plan, a host-only call) gives them -- their routed
experts and their slice of the shared expert's tokens -- and compute it
with the oracle; the all-reduce of the partial outputs must be the whole
block's output.  This covers the multi-rank path's partition and reduction
without a GPU; the kernels' shard handling is covered by the GPU tests."""
import math
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _block(seed=5, T=37):
    from oracle.moe_oracle import MoEShape, router
    rng = np.random.default_rng(seed)
    D, E, I = 32, 16, 16
    shape = MoEShape(dim=D, n_routed_experts=E, n_expert_groups=4, n_limited_groups=2,
                     n_activated_experts=4, moe_inter_dim=I)
    x = rng.standard_normal((T, D)).astype(np.float32)
    w_r = (rng.standard_normal((E, D)) / math.sqrt(D)).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    mats = [tuple((rng.standard_normal(s) / math.sqrt(s[1])).astype(np.float32)
                  for s in ((I, D), (I, D), (D, I))) for _ in range(E + 1)]
    return shape, x, router(x, w_r, b, shape), mats


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle.moe_oracle import expert_ffn
        from sparse_moe_layer_sum_b200.moe import BlockShape, ep_plan
        shape, x, r, mats = _block()
        T, E = x.shape[0], shape.n_routed_experts
        bs = BlockShape(dim=32, n_routed=E, n_groups=4, topk_groups=2, topk=4, inter=16)
        e0, e1, t0, t1 = ep_plan(bs, T, rank, world)
        # this rank's partial output: its experts' weighted rows, its slice
        # of the shared expert
        y = np.zeros_like(x, dtype=np.float64)
        for t in range(T):
            for j in range(4):
                e = int(r.indices[t, j])
                if e0 <= e < e1:
                    y[t] += r.weights[t, j] * expert_ffn(x[t:t + 1], *mats[e], "f32")[0]
        y[t0:t1] += expert_ffn(x[t0:t1], *mats[E], "f32")
        yt = torch.from_numpy(y)
        dist.all_reduce(yt)
        out[rank] = (yt.numpy(), (e0, e1, t0, t1))
    finally:
        dist.destroy_process_group()


def test_two_ranks_sum_to_the_block_output():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    from oracle.moe_oracle import moe_forward
    shape, x, r, mats = _block()
    full = moe_forward(x, r, lambda e: mats[e], lambda: mats[16], 16, "f32")
    for rank in range(world):
        assert np.allclose(out[rank][0], full, rtol=1e-12, atol=1e-12)
    # the plans partition the experts and the tokens
    plans = sorted(out[k][1] for k in range(world))
    assert plans[0][0] == 0 and plans[-1][1] == 16 and plans[0][1] == plans[1][0]
    assert plans[0][2] == 0 and plans[-1][3] == x.shape[0] and plans[0][3] == plans[1][2]

"""moe_dispatch_build_noalloc against moe_dispatch_build.

The no-allocation entry point serves callers that hold only their input and
output buffers and cannot obtain device memory for a workspace (a host
framework that passes tensors but no allocator, or a process whose device
memory is owned entirely by another allocator).  It keeps its scratch in a
fixed array inside the library instead.  This file is collected last so that
a run stopping at the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

from sparse_moe_layer_sum_b200 import _lib
from sparse_moe_layer_sum_b200.inputs import random_topk_indices
from sparse_moe_layer_sum_b200.moe import BlockShape

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_moe_layer_sum_b200 import build
    build.build_all()


def _outputs(T, E, k, dev):
    i32 = torch.int32
    return (torch.full((E,), -7, dtype=i32, device=dev), torch.full((E + 1,), -7, dtype=i32, device=dev),
            torch.full((T * k,), -7, dtype=i32, device=dev), torch.full((T * k,), -7, dtype=i32, device=dev))


def _with_workspace(cfg, idx, T, E, k):
    counts, offsets, st, so = _outputs(T, E, k, idx.device)
    need = _lib.fn("moe_dispatch", "moe_dispatch_workspace_size")(ctypes.byref(cfg), T)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=idx.device)
    rc = _lib.fn("moe_dispatch", "moe_dispatch_build")(
        ctypes.byref(cfg), T, idx.data_ptr(), counts.data_ptr(), offsets.data_ptr(),
        st.data_ptr(), so.data_ptr(), ws.data_ptr(), ws.numel(), None,
        torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return counts, offsets, st, so


def _no_alloc(cfg, idx, T, E, k, status):
    counts, offsets, st, so = _outputs(T, E, k, idx.device)
    rc = _lib.fn("moe_dispatch", "moe_dispatch_build_noalloc")(
        ctypes.byref(cfg), T, idx.data_ptr(), counts.data_ptr(), offsets.data_ptr(),
        st.data_ptr(), so.data_ptr(), status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return counts, offsets, st, so


def test_no_alloc_dispatch_matches_workspace_dispatch_twice():
    E, k = 256, 8
    cfg = BlockShape(dim=7168, n_routed=E, n_groups=8, topk_groups=4, topk=k, inter=2048).cfg()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # two calls in a row on different batches: the shared scratch keeps the
    # first call's contents and must not leak into the second
    for T, seed in ((4096, 1), (1000, 2)):
        idx = random_topk_indices(T, E, k, seed=seed, device="cuda")
        ref = _with_workspace(cfg, idx, T, E, k)
        got = _no_alloc(cfg, idx, T, E, k, status)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):  # integer outputs: identical
            assert torch.equal(a, b)
        assert int(status.item()) == 0
    # an empty batch, and a batch whose histograms fill the scratch array
    # exactly (ceil(T / 64) * E = 262144 ints)
    for T, seed in ((0, 3), (64 * (262144 // E), 4)):
        idx = random_topk_indices(T, E, k, seed=seed, device="cuda")
        ref = _with_workspace(cfg, idx, T, E, k)
        got = _no_alloc(cfg, idx, T, E, k, status)
        torch.cuda.synchronize()
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
        assert int(status.item()) == 0
    # beyond the fixed scratch size: a clear error and nothing launched
    big = 64 * (262144 // E + 1)
    rc = _lib.fn("moe_dispatch", "moe_dispatch_build_noalloc")(
        ctypes.byref(cfg), big, None, None, None, None, None, None, None)
    assert rc == -3  # MOE_ERR_WORKSPACE

"""Oracle pins for the token grouping (histogram, scan, stable scatter).

The moe-forward excerpt of "DeepSeek-V3.2-Exp · Mixture of experts" counts
tokens per expert with a bincount and groups them with ``torch.where`` in
row-major order.  The oracle's vectorised version is checked against that
definition written as plain loops on small inputs.
"""
import numpy as np
import pytest

from oracle.moe_oracle import dispatch


def _definition(indices, E):
    T, k = indices.shape
    counts = [0] * E
    for t in range(T):
        for j in range(k):
            counts[indices[t, j]] += 1
    rows = []          # expert-major, ascending token within an expert
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if indices[t, j] == e:
                    rows.append((t, j))
    return counts, rows


def _random_topk(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)


@pytest.mark.parametrize("T,E,k,seed", [(1, 4, 2, 0), (37, 16, 4, 1), (200, 64, 8, 2), (5, 256, 8, 3)])
def test_dispatch_matches_definition(T, E, k, seed):
    idx = _random_topk(T, E, k, seed)
    d = dispatch(idx, E)
    counts, rows = _definition(idx, E)
    assert d.counts.tolist() == counts
    assert d.offsets[0] == 0 and d.offsets[-1] == T * k
    assert np.all(np.diff(d.offsets) == d.counts)
    assert d.sorted_token.tolist() == [t for t, _ in rows]
    for pos, (t, j) in enumerate(rows):
        assert d.slot_of[t * k + j] == pos


def test_skewed_and_empty_experts():
    # every token picks experts 0..3: the other experts are empty
    idx = np.tile(np.arange(4), (50, 1))
    d = dispatch(idx, 16)
    assert d.counts.tolist() == [50] * 4 + [0] * 12
    assert d.offsets.tolist() == [0, 50, 100, 150] + [200] * 13
    assert d.sorted_token.tolist() == list(range(50)) * 4


def test_empty_batch():
    d = dispatch(np.zeros((0, 8), dtype=np.int64), 256)
    assert d.counts.sum() == 0 and d.offsets.tolist() == [0] * 257
    assert d.sorted_token.size == 0 and d.slot_of.size == 0

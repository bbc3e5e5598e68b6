"""Pins for the oracle's permutation into expert-contiguous order (CPU only).

"MindIE-SD Fused MoE", execution flow: dispatch reorders tokens by expert and counts the
tokens of each expert; combine restores token order.  Pins: a stable library sort, the
exclusive-scan identity and the inverse-permutation identity.
"""
import numpy as np
import pytest

import oracle


@pytest.mark.parametrize("T,K,E,seed", [(1, 1, 1, 0), (16, 2, 8, 1), (37, 3, 6, 2),
                                        (500, 8, 256, 3), (64, 8, 128, 4)])
def test_permutation_invariants(T, K, E, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, row_src, row_of = oracle.permute(idx, E)
    A = T * K
    assert counts.sum() == A
    assert np.array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    # stable sort by expert of the routed rows a = t*K + j (numpy, an independent routine)
    ref = np.argsort(idx.ravel(), kind="stable").astype(np.int32)
    assert np.array_equal(row_src, ref)
    assert np.array_equal(row_of.ravel()[row_src], np.arange(A))
    for e in range(E):
        rows = row_src[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[rows] == e)
        assert np.all(np.diff(rows // K) > 0)      # ascending token inside an expert


def test_empty_experts_have_empty_ranges():
    idx = np.array([[3, 1], [3, 1], [1, 3]], np.int32)
    counts, offsets, row_src, _ = oracle.permute(idx, 6)
    assert list(counts) == [0, 3, 0, 3, 0, 0]
    assert list(offsets) == [0, 0, 3, 3, 6, 6, 6]
    assert list(row_src) == [1, 3, 4, 0, 2, 5]

"""tv_tree_shape (host code in the library) against the oracle's budget DP:
the same tree, numbering and value, bit for bit; argument checks."""
import numpy as np
import pytest

import oracle
import tree_speculative_decoding_07_b200 as tv


@pytest.mark.parametrize("accept,budget,depth", [
    ([0.6, 0.25, 0.1], 7, 6), ([0.55, 0.2, 0.1, 0.05], 64, 6), ([0.7], 6, 0), ([0.8, 0.1], 40, 0),
    ([0.3, 0.3, 0.3], 30, 4), ([0.9, 0.05, 0.02], 128, 0), ([0.0, 0.0], 5, 0), ([1.0, 1.0], 9, 3),
])
def test_library_dp_equals_oracle(accept, budget, depth):
    p, r, v = tv.tree_shape(accept, budget, depth)
    po, ro, vo = oracle.tree_shape_dp(accept, budget, depth or None)
    np.testing.assert_array_equal(p, po)
    np.testing.assert_array_equal(r, ro)
    assert v == vo


def test_tree_shape_rejects_bad_arguments():
    parent = np.zeros(8, np.int32)
    rank = np.zeros(8, np.int32)
    n = np.zeros(1, np.int32)
    val = np.zeros(1)
    acc = np.array([0.5, 0.2])
    assert tv.tv_tree_shape(acc, 2, 0, 0, parent, rank, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_shape(acc, 2, 8, -1, parent, rank, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_shape(np.array([0.5, 1.5]), 2, 8, 0, parent, rank, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_shape(np.array([0.5, np.nan]), 2, 8, 0, parent, rank, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_shape(acc, 2, 8, 0, None, rank, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_shape(acc, 2, 257, 0, parent, rank, n, val) == tv.TV_ERR_UNSUPPORTED
    assert tv.tv_tree_shape(np.full(33, 0.01), 33, 8, 0, parent, rank, n, val) == tv.TV_ERR_UNSUPPORTED
    assert tv.tv_tree_shape(acc, 2, 8, 0, parent, rank, n, val) == tv.TV_OK and 1 <= n[0] <= 8
    assert parent[0] == -1 and (parent[n[0]:] == -1).all()

"""Pins for the oracle's tree mask (glossary page, "Tree attention";
blog section 3, "Tree Attention Verification Matrix")."""
import numpy as np
import pytest

import oracle
from helpers import golden_lines


def test_mask_matches_page_matrix():
    lines = list(golden_lines("tree_mask_5node.txt"))
    parent = [int(x) for x in lines[0][1:]]
    expected = np.array([[int(x) for x in row[1:]] for row in lines[1:]], dtype=np.uint8)
    assert [row[0] for row in lines[1:]] == ["T0", "A1", "A2", "B1", "B2"]
    np.testing.assert_array_equal(oracle.tree_mask(parent), expected)


def test_chain_mask_is_causal():
    n = 9
    m = oracle.tree_mask([-1] + list(range(n - 1)))
    np.testing.assert_array_equal(m, np.tril(np.ones((n, n), dtype=np.uint8)))


def test_star_mask():
    n = 7
    m = oracle.tree_mask([-1] + [0] * (n - 1))
    expected = np.eye(n, dtype=np.uint8)
    expected[:, 0] = 1
    np.testing.assert_array_equal(m, expected)


def test_mask_is_reflexive_transitive_and_counts_depth():
    rng = np.random.default_rng(0)
    for _ in range(50):
        n = int(rng.integers(1, 40))
        parent = [-1] + [int(rng.integers(0, i)) for i in range(1, n)]
        m = oracle.tree_mask(parent).astype(bool)
        depth = [0] * n
        for i in range(1, n):
            depth[i] = depth[parent[i]] + 1
        assert m.diagonal().all()
        assert (m.sum(1) == np.array(depth) + 1).all()          # own path: depth + 1 nodes
        assert not np.triu(m, 1).any()                           # ancestors precede
        for i in range(1, n):                                    # row i = row parent + {i}
            expect = m[parent[i]].copy()
            expect[i] = True
            assert (m[i] == expect).all()


@pytest.mark.parametrize("parent", [[0], [-1, 1], [-1, 0, 3, 1], [-1, -1]])
def test_invalid_trees_rejected(parent):
    with pytest.raises(ValueError):
        oracle.tree_mask(parent)

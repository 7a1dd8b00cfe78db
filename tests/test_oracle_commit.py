"""Pins for the oracle's KV commit (oracle.c or_commit_path).

After verification the accepted path joins the cached prefix and every other
tree entry is dropped (blog "Speculative decoding x tree attention", section
"KV cache management and prefix sharing"; glossary "Tree-based speculative
decoding", section "KV cache management challenges").  Reading: the root stays
at L, accepted node path[k] moves to L + 1 + k, the new length is L + 1 + len.

The pins: the pages' 5-node tree worked by hand; an already-in-place path moves
nothing; a move whose destination is another move's source; and the property
that ties the commit to tree attention -- every accepted node's tree attention
before the commit equals plain causal attention at its new position after it.
"""
import numpy as np

import oracle


def _cache(nb, hkv, d, seed, dtype=np.float32):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((nb, 16, hkv, d)).astype(dtype), rng.standard_normal((nb, 16, hkv, d)).astype(dtype)


def _rows(cache, bt_row, positions):
    flat = cache.reshape(-1, *cache.shape[2:])
    return np.stack([flat[bt_row[t // 16] * 16 + t % 16] for t in positions])


def test_pages_five_node_tree_accepting_b1_b2():
    # T0 -> A1 -> A2, T0 -> B1 -> B2 (nodes 0..4); the walk accepts B1 then B2
    k, v = _cache(4, 2, 8, 1)
    bt = np.array([[2, 0, 3, 1]], np.int32)  # a permuted block table
    L = 21
    path = np.array([[3, 4, -1, -1, -1]], np.int32)
    k2, v2, npl, st = oracle.commit_path(k, v, bt, [L], path, [2])
    assert st == 0 and npl[0] == L + 3
    # B1 (was at L + 3) now at L + 1, B2 (was at L + 4) now at L + 2
    np.testing.assert_array_equal(_rows(k2, bt[0], [L + 1, L + 2]), _rows(k, bt[0], [L + 3, L + 4]))
    np.testing.assert_array_equal(_rows(v2, bt[0], [L + 1, L + 2]), _rows(v, bt[0], [L + 3, L + 4]))
    # the prefix, the root and everything past the new length are untouched
    keep = [t for t in range(64) if t not in (L + 1, L + 2)]
    np.testing.assert_array_equal(_rows(k2, bt[0], keep), _rows(k, bt[0], keep))
    np.testing.assert_array_equal(_rows(v2, bt[0], keep), _rows(v, bt[0], keep))


def test_path_already_in_place_moves_nothing():
    k, v = _cache(3, 2, 8, 2)
    bt = np.array([[1, 2, 0]], np.int32)
    k2, v2, npl, st = oracle.commit_path(k, v, bt, [7], np.array([[1, 2, 3, -1, -1, -1]], np.int32), [3])
    assert st == 0 and npl[0] == 11
    np.testing.assert_array_equal(k2, k)
    np.testing.assert_array_equal(v2, v)


def test_destination_that_is_another_source():
    # path [2, 5]: node 2 goes to L + 1, node 5 to L + 2, which was node 2's slot
    k, v = _cache(2, 1, 4, 3)
    bt = np.array([[0, 1]], np.int32)
    L = 9
    k2, v2, npl, st = oracle.commit_path(k, v, bt, [L], np.array([[2, 5, -1, -1, -1, -1]], np.int32), [2])
    assert st == 0 and npl[0] == L + 3
    np.testing.assert_array_equal(_rows(k2, bt[0], [L + 1, L + 2]), _rows(k, bt[0], [L + 2, L + 5]))
    np.testing.assert_array_equal(_rows(v2, bt[0], [L + 1, L + 2]), _rows(v, bt[0], [L + 2, L + 5]))


def test_flagged_and_malformed_paths_leave_the_sequence_alone():
    k, v = _cache(2, 1, 4, 4)
    bt = np.array([[0, 1], [1, 0], [0, 1], [1, 0]], np.int32)
    path = np.array([[1, 2, -1, -1],     # flagged by the walk (len -1): no commit
                     [2, 2, -1, -1],     # not strictly increasing
                     [0, 1, -1, -1],     # the root is not a path node
                     [1, 4, -1, -1]], np.int32)  # past the tree
    k2, v2, npl, st = oracle.commit_path(k, v, bt, [5, 5, 5, 5], path, [-1, 2, 2, 2])
    assert st == 3  # the malformed ones report a tree error
    np.testing.assert_array_equal(npl, [5, 5, 5, 5])
    np.testing.assert_array_equal(k2, k)
    np.testing.assert_array_equal(v2, v)
    # a block id out of range inside the tree's span
    k2, v2, npl, st = oracle.commit_path(k, v, np.array([[0, 7]], np.int32), [10], np.array([[1, 2, -1, -1, -1, -1, -1, -1]], np.int32), [2])
    assert st == 4 and npl[0] == 10
    np.testing.assert_array_equal(k2, k)


def _path_to(parent, node):
    out = []
    while node > 0:
        out.append(node)
        node = parent[node]
    return out[::-1]


def test_commit_turns_tree_attention_into_causal_attention():
    """For every accepted node c_k: tree attention of c_k over (prefix, root,
    c_1..c_k) before the commit == causal attention of the same query at
    position L + k over the committed sequence (positions 0 .. L + k)."""
    rng = np.random.default_rng(5)
    B, N, Hq, Hkv, D, L = 1, 12, 4, 2, 16, 37
    parent = np.array([-1, 0, 0, 1, 1, 3, 2, 5, 5, 7, 6, 9], np.int32)
    nb = 8
    k, v = _cache(nb, Hkv, D, 6)
    bt = rng.permutation(nb).astype(np.int32)[None, :]
    q = rng.standard_normal((B, N, Hq, D)).astype(np.float32)
    leaf = 11
    acc = _path_to(parent, leaf)  # root excluded
    assert acc == [1, 3, 5, 7, 9, 11]
    before = oracle.tree_attention(q, k, v, bt, np.array([L], np.int32), parent[None, :], Hkv, "f32")
    path = np.full((1, N), -1, np.int32)
    path[0, :len(acc)] = acc
    k2, v2, npl, st = oracle.commit_path(k, v, bt, [L], path, [len(acc)])
    assert st == 0 and npl[0] == L + 1 + len(acc)
    for kk, c in enumerate(acc, start=1):
        # one-node "tree" at position L + kk whose prefix is positions 0 .. L + kk - 1
        after = oracle.tree_attention(q[:, c:c + 1], k2, v2, bt, np.array([L + kk], np.int32),
                                      np.array([[-1]], np.int32), Hkv, "f32")
        np.testing.assert_allclose(after[0, 0], before[0, c], rtol=0, atol=1e-12)
    # the root itself is committed in place: same check at position L
    after0 = oracle.tree_attention(q[:, 0:1], k2, v2, bt, np.array([L], np.int32), np.array([[-1]], np.int32), Hkv,
                                   "f32")
    np.testing.assert_allclose(after0[0, 0], before[0, 0], rtol=0, atol=1e-12)


def test_rows_move_as_bytes_for_bf16():
    k, v = _cache(2, 2, 8, 7)
    kb, vb = (k.view(np.uint32) >> 16).astype(np.uint16), (v.view(np.uint32) >> 16).astype(np.uint16)
    bt = np.array([[0, 1]], np.int32)
    k2, v2, npl, st = oracle.commit_path(kb, vb, bt, [3], np.array([[2, 4, -1, -1, -1]], np.int32), [2])
    assert st == 0 and k2.dtype == kb.dtype
    np.testing.assert_array_equal(_rows(k2, bt[0], [4, 5]), _rows(kb, bt[0], [5, 7]))

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


@pytest.mark.parametrize("seed", range(12))
def test_library_select_equals_oracle(seed):
    rng = np.random.default_rng(100 + seed)
    M = int(rng.integers(0, 300))
    par = np.array([int(rng.integers(-1, c)) if c else -1 for c in range(M)], np.int32)
    prob = rng.random(M)
    if seed % 3 == 0:
        prob = np.round(prob * 4) / 4  # many exact ties
    tok = rng.integers(0, 128256, M).astype(np.int32)
    for budget in (1, 2, 17, 64, 1024):
        got = tv.tree_select(par, tok, prob, budget)
        ref = oracle.select_tree(par, tok, prob, budget)
        for g, r in zip(got[:3], ref[:3]):
            np.testing.assert_array_equal(g, r)
        assert got[3] == ref[3]


def test_tree_select_rejects_bad_arguments():
    out = [np.zeros(8, np.int32) for _ in range(3)]
    n = np.zeros(1, np.int32)
    val = np.zeros(1)
    par, tok, prob = np.array([-1, 0], np.int32), np.array([1, 2], np.int32), np.array([0.5, 0.5])
    assert tv.tv_tree_select(par, tok, prob, 2, 8, *out, n, val) == tv.TV_OK and n[0] == 3
    assert tv.tv_tree_select(np.array([-1, 1], np.int32), tok, prob, 2, 8, *out, n, val) == tv.TV_ERR_TREE
    assert tv.tv_tree_select(par, tok, np.array([0.5, 1.5]), 2, 8, *out, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_select(par, tok, prob, 2, 0, *out, n, val) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_select(par, tok, prob, 2, 1025, *out, n, val) == tv.TV_ERR_UNSUPPORTED
    assert tv.tv_tree_select(None, None, None, 0, 8, *out, n, val) == tv.TV_OK and n[0] == 1


def test_batch_select_equals_per_sequence_oracle():
    rng = np.random.default_rng(7)
    B, budget = 9, 24
    sizes = rng.integers(0, 60, B)
    sizes[0] = 0
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    par, tok, prob = [], [], []
    for m in sizes:
        par += [int(rng.integers(-1, c)) if c else -1 for c in range(m)]
        tok += list(rng.integers(0, 1000, m))
        prob += list(np.round(rng.random(m) * 8) / 8)
    parent, tokens, index, counts, val = tv.tree_select_batch(off, par, tok, prob, budget)
    for b in range(B):
        o, m = off[b], sizes[b]
        rp, rt, ri, rv = oracle.select_tree(par[o:o + m], tok[o:o + m], prob[o:o + m], budget)
        n = len(rp)
        assert counts[b] == n and val[b] == rv
        np.testing.assert_array_equal(parent[b, :n], rp)
        np.testing.assert_array_equal(tokens[b, :n], rt)
        np.testing.assert_array_equal(index[b, :n], ri)
        assert (parent[b, n:] == -1).all()
    # a bad sequence anywhere: nothing is written
    bad_par = list(par)
    bad_par[off[3] + 1] = 5
    counts2 = np.full(B, 77, np.int32)
    out = [np.full((B, budget), 77, np.int32) for _ in range(3)]
    val2 = np.zeros(B)
    s = tv.lib().tv_tree_select_batch(B, tv._hptr(off), tv._hptr(np.array(bad_par, np.int32)),
                                      tv._hptr(np.array(tok, np.int32)), tv._hptr(np.array(prob)), budget,
                                      *[tv._hptr(x) for x in out], tv._hptr(counts2), tv._hptr(val2))
    assert s == tv.TV_ERR_TREE and (counts2 == 77).all() and all((x == 77).all() for x in out)


@pytest.mark.parametrize("accept,budget,depth,cost,alpha", [
    ([0.8], 40, 0, 0.0, 0.1), ([0.9], 40, 0, 0.0, 0.1), ([0.6, 0.25, 0.1], 48, 6, 0.3, 0.05),
    ([0.55, 0.2, 0.1, 0.05], 64, 0, 0.1, 0.15), ([0.7, 0.2], 30, 3, 0.0, 0.0), ([1.0], 50, 0, 0.0, 0.1),
    ([0.5, 0.5], 20, 4, 1.0, 0.02),
])
def test_library_cost_aware_shape_equals_oracle(accept, budget, depth, cost, alpha):
    p, r, v, sp = tv.tree_shape_for_cost(accept, budget, depth, cost, alpha)
    po, ro, vo, spo = oracle.tree_shape_for_cost(accept, budget, depth or None, cost, alpha)
    np.testing.assert_array_equal(p, po)
    np.testing.assert_array_equal(r, ro)
    assert v == vo and sp == spo


def test_cost_aware_shape_rejects_bad_costs():
    out = [np.zeros(8, np.int32), np.zeros(8, np.int32), np.zeros(1, np.int32), np.zeros(1), np.zeros(1)]
    acc = np.array([0.5])
    f = tv.lib().tv_tree_shape_for_cost
    assert f(tv._hptr(acc), 1, 8, 0, 0.0, 0.1, *[tv._hptr(x) for x in out]) == tv.TV_OK
    assert f(tv._hptr(acc), 1, 8, 0, -1.0, 0.1, *[tv._hptr(x) for x in out]) == tv.TV_ERR_INVALID_ARG
    assert f(tv._hptr(acc), 1, 8, 0, 0.0, float("nan"), *[tv._hptr(x) for x in out]) == tv.TV_ERR_INVALID_ARG
    assert f(tv._hptr(acc), 1, 8, 0, float("inf"), 0.1, *[tv._hptr(x) for x in out]) == tv.TV_ERR_INVALID_ARG
    assert f(tv._hptr(acc), 1, 300, 0, 0.0, 0.1, *[tv._hptr(x) for x in out]) == tv.TV_ERR_UNSUPPORTED


@pytest.mark.parametrize("seed", range(6))
def test_library_merge_equals_oracle(seed):
    rng = np.random.default_rng(300 + seed)
    K = int(rng.integers(0, 9))
    seqs = [list(rng.integers(0, 4 if seed % 2 else 128256, rng.integers(0, 12))) for _ in range(K)]
    parent, tokens, node_of = tv.tree_merge(seqs)
    rp, rt, rn = oracle.merge_sequences(seqs)
    np.testing.assert_array_equal(parent, rp)
    np.testing.assert_array_equal(tokens, rt)
    assert [list(x) for x in node_of] == rn


def test_merge_rejects_bad_arguments():
    out = [np.zeros(4, np.int32), np.zeros(4, np.int32), np.zeros(8, np.int32), np.zeros(1, np.int32)]
    off = np.array([0, 2, 4], np.int32)
    tok = np.array([1, 2, 3, 4], np.int32)
    f = tv.lib().tv_tree_merge
    h = [tv._hptr(x) for x in out]
    assert f(2, tv._hptr(off), tv._hptr(tok), 8, *[tv._hptr(x) for x in
             (np.zeros(8, np.int32), np.zeros(8, np.int32), np.zeros(8, np.int32), out[3])]) == tv.TV_OK
    assert out[3][0] == 5
    assert f(2, tv._hptr(off), tv._hptr(tok), 4, *h) == tv.TV_ERR_UNSUPPORTED  # 5 nodes do not fit in 4
    assert f(2, tv._hptr(np.array([1, 2, 4], np.int32)), tv._hptr(tok), 8, *h) == tv.TV_ERR_INVALID_ARG
    assert f(2, tv._hptr(off), tv._hptr(np.array([1, -2, 3, 4], np.int32)), 8, *h) == tv.TV_ERR_INVALID_ARG
    assert f(2, tv._hptr(off), tv._hptr(tok), 0, *h) == tv.TV_ERR_INVALID_ARG

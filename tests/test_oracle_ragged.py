"""Pins for the oracle's ragged-tree and chain forms.

A batch may hold trees of different sizes (mixed serving) and chains (linear
speculation, glossary "Tree-based speculative decoding", section "linear vs
tree": a chain is the tree whose every node has one child, and its mask is the
causal one).  The oracle treats sequence b as its own problem over its first
node_counts[b] nodes.  Pins: full counts reproduce the batched call bit for
bit; padding nodes hung as extra leaves do not change any real node's
attention (a leaf is nobody's ancestor); a root-only tree draws the bonus
straight from p by the inverse CDF; an empty tree produces nothing; chain
parents give the lower-triangular mask."""
import numpy as np

import oracle
from helpers import contiguous_table, dense_kv_to_paged


def _case(seed, B, N, Hq, Hkv, D, prefix_lens):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, N, Hq, D)).astype(np.float32)
    bt, _ = contiguous_table(prefix_lens, N)
    ks = [rng.standard_normal((L + N, Hkv, D)).astype(np.float32) for L in prefix_lens]
    vs = [rng.standard_normal((L + N, Hkv, D)).astype(np.float32) for L in prefix_lens]
    parent = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    return rng, q, dense_kv_to_paged(ks, bt), dense_kv_to_paged(vs, bt), bt, np.array(prefix_lens, np.int32), parent


def test_chain_parents_give_the_causal_mask():
    for N in (1, 2, 7, 40):
        par = oracle.chain_parents(3, N)
        assert par.shape == (3, N)
        np.testing.assert_array_equal(oracle.tree_mask(par[1]), np.tril(np.ones((N, N), np.uint8)))


def test_full_counts_reproduce_the_batched_call():
    rng, q, kc, vc, bt, pl, parent = _case(1, 3, 9, 4, 2, 16, [5, 40, 17])
    counts = np.full(3, 9)
    full = oracle.tree_attention(q, kc, vc, bt, pl, parent, 2, "f32")
    np.testing.assert_array_equal(oracle.tree_attention_ragged(q, kc, vc, bt, pl, parent, counts, 2, "f32"), full)
    V = 50
    p = oracle.softmax_rows(rng.normal(0, 2, (3, 9, V)))
    qd = oracle.softmax_rows(rng.normal(0, 2, (3, 9, V)))
    tok = rng.integers(0, V, (3, 9)).astype(np.int32)
    u = rng.random((3, 9)).astype(np.float32)
    a = oracle.verify_sample(p, qd, tok, parent, u)
    r = oracle.verify_sample_ragged(p, qd, tok, parent, u, counts)
    for key in ("accepted_path", "accepted_len", "bonus_token", "near", "rows"):
        np.testing.assert_array_equal(r[key], a[key])


def test_padding_leaves_do_not_change_real_rows():
    """Fill each sequence's padding with leaves under the root and run the
    batched definition: every real node's row equals the ragged result."""
    B, N = 4, 12
    rng, q, kc, vc, bt, pl, parent = _case(2, B, N, 4, 2, 16, [3, 30, 64, 1])
    counts = np.array([12, 5, 1, 8])
    padded = parent.copy()
    for b in range(B):
        padded[b, counts[b]:] = 0
    full = oracle.tree_attention(q, kc, vc, bt, pl, padded, 2, "f32")
    garbage = parent.copy()
    for b in range(B):
        garbage[b, counts[b]:] = 99  # ignored by the ragged form
    rag = oracle.tree_attention_ragged(q, kc, vc, bt, pl, garbage, counts, 2, "f32")
    for b in range(B):
        np.testing.assert_array_equal(rag[b, :counts[b]], full[b, :counts[b]])
        assert np.isnan(rag[b, counts[b]:]).all()


def test_root_only_tree_draws_the_bonus_from_p():
    rng = np.random.default_rng(3)
    B, N, V = 6, 5, 40
    p = oracle.softmax_rows(rng.normal(0, 2, (B, N, V)))
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    r = oracle.verify_sample_ragged(p, p, tok, None, u, np.ones(B, int))
    assert (r["accepted_len"] == 0).all() and (r["accepted_path"] == -1).all()
    for b in range(B):
        c = np.cumsum(p[b, 0].astype(np.float64))
        assert r["bonus_token"][b] == int(np.searchsorted(c, float(u[b, 0]) * c[-1], side="right"))


def test_empty_trees_produce_nothing():
    rng, q, kc, vc, bt, pl, parent = _case(4, 2, 6, 2, 1, 8, [10, 20])
    counts = np.array([0, 6])
    out = oracle.tree_attention_ragged(q, kc, vc, bt, pl, parent, counts, 1, "f32")
    assert np.isnan(out[0]).all() and not np.isnan(out[1]).any()
    V = 30
    p = oracle.softmax_rows(rng.normal(0, 1, (2, 6, V)))
    r = oracle.verify_sample_ragged(p, p, np.zeros((2, 6), np.int32), parent, np.full((2, 6), 0.3, np.float32),
                                    counts)
    assert r["accepted_len"][0] == 0 and r["bonus_token"][0] == -1 and (r["accepted_path"][0] == -1).all()
    k2, v2, npl, st = oracle.commit_path_ragged(kc, vc, bt, pl, np.full((2, 6), -1, np.int32), [0, 0], counts)
    assert st == 0 and list(npl) == [10, 21]
    np.testing.assert_array_equal(k2, kc)


def test_chain_walk_equals_explicit_chain_parents():
    rng = np.random.default_rng(5)
    B, N, V = 20, 7, 25
    lp = rng.normal(0, 1, (B, N, V))
    p = oracle.softmax_rows(lp)
    qd = oracle.softmax_rows(lp + rng.normal(0, 0.5, (B, N, V)))
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    counts = rng.integers(0, N + 1, B)
    a = oracle.verify_sample_ragged(p, qd, tok, None, u, counts)
    b = oracle.verify_sample_ragged(p, qd, tok, oracle.chain_parents(B, N), u, counts)
    for key in ("accepted_path", "accepted_len", "bonus_token"):
        np.testing.assert_array_equal(a[key], b[key])
    # on a chain the accepted path is always 1, 2, ..., len
    for i in range(B):
        n = a["accepted_len"][i]
        np.testing.assert_array_equal(a["accepted_path"][i, :n], np.arange(1, n + 1))

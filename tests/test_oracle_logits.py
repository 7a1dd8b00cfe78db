"""Pins for the oracle's fused-logits acceptance walk (verify_sample_logits).

p and q are the models' output distributions (blog "Speculative decoding x
tree attention", section 2; glossary "Tree-based speculative decoding",
section "SpecInfer"), so a verifier that takes logits first applies a softmax
per row.  Pins: softmax_rows against a closed form and its invariances, and the
walk on logits = log p reproducing the walk on p."""
import numpy as np

import oracle


def test_softmax_rows_closed_form_and_invariances():
    x = np.array([[0.0, np.log(3.0), np.log(6.0)]])
    np.testing.assert_allclose(oracle.softmax_rows(x), [[0.1, 0.3, 0.6]], rtol=1e-7)
    rng = np.random.default_rng(1)
    l = rng.normal(0, 3, (4, 1000))
    p = oracle.softmax_rows(l)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-6)
    assert (p > 0).all()
    # shifting a row by a constant leaves its distribution unchanged
    np.testing.assert_allclose(oracle.softmax_rows(l + 17.0), p, rtol=2e-7)
    # order is preserved
    assert (np.argsort(p, axis=1) == np.argsort(l, axis=1)).all()


def test_walk_on_log_probabilities_equals_walk_on_probabilities():
    rng = np.random.default_rng(2)
    B, N, V = 40, 9, 257
    parent = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    lp = rng.normal(0, 2, (B, N, V))
    lq = lp + rng.normal(0, 1, (B, N, V))
    p, q = oracle.softmax_rows(lp), oracle.softmax_rows(lq)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        for i in range(1, N):
            w = q[b, parent[b, i]].astype(np.float64)
            tokens[b, i] = int(rng.choice(V, p=w / w.sum()))
    u = rng.random((B, N)).astype(np.float32)
    ref = oracle.verify_sample(p, q, tokens, parent, u)
    got = oracle.verify_sample_logits(np.log(p.astype(np.float64)), np.log(q.astype(np.float64)), tokens, parent, u)
    same = ((ref["accepted_len"] == got["accepted_len"]) & (ref["bonus_token"] == got["bonus_token"])
            & (ref["accepted_path"] == got["accepted_path"]).all(axis=1))
    flagged = (ref["near"] > 0) | (got["near"] > 0)
    assert (same | flagged).all()
    assert same.mean() > 0.9

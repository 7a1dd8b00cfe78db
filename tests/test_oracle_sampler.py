"""Pins for the oracle's acceptance walk.

Rule: accept draft x when r < min(1, p(x)/q(x)); on rejection resample from
max(0, p - q) normalised (blog, section 2, "Rejection Sampling Acceptance
Condition"); siblings are retried root-down against the renormalised
residual (glossary, "SpecInfer").  Pinned by a hand-worked example
(tests/golden), degenerate cases, the losslessness claim (the output follows
p exactly: blog section 2, last paragraph; LLM primer chapter 9.1) as a
chi-square test, and the chain closed form (1 - a^(g+1)) / (1 - a) for the
expected number of emitted tokens (glossary, "linear vs tree" table)."""
import numpy as np
import pytest
from scipy import stats

import oracle
import synth
from helpers import golden_lines


def _walk(p, q, tokens, parent, u, eps=1e-6):
    return oracle.verify_sample(np.asarray(p, np.float32), np.asarray(q, np.float32),
                                np.asarray(tokens, np.int32), np.asarray(parent, np.int32),
                                np.asarray(u, np.float32), eps)


def test_worked_example():
    p_root = [0.5, 0.3, 0.2, 0.0]
    q_root = [0.25] * 4
    for case, r1, r2, u0, exp_len, exp_p0, exp_bonus in golden_lines("sampler_worked_example.txt"):
        toks = [0, 3, 2] if case == "A" else [0, 3, 1]
        p = np.zeros((1, 3, 4)); q = np.zeros((1, 3, 4))
        p[0, 0] = p_root; q[0, 0] = q_root
        p[0, 1] = [0.25] * 4; q[0, 1] = [0.25] * 4
        p[0, 2] = [0, 0, 1, 0]; q[0, 2] = [0.25] * 4
        res = _walk(p, q, [toks], [[-1, 0, 0]], [[float(u0), float(r1), float(r2)]])
        assert res["rc"] == 0
        assert res["accepted_len"][0] == int(exp_len), (case, r1, r2)
        assert res["accepted_path"][0, 0] == int(exp_p0)
        assert res["bonus_token"][0] == int(exp_bonus)


def test_equal_distributions_always_accept_first_child():
    rng = np.random.default_rng(0)
    B, V = 64, 10
    parent = [-1, 0, 0, 1, 1, 3, 2]
    N = len(parent)
    p = rng.dirichlet(np.ones(V), size=(B, N))
    toks = rng.integers(0, V, size=(B, N))
    u = rng.random((B, N)) * 0.999
    res = _walk(p, p, toks, [parent] * B, u)
    for b in range(B):
        assert list(res["accepted_path"][b, :3]) == [1, 3, 5]     # first child at every level
        assert res["accepted_len"][b] == 3


def test_onehot_draft_on_zero_target_always_rejects():
    V = 6
    p = np.zeros((1, 3, V)); q = np.zeros((1, 3, V))
    p[0, 0] = [0.0, 0.4, 0.6, 0, 0, 0]
    q[0, 0] = [1.0, 0, 0, 0, 0, 0]
    p[0, 1:] = 1.0 / V; q[0, 1:] = 1.0 / V
    for u1 in (0.0, 0.5, 0.999):
        res = _walk(p, q, [[0, 0, 0]], [[-1, 0, 0]], [[0.5, u1, u1]])
        assert res["accepted_len"][0] == 0
        # residual after the first rejection is p itself (q's mass sits on a p = 0 token)
        assert res["bonus_token"][0] == 2


def test_zero_uniform_accepts_iff_target_positive():
    V = 5
    p = np.full((1, 2, V), 0.2); q = np.full((1, 2, V), 0.2)
    p[0, 0] = [0.0, 0.1, 0.2, 0.3, 0.4]
    for tok in range(V):
        res = _walk(p, q, [[0, tok]], [[-1, 0]], [[0.5, 0.0]])
        assert res["accepted_len"][0] == (1 if p[0, 0, tok] > 0 else 0)


def test_leaf_draws_from_plain_target_with_cdf_rule():
    V = 4
    p = np.array([[[0.1, 0.2, 0.3, 0.4]]]); q = np.full((1, 1, V), 0.25)
    edges = np.cumsum(p[0, 0])
    for u0 in np.linspace(0.0, 0.99, 23):
        u32 = float(np.float32(u0))
        res = _walk(p, q, [[0]], [[-1]], [[u32]])
        # first index whose running sum exceeds u0 * total
        expect = int(np.argmax(edges > u32 * edges[-1]))
        assert res["bonus_token"][0] == expect


def test_invalid_tree_and_token_are_reported():
    p = np.full((2, 3, 4), 0.25)
    res = _walk(p, p, [[0, 1, 9], [0, 1, 2]], [[-1, 0, 0], [-1, 2, 0]], np.zeros((2, 3)))
    assert res["rc"] == oracle.ERR_TREE
    assert list(res["accepted_len"]) == [-1, -1]
    assert list(res["bonus_token"]) == [-1, -1]


def _iid_tree_inputs(n_walks, V, seed):
    """Root with 3 children drawn i.i.d. from q_root, each child with 2
    children drawn i.i.d. from its own q; p depends only on the token path."""
    rng = np.random.default_rng(seed)
    parent = [-1, 0, 0, 0, 1, 1, 2, 2, 3, 3]
    N = len(parent)
    p_root = rng.dirichlet(np.ones(V) * 0.8)
    q_root = rng.dirichlet(np.ones(V) * 0.8)
    p_child = rng.dirichlet(np.ones(V) * 0.8, size=V)       # p(. | x1)
    q_child = rng.dirichlet(np.ones(V) * 0.8, size=V)
    toks = np.zeros((n_walks, N), dtype=np.int32)
    toks[:, 1:4] = rng.choice(V, size=(n_walks, 3), p=q_root)
    for c, par in enumerate(parent):
        if par >= 1:
            x1 = toks[:, par]
            cdf = np.cumsum(q_child[x1], axis=1)
            r = rng.random(n_walks)[:, None]
            toks[:, c] = np.minimum((cdf <= r).sum(1), V - 1)
    p = np.empty((n_walks, N, V), np.float32)
    q = np.empty((n_walks, N, V), np.float32)
    p[:, 0] = p_root; q[:, 0] = q_root
    for c in range(1, N):
        if parent[c] == 0:
            p[:, c] = p_child[toks[:, c]]; q[:, c] = q_child[toks[:, c]]
        else:   # grandchildren are leaves; their p is only used for the bonus draw
            p[:, c] = p_root; q[:, c] = q_root
    u = synth.uniforms(n_walks * N, seed, synth.STREAM_UNIFORM).reshape(n_walks, N)
    return p, q, toks, np.array([parent] * n_walks, np.int32), u, p_root, p_child


def _chi2_ok(counts, probs, alpha=1e-3):
    n = counts.sum()
    keep = probs > 0
    assert counts[~keep].sum() == 0
    stat = ((counts[keep] - n * probs[keep]) ** 2 / (n * probs[keep])).sum()
    return stat < stats.chi2.ppf(1 - alpha, keep.sum() - 1), stat


def lossless_check(verify, n_walks=200_000, V=8, seed=123):
    """Returns (ok_first, ok_second) for a walk function with the oracle's
    signature.  Used on the oracle here and on the GPU kernel elsewhere."""
    p, q, toks, par, u, p_root, p_child = _iid_tree_inputs(n_walks, V, seed)
    res = verify(p, q, toks, par, u)
    alen, path, bonus = res["accepted_len"], res["accepted_path"], res["bonus_token"]
    first = np.where(alen >= 1, toks[np.arange(n_walks), np.maximum(path[:, 0], 0)], bonus)
    ok1, _ = _chi2_ok(np.bincount(first, minlength=V), p_root)
    # second emitted token given an accepted first token x1 (most frequent one)
    acc = alen >= 1
    x1_all = toks[np.arange(n_walks), np.maximum(path[:, 0], 0)]
    x1 = np.bincount(x1_all[acc], minlength=V).argmax()
    sel = acc & (x1_all == x1)
    second = np.where(alen[sel] >= 2, toks[np.arange(n_walks)[sel], np.maximum(path[sel, 1], 0)], bonus[sel])
    ok2, _ = _chi2_ok(np.bincount(second, minlength=V), p_child[x1])
    return ok1, ok2


def test_lossless_chi_square():
    ok1, ok2 = lossless_check(lambda *a: _walk(*a))
    assert ok1 and ok2


@pytest.mark.parametrize("a,gamma", [(0.7, 5), (0.45, 3)])
def test_chain_expected_emitted_tokens(a, gamma):
    # every position: sum_x min(p, q) = a, drafts drawn i.i.d. from q
    n, V = 100_000, 6
    rng = np.random.default_rng(int(a * 100) + gamma)
    N = gamma + 1
    q_pos = np.zeros((N, V)); p_pos = np.zeros((N, V))
    for i in range(N):
        qi = rng.dirichlet(np.ones(V - 1))
        q_pos[i, :-1] = qi
        p_pos[i, :-1] = a * qi
        p_pos[i, -1] = 1.0 - a             # the last token is never drafted
    toks = np.zeros((n, N), np.int32)
    for c in range(1, N):
        toks[:, c] = rng.choice(V, size=n, p=q_pos[c - 1])
    p = np.broadcast_to(p_pos, (n, N, V)).astype(np.float32)
    q = np.broadcast_to(q_pos, (n, N, V)).astype(np.float32)
    u = rng.random((n, N)).astype(np.float32)
    res = _walk(p, q, toks, np.array([[-1] + list(range(gamma))] * n), u)
    emitted = res["accepted_len"] + 1.0
    expect = (1 - a ** (gamma + 1)) / (1 - a)
    se = emitted.std() / np.sqrt(n)
    assert abs(emitted.mean() - expect) < 4 * se, (emitted.mean(), expect, se)


def test_cdf_tie_break_is_strict():
    # bucket edges exactly representable: u0 * total == C_0 picks the next index,
    # and a zero-mass index is never drawn even at u0 = 0
    p = np.array([[[0.25, 0.25, 0.5]]]); q = np.full((1, 1, 3), 1 / 3)
    assert _walk(p, q, [[0]], [[-1]], [[0.25]])["bonus_token"][0] == 1
    assert _walk(p, q, [[0]], [[-1]], [[0.5]])["bonus_token"][0] == 2
    p = np.array([[[0.0, 0.5, 0.5, 0.0]]]); q = np.full((1, 1, 4), 0.25)
    assert _walk(p, q, [[0]], [[-1]], [[0.0]])["bonus_token"][0] == 1

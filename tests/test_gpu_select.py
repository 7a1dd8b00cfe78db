"""The dynamic tree selected on the GPU (tv_tree_select_device) against the
oracle's select_tree, bit for bit: the trees (parent, token and candidate of
every node), their sizes and their values (fp64 sums of fp64 path products).
Cases: ragged candidate counts (0 .. 1500 per sequence), EAGLE-2-like
level-by-level growth, heavy score ties (probabilities on a coarse grid,
zeros and ones), a chain as deep as the candidate set, budgets from 1 to
1024; malformed sequences are reported and leave the others intact."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _grown(rng, M, width=8, coarse=False):
    """Candidates grown level by level: each level expands the best few nodes
    of the previous one with `width` children (parents before children)."""
    par, prob = [], []
    frontier = [-1]
    while len(par) < M:
        nxt = []
        for u in frontier:
            for _ in range(width):
                if len(par) >= M:
                    break
                par.append(u)
                p = rng.integers(0, 5) / 4.0 if coarse else float(np.float32(rng.random() ** 2))
                prob.append(p)
                nxt.append(len(par) - 1)
        frontier = nxt[: max(1, len(nxt) // 3)]
    return np.array(par, np.int32), np.array(prob, np.float32)


def _random(rng, M, coarse=False):
    par = np.array([int(rng.integers(-1, c)) if c else -1 for c in range(M)], np.int32)
    prob = (rng.integers(0, 5, M) / 4.0 if coarse else rng.random(M) ** 3).astype(np.float32)
    return par, prob


def _run(seqs, budget, status=None):
    counts = [len(p) for p, _, _ in seqs]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    par = np.concatenate([p for p, _, _ in seqs] + [np.zeros(0, np.int32)]).astype(np.int32)
    tok = np.concatenate([t for _, t, _ in seqs] + [np.zeros(0, np.int32)]).astype(np.int32)
    prob = np.concatenate([q for _, _, q in seqs] + [np.zeros(0, np.float32)]).astype(np.float32)
    pad = lambda a: a if a.size else np.zeros(1, a.dtype)
    parent, tokens, index, n, val = tv.tree_select_device(dev(off), dev(pad(par)), dev(pad(tok)), dev(pad(prob)),
                                                          budget, dev_status=status)
    torch.cuda.synchronize()
    return (parent.cpu().numpy(), tokens.cpu().numpy(), index.cpu().numpy(), n.cpu().numpy(), val.cpu().numpy())


def _check(seqs, budget):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    parent, tokens, index, n, val = _run(seqs, budget, status)
    assert int(status.item()) == 0
    for b, (par, tok, prob) in enumerate(seqs):
        rp, rt, ri, rv = oracle.select_tree(par, tok, prob.astype(np.float64), budget)
        k = len(rp)
        assert n[b] == k, (b, n[b], k)
        np.testing.assert_array_equal(parent[b, :k], rp)
        np.testing.assert_array_equal(tokens[b, :k], rt)
        np.testing.assert_array_equal(index[b, :k], ri)
        assert (parent[b, k:] == -1).all() and (tokens[b, k:] == -1).all() and (index[b, k:] == -1).all()
        assert val[b] == rv, (b, val[b], rv)   # bit for bit


@pytest.mark.parametrize("coarse", [False, True], ids=["continuous", "ties"])
@pytest.mark.parametrize("budget", [1, 2, 16, 64, 1024])
def test_grown_candidates_match_oracle(budget, coarse):
    rng = np.random.default_rng(100 + budget + coarse)
    seqs = []
    for b, M in enumerate([0, 1, 7, 60, 255, 256, 257, 600, 1500]):
        par, prob = _grown(rng, M, coarse=coarse) if b % 2 else _random(rng, M, coarse=coarse)
        tok = rng.integers(0, 128256, M).astype(np.int32)
        seqs.append((par, tok, prob))
    _check(seqs, budget)


def test_deep_chain_and_extreme_probabilities():
    rng = np.random.default_rng(7)
    M = 1200
    chain = np.arange(-1, M - 1, dtype=np.int32)
    ones = np.ones(M, np.float32)
    zeros = np.zeros(M, np.float32)
    star = np.full(M, -1, np.int32)
    tok = rng.integers(0, 1000, M).astype(np.int32)
    _check([(chain, tok, ones), (chain, tok, zeros), (star, tok, ones), (star, tok, zeros)], 700)


def test_malformed_sequences_are_reported():
    rng = np.random.default_rng(8)
    good_par, good_prob = _random(rng, 50)
    tok = rng.integers(0, 1000, 50).astype(np.int32)
    bad_par = good_par.copy()
    bad_par[10] = 20                   # parent after child
    bad_prob = good_prob.copy()
    bad_prob[3] = 1.5                  # not a probability
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    parent, tokens, index, n, val = _run([(good_par, tok, good_prob), (bad_par, tok, good_prob),
                                          (good_par, tok, bad_prob)], 16, status)
    assert int(status.item()) in (tv.TV_ERR_TREE, tv.TV_ERR_INVALID_ARG)
    assert n[1] == -1 and n[2] == -1 and (parent[1] == -1).all() and (parent[2] == -1).all()
    rp, _, _, rv = oracle.select_tree(good_par, tok, good_prob.astype(np.float64), 16)
    assert n[0] == len(rp) and val[0] == rv


def test_selected_tree_drives_the_walk():
    """The selected tree, still on the device, feeds the acceptance walk."""
    rng = np.random.default_rng(9)
    par, prob = _grown(rng, 200)
    tok = rng.integers(0, 1000, 200).astype(np.int32)
    off = torch.tensor([0, 200], dtype=torch.int32, device="cuda")
    parent, tokens, index, n, val = tv.tree_select_device(off, dev(par), dev(tok), dev(prob), 32)
    N = 32
    lp = rng.normal(0, 2, (1, N, 1000)).astype(np.float32)
    p = oracle.softmax_rows(lp)
    q = oracle.softmax_rows(lp + rng.normal(0, 1, (1, N, 1000)))
    u = rng.random((1, N)).astype(np.float32)
    tokens_dev = tokens.clone()
    tokens_dev[:, 0] = 0
    path, alen, bonus = tv.verify_sample(dev(p), dev(q), tokens_dev, parent, dev(u), node_counts=n)
    torch.cuda.synchronize()
    ref = oracle.verify_sample_ragged(p, q, tokens_dev.cpu().numpy(), parent.cpu().numpy(), u, n.cpu().numpy())
    if ref["near"][0] == 0:
        assert int(alen[0]) == ref["accepted_len"][0] and int(bonus[0]) == ref["bonus_token"][0]

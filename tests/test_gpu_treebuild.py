"""Top-k branching on the GPU (tv_tree_fill_topk) against the oracle's
fill_topk_tokens, bit for bit (token ids are integers): the 64-node top-k tree
[4, 3, 2, 2, 1, 1] on its full 128256-entry draft rows, random trees with
ragged counts, default ranks, chains, odd vocabularies, heavy ties and
negative logits; malformed inputs; and shape -> tokens -> walk end to end."""
import numpy as np
import pytest
import torch

import oracle
import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import compare_sampler, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _fill(q, parent, rank, counts=None, status=None, prefill=-1):
    B, N = q.shape[:2]
    out = torch.full((B, N), prefill, dtype=torch.int32, device="cuda")
    tv.fill_topk(dev(np.ascontiguousarray(q, np.float32)), None if parent is None else dev(parent),
                 None if rank is None else dev(rank), tree_tokens=out,
                 node_counts=None if counts is None else dev(counts), dev_status=status)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _sibling_ranks(parent):
    rank = np.full(parent.shape, -1, np.int32)
    for b in range(parent.shape[0]):
        seen = {}
        for c in range(1, parent.shape[1]):
            rank[b, c] = seen.get(int(parent[b, c]), 0)
            seen[int(parent[b, c])] = rank[b, c] + 1
    return rank


def _check(q, parent, rank, counts=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fill(q, parent, rank, counts, status)
    assert int(status.item()) == 0
    par = oracle.chain_parents(q.shape[0], q.shape[1]) if parent is None else parent
    rk = _sibling_ranks(par) if rank is None else rank
    ref = oracle.fill_topk_tokens(q, par, rk, counts)
    B, N = got.shape
    for b in range(B):
        n = N if counts is None else int(counts[b])
        np.testing.assert_array_equal(got[b, 1:n], ref[b, 1:n])
        assert got[b, 0] == -1 and (got[b, n:] == -1).all()  # root and padding untouched
    return got


def test_topk_tree_on_full_draft_rows():
    wl = synth.make("l8b")
    _, q = wl.pq()
    par, rank = synth.topk_tree([4, 3, 2, 2, 1, 1], 64)
    parent = np.array([par], np.int32)
    got = _check(q, parent, np.array([rank], np.int32))
    # the workload's own tokens were built by the same rule
    np.testing.assert_array_equal(got[0, 1:], wl.tree_tokens[0, 1:])


@pytest.mark.parametrize("V", [1, 7, 1000, 4099, 65536, 151936])
def test_random_trees_ragged_counts(V):
    rng = np.random.default_rng(V)
    B, N = 12, 24
    parent = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    rank = _sibling_ranks(parent)
    rank = np.where(rank >= 0, np.minimum(rank, V - 1), -1).astype(np.int32)
    counts = rng.integers(0, N + 1, B).astype(np.int32)
    counts[:2] = [0, N]
    q = rng.dirichlet(np.ones(V), size=(B, N)).astype(np.float32)
    _check(q, parent, rank, counts)
    _check(q, parent, None if V >= 8 else rank, counts)  # default ranks: sibling order


def test_ties_chains_and_negative_logits():
    rng = np.random.default_rng(3)
    B, N, V = 6, 16, 3001
    q = rng.integers(0, 4, (B, N, V)).astype(np.float32)  # heavy ties
    _check(q, None, None)                                  # chains, rank 0
    logits = rng.normal(-3, 2, (B, N, V)).astype(np.float32)
    parent = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    _check(logits, parent, _sibling_ranks(parent))


def test_malformed_inputs_report_and_clear():
    V = 500
    q = np.random.default_rng(4).random((3, 40, V)).astype(np.float32)
    parent = np.zeros((3, 40), np.int32)
    parent[:, 0] = -1
    parent[1, 5] = 7            # not topological
    rank = _sibling_ranks(parent)  # sequences 0 and 2: the root has 39 children (> 32)
    rank[2] = np.where(rank[2] >= 0, 0, -1)
    rank[2, 3] = 40             # sequence 2: a rank past 31
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fill(q, parent, rank, status=status, prefill=7)
    assert int(status.item()) == tv.TV_ERR_TREE
    assert (got[:, 1:] == -1).all() and (got[:, 0] == 7).all()


def test_shape_tokens_walk_end_to_end():
    """tv_tree_shape builds the shape, tv_tree_fill_topk its tokens from the
    draft rows, and the acceptance walk runs on the result."""
    acc = [0.55, 0.2, 0.1, 0.05]
    par, rank, _ = tv.tree_shape(acc, 40, 6)
    N, V, B = len(par), 32000, 8
    rng = np.random.default_rng(5)
    lq = rng.normal(0, 3, (B, N, V))
    q = oracle.softmax_rows(lq)
    p = oracle.softmax_rows(lq + rng.normal(0, 1, (B, N, V)))
    parent = np.tile(par, (B, 1)).astype(np.int32)
    ranks = np.tile(rank, (B, 1)).astype(np.int32)
    tokens = _check(q, parent, ranks)
    tokens[:, 0] = 0
    u = rng.random((B, N)).astype(np.float32)
    path, alen, bonus = tv.verify_sample(dev(p), dev(q), dev(tokens), dev(parent), dev(u))
    torch.cuda.synchronize()
    got = {"accepted_path": path.cpu().numpy(), "accepted_len": alen.cpu().numpy(), "bonus_token": bonus.cpu().numpy()}
    compare_sampler(got, oracle.verify_sample(p, q, tokens, parent, u))


@pytest.mark.parametrize("V", [40, 5000, 151936])
def test_wide_nodes_take_several_passes(V):
    """A root with 32 children (ranks 0..31) and a node with 12 (ranks past 8
    take more than one pass over the row), on tie-heavy rows."""
    N = 45
    parent = np.array([[-1] + [0] * 32 + [1] * 12] * 2, np.int32)
    rng = np.random.default_rng(V)
    q = rng.integers(0, 10, (2, N, V)).astype(np.float32)
    q[1] = rng.random((N, V)).astype(np.float32)
    _check(q, parent, _sibling_ranks(parent))
    _check(q, parent, None)

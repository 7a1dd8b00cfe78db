"""Pins for the oracle's tree construction: top-k branching and the
budget-constrained shape (glossary "Tree-based speculative decoding", the
section on tree-structure optimisation: "Top-k branching" and
"Budget-constrained optimisation", solved by dynamic programming).

Pins: top-k against a brute-force sort and hand-made ties; the filled tokens
on a hand-worked tree; the DP against exhaustive enumeration of every tree
within the budget; a width-1 budget against the pages' chain formula
(1 - a^(g+1)) / (1 - a) (glossary, "linear vs tree" table); the depth cap;
monotonicity in the budget."""
import itertools

import numpy as np
import pytest

import oracle


def test_topk_rows_against_brute_force_and_ties():
    x = np.array([[0.1, 0.5, 0.2, 0.5, 0.0, 0.2]], np.float32)
    idx, val = oracle.topk_rows(x, 4)
    assert idx.tolist() == [[1, 3, 2, 5]]  # equal values: lower index first
    np.testing.assert_array_equal(val, x[:, [1, 3, 2, 5]])
    rng = np.random.default_rng(1)
    y = rng.integers(0, 5, (20, 30)).astype(np.float32)  # many ties
    idx, _ = oracle.topk_rows(y, 7)
    for r in range(20):
        want = sorted(range(30), key=lambda i: (-y[r, i], i))[:7]
        assert idx[r].tolist() == want


def test_fill_topk_tokens_hand_example():
    # root -> {1 (rank 0), 2 (rank 1)}, 1 -> {3 (rank 0)}; node 2 and 3 are leaves
    q = np.zeros((1, 4, 6), np.float32)
    q[0, 0] = [0.1, 0.3, 0.05, 0.3, 0.2, 0.05]    # order 1, 3, 4, 0, ...
    q[0, 1] = [0.0, 0.0, 0.0, 0.0, 0.0, 1.0]      # order 5, ...
    q[0, 2] = q[0, 3] = 1.0 / 6                    # leaves: never read
    parent = np.array([[-1, 0, 0, 1]], np.int32)
    rank = np.array([[-1, 0, 1, 0]], np.int32)
    assert oracle.fill_topk_tokens(q, parent, rank).tolist() == [[0, 1, 3, 5]]
    # ragged: a one-node tree has only its root
    assert oracle.fill_topk_tokens(q, parent, rank, node_counts=[1]).tolist() == [[0, -1, -1, -1]]


def _all_trees(budget, k, depth):
    """Every tree (as (parent, rank)) with at most `budget` nodes, children of
    ranks 0..m-1 (m <= k) and depth <= `depth`."""
    def subtrees(n, d):
        # ordered child lists for a root with exactly n nodes
        if n == 1:
            yield []
            return
        if d == 0:
            return
        for m in range(1, k + 1):
            for sizes in itertools.product(range(1, n), repeat=m):
                if sum(sizes) != n - 1:
                    continue
                for kids in itertools.product(*[list(subtrees(s, d - 1)) for s in sizes]):
                    yield list(kids)

    for n in range(1, budget + 1):
        for t in subtrees(n, depth):
            parent, rank = [-1], [-1]

            def walk(children, me):
                for r, ch in enumerate(children):
                    parent.append(me)
                    rank.append(r)
                    walk(ch, len(parent) - 1)

            walk(t, 0)
            yield parent, rank


@pytest.mark.parametrize("accept,budget,depth", [
    ([0.6, 0.25, 0.1], 7, 6), ([0.9, 0.05], 7, 3), ([0.5, 0.3, 0.15], 6, 2), ([0.35, 0.3, 0.2], 7, 6),
    ([0.8], 5, 4),
])
def test_dp_equals_exhaustive_search(accept, budget, depth):
    best = max(oracle.tree_value(p, r, accept) for p, r in _all_trees(budget, len(accept), depth))
    parent, rank, value = oracle.tree_shape_dp(accept, budget, depth)
    assert abs(value - best) <= 1e-12
    assert abs(oracle.tree_value(parent, rank, accept) - value) <= 1e-12
    # the returned tree obeys the constraints and is numbered parent-first
    n = len(parent)
    assert n <= budget and parent[0] == -1 and all(0 <= parent[c] < c for c in range(1, n))
    depth_of = [0] * n
    for c in range(1, n):
        depth_of[c] = depth_of[parent[c]] + 1
    assert max(depth_of) <= depth
    for u in range(n):
        ranks = sorted(rank[c] for c in range(1, n) if parent[c] == u)
        assert ranks == list(range(len(ranks))) and len(ranks) <= len(accept)


@pytest.mark.parametrize("a,n", [(0.5, 2), (0.7, 6), (0.9, 12), (0.3, 9)])
def test_width_one_budget_is_the_chain_formula(a, n):
    parent, rank, value = oracle.tree_shape_dp([a], n)
    assert parent.tolist() == [-1] + list(range(n - 1))
    # emitted tokens per step = accepted + the bonus: (1 - a^(g+1)) / (1 - a), g = n - 1 drafts
    assert abs((1.0 + value) - (1 - a ** n) / (1 - a)) <= 1e-12


def test_depth_cap_and_budget_monotonicity():
    parent, rank, value = oracle.tree_shape_dp([0.8], 10, max_depth=3)
    assert len(parent) == 4 and abs(value - (0.8 + 0.64 + 0.512)) <= 1e-12
    acc = [0.55, 0.2, 0.1, 0.05]
    vals = [oracle.tree_shape_dp(acc, n, 5)[2] for n in range(1, 25)]
    assert all(b >= a for a, b in zip(vals, vals[1:]))


def test_ties_follow_the_stated_rule():
    """Equal values: the smaller subtree goes to the lower rank, then the
    smaller tree wins (the reading the library documents)."""
    # root children sized (1, 2) or (2, 1) tie at 0.5 * 1 + 0.5 * 1.5 = 1.25: the rank-0 child stays a leaf
    parent, rank, value = oracle.tree_shape_dp([0.5, 0.5], 4, 2)
    assert value == 1.25
    assert parent.tolist() == [-1, 0, 0, 2] and rank.tolist() == [-1, 0, 1, 0]
    # a rank that is never accepted adds nothing: the tree without it is smaller
    parent, rank, value = oracle.tree_shape_dp([0.5, 0.0], 3, 1)
    assert parent.tolist() == [-1, 0] and value == 0.5


def _closed_subsets(par, size):
    M = len(par)
    for k in range(size + 1):
        for sub in itertools.combinations(range(M), k):
            ss = set(sub)
            if all(par[c] < 0 or par[c] in ss for c in sub):
                yield sub


@pytest.mark.parametrize("seed", range(8))
def test_select_tree_is_the_best_closed_subset(seed):
    rng = np.random.default_rng(seed)
    M = int(rng.integers(3, 10))
    par = [-1] + [int(rng.integers(-1, c)) for c in range(1, M)]
    prob = rng.random(M) * 0.9 + 0.05
    tok = rng.integers(0, 100, M)
    score = np.zeros(M)
    for c in range(M):
        score[c] = (score[par[c]] if par[c] >= 0 else 1.0) * prob[c]
    for budget in (1, 2, 4, M + 3):
        parent, tokens, index, value = oracle.select_tree(par, tok, prob, budget)
        best = max(sum(score[c] for c in sub) for sub in _closed_subsets(par, budget - 1))
        assert abs(value - best) <= 1e-12
        n = len(parent)
        assert n == min(budget, M + 1) and parent[0] == -1 and index[0] == -1
        for j in range(1, n):
            c = index[j]
            assert 0 <= parent[j] < j and tokens[j] == tok[c]
            assert (par[c] < 0 and parent[j] == 0) or index[parent[j]] == par[c]


def test_select_tree_ties_and_hand_example():
    # root -> a (0.5), b (0.5); a -> c (1.0): scores a 0.5, b 0.5, c 0.5 -> order a, b, c by index
    parent, tokens, index, value = oracle.select_tree([-1, -1, 0], [7, 8, 9], [0.5, 0.5, 1.0], 3)
    assert index.tolist() == [-1, 0, 1] and parent.tolist() == [-1, 0, 0] and tokens.tolist() == [-1, 7, 8]
    assert value == 1.0
    parent, tokens, index, value = oracle.select_tree([-1, -1, 0], [7, 8, 9], [0.5, 0.4, 0.9], 3)
    assert index.tolist() == [-1, 0, 2] and parent.tolist() == [-1, 0, 1] and abs(value - 0.95) < 1e-15


@pytest.mark.parametrize("p,lo,hi", [(0.8, 6, 8), (0.9, 10, 12)])
def test_chain_speedup_peaks_where_the_pages_say(p, lo, hi):
    """LLM Primer VI ch. 9, 9.3: the speedup (1 + E) / (T_draft/T_decode + 1 + alpha N)
    peaks near N = 6-8 draft tokens for p = 0.8 and N = 10-12 for p = 0.9 (alpha in
    0.05-0.15; taken here at 0.1 with free drafting)."""
    parent, rank, value, sp = oracle.tree_shape_for_cost([p], 40, None, 0.0, 0.1)
    N = len(parent) - 1
    assert lo <= N <= hi
    assert abs(sp - ((1 - p ** (N + 1)) / (1 - p)) / (1 + 0.1 * N)) <= 1e-12
    # every other chain length is no better
    for n in range(1, 41):
        assert ((1 - p ** n) / (1 - p)) / (1 + 0.1 * (n - 1)) <= sp + 1e-12


def test_speedup_limits():
    # p -> 1: the speedup grows towards 1/alpha and never reaches it (the pages' ceiling)
    parent, rank, value, sp = oracle.tree_shape_for_cost([1.0], 60, None, 0.0, 0.1)
    assert len(parent) == 60 and sp < 10.0 and sp > 8.5
    # no verification overhead and free drafting: the largest best tree wins
    acc = [0.6, 0.25, 0.1]
    _, _, v_all = oracle.tree_shape_dp(acc, 12, 4)
    parent, rank, value, sp = oracle.tree_shape_for_cost(acc, 12, 4, 0.0, 0.0)
    assert value == v_all and sp == 1.0 + v_all
    # drafting that costs a whole decode step halves the speedup of a one-node tree
    assert oracle.step_speedup(0.0, 1, 1.0, 0.1) == 0.5


def test_merging_two_drafts_gives_the_pages_five_node_tree():
    """Two drafts A1 A2 and B1 B2 merge into the blog's tree T0 -> A1 -> A2,
    T0 -> B1 -> B2 (section 3, "Tree Attention Verification Matrix"), whose
    ancestor mask is the one the pages print."""
    from helpers import golden_lines
    A1, A2, B1, B2 = 101, 102, 201, 202
    parent, tokens, node_of = oracle.merge_sequences([[A1, A2], [B1, B2]])
    assert tokens.tolist() == [-1, A1, A2, B1, B2]
    assert parent.tolist() == [-1, 0, 1, 0, 3]
    assert node_of == [[1, 2], [3, 4]]
    rows = list(golden_lines("tree_mask_5node.txt"))
    assert [int(x) for x in rows[0][1:]] == parent.tolist()  # the golden file's parent line
    want = [[int(x) for x in row[1:]] for row in rows[1:]]
    assert oracle.tree_mask(parent).tolist() == want


def test_merged_prefixes_are_shared():
    rng = np.random.default_rng(9)
    seqs = [list(rng.integers(0, 3, rng.integers(0, 7))) for _ in range(12)]
    seqs.append(list(seqs[0]))  # a repeated draft adds nothing
    parent, tokens, node_of = oracle.merge_sequences(seqs)
    prefixes = {tuple(s[:j + 1]) for s in seqs for j in range(len(s))}
    assert len(parent) == 1 + len(prefixes)
    assert all(0 <= parent[c] < c for c in range(1, len(parent)))
    for s, nodes in zip(seqs, node_of):
        # every draft is a root path of the tree
        u = 0
        for t, v in zip(s, nodes):
            assert parent[v] == u and tokens[v] == t
            u = v
    # siblings carry distinct tokens
    seen = set()
    for c in range(1, len(parent)):
        assert (parent[c], tokens[c]) not in seen
        seen.add((parent[c], tokens[c]))


def test_tree_versus_chain_matches_the_pages():
    """Glossary, "linear vs tree" table and FAQ Q1: a tree yields 20-80 % more
    expected accepted tokens than a chain, and pays mostly at moderate
    acceptance (0.5-0.8); at 0.9 and above a chain is enough.  Under the
    positional model, at 32 nodes: moderate first-rank acceptance gives trees
    20-80 % ahead of the chain of the same size; at 0.95 the best tree is a chain."""
    for acc in ([0.6, 0.2, 0.1], [0.5, 0.25, 0.1, 0.05], [0.7, 0.15, 0.05]):
        _, _, v = oracle.tree_shape_dp(acc, 32)
        a = acc[0]
        chain = (1 - a ** 32) / (1 - a)  # tokens per step of a 32-node chain, the pages' formula
        assert 1.2 <= (1 + v) / chain <= 1.8, acc
    for n in (16, 32, 64):
        parent, _, _ = oracle.tree_shape_dp([0.95, 0.03, 0.01], n)
        assert parent.tolist() == [-1] + list(range(n - 1))


def test_selection_is_the_first_candidates_of_the_score_order():
    """With probabilities in [0, 1] every parent precedes its children in the
    (score descending, index ascending) order, so the selected set is exactly
    the first budget - 1 candidates of that order (the property the GPU
    selection relies on), here checked on the oracle's own output."""
    rng = np.random.default_rng(31)
    for trial in range(40):
        M = int(rng.integers(0, 300))
        par = np.array([int(rng.integers(-1, c)) if c else -1 for c in range(M)], np.int32)
        prob = (rng.integers(0, 5, M) / 4.0) if trial % 2 else rng.random(M) ** 2
        tok = np.arange(M, dtype=np.int32)
        budget = int(rng.integers(1, 80))
        _, _, index, _ = oracle.select_tree(par, tok, prob, budget)
        score = np.zeros(M)
        for c in range(M):
            score[c] = (score[par[c]] if par[c] >= 0 else 1.0) * prob[c]
        order = sorted(range(M), key=lambda c: (-score[c], c))
        assert list(index[1:]) == order[: budget - 1]

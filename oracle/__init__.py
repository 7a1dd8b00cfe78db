"""CPU oracle for the tree-verification step (fp64, plain C).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may call it; the library under test never does.
It shares no code with the CUDA path; both read inputs from ``synth``.

Functions and what each follows (all pages are about tree-based speculative
decoding):

* :func:`tree_mask` -- the mask definition M[i][j] = 1 iff node j is node i or
  an ancestor of i (glossary page, "Tree attention"), whose 5-node instance is
  the blog's "Tree Attention Verification Matrix" (section 3).
* :func:`tree_attention` -- every node attends to the whole prefix plus its own
  root path in one pass (glossary, "Tree attention"); plain masked softmax
  attention with a dense mask, accumulated in fp64.
* :func:`verify_sample` -- the acceptance rule min(1, p/q) and the
  renormalised residual max(0, p - q) (blog section 2, "Rejection Sampling
  Acceptance Condition"), applied root-down with sibling retries (glossary,
  "SpecInfer").

* :func:`verify_sample_logits` -- the same walk on the row softmax of the two
  models' logits (p and q are the models' output distributions).
* :func:`commit_path` -- the accepted path joins the cached prefix (blog,
  "KV cache management and prefix sharing"; glossary, "KV cache management
  challenges").
* :func:`tree_attention_ragged`, :func:`verify_sample_ragged`,
  :func:`commit_path_ragged`, :func:`chain_parents` -- ragged batches (each
  sequence its own tree) and chains (linear speculation).
* :func:`topk_rows`, :func:`fill_topk_tokens` -- top-k branching (glossary,
  tree-structure optimisation, "Top-k branching").
* :func:`tree_shape_dp`, :func:`tree_value` -- the budget-constrained tree shape
  by dynamic programming (glossary, "Budget-constrained optimisation").
* :func:`step_speedup`, :func:`tree_shape_for_cost` -- the step's speedup
  over plain decoding and the tree size that maximises it (LLM Primer VI
  ch. 9, 9.3).
* :func:`merge_sequences` -- SpecInfer's token tree: several drafts' sequences
  merged on their common prefixes (glossary, "SpecInfer").
* :func:`select_tree` -- the dynamic tree: the best-scoring ancestor-closed
  candidates under a node budget (LLM Primer VI ch. 9, 9.2, EAGLE-2).

Every function is pinned by ``tests/test_oracle_*.py`` against values the
pages print, closed forms, exhaustive search and library routines.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

OK, ERR_ARG, ERR_TREE, ERR_BLOCK = 0, 1, 3, 4


def build(force: bool = False, extra_flags=(), out: str | None = None) -> str:
    """Compile the oracle with gcc (fp64, OpenMP, no fast-math)."""
    src = os.path.join(_HERE, "oracle.c")
    out = out or _LIB_PATH
    if force or extra_flags or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", *extra_flags, "-o", out, src, "-lm"])
    return out


def _bind(path):
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    L.or_tree_mask.argtypes = [i32, P, P]
    L.or_tree_attention.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, dbl, i64, P, P]
    L.or_verify_sample.argtypes = [i32, i32, i64, P, P, P, P, P, dbl, P, P, P, P, P]
    L.or_commit_path.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P]
    L.or_set_threads.argtypes = [ctypes.c_int]
    L.or_max_threads.restype = ctypes.c_int
    return L


_lib = None


def lib():
    """The oracle library; ``ORACLE_LIB`` may name another build of
    ``oracle.c`` (the mutation tests point it at planted-mistake builds)."""
    global _lib
    if _lib is None:
        _lib = _bind(os.environ.get("ORACLE_LIB") or build())
    return _lib


def load_variant(path: str):
    """Bind a separately compiled oracle build (used by the mutation tests)."""
    return _bind(path)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    lib().or_set_threads(int(n))


def max_threads() -> int:
    return int(lib().or_max_threads())


def tree_mask(parent, L=None) -> np.ndarray:
    parent = np.ascontiguousarray(parent, dtype=np.int32)
    n = parent.shape[0]
    m = np.zeros((n, n), dtype=np.uint8)
    rc = (L or lib()).or_tree_mask(n, _p(parent), _p(m))
    if rc:
        raise ValueError(f"invalid tree (code {rc})")
    return m


def tree_attention(query, k_cache, v_cache, block_table, prefix_lens, parent_idx, num_kv_heads,
                   dtype: str, scale: float | None = None, rows=None, L=None) -> np.ndarray:
    """fp64 tree attention.

    query [B][N][Hq][D], caches [num_blocks][bs][Hkv][D] (float32 arrays, or
    uint16 bfloat16 bits when dtype == "bf16"), block_table [B][max_blocks],
    prefix_lens [B], parent_idx [B][N].  ``rows`` is an optional int array of
    (b, i, h) triples; the result is then [n_rows][D], else [B][N][Hq][D]."""
    B, N, Hq, D = query.shape
    nb, bs, Hkv, D2 = k_cache.shape
    assert D2 == D and Hkv == num_kv_heads
    code = 0 if dtype == "bf16" else 1
    want = np.uint16 if code == 0 else np.float32
    q = np.ascontiguousarray(query, dtype=want)
    kc = np.ascontiguousarray(k_cache, dtype=want)
    vc = np.ascontiguousarray(v_cache, dtype=want)
    bt = np.ascontiguousarray(block_table, dtype=np.int32)
    pl = np.ascontiguousarray(prefix_lens, dtype=np.int32)
    pa = np.ascontiguousarray(parent_idx, dtype=np.int32)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is not None:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))
        out = np.zeros((r.shape[0], D), dtype=np.float64)
        n_rows = r.shape[0]
    else:
        r = None
        out = np.zeros((B, N, Hq, D), dtype=np.float64)
        n_rows = B * N * Hq
    rc = (L or lib()).or_tree_attention(B, N, Hq, Hkv, D, bs, bt.shape[1], nb, code, _p(q), _p(kc), _p(vc),
                                        _p(bt), _p(pl), _p(pa), float(scale), n_rows, _p(r), _p(out))
    if rc:
        raise ValueError(f"oracle tree_attention failed (code {rc})")
    return out


def verify_sample(p, q, tree_tokens, parent_idx, uniforms, eps: float = 1e-6, L=None):
    """Literal root-down acceptance walk in fp64.

    Returns a dict with accepted_path [B][N] (-1 padded), accepted_len [B],
    bonus_token [B], near [B] (threshold events within ``eps``), rows [B]
    (vocabulary rows read in full) and rc (0, or 3 when some tree was
    invalid)."""
    B, N, V = p.shape
    pp = np.ascontiguousarray(p, dtype=np.float32)
    qq = np.ascontiguousarray(q, dtype=np.float32)
    tt = np.ascontiguousarray(tree_tokens, dtype=np.int32)
    pa = np.ascontiguousarray(parent_idx, dtype=np.int32)
    uu = np.ascontiguousarray(uniforms, dtype=np.float32)
    path = np.zeros((B, N), dtype=np.int32)
    alen = np.zeros(B, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    near = np.zeros(B, dtype=np.int32)
    rows = np.zeros(B, dtype=np.int32)
    rc = (L or lib()).or_verify_sample(B, N, V, _p(pp), _p(qq), _p(tt), _p(pa), _p(uu), float(eps),
                                       _p(path), _p(alen), _p(bonus), _p(near), _p(rows))
    return {"accepted_path": path, "accepted_len": alen, "bonus_token": bonus, "near": near, "rows": rows, "rc": rc}


def commit_path(k_cache, v_cache, block_table, prefix_lens, accepted_path, accepted_len, L=None):
    """Move each sequence's accepted path into the cached prefix, in place on
    copies of the caches (oracle.c or_commit_path).  Caches [nb][16][Hkv][D]
    of any dtype (rows are moved as bytes).  Returns (k, v, new_prefix_lens,
    status)."""
    L = L or lib()
    k = np.ascontiguousarray(k_cache).copy()
    v = np.ascontiguousarray(v_cache).copy()
    bt = np.ascontiguousarray(block_table, np.int32)
    pl = np.ascontiguousarray(prefix_lens, np.int32)
    path = np.ascontiguousarray(accepted_path, np.int32)
    ln = np.ascontiguousarray(accepted_len, np.int32)
    nb, bs, hkv, d = k.shape
    assert bs == 16 and v.shape == k.shape
    B, N = path.shape
    new_pl = np.zeros(B, np.int32)
    st = L.or_commit_path(B, N, hkv, d, bt.shape[1], nb, k.dtype.itemsize, _p(k), _p(v), _p(bt), _p(pl), _p(path),
                          _p(ln), _p(new_pl))
    return k, v, new_pl, int(st)


def chain_parents(B: int, N: int) -> np.ndarray:
    """Parent arrays of B chains of N nodes (linear speculation: node i's parent
    is i - 1), the tree a NULL parent array stands for in the library."""
    return np.tile(np.arange(-1, N - 1, dtype=np.int32), (B, 1))


def _seq_parent(parent_idx, b: int, n: int) -> np.ndarray:
    return chain_parents(1, n) if parent_idx is None else np.asarray(parent_idx, np.int32)[b:b + 1, :n]


def tree_attention_ragged(query, k_cache, v_cache, block_table, prefix_lens, parent_idx, node_counts, num_kv_heads,
                          dtype: str, scale: float | None = None) -> np.ndarray:
    """Ragged trees in one batch: sequence b's tree is its first node_counts[b]
    nodes, and by the definition of tree attention (glossary, "Tree attention")
    each sequence is its own problem, so this is :func:`tree_attention` on each
    sequence's slice.  parent_idx None means chains.  Rows of padding nodes are
    NaN (not defined)."""
    B, N, Hq, D = query.shape
    out = np.full((B, N, Hq, D), np.nan)
    for b in range(B):
        n = int(node_counts[b])
        if n == 0:
            continue
        out[b, :n] = tree_attention(query[b:b + 1, :n], k_cache, v_cache, np.asarray(block_table)[b:b + 1],
                                    np.asarray(prefix_lens)[b:b + 1], _seq_parent(parent_idx, b, n), num_kv_heads,
                                    dtype, scale)[0]
    return out


def verify_sample_ragged(p, q, tree_tokens, parent_idx, uniforms, node_counts, eps: float = 1e-6,
                         logits: bool = False):
    """The walk on ragged trees: sequence b's tree is its first node_counts[b]
    nodes (children past it do not exist); each sequence walks on its own
    slice with :func:`verify_sample` (or :func:`verify_sample_logits`).  A
    sequence with no nodes accepts nothing and draws no token (length 0,
    bonus -1).  parent_idx None means chains."""
    B, N = np.asarray(tree_tokens).shape
    res = {"accepted_path": np.full((B, N), -1, np.int32), "accepted_len": np.zeros(B, np.int32),
           "bonus_token": np.full(B, -1, np.int32), "near": np.zeros(B, np.int32), "rows": np.zeros(B, np.int32),
           "rc": 0}
    walk = verify_sample_logits if logits else verify_sample
    for b in range(B):
        n = int(node_counts[b])
        if n == 0:
            continue
        r = walk(np.asarray(p)[b:b + 1, :n], np.asarray(q)[b:b + 1, :n], np.asarray(tree_tokens)[b:b + 1, :n],
                 _seq_parent(parent_idx, b, n), np.asarray(uniforms)[b:b + 1, :n], eps=eps)
        res["accepted_path"][b, :n] = r["accepted_path"][0]
        for key in ("accepted_len", "bonus_token", "near", "rows"):
            res[key][b] = r[key][0]
        res["rc"] = res["rc"] or r["rc"]
    return res


def commit_path_ragged(k_cache, v_cache, block_table, prefix_lens, accepted_path, accepted_len, node_counts):
    """The KV commit on ragged trees: each sequence is committed on its own
    with :func:`commit_path` over its node_counts[b]-node tree (its blocks are
    its own, so the order does not matter).  Returns (k, v, new_prefix_lens,
    status)."""
    k = np.ascontiguousarray(k_cache).copy()
    v = np.ascontiguousarray(v_cache).copy()
    pl = np.asarray(prefix_lens, np.int32)
    path = np.asarray(accepted_path, np.int32)
    alen = np.asarray(accepted_len, np.int32)
    B = path.shape[0]
    new_pl = pl.copy()
    st = 0
    for b in range(B):
        n = int(node_counts[b])
        if n == 0 or alen[b] < 0:
            continue
        k, v, npl, s = commit_path(k, v, np.asarray(block_table)[b:b + 1], pl[b:b + 1], path[b:b + 1, :n],
                                   alen[b:b + 1])
        new_pl[b] = npl[0]
        st = st or s
    return k, v, new_pl, st


def topk_rows(x, k: int):
    """Top-k of each row of x [..][V]: (indices, values), values descending and
    equal values by ascending index (a stable sort of -x)."""
    x = np.asarray(x)
    V = x.shape[-1]
    flat = x.reshape(-1, V)
    idx = np.empty((flat.shape[0], k), np.int32)
    for r in range(flat.shape[0]):
        idx[r] = np.argsort(-flat[r].astype(np.float64), kind="stable")[:k]
    vals = np.take_along_axis(flat, idx.astype(np.int64), axis=1)
    return idx.reshape(x.shape[:-1] + (k,)), vals.reshape(x.shape[:-1] + (k,))


def fill_topk_tokens(q, parent_idx, rank, node_counts=None) -> np.ndarray:
    """Top-k branching (glossary "Tree-based speculative decoding", section on
    tree-structure optimisation, "Top-k branching": each node expands the draft
    model's top-k tokens as its children).  Child c of node u with rank r gets
    the r-th most probable token of u's draft distribution q[b][u] (r = 0 the
    most probable; ties by lower token id).  Returns tree_tokens [B][N] with
    the root's entry 0 and padding nodes -1."""
    q = np.asarray(q)
    B, N, V = q.shape
    par = np.asarray(parent_idx, np.int32)
    rk = np.asarray(rank, np.int32)
    tokens = np.full((B, N), -1, np.int32)
    for b in range(B):
        n = N if node_counts is None else int(node_counts[b])
        if n == 0:
            continue
        tokens[b, 0] = 0
        for u in range(n):
            kids = [c for c in range(1, n) if par[b, c] == u]
            if not kids:
                continue
            kk = max(int(rk[b, c]) for c in kids) + 1
            idx, _ = topk_rows(q[b, u], kk)
            for c in kids:
                tokens[b, c] = idx[int(rk[b, c])]
    return tokens


def tree_value(parent, rank, accept) -> float:
    """Expected accepted tokens of a tree under positional acceptance: the sum
    over non-root nodes of the product, along the root path, of accept[rank] of
    each edge (the rank-r candidate of a node is accepted with probability
    accept[r], whatever the depth)."""
    n = len(parent)
    reach = np.zeros(n)
    reach[0] = 1.0
    for c in range(1, n):
        reach[c] = reach[parent[c]] * accept[rank[c]]
    return float(reach[1:].sum())


def tree_shape_dp(accept, budget: int, max_depth: int | None = None):
    """Budget-constrained tree shape (glossary, "Budget-constrained
    optimisation": allocate branches under a node budget so that the whole
    tree's expected accepted tokens is largest; solved by dynamic programming,
    as Sequoia does).  accept[r] is the probability that a node's rank-r
    candidate is accepted (positional acceptance, independent of depth); a node
    has children of ranks 0..m-1 (m <= len(accept)); the tree has at most
    `budget` nodes (root included) and depth at most max_depth.

    F[d][n]: best value of a subtree of exactly n nodes with at most d levels
    below its root; G[i][s]: best value of children of ranks i.. holding s
    nodes in all.  F[d][n] = G[0][n - 1] with G[i][s] = max over t of
    accept[i] * (1 + F[d-1][t]) + G[i+1][s-t].  Ties go to the smallest t and
    the smallest total size.  Returns (parent, rank, value): nodes numbered by
    depth, then by the ranks along their path."""
    accept = [float(a) for a in accept]
    k = len(accept)
    D = budget - 1 if max_depth is None else min(max_depth, budget - 1)
    NEG = float("-inf")
    F = [[NEG] * (budget + 1) for _ in range(D + 1)]
    choice = [None] * (D + 1)  # choice[d][i][s] = t
    for d in range(D + 1):
        F[d][1] = 0.0
        if d == 0:
            continue
        G = [[NEG] * budget for _ in range(k + 1)]
        ch = [[0] * budget for _ in range(k + 1)]
        G[k][0] = 0.0
        for i in range(k - 1, -1, -1):
            G[i][0] = 0.0
            for s in range(1, budget):
                best, arg = NEG, 0
                for t in range(1, s + 1):
                    if F[d - 1][t] == NEG or G[i + 1][s - t] == NEG:
                        continue
                    v = accept[i] * (1.0 + F[d - 1][t]) + G[i + 1][s - t]
                    if v > best:
                        best, arg = v, t
                G[i][s], ch[i][s] = best, arg
        for n in range(2, budget + 1):
            F[d][n] = G[0][n - 1]
        choice[d] = ch
    n_best = max(range(1, budget + 1), key=lambda n: (F[D][n], -n))
    # rebuild: children of a node with d levels and n nodes, rank by rank
    paths = []  # (path of ranks, ) for every node

    def build(path, d, n):
        paths.append(path)
        s, i = n - 1, 0
        while s > 0:
            t = choice[d][i][s]
            build(path + (i,), d - 1, t)
            s -= t
            i += 1

    build((), D, n_best)
    paths.sort(key=lambda pth: (len(pth), pth))
    index = {pth: j for j, pth in enumerate(paths)}
    parent = np.array([-1] + [index[pth[:-1]] for pth in paths[1:]], np.int32)
    rank = np.array([-1] + [pth[-1] for pth in paths[1:]], np.int32)
    return parent, rank, F[D][n_best]


def step_speedup(expected_accepted: float, num_nodes: int, draft_cost: float, alpha: float) -> float:
    """Speedup of one speculative step over plain decoding (LLM Primer VI
    ch. 9, 9.3): tokens emitted per step over the step's cost in decode steps,
    (1 + E) / (draft_cost + 1 + alpha * N), where E is the expected accepted
    tokens, the 1 is the bonus token, N = num_nodes - 1 draft tokens,
    draft_cost = T_draft / T_decode and alpha the verification overhead per
    position."""
    return (1.0 + expected_accepted) / (draft_cost + 1.0 + alpha * (num_nodes - 1))


def tree_shape_for_cost(accept, max_budget: int, max_depth: int | None, draft_cost: float, alpha: float):
    """The tree size that pays (LLM Primer VI ch. 9, 9.3: a fixed N misses the
    optimum; the glossary: Sequoia sizes the tree for the hardware): for every
    budget n = 1..max_budget take :func:`tree_shape_dp`'s tree and its
    :func:`step_speedup`; return the first best one as (parent, rank, value,
    speedup)."""
    best = None
    for n in range(1, max_budget + 1):
        parent, rank, value = tree_shape_dp(accept, n, max_depth)
        sp = step_speedup(value, len(parent), draft_cost, alpha)
        if best is None or sp > best[3]:
            best = (parent, rank, value, sp)
    return best


def merge_sequences(seqs):
    """SpecInfer's token tree (glossary "Tree-based speculative decoding",
    section "SpecInfer", token tree construction): every draft model generates
    its own candidate sequence and the sequences are merged, candidates with a
    common prefix sharing those nodes.  Node 0 is the root (the last committed
    token); nodes are created in input order, each the first time its prefix
    appears.  Returns (parent_idx, tree_tokens, node_of): node_of[k][j] is the
    node of token j of sequence k."""
    parent, tokens = [-1], [-1]
    child = {}
    node_of = []
    for seq in seqs:
        u = 0
        path = []
        for t in seq:
            key = (u, int(t))
            if key not in child:
                child[key] = len(parent)
                parent.append(u)
                tokens.append(int(t))
            u = child[key]
            path.append(u)
        node_of.append(path)
    return np.array(parent, np.int32), np.array(tokens, np.int32), node_of


def select_tree(cand_parent, cand_token, cand_prob, budget: int):
    """Dynamic tree selection from a grown candidate set (EAGLE-2's dynamic
    draft tree, LLM Primer VI ch. 9, 9.2; scored as the glossary's
    budget-constrained optimisation, "the whole tree's expected accepted
    tokens under a node budget").  Candidates 0..M-1 are topological
    (cand_parent[c] < c, -1 = a child of the root); a candidate's score is the
    product of cand_prob along its path (the draft's estimate that it is
    accepted).  Take candidates by descending score, equal scores by lower
    index, each one only if its parent is already in, until the tree holds
    `budget` nodes with the root.  Returns (parent_idx, tree_tokens,
    cand_index, value): node 0 is the root (parent -1, token -1, index -1),
    nodes 1.. the selected candidates in the order taken; value = the sum of
    their scores."""
    par = [int(x) for x in cand_parent]
    prob = [float(x) for x in cand_prob]
    M = len(par)
    score = [0.0] * M
    for c in range(M):
        score[c] = (score[par[c]] if par[c] >= 0 else 1.0) * prob[c]
    order = sorted(range(M), key=lambda c: (-score[c], c))
    node_of = {}
    taken = []
    for c in order:
        if len(taken) >= budget - 1:
            break
        if par[c] < 0 or par[c] in node_of:
            node_of[c] = len(taken) + 1
            taken.append(c)
    parent = np.array([-1] + [0 if par[c] < 0 else node_of[par[c]] for c in taken], np.int32)
    tokens = np.array([-1] + [int(cand_token[c]) for c in taken], np.int32)
    index = np.array([-1] + taken, np.int32)
    value = 0.0
    for c in taken:
        value += score[c]
    return parent, tokens, index, value


def softmax_rows(logits) -> np.ndarray:
    """Plain softmax over the last axis in fp64 (max-shifted), rounded to fp32:
    the distributions a verifier that takes logits works from."""
    x = np.asarray(logits, dtype=np.float64)
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)


def verify_sample_logits(target_logits, draft_logits, tree_tokens, parent_idx, uniforms, eps: float = 1e-6,
                         L=None):
    """The acceptance walk on p = softmax(target_logits), q =
    softmax(draft_logits) (row-wise, temperature 1): the fused-logits form of
    the step (the glossary's and the blog's p and q are the two models' output
    distributions).  Same outputs as verify_sample."""
    return verify_sample(softmax_rows(target_logits), softmax_rows(draft_logits), tree_tokens, parent_idx, uniforms,
                         eps=eps, L=L)

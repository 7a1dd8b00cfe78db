"""Seeded synthetic inputs for the tree-verification step.

Both sides of every parity check read their inputs from here: the CUDA
library (through the tests and ``bench.py``) and the CPU oracle.  The module
holds no arithmetic of the method itself; it only draws shapes, trees, KV
caches and distributions from Philox4x32-10 (see ``synth.c``).

Workloads follow the five shapes the verification step is quoted on:

====  =====================================================================
name  shape
====  =====================================================================
tiny  batch 1, prefix 128, Hq 8 / Hkv 2, D 64, fp32, the 5-node tree
      T0->A1->A2, T0->B1->B2, vocab 1000, p and q independent softmax(N(0,2))
l8b   batch 1, prefix 4096 (contiguous), Hq 32 / Hkv 8, D 128, bf16,
      64-node top-k [4,3,2,2,1,1] tree, vocab 128256,
      p = softmax(N(0,3)), q = softmax(logits + N(0,1))
l70b  batch 8, prefix 8192 each, Hq 64 / Hkv 8, D 128, bf16, paged with a
      permuted block table, 32-node DFS trees (1..4 children, depth 5),
      vocab 128256, p/q as l8b
mix   batch 64, prefix ~ U{512..32768}, Hq 32 / Hkv 8, D 128, bf16, paged,
      16-node trees of depth U{2..6}, vocab 151936,
      p = softmax(N(0,4)), q = softmax(logits + N(0,1.5))
long  batch 1, prefix 131072, Hq 64 / Hkv 8, D 128, bf16, paged, 128-node
      greedy budget tree (depth <= 6, <= 4 children), vocab 128256, p/q as l8b
====  =====================================================================

One more shape, outside the five (``RAGGED_NAMES``): mixed serving with trees
of different sizes in one call.

======  ===================================================================
ragged  batch 32, prefix ~ U{512..32768}, Hq 32 / Hkv 8, D 128, bf16, paged,
        capacity 32 nodes, n_b ~ U{1..32} nodes per sequence; every fourth
        sequence a chain (linear speculation), the rest DFS trees of depth
        U{2..6}; padding slots hold parent -1 and token -1; vocab 151936,
        p/q as mix
======  ===================================================================
"""
from __future__ import annotations

import ctypes
import heapq
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

# stream ids (the Philox key's second word)
STREAM_QUERY = 1
STREAM_K = 2
STREAM_V = 3
STREAM_LOGIT = 4
STREAM_NOISE = 5
STREAM_UNIFORM = 6
STREAM_TREE = 7
STREAM_TOKEN = 8
STREAM_PERM = 9
STREAM_LEN = 10

BLOCK_SIZE = 16


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` with gcc (OpenMP) if missing or stale."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", _LIB_PATH, src, "-lm"])
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i64, u64, u32, i32, dbl = ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_double
        L.sy_philox4x32_10.argtypes = [P, P, P]
        L.sy_uniform_f32.argtypes = [P, i64, u64, u32, i64]
        L.sy_words_u32.argtypes = [P, i64, u64, u32, i64]
        L.sy_normal_f32.argtypes = [P, i64, u64, u32, i64, dbl]
        L.sy_normal_bf16.argtypes = [P, i64, u64, u32, i64, dbl]
        L.sy_paged_cache.argtypes = [P, ctypes.c_int, i32, i32, i32, i32, i32, P, P, i64, u64, u32, dbl]
        L.sy_pq_rows.argtypes = [P, P, i64, P, i64, u64, u32, u32, ctypes.c_int, dbl, dbl]
        L.sy_logit_rows.argtypes = [P, P, i64, P, i64, u64, u32, u32, ctypes.c_int, dbl, dbl]
        L.sy_categorical.argtypes = [P, i64, dbl]
        L.sy_categorical.restype = i64
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- primitives

def philox4x32_10(ctr, key) -> np.ndarray:
    c = np.asarray(ctr, dtype=np.uint32).copy()
    k = np.asarray(key, dtype=np.uint32).copy()
    out = np.zeros(4, dtype=np.uint32)
    lib().sy_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniforms(n: int, seed: int, stream: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    if n:
        lib().sy_uniform_f32(_ptr(out), n, seed, stream, offset)
    return out


def words(n: int, seed: int, stream: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.uint32)
    if n:
        lib().sy_words_u32(_ptr(out), n, seed, stream, offset)
    return out


def normals(n: int, seed: int, stream: int, offset: int = 0, std: float = 1.0, bf16: bool = False) -> np.ndarray:
    if bf16:
        out = np.empty(n, dtype=np.uint16)
        if n:
            lib().sy_normal_bf16(_ptr(out), n, seed, stream, offset, std)
    else:
        out = np.empty(n, dtype=np.float32)
        if n:
            lib().sy_normal_f32(_ptr(out), n, seed, stream, offset, std)
    return out


def pq_rows(row_ids, V: int, seed: int, mode: int, sp: float, sn: float):
    row_ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    R = row_ids.shape[0]
    p = np.empty((R, V), dtype=np.float32)
    q = np.empty((R, V), dtype=np.float32)
    if R:
        lib().sy_pq_rows(_ptr(p), _ptr(q), R, _ptr(row_ids), V, seed, STREAM_LOGIT, STREAM_NOISE, mode, sp, sn)
    return p, q


def logit_rows(row_ids, V: int, seed: int, mode: int, sp: float, sn: float):
    """The logits whose row softmaxes pq_rows returns (target, draft), float32."""
    row_ids = np.ascontiguousarray(np.asarray(row_ids, dtype=np.int64))
    R = row_ids.shape[0]
    la = np.empty((R, V), dtype=np.float32)
    lb = np.empty((R, V), dtype=np.float32)
    if R:
        lib().sy_logit_rows(_ptr(la), _ptr(lb), R, _ptr(row_ids), V, seed, STREAM_LOGIT, STREAM_NOISE, mode, sp, sn)
    return la, lb


def categorical(w: np.ndarray, u: float) -> int:
    w = np.ascontiguousarray(w, dtype=np.float32)
    return int(lib().sy_categorical(_ptr(w), w.shape[0], float(u)))


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns (uint16) to float32."""
    return (a.astype(np.uint32) << 16).view(np.float32)


class _Draws:
    """Sequential reader over one Philox stream (offset = base + k)."""

    def __init__(self, seed: int, stream: int, base: int):
        self.seed, self.stream, self.base, self.k = seed, stream, base, 0

    def uniform(self) -> float:
        u = float(uniforms(1, self.seed, self.stream, self.base + self.k)[0])
        self.k += 1
        return u

    def randint(self, lo: int, hi: int) -> int:
        """Integer uniform in [lo, hi] inclusive."""
        return lo + min(int(self.uniform() * (hi - lo + 1)), hi - lo)


# ---------------------------------------------------------------- trees

def topk_tree(branching, budget: int):
    """Top-k tree with per-depth branching, truncated to ``budget`` nodes.

    The full tree gives node at depth d (1-based) ``branching[d-1]`` children
    ranked 0..k-1.  Nodes are kept by priority (sum of sibling ranks along the
    path, then depth, then the rank path itself) and numbered breadth-first.
    Returns (parent, rank) lists; the root has parent -1 and rank -1.
    """
    paths = [()]
    frontier = [()]
    for k in branching:
        nxt = []
        for pth in frontier:
            for r in range(k):
                nxt.append(pth + (r,))
        paths.extend(nxt)
        frontier = nxt
    kept = sorted(paths[1:], key=lambda pth: (sum(pth), len(pth), pth))[: budget - 1]
    kept = sorted(kept, key=lambda pth: (len(pth), pth))
    index = {(): 0}
    parent, rank = [-1], [-1]
    for pth in kept:
        index[pth] = len(parent)
        parent.append(index[pth[:-1]])
        rank.append(pth[-1])
    return parent, rank


def dfs_tree(draws: _Draws, n_nodes: int, max_depth: int, kmin: int = 1, kmax: int = 4):
    """Depth-first growth: each node below ``max_depth`` draws U{kmin..kmax}
    children, nodes are numbered in creation order, growth stops at
    ``n_nodes``.  If the pass ends short, further passes over the existing
    nodes in index order give each node above the depth cap one more child
    until the budget is met."""
    parent, depth = [-1], [0]

    def grow(u):
        if depth[u] >= max_depth:
            return
        k = draws.randint(kmin, kmax)
        for _ in range(k):
            if len(parent) >= n_nodes:
                return
            parent.append(u)
            depth.append(depth[u] + 1)
            grow(len(parent) - 1)

    grow(0)
    while len(parent) < n_nodes:
        for u in range(len(parent)):
            if len(parent) >= n_nodes:
                break
            if depth[u] < max_depth:
                parent.append(u)
                depth.append(depth[u] + 1)
    return parent


# ---------------------------------------------------------------- workloads

@dataclass
class Workload:
    name: str
    batch: int
    num_nodes: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str            # "f32" or "bf16"
    vocab: int
    prefix_lens: np.ndarray        # int32 [B]
    block_table: np.ndarray        # int32 [B][max_blocks], -1 = unused
    num_blocks: int
    parent_idx: np.ndarray         # int32 [B][N]
    tree_tokens: np.ndarray        # int32 [B][N]
    seed: int
    kv_std: float
    pq_mode: int
    pq_sp: float
    pq_sn: float
    paged: bool
    row_keys: np.ndarray           # int64 [B][N]: generator row key of each node's p/q
    extra: dict = field(default_factory=dict)
    node_counts: np.ndarray | None = None  # int32 [B] nodes per sequence (ragged workloads)
    tree_k_scale: float = 1.0      # keys of the tree block (positions L_b..L_b+n_b-1) are multiplied by this

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def counts(self) -> np.ndarray:
        """Nodes per sequence (num_nodes for every sequence unless ragged)."""
        if self.node_counts is None:
            return np.full(self.batch, self.num_nodes, dtype=np.int32)
        return self.node_counts

    @property
    def seq_tokens(self) -> np.ndarray:
        return (self.prefix_lens + self.counts).astype(np.int32)

    # ---- attention inputs
    def query(self) -> np.ndarray:
        n = self.batch * self.num_nodes * self.num_q_heads * self.head_dim
        a = normals(n, self.seed, STREAM_QUERY, 0, 1.0, bf16=(self.dtype == "bf16"))
        return a.reshape(self.batch, self.num_nodes, self.num_q_heads, self.head_dim)

    def _cache(self, stream: int) -> np.ndarray:
        shape = (self.num_blocks, BLOCK_SIZE, self.num_kv_heads, self.head_dim)
        bf = self.dtype == "bf16"
        out = np.zeros(shape, dtype=np.uint16 if bf else np.float32)
        bt = np.ascontiguousarray(self.block_table, dtype=np.int32)
        st = np.ascontiguousarray(self.seq_tokens, dtype=np.int32)
        lib().sy_paged_cache(_ptr(out), 0 if bf else 1, self.batch, self.max_blocks, BLOCK_SIZE,
                             self.num_kv_heads, self.head_dim, _ptr(bt), _ptr(st),
                             self.max_blocks * BLOCK_SIZE, self.seed, stream, self.kv_std)
        return out

    def k_cache(self) -> np.ndarray:
        k = self._cache(STREAM_K)
        if self.tree_k_scale != 1.0:
            # scale the tree block's keys in place; a power-of-two factor is exact in bf16 and fp32
            bf = self.dtype == "bf16"
            for b in range(self.batch):
                L, n = int(self.prefix_lens[b]), int(self.counts[b])
                for t in range(L, L + n):
                    blk, slot = int(self.block_table[b, t // BLOCK_SIZE]), t % BLOCK_SIZE
                    row = bf16_to_f32(k[blk, slot]) if bf else k[blk, slot]
                    row = (row * np.float32(self.tree_k_scale)).astype(np.float32)
                    k[blk, slot] = (row.view(np.uint32) >> 16).astype(np.uint16) if bf else row
        return k

    def v_cache(self) -> np.ndarray:
        return self._cache(STREAM_V)

    # ---- sampler inputs
    def pq(self):
        """(p, q) float32 [B][N][V]; generated once and cached."""
        if "pq" not in self.extra:
            p, q = pq_rows(self.row_keys.reshape(-1), self.vocab, self.seed, self.pq_mode, self.pq_sp, self.pq_sn)
            shape = (self.batch, self.num_nodes, self.vocab)
            self.extra["pq"] = (p.reshape(shape), q.reshape(shape))
        return self.extra["pq"]

    def logits(self):
        """(target, draft) logits float32 [B][N][V] whose row softmaxes are pq()."""
        if "logits" not in self.extra:
            la, lb = logit_rows(self.row_keys.reshape(-1), self.vocab, self.seed, self.pq_mode, self.pq_sp, self.pq_sn)
            shape = (self.batch, self.num_nodes, self.vocab)
            self.extra["logits"] = (la.reshape(shape), lb.reshape(shape))
        return self.extra["logits"]

    def uniforms(self) -> np.ndarray:
        return uniforms(self.batch * self.num_nodes, self.seed, STREAM_UNIFORM).reshape(self.batch, self.num_nodes)


def _block_table(prefix_lens, n_nodes, permute, seed):
    """n_nodes: one tree size for all sequences, or one per sequence."""
    B = len(prefix_lens)
    nn = np.broadcast_to(np.asarray(n_nodes), (B,))
    nblk = [(int(L) + int(n) + BLOCK_SIZE - 1) // BLOCK_SIZE for L, n in zip(prefix_lens, nn)]
    total = sum(nblk)
    ids = np.arange(total, dtype=np.int64)
    if permute:  # Fisher-Yates driven by the PERM stream
        w = words(total, seed, STREAM_PERM)
        for i in range(total - 1, 0, -1):
            j = int(w[i]) % (i + 1)
            ids[i], ids[j] = ids[j], ids[i]
    mb = max(nblk)
    bt = np.full((B, mb), -1, dtype=np.int32)
    off = 0
    for b in range(B):
        bt[b, : nblk[b]] = ids[off: off + nblk[b]]
        off += nblk[b]
    return bt, total


CONFIG_NAMES = ("tiny", "l8b", "l70b", "mix", "long")
RAGGED_NAMES = ("ragged",)


UNIT_TREE_K_SCALE = 4.0


def make(name: str, seed: int | None = None, need_tokens: bool = True, unit_kv: bool = False) -> Workload:
    """Build the tree, lengths and block table of a named workload.

    Heavy tensors (KV cache, p/q) are produced on demand by the Workload
    methods so callers only pay for what they use.  ``seed`` defaults to the
    workload's index + 1.

    ``unit_kv`` gives the same shapes, tree and block table with K and V drawn
    from N(0, 1) instead of N(0, 1/128), and the tree block's keys multiplied
    by ``UNIT_TREE_K_SCALE``: attention outputs are then of order one and each
    row's ancestors carry a visible share of its softmax mass, so a wrong mask
    word, split merge or row mapping changes the output far beyond bf16
    rounding (with the default scales every output is an average of
    thousands of small values and such mistakes stay below 1e-2)."""
    if name in RAGGED_NAMES:
        wl = _make_ragged(name, 10 + RAGGED_NAMES.index(name) if seed is None else seed, need_tokens)
        return _unit(wl) if unit_kv else wl
    if name not in CONFIG_NAMES:
        raise ValueError(f"unknown workload {name!r}; choose from {CONFIG_NAMES + RAGGED_NAMES}")
    if seed is None:
        seed = CONFIG_NAMES.index(name) + 1
    if name == "tiny":
        B, N, Hq, Hkv, D, dt, V = 1, 5, 8, 2, 64, "f32", 1000
        prefix = np.array([128], dtype=np.int32)
        parents = np.array([[-1, 0, 1, 0, 3]], dtype=np.int32)
        mode, sp, sn, kv_std, paged = 0, 2.0, 0.0, 1.0, False
    elif name == "l8b":
        B, N, Hq, Hkv, D, dt, V = 1, 64, 32, 8, 128, "bf16", 128256
        prefix = np.array([4096], dtype=np.int32)
        par, rank = topk_tree([4, 3, 2, 2, 1, 1], 64)
        parents = np.array([par], dtype=np.int32)
        mode, sp, sn, kv_std, paged = 1, 3.0, 1.0, 1.0 / np.sqrt(128.0), False
    elif name == "l70b":
        B, N, Hq, Hkv, D, dt, V = 8, 32, 64, 8, 128, "bf16", 128256
        prefix = np.full(B, 8192, dtype=np.int32)
        parents = np.array([dfs_tree(_Draws(seed, STREAM_TREE, b << 20), N, 5) for b in range(B)], dtype=np.int32)
        mode, sp, sn, kv_std, paged = 1, 3.0, 1.0, 1.0 / np.sqrt(128.0), True
    elif name == "mix":
        B, N, Hq, Hkv, D, dt, V = 64, 16, 32, 8, 128, "bf16", 151936
        u = uniforms(B, seed, STREAM_LEN)
        prefix = (512 + np.minimum((u * (32768 - 512 + 1)).astype(np.int64), 32768 - 512)).astype(np.int32)
        plist = []
        for b in range(B):
            dr = _Draws(seed, STREAM_TREE, b << 20)
            depth = dr.randint(2, 6)
            plist.append(dfs_tree(dr, N, depth))
        parents = np.array(plist, dtype=np.int32)
        mode, sp, sn, kv_std, paged = 1, 4.0, 1.5, 1.0 / np.sqrt(128.0), True
    else:  # long
        B, N, Hq, Hkv, D, dt, V = 1, 128, 64, 8, 128, "bf16", 128256
        prefix = np.array([131072], dtype=np.int32)
        mode, sp, sn, kv_std, paged = 1, 3.0, 1.0, 1.0 / np.sqrt(128.0), True
        parents = None

    row_keys = (np.arange(B, dtype=np.int64)[:, None] * N + np.arange(N, dtype=np.int64)[None, :])
    extra = {}
    if name == "long":
        parents, tokens, row_keys = _greedy_budget_tree(seed, N, V, mode, sp, sn, max_depth=6, width=4)
        parents = parents[None, :]
        tokens = tokens[None, :]
        row_keys = row_keys[None, :]
    bt, nb = _block_table(prefix, N, paged, seed)
    wl = Workload(name, B, N, Hq, Hkv, D, dt, V, prefix, bt, nb, parents, None, seed, float(kv_std),
                  mode, sp, sn, paged, row_keys, extra)
    if name == "long":
        wl.tree_tokens = tokens.astype(np.int32)
    elif not need_tokens:
        wl.tree_tokens = np.zeros((B, N), dtype=np.int32)
    else:
        p, q = wl.pq()
        toks = np.zeros((B, N), dtype=np.int32)
        if name == "l8b":
            # children take the distinct top-k tokens of the parent's draft distribution, by rank
            for u_node in range(N):
                kids = [c for c in range(N) if parents[0, c] == u_node]
                if kids:
                    order = np.argsort(-q[0, u_node], kind="stable")
                    for c in kids:
                        toks[0, c] = order[rank[c]]
        else:
            # token of node c drawn from the draft distribution of its parent
            u = uniforms(B * N, seed, STREAM_TOKEN).reshape(B, N)
            for b in range(B):
                for c in range(1, N):
                    toks[b, c] = categorical(q[b, parents[b, c]], float(u[b, c]))
        wl.tree_tokens = toks
    return _unit(wl) if unit_kv else wl


def _unit(wl: Workload) -> Workload:
    wl.kv_std = 1.0
    wl.tree_k_scale = UNIT_TREE_K_SCALE
    return wl


def _make_ragged(name: str, seed: int, need_tokens: bool) -> Workload:
    B, N, Hq, Hkv, D, dt, V = 32, 32, 32, 8, 128, "bf16", 151936
    u = uniforms(2 * B, seed, STREAM_LEN)
    prefix = (512 + np.minimum((u[:B] * (32768 - 512 + 1)).astype(np.int64), 32768 - 512)).astype(np.int32)
    counts = (1 + np.minimum((u[B:] * N).astype(np.int64), N - 1)).astype(np.int32)
    parents = np.full((B, N), -1, dtype=np.int32)
    for b in range(B):
        n = int(counts[b])
        if b % 4 == 3:
            parents[b, :n] = np.arange(-1, n - 1)
        else:
            dr = _Draws(seed, STREAM_TREE, b << 20)
            parents[b, :n] = dfs_tree(dr, n, dr.randint(2, 6))
    row_keys = np.arange(B, dtype=np.int64)[:, None] * N + np.arange(N, dtype=np.int64)[None, :]
    bt, nb = _block_table(prefix, counts, True, seed)
    wl = Workload(name, B, N, Hq, Hkv, D, dt, V, prefix, bt, nb, parents, None, seed, float(1.0 / np.sqrt(128.0)),
                  1, 4.0, 1.5, True, row_keys, {}, counts)
    toks = np.full((B, N), -1, dtype=np.int32)
    toks[:, 0] = 0
    if need_tokens:
        p, q = wl.pq()
        ut = uniforms(B * N, seed, STREAM_TOKEN).reshape(B, N)
        for b in range(B):
            for c in range(1, int(counts[b])):
                toks[b, c] = categorical(q[b, parents[b, c]], float(ut[b, c]))
    wl.tree_tokens = toks
    return wl


def _greedy_budget_tree(seed, N, V, mode, sp, sn, max_depth, width):
    """Greedy budget tree: candidates are the top-``width`` tokens of each
    node's draft distribution, scored by the product of draft probabilities
    along the path; the best candidate becomes a node (max-heap, ties by
    insertion order) until N nodes exist; nodes deeper than ``max_depth`` are
    not expanded.  Nodes are renumbered breadth-first (children in creation
    order).  Each node's p/q key is its creation index."""
    created_parent, created_token, created_depth = [-1], [0], [0]
    heap = []
    tie = 0

    def push_children(node_id, score):
        nonlocal tie
        if created_depth[node_id] >= max_depth:
            return
        _, q = pq_rows([node_id], V, seed, mode, sp, sn)
        order = np.argsort(-q[0], kind="stable")[:width]
        for tok in order:
            s = score * float(q[0, tok])
            heapq.heappush(heap, (-s, tie, node_id, int(tok)))
            tie += 1

    push_children(0, 1.0)
    while len(created_parent) < N and heap:
        negs, _, par, tok = heapq.heappop(heap)
        nid = len(created_parent)
        created_parent.append(par)
        created_token.append(tok)
        created_depth.append(created_depth[par] + 1)
        push_children(nid, -negs)
    # breadth-first renumbering
    kids = {i: [] for i in range(len(created_parent))}
    for i in range(1, len(created_parent)):
        kids[created_parent[i]].append(i)
    order, queue = [], [0]
    while queue:
        u = queue.pop(0)
        order.append(u)
        queue.extend(kids[u])
    new_of = {old: new for new, old in enumerate(order)}
    parents = np.array([-1 if created_parent[o] < 0 else new_of[created_parent[o]] for o in order], dtype=np.int32)
    tokens = np.array([created_token[o] for o in order], dtype=np.int32)
    keys = np.array(order, dtype=np.int64)
    return parents, tokens, keys


def grown_candidates(batch: int, per_seq: int, width: int, seed: int):
    """Candidate sets for dynamic tree selection, grown as a draft model would
    grow them level by level: each level gives `width` children to the best
    third of the previous level's nodes (by path probability), each child's
    probability drawn from Philox as u**2 (a draft's top-k tail).  Returns
    (offsets [B+1], parent [sum], token [sum], prob [sum] float32); parent
    indices are local to the sequence (-1 = a child of the root)."""
    par_all, tok_all, prob_all, offs = [], [], [], [0]
    for b in range(batch):
        u = uniforms(2 * per_seq, seed, STREAM_TREE, b << 20)
        par, prob, score = [], [], []
        frontier = [(-1, 1.0)]
        while len(par) < per_seq:
            nxt = []
            for node, s in frontier:
                for _ in range(width):
                    if len(par) >= per_seq:
                        break
                    pr = float(np.float32(u[len(par)] ** 2))
                    par.append(node)
                    prob.append(pr)
                    nxt.append((len(par) - 1, s * pr))
            nxt.sort(key=lambda t: -t[1])
            frontier = nxt[: max(1, len(nxt) // 3)]
        par_all += par
        prob_all += prob
        tok_all += [int(w % 128256) for w in words(per_seq, seed, STREAM_TOKEN, b << 20)]
        offs.append(offs[-1] + per_seq)
    return (np.array(offs, np.int32), np.array(par_all, np.int32), np.array(tok_all, np.int32),
            np.array(prob_all, np.float32))

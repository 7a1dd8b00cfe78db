"""libtreeverify: the target model's verification step of tree-based
speculative decoding, as a CUDA library for one B200 (sm_100a).

This module is a thin ctypes binding over the C ABI in
``include/treeverify.h``: the functions named ``tv_*`` take the same
arguments as the C calls (device pointers taken from torch tensors, the
current torch CUDA stream unless another is given) and return the C status.
All computation happens in the library's kernels; torch only provides
device memory and streams.

Convenience wrappers :func:`tree_attention` and :func:`verify_sample`
allocate outputs/workspace with torch and raise on a non-OK status.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtreeverify.so")

TV_OK, TV_ERR_INVALID_ARG, TV_ERR_UNSUPPORTED, TV_ERR_TREE = 0, 1, 2, 3
TV_ERR_BLOCK_TABLE, TV_ERR_WORKSPACE, TV_ERR_CUDA, TV_ERR_TIMEOUT = 4, 5, 6, 7
TV_BF16, TV_F32 = 0, 1
TV_STATIC_SCRATCH_BYTES = 2 << 20


class TvAttnDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_nodes", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_blocks", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("node_counts", ctypes.c_void_p)]


class TvAttnPlan(ctypes.Structure):
    _fields_ = [("kernel", ctypes.c_int32), ("num_splits", ctypes.c_int32), ("row_tiles", ctypes.c_int32),
                ("grid_ctas", ctypes.c_int32), ("launches", ctypes.c_int32), ("workspace_bytes", ctypes.c_size_t)]


class TvSampleDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_nodes", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("node_counts", ctypes.c_void_p)]


class TvSamplePlan(ctypes.Structure):
    _fields_ = [("cluster_ctas", ctypes.c_int32), ("threads", ctypes.c_int32), ("slice", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32), ("launches", ctypes.c_int32)]


class TreeVerifyError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {tv_status_string(status)} (status {status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libtreeverify.so; raises if the library has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libtreeverify.so not built at {LIB_PATH}; run __graft_entry__.build() "
                              "or python -m tree_speculative_decoding_07_b200.build_lib")
        L = ctypes.CDLL(LIB_PATH)
        P, sz = ctypes.c_void_p, ctypes.c_size_t
        L.tv_tree_attention_plan.argtypes = [ctypes.POINTER(TvAttnDesc), ctypes.POINTER(TvAttnPlan)]
        L.tv_tree_attention_workspace_size.argtypes = [ctypes.POINTER(TvAttnDesc)]
        L.tv_tree_attention_workspace_size.restype = sz
        L.tv_tree_attention.argtypes = [ctypes.POINTER(TvAttnDesc), P, P, P, P, P, P, P, P, sz, P, P]
        L.tv_tree_attention_static.argtypes = [ctypes.POINTER(TvAttnDesc), P, P, P, P, P, P, P, P, P]
        L.tv_verify_sample_plan.argtypes = [ctypes.POINTER(TvSampleDesc), ctypes.POINTER(TvSamplePlan)]
        L.tv_verify_sample_workspace_size.argtypes = [ctypes.POINTER(TvSampleDesc)]
        L.tv_verify_sample_workspace_size.restype = sz
        L.tv_verify_sample.argtypes = [ctypes.POINTER(TvSampleDesc), P, P, P, P, P, P, P, P, P, sz, P, P]
        L.tv_commit_path.argtypes = [ctypes.POINTER(TvAttnDesc), P, P, P, P, P, P, P, P, P]
        L.tv_verify_sample_logits.argtypes = [ctypes.POINTER(TvSampleDesc), P, P, P, P, P, P, P, P, P, sz, P, P]
        L.tv_tree_fill_topk.argtypes = [ctypes.POINTER(TvSampleDesc), P, P, P, P, P, P]
        L.tv_tree_shape.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P, P, P]
        L.tv_tree_select.argtypes = [P, P, P, ctypes.c_int32, ctypes.c_int32, P, P, P, P, P]
        L.tv_tree_merge.argtypes = [ctypes.c_int32, P, P, ctypes.c_int32, P, P, P, P]
        L.tv_tree_shape_for_cost.argtypes = [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_double,
                                             ctypes.c_double, P, P, P, P, P]
        L.tv_tree_select_batch.argtypes = [ctypes.c_int32, P, P, P, P, ctypes.c_int32, P, P, P, P, P]
        L.tv_tree_select_device.argtypes = [ctypes.c_int32, ctypes.c_int32, P, P, P, P, ctypes.c_int32, P, P, P, P,
                                            P, P, P]
        L.tv_status_string.argtypes = [ctypes.c_int32]
        L.tv_status_string.restype = ctypes.c_char_p
        L.tv_version.restype = ctypes.c_int32
        for name in ("tv_tree_attention_plan", "tv_tree_attention", "tv_tree_attention_static",
                     "tv_verify_sample_plan", "tv_verify_sample", "tv_commit_path", "tv_verify_sample_logits",
                     "tv_tree_fill_topk", "tv_tree_shape", "tv_tree_select", "tv_tree_select_batch", "tv_tree_select_device",
                     "tv_tree_shape_for_cost", "tv_tree_merge"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(t) -> ctypes.c_void_p | None:
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p | None:
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------ C ABI, same names

def tv_version() -> int:
    return int(lib().tv_version())


def tv_status_string(status: int) -> str:
    return lib().tv_status_string(int(status)).decode()


def tv_tree_attention_plan(desc: TvAttnDesc) -> TvAttnPlan:
    plan = TvAttnPlan()
    s = lib().tv_tree_attention_plan(ctypes.byref(desc), ctypes.byref(plan))
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_attention_plan")
    return plan


def tv_tree_attention_workspace_size(desc: TvAttnDesc) -> int:
    return int(lib().tv_tree_attention_workspace_size(ctypes.byref(desc)))


def tv_tree_attention(desc, q, paged_k, paged_v, block_table, prefix_lens, parent_idx, out,
                      workspace=None, workspace_bytes: int = 0, dev_status=None, stream=None) -> int:
    return int(lib().tv_tree_attention(ctypes.byref(desc), _ptr(q), _ptr(paged_k), _ptr(paged_v), _ptr(block_table),
                                       _ptr(prefix_lens), _ptr(parent_idx), _ptr(out), _ptr(workspace),
                                       int(workspace_bytes), _ptr(dev_status), _stream(stream)))


def tv_tree_attention_static(desc, q, paged_k, paged_v, block_table, prefix_lens, parent_idx, out,
                             dev_status=None, stream=None) -> int:
    """tv_tree_attention with the library's fixed scratch array instead of a
    caller workspace, for callers that cannot allocate device memory when they
    call.  The first call on a device must come before any stream capture;
    overlapping calls race on the shared array."""
    return int(lib().tv_tree_attention_static(ctypes.byref(desc), _ptr(q), _ptr(paged_k), _ptr(paged_v),
                                              _ptr(block_table), _ptr(prefix_lens), _ptr(parent_idx), _ptr(out),
                                              _ptr(dev_status), _stream(stream)))


def tv_verify_sample_plan(desc: TvSampleDesc) -> TvSamplePlan:
    plan = TvSamplePlan()
    s = lib().tv_verify_sample_plan(ctypes.byref(desc), ctypes.byref(plan))
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_verify_sample_plan")
    return plan


def tv_verify_sample_workspace_size(desc: TvSampleDesc) -> int:
    return int(lib().tv_verify_sample_workspace_size(ctypes.byref(desc)))


def tv_verify_sample(desc, p, q, tree_tokens, parent_idx, uniforms, accepted_path, accepted_len, bonus_token,
                     workspace=None, workspace_bytes: int = 0, dev_status=None, stream=None) -> int:
    return int(lib().tv_verify_sample(ctypes.byref(desc), _ptr(p), _ptr(q), _ptr(tree_tokens), _ptr(parent_idx),
                                      _ptr(uniforms), _ptr(accepted_path), _ptr(accepted_len), _ptr(bonus_token),
                                      _ptr(workspace), int(workspace_bytes), _ptr(dev_status), _stream(stream)))


def tv_verify_sample_logits(desc, target_logits, draft_logits, tree_tokens, parent_idx, uniforms, accepted_path,
                            accepted_len, bonus_token, workspace=None, workspace_bytes: int = 0, dev_status=None,
                            stream=None) -> int:
    return int(lib().tv_verify_sample_logits(ctypes.byref(desc), _ptr(target_logits), _ptr(draft_logits),
                                             _ptr(tree_tokens), _ptr(parent_idx), _ptr(uniforms),
                                             _ptr(accepted_path), _ptr(accepted_len), _ptr(bonus_token),
                                             _ptr(workspace), int(workspace_bytes), _ptr(dev_status),
                                             _stream(stream)))


def tv_tree_fill_topk(desc, q, parent_idx, rank, tree_tokens, dev_status=None, stream=None) -> int:
    return int(lib().tv_tree_fill_topk(ctypes.byref(desc), _ptr(q), _ptr(parent_idx), _ptr(rank), _ptr(tree_tokens),
                                       _ptr(dev_status), _stream(stream)))


def tv_tree_shape(accept, num_ranks: int, budget: int, max_depth: int, parent_idx, rank, num_nodes,
                  expected_accepted) -> int:
    """Host pointers (numpy arrays or ctypes addresses)."""
    return int(lib().tv_tree_shape(_hptr(accept), int(num_ranks), int(budget), int(max_depth), _hptr(parent_idx),
                                   _hptr(rank), _hptr(num_nodes), _hptr(expected_accepted)))


def tv_tree_select(cand_parent, cand_token, cand_prob, num_candidates: int, budget: int, parent_idx, tree_tokens,
                   cand_index, num_nodes, expected_accepted) -> int:
    """Host pointers (numpy arrays or ctypes addresses)."""
    return int(lib().tv_tree_select(_hptr(cand_parent), _hptr(cand_token), _hptr(cand_prob), int(num_candidates),
                                    int(budget), _hptr(parent_idx), _hptr(tree_tokens), _hptr(cand_index),
                                    _hptr(num_nodes), _hptr(expected_accepted)))


def tree_select(cand_parent, cand_token, cand_prob, budget: int):
    """Dynamic tree selection; returns (parent_idx, tree_tokens, cand_index,
    expected_accepted) as numpy arrays trimmed to the tree's size."""
    import numpy as np
    par = np.ascontiguousarray(cand_parent, dtype=np.int32)
    tok = np.ascontiguousarray(cand_token, dtype=np.int32)
    prob = np.ascontiguousarray(cand_prob, dtype=np.float64)
    parent = np.empty(max(int(budget), 1), np.int32)
    tokens = np.empty_like(parent)
    index = np.empty_like(parent)
    n = np.zeros(1, np.int32)
    val = np.zeros(1, np.float64)
    s = tv_tree_select(par, tok, prob, par.size, budget, parent, tokens, index, n, val)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_select")
    k = int(n[0])
    return parent[:k].copy(), tokens[:k].copy(), index[:k].copy(), float(val[0])


def tree_shape_for_cost(accept, max_budget: int, max_depth: int = 0, draft_cost: float = 0.0, alpha: float = 0.1):
    """The tree size with the best step speedup; returns (parent_idx, rank,
    expected_accepted, speedup), the arrays trimmed to the tree's size."""
    import numpy as np
    acc = np.ascontiguousarray(accept, dtype=np.float64)
    parent = np.empty(max(int(max_budget), 1), np.int32)
    rank = np.empty_like(parent)
    n = np.zeros(1, np.int32)
    val = np.zeros(1, np.float64)
    sp = np.zeros(1, np.float64)
    s = int(lib().tv_tree_shape_for_cost(_hptr(acc), acc.size, int(max_budget), int(max_depth), float(draft_cost),
                                         float(alpha), _hptr(parent), _hptr(rank), _hptr(n), _hptr(val), _hptr(sp)))
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_shape_for_cost")
    k = int(n[0])
    return parent[:k].copy(), rank[:k].copy(), float(val[0]), float(sp[0])


def tree_merge(seqs, max_nodes: int = 1024):
    """SpecInfer's token tree from several drafts' sequences; returns
    (parent_idx, tree_tokens, node_of) with node_of a list of per-sequence
    node arrays."""
    import numpy as np
    lens = [len(s) for s in seqs]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    tok = np.ascontiguousarray(np.concatenate([np.asarray(s, np.int64) for s in seqs]) if seqs else np.zeros(0),
                               dtype=np.int32)
    parent = np.empty(int(max_nodes), np.int32)
    tokens = np.empty_like(parent)
    node_of = np.empty(max(tok.size, 1), np.int32)
    n = np.zeros(1, np.int32)
    s = int(lib().tv_tree_merge(len(seqs), _hptr(off), _hptr(tok), int(max_nodes), _hptr(parent), _hptr(tokens),
                                _hptr(node_of), _hptr(n)))
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_merge")
    k = int(n[0])
    return parent[:k].copy(), tokens[:k].copy(), [node_of[off[i]:off[i + 1]].copy() for i in range(len(seqs))]


def tree_select_batch(cand_offsets, cand_parent, cand_token, cand_prob, budget: int):
    """tv_tree_select over a batch; returns (parent_idx, tree_tokens, cand_index)
    as [B][budget] int32 arrays, node_counts [B] and expected_accepted [B]."""
    import numpy as np
    off = np.ascontiguousarray(cand_offsets, dtype=np.int32)
    B = off.size - 1
    par = np.ascontiguousarray(cand_parent, dtype=np.int32)
    tok = np.ascontiguousarray(cand_token, dtype=np.int32)
    prob = np.ascontiguousarray(cand_prob, dtype=np.float64)
    parent = np.empty((B, int(budget)), np.int32)
    tokens = np.empty_like(parent)
    index = np.empty_like(parent)
    counts = np.empty(B, np.int32)
    val = np.empty(B, np.float64)
    s = int(lib().tv_tree_select_batch(B, _hptr(off), _hptr(par), _hptr(tok), _hptr(prob), int(budget),
                                       _hptr(parent), _hptr(tokens), _hptr(index), _hptr(counts), _hptr(val)))
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_select_batch")
    return parent, tokens, index, counts, val


def tv_tree_select_device(batch: int, max_candidates: int, cand_offsets, cand_parent, cand_token, cand_prob,
                          budget: int, parent_idx, tree_tokens, cand_index, node_counts, expected_accepted,
                          dev_status=None, stream=None) -> int:
    """Device pointers (torch tensors or addresses)."""
    return int(lib().tv_tree_select_device(int(batch), int(max_candidates), _ptr(cand_offsets), _ptr(cand_parent),
                                           _ptr(cand_token), _ptr(cand_prob), int(budget), _ptr(parent_idx),
                                           _ptr(tree_tokens), _ptr(cand_index), _ptr(node_counts),
                                           _ptr(expected_accepted), _ptr(dev_status), _stream(stream)))


def tree_select_device(cand_offsets, cand_parent, cand_token, cand_prob, budget: int, max_candidates=None,
                       dev_status=None, stream=None):
    """tv_tree_select_device on CUDA tensors (offsets [B+1] int32, candidates
    int32 / float32); returns (parent_idx, tree_tokens, cand_index) as
    [B][budget] int32 tensors, node_counts [B] and expected_accepted [B]
    (float64), all on the device."""
    import torch
    B = cand_offsets.numel() - 1
    if max_candidates is None:
        max_candidates = int((cand_offsets[1:] - cand_offsets[:-1]).max().item()) if B > 0 else 0
    dev = cand_offsets.device
    parent = torch.empty((B, int(budget)), dtype=torch.int32, device=dev)
    tokens = torch.empty_like(parent)
    index = torch.empty_like(parent)
    counts = torch.empty((B,), dtype=torch.int32, device=dev)
    val = torch.empty((B,), dtype=torch.float64, device=dev)
    s = tv_tree_select_device(B, max_candidates, cand_offsets, cand_parent, cand_token, cand_prob, budget, parent,
                              tokens, index, counts, val, dev_status, stream)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_select_device")
    return parent, tokens, index, counts, val


def _hptr(a):
    if a is None:
        return None
    if isinstance(a, int):
        return ctypes.c_void_p(a)
    return ctypes.c_void_p(a.ctypes.data)


def tree_shape(accept, budget: int, max_depth: int = 0):
    """Budget-constrained tree shape; returns (parent_idx, rank, expected_accepted)
    as numpy arrays trimmed to the tree's size."""
    import numpy as np
    acc = np.ascontiguousarray(accept, dtype=np.float64)
    parent = np.empty(max(int(budget), 1), np.int32)
    rank = np.empty_like(parent)
    n = np.zeros(1, np.int32)
    val = np.zeros(1, np.float64)
    s = tv_tree_shape(acc, acc.size, budget, max_depth, parent, rank, n, val)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_shape")
    return parent[:n[0]].copy(), rank[:n[0]].copy(), float(val[0])


def fill_topk(q, parent_idx=None, rank=None, tree_tokens=None, node_counts=None, dev_status=None, stream=None):
    """Run tv_tree_fill_topk; returns tree_tokens (allocated, filled with -1, when
    not given)."""
    import torch
    _check_cuda(q, parent_idx, rank, tree_tokens, node_counts, dev_status)
    if q.dtype != torch.float32:
        raise TypeError("q must be float32")
    B, N, V = q.shape
    if tree_tokens is None:
        tree_tokens = torch.full((B, N), -1, dtype=torch.int32, device=q.device)
    desc = TvSampleDesc(B, N, V, _ptr(node_counts))
    s = tv_tree_fill_topk(desc, q, parent_idx, rank, tree_tokens, dev_status, stream)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_fill_topk")
    return tree_tokens


def tv_commit_path(desc, paged_k, paged_v, block_table, prefix_lens, accepted_path, accepted_len, new_prefix_lens,
                   dev_status=None, stream=None) -> int:
    return int(lib().tv_commit_path(ctypes.byref(desc), _ptr(paged_k), _ptr(paged_v), _ptr(block_table),
                                    _ptr(prefix_lens), _ptr(accepted_path), _ptr(accepted_len),
                                    _ptr(new_prefix_lens), _ptr(dev_status), _stream(stream)))


# ------------------------------------------------------------ torch conveniences

def attn_desc(q, k_cache, block_table, softmax_scale: float = 0.0, node_counts=None) -> TvAttnDesc:
    """Descriptor from tensors: q [B][N][Hq][D], cache [nb][16][Hkv][D],
    block_table [B][max_blocks], optional node_counts [B] int32 (ragged trees)."""
    import torch
    B, N, Hq, D = q.shape
    nb, bs, Hkv, D2 = k_cache.shape
    if D2 != D:
        raise ValueError("head_dim mismatch between q and cache")
    dt = {torch.bfloat16: TV_BF16, torch.float32: TV_F32}.get(q.dtype)
    if dt is None:
        raise TypeError(f"unsupported dtype {q.dtype}")
    return TvAttnDesc(B, N, Hq, Hkv, D, bs, block_table.shape[1], nb, dt, float(softmax_scale), _ptr(node_counts))


def _check_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


def tree_attention(q, k_cache, v_cache, block_table, prefix_lens, parent_idx, softmax_scale: float = 0.0,
                   out=None, workspace=None, dev_status=None, stream=None, node_counts=None):
    """Run tv_tree_attention; allocates `out` (and workspace) when not given.
    parent_idx None: every tree is a chain; node_counts [B]: ragged trees."""
    import torch
    _check_cuda(q, k_cache, v_cache, block_table, prefix_lens, parent_idx, out, workspace, dev_status, node_counts)
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    for t in (block_table, prefix_lens, parent_idx, node_counts):
        if t is not None and t.dtype != torch.int32:
            raise TypeError("block_table, prefix_lens, parent_idx and node_counts must be int32")
    desc = attn_desc(q, k_cache, block_table, softmax_scale, node_counts)
    if out is None:
        out = torch.empty_like(q)
    ws_bytes = tv_tree_attention_workspace_size(desc)
    if ws_bytes and workspace is None:
        workspace = torch.zeros(ws_bytes, dtype=torch.uint8, device=q.device)
    s = tv_tree_attention(desc, q, k_cache, v_cache, block_table, prefix_lens, parent_idx, out, workspace,
                          workspace.numel() if workspace is not None else 0, dev_status, stream)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_tree_attention")
    return out


def verify_sample(p, q, tree_tokens, parent_idx, uniforms, accepted_path=None, accepted_len=None,
                  bonus_token=None, dev_status=None, stream=None, logits: bool = False, node_counts=None):
    """Run tv_verify_sample (or, with logits=True, tv_verify_sample_logits on the
    two models' logits); returns (accepted_path, accepted_len, bonus_token).
    parent_idx None: every tree is a chain; node_counts [B]: ragged trees."""
    import torch
    _check_cuda(p, q, tree_tokens, parent_idx, uniforms, dev_status, node_counts)
    if p.dtype != torch.float32 or q.dtype != torch.float32 or uniforms.dtype != torch.float32:
        raise TypeError("p, q and uniforms must be float32")
    B, N, V = p.shape
    dev = p.device
    if accepted_path is None:
        accepted_path = torch.empty((B, N), dtype=torch.int32, device=dev)
    if accepted_len is None:
        accepted_len = torch.empty((B,), dtype=torch.int32, device=dev)
    if bonus_token is None:
        bonus_token = torch.empty((B,), dtype=torch.int32, device=dev)
    desc = TvSampleDesc(B, N, V, _ptr(node_counts))
    call = tv_verify_sample_logits if logits else tv_verify_sample
    s = call(desc, p, q, tree_tokens, parent_idx, uniforms, accepted_path, accepted_len, bonus_token, None, 0,
             dev_status, stream)
    if s != TV_OK:
        raise TreeVerifyError(s, call.__name__)
    return accepted_path, accepted_len, bonus_token


def commit_path(k_cache, v_cache, block_table, prefix_lens, accepted_path, accepted_len, new_prefix_lens=None,
                dev_status=None, stream=None, node_counts=None):
    """Run tv_commit_path on the caches in place; returns new_prefix_lens."""
    import torch
    _check_cuda(k_cache, v_cache, block_table, prefix_lens, accepted_path, accepted_len, new_prefix_lens, dev_status,
                node_counts)
    for t in (block_table, prefix_lens, accepted_path, accepted_len):
        if t.dtype != torch.int32:
            raise TypeError("block_table, prefix_lens, accepted_path and accepted_len must be int32")
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise TypeError("k_cache and v_cache must match")
    nb, bs, hkv, d = k_cache.shape
    B, N = accepted_path.shape
    dt = {torch.bfloat16: TV_BF16, torch.float32: TV_F32}.get(k_cache.dtype)
    if dt is None:
        raise TypeError(f"unsupported dtype {k_cache.dtype}")
    desc = TvAttnDesc(B, N, hkv, hkv, d, bs, block_table.shape[1], nb, dt, 0.0, _ptr(node_counts))
    if new_prefix_lens is None:
        new_prefix_lens = torch.empty_like(prefix_lens)
    s = tv_commit_path(desc, k_cache, v_cache, block_table, prefix_lens, accepted_path, accepted_len,
                       new_prefix_lens, dev_status, stream)
    if s != TV_OK:
        raise TreeVerifyError(s, "tv_commit_path")
    return new_prefix_lens

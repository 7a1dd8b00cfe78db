"""Ragged trees and chains on the GPU (per-sequence node counts in one call;
a missing parent array meaning chains), against the oracle's ragged forms.

Padding nodes carry garbage parents and tokens, their output rows are
prefilled with a sentinel that must survive, and each sequence's block table
stops at its own tree: the kernels must not read past n_b."""
import numpy as np
import pytest
import torch

import oracle
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import attention_errors, attention_ok, compare_sampler, dev, host_f32, random_attn

pytestmark = pytest.mark.gpu

SENTINEL = 3.0


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _trim_table(a, counts):
    """Unmap every block past each sequence's prefix + tree."""
    bt = a.block_table.copy()
    for b, n in enumerate(counts):
        used = (int(a.prefix_lens[b]) + int(n) + 15) // 16
        bt[b, used:] = -1
    return bt


def _run_attn(a, parents, counts, status=None):
    out = torch.full(a.q.shape, SENTINEL, dtype=torch.bfloat16 if a.dtype == "bf16" else torch.float32,
                     device="cuda")
    bt = _trim_table(a, counts)
    tv.tree_attention(dev(a.q), dev(a.k), dev(a.v), dev(bt), dev(a.prefix_lens),
                      None if parents is None else dev(parents), out=out, dev_status=status,
                      node_counts=dev(np.asarray(counts, np.int32)))
    torch.cuda.synchronize()
    return host_f32(out), bt


def _check_rows(got, ref, heads, G, dtype, what):
    """got, ref: [R][D] rows whose query heads are `heads` (blocks = KV heads)."""
    e = attention_errors(got, ref, np.asarray(heads) // G, dtype)
    assert attention_ok(e, dtype), (what, e)


def _check_attn(a, parents, counts):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got, bt = _run_attn(a, parents, counts, status)
    assert int(status.item()) == 0
    ref = oracle.tree_attention_ragged(a.q, a.k, a.v, bt, a.prefix_lens, parents, counts, a.num_kv_heads, a.dtype)
    Hq, D = a.q.shape[2], a.q.shape[3]
    for b, n in enumerate(counts):
        assert (got[b, n:] == SENTINEL).all(), f"padding rows of sequence {b} were written"
        if n == 0:
            continue
        heads = np.tile(np.arange(Hq), n)
        _check_rows(got[b, :n].reshape(-1, D), ref[b, :n].reshape(-1, D), heads, Hq // a.num_kv_heads, a.dtype, b)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128)])
def test_ragged_trees_match_oracle(dtype, D):
    counts = [40, 0, 1, 33, 17, 32]  # with G = 4: 160, 0, 4, 132, 68, 128 query rows
    a = random_attn(41, 6, 40, 8, 2, D, [0, 15, 16, 100, 3000, 333], dtype=dtype)
    parents = a.parent_idx.copy()
    for b, n in enumerate(counts):
        parents[b, n:] = 999  # garbage the kernels must ignore
    _check_attn(a, parents, counts)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f32", 64)])
def test_chains_match_oracle(dtype, D):
    counts = [8, 1, 64, 30]
    a = random_attn(42, 4, 64, 16, 4, D, [700, 0, 4100, 31], dtype=dtype)
    _check_attn(a, None, counts)


def test_bad_node_count_is_reported():
    a = random_attn(43, 3, 12, 8, 2, 128, [50, 60, 70])
    counts = np.array([5, 13, -1], np.int32)  # 13 > capacity, -1 < 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full(a.q.shape, SENTINEL, dtype=torch.bfloat16, device="cuda")
    tv.tree_attention(dev(a.q), dev(a.k), dev(a.v), dev(a.block_table), dev(a.prefix_lens), dev(a.parent_idx),
                      out=out, dev_status=status, node_counts=dev(counts))
    torch.cuda.synchronize()
    assert int(status.item()) == tv.TV_ERR_INVALID_ARG
    got = host_f32(out)
    assert np.isnan(got[1]).all() and np.isnan(got[2]).all()
    ref = oracle.tree_attention_ragged(a.q, a.k, a.v, a.block_table, a.prefix_lens, a.parent_idx, [5, 0, 0], 2,
                                       "bf16")
    _check_rows(got[0, :5].reshape(-1, 128), ref[0, :5].reshape(-1, 128), np.tile(np.arange(8), 5), 4, "bf16", 0)


def _walk_case(seed, B, N, V, chain=False):
    rng = np.random.default_rng(seed)
    lp = rng.normal(0, 2, (B, N, V)).astype(np.float32)
    lq = (lp + rng.normal(0, 1, (B, N, V))).astype(np.float32)
    p, q = oracle.softmax_rows(lp), oracle.softmax_rows(lq)
    parents = None if chain else np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)],
                                          np.int32)
    counts = rng.integers(0, N + 1, B).astype(np.int32)
    counts[:3] = [0, 1, N]
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    for b in range(B):
        tok[b, counts[b]:] = -7  # out of range: must be ignored
        if parents is not None:
            parents[b, counts[b]:] = 999
    return lp, lq, p, q, tok, parents, u, counts


def _gpu_walk(p, q, tok, parents, u, counts, logits=False, status=None):
    path, alen, bonus = tv.verify_sample(dev(p), dev(q), dev(tok), None if parents is None else dev(parents), dev(u),
                                         dev_status=status, logits=logits, node_counts=dev(counts))
    torch.cuda.synchronize()
    return {"accepted_path": path.cpu().numpy(), "accepted_len": alen.cpu().numpy(),
            "bonus_token": bonus.cpu().numpy()}


@pytest.mark.parametrize("chain", [False, True])
@pytest.mark.parametrize("logits", [False, True])
def test_ragged_walk_matches_oracle(chain, logits):
    lp, lq, p, q, tok, parents, u, counts = _walk_case(44 + chain, 40, 20, 5003, chain)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _gpu_walk(lp if logits else p, lq if logits else q, tok, parents, u, counts, logits, status)
    assert int(status.item()) == 0
    ref = oracle.verify_sample_ragged(lp if logits else p, lq if logits else q, tok, parents, u, counts,
                                      logits=logits)
    compare_sampler(got, ref)
    assert got["accepted_len"][0] == 0 and got["bonus_token"][0] == -1 and (got["accepted_path"][0] == -1).all()


def test_ragged_commit_matches_oracle():
    counts = np.array([9, 0, 1, 16, 5], np.int32)
    a = random_attn(45, 5, 16, 4, 2, 128, [20, 33, 16, 400, 7])
    parents = a.parent_idx.copy()
    rng = np.random.default_rng(9)
    path = np.full((5, 16), -1, np.int32)
    alen = np.zeros(5, np.int32)
    for b, n in enumerate(counts):
        parents[b, n:] = 999
        if n <= 1:
            continue
        node = int(rng.integers(1, n))
        nodes = []
        while node > 0:
            nodes.append(node)
            node = int(parents[b, node])
        nodes = nodes[::-1]
        path[b, :len(nodes)] = nodes
        alen[b] = len(nodes)
    bt = _trim_table(a, counts)
    dk, dv = dev(a.k), dev(a.v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    new = tv.commit_path(dk, dv, dev(bt), dev(a.prefix_lens), dev(path), dev(alen), dev_status=status,
                         node_counts=dev(counts))
    torch.cuda.synchronize()
    rk, rv, rnew, rst = oracle.commit_path_ragged(a.k, a.v, bt, a.prefix_lens, path, alen, counts)
    assert rst == 0 and int(status.item()) == 0
    np.testing.assert_array_equal(new.cpu().numpy(), rnew)
    np.testing.assert_array_equal(dk.view(torch.int16).cpu().numpy().view(np.uint16), rk)
    np.testing.assert_array_equal(dv.view(torch.int16).cpu().numpy().view(np.uint16), rv)


def test_ragged_serving_workload():
    """The mixed-serving shape (32 sequences, 1..32 nodes each, every fourth a
    chain, prefixes up to 32K, vocab 151936) at full size: attention on sampled
    rows (every sequence's root and last node, head 0 and the last head), the
    whole walk, and the commit of the walk's paths."""
    import synth
    wl = synth.make("ragged")
    counts = wl.counts
    q, k, v = wl.query(), wl.k_cache(), wl.v_cache()
    out = torch.full(q.shape, SENTINEL, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dk, dv, dbt, dpl, dcnt = dev(k), dev(v), dev(wl.block_table), dev(wl.prefix_lens), dev(counts)
    tv.tree_attention(dev(q), dk, dv, dbt, dpl, dev(wl.parent_idx), out=out, dev_status=status, node_counts=dcnt)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = host_f32(out)
    Hq = wl.num_q_heads
    for b in range(wl.batch):
        n = int(counts[b])
        assert (got[b, n:] == SENTINEL).all()
        nodes = sorted({0, n - 1})
        rows = np.array([(0, i, h) for i in nodes for h in (0, Hq - 1)], np.int32)
        ref = oracle.tree_attention(q[b:b + 1, :n], k, v, wl.block_table[b:b + 1], wl.prefix_lens[b:b + 1],
                                    wl.parent_idx[b:b + 1, :n], wl.num_kv_heads, "bf16", rows=rows)
        g = np.stack([got[b, i, h] for _, i, h in rows])
        _check_rows(g, ref, rows[:, 2], Hq // wl.num_kv_heads, "bf16", b)
    p, qd = wl.pq()
    u = wl.uniforms()
    walk = _gpu_walk(p, qd, wl.tree_tokens, wl.parent_idx, u, counts, status=status)
    assert int(status.item()) == 0
    ref = oracle.verify_sample_ragged(p, qd, wl.tree_tokens, wl.parent_idx, u, counts)
    compare_sampler(walk, ref, oracle.verify_sample_ragged(p, qd, wl.tree_tokens, wl.parent_idx, u, counts, eps=1e-9))
    new = tv.commit_path(dk, dv, dbt, dpl, dev(walk["accepted_path"]), dev(walk["accepted_len"]), dev_status=status,
                         node_counts=dcnt)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    np.testing.assert_array_equal(new.cpu().numpy(), wl.prefix_lens + 1 + walk["accepted_len"])

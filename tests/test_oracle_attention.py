"""Pins for the oracle's tree attention.

Every node attends to the whole prefix and to its own root path (glossary
page, "Tree attention").  Pinned by closed forms (one visible key, equal
logits, a two-key softmax), by the library routine
``torch.nn.functional.scaled_dot_product_attention`` in float64 (a chain is
ordinary causal attention; N = 1 is plain decode; any tree is SDPA under the
ancestor mask), and by invariances of the definition."""
import math

import numpy as np
import pytest
import torch

import oracle
from helpers import contiguous_table, dense_kv_to_paged


def _run(q, kv_k, kv_v, parent, prefix_lens, num_kv_heads, perm=None, scale=None, dtype="f32"):
    """q [B][N][Hq][D]; kv_k/kv_v lists over b of [L_b+N][Hkv][D]."""
    B, N = q.shape[:2]
    bt, nb = contiguous_table(prefix_lens, N)
    if perm is not None:
        bt = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    kc = dense_kv_to_paged(kv_k, bt)
    vc = dense_kv_to_paged(kv_v, bt)
    par = np.array(parent, dtype=np.int32).reshape(B, N)
    return oracle.tree_attention(q, kc, vc, bt, np.array(prefix_lens, np.int32), par, num_kv_heads, dtype, scale)


def _rand_case(rng, B, N, Hq, Hkv, D, prefix_lens):
    q = rng.standard_normal((B, N, Hq, D)).astype(np.float32)
    ks = [rng.standard_normal((L + N, Hkv, D)).astype(np.float32) for L in prefix_lens]
    vs = [rng.standard_normal((L + N, Hkv, D)).astype(np.float32) for L in prefix_lens]
    return q, ks, vs


def _sdpa(q, k, v, mask, scale):
    """float64 torch SDPA for one (b, h): q [N][D], k/v [T][D], mask [N][T] bool."""
    qt = torch.tensor(q, dtype=torch.float64)[None, None]
    kt = torch.tensor(k, dtype=torch.float64)[None, None]
    vt = torch.tensor(v, dtype=torch.float64)[None, None]
    mt = torch.tensor(mask)[None, None]
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mt, scale=scale)[0, 0].numpy()


def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(1)
    q, ks, vs = _rand_case(rng, 1, 1, 2, 1, 8, [0])
    out = _run(q, ks, vs, [-1], [0], 1)
    np.testing.assert_array_equal(out[0, 0, 0], vs[0][0, 0].astype(np.float64))
    np.testing.assert_array_equal(out[0, 0, 1], vs[0][0, 0].astype(np.float64))


def test_equal_logits_average_visible_values():
    rng = np.random.default_rng(2)
    L, N = 5, 5
    parent = [-1, 0, 1, 0, 3]
    q = np.zeros((1, N, 2, 4), dtype=np.float32)
    _, ks, vs = _rand_case(rng, 1, N, 2, 2, 4, [L])
    out = _run(q, ks, vs, parent, [L], 2)
    for i in range(N):
        anc = []
        j = i
        while j >= 0:
            anc.append(L + j)
            j = parent[j]
        visible = list(range(L)) + sorted(anc)
        for h in range(2):
            expect = vs[0][visible, h].astype(np.float64).mean(0)
            np.testing.assert_allclose(out[0, i, h], expect, rtol=1e-14, atol=1e-15)


def test_two_key_softmax_closed_form():
    # D = 1, scale 1: logits 0 and ln 3 -> weights 1/4 and 3/4
    q = np.array([[[[1.0]]]], dtype=np.float32)
    k = [np.array([[[0.0]], [[math.log(3.0)]]], dtype=np.float32)]
    v = [np.array([[[2.0]], [[10.0]]], dtype=np.float32)]
    out = _run(q, k, v, [-1], [1], 1, scale=1.0)
    lg = float(np.float32(math.log(3.0)))
    w1 = math.exp(lg) / (1.0 + math.exp(lg))
    assert abs(out[0, 0, 0, 0] - (2.0 * (1 - w1) + 10.0 * w1)) < 1e-12
    assert abs(out[0, 0, 0, 0] - 8.0) < 1e-6


@pytest.mark.parametrize("N,L,G", [(1, 37, 1), (6, 0, 2), (8, 21, 4)])
def test_chain_equals_causal_attention(N, L, G):
    rng = np.random.default_rng(3 + N)
    Hkv, D = 2, 16
    Hq = Hkv * G
    q, ks, vs = _rand_case(rng, 1, N, Hq, Hkv, D, [L])
    out = _run(q, ks, vs, [-1] + list(range(N - 1)), [L], Hkv)
    scale = 1.0 / math.sqrt(D)
    causal = np.zeros((N, L + N), dtype=bool)
    for i in range(N):
        causal[i, : L + i + 1] = True
    for h in range(Hq):
        ref = _sdpa(q[0, :, h], ks[0][:, h // G], vs[0][:, h // G], causal, scale)
        np.testing.assert_allclose(out[0, :, h], ref, rtol=1e-12, atol=1e-12)


def test_single_node_is_plain_decode():
    rng = np.random.default_rng(7)
    q, ks, vs = _rand_case(rng, 2, 1, 4, 4, 32, [50, 3])
    out = _run(q, ks, vs, [-1, -1], [50, 3], 4)
    for b, L in enumerate([50, 3]):
        for h in range(4):
            ref = _sdpa(q[b, :, h], ks[b][:, h], vs[b][:, h], np.ones((1, L + 1), bool), 1 / math.sqrt(32))
            np.testing.assert_allclose(out[b, 0, h], ref[0], rtol=1e-12, atol=1e-12)


def test_random_trees_equal_masked_sdpa():
    rng = np.random.default_rng(11)
    B, N, Hq, Hkv, D = 3, 12, 4, 2, 8
    prefix = [0, 17, 40]
    parents = []
    for b in range(B):
        parents.append([-1] + [int(rng.integers(0, i)) for i in range(1, N)])
    q, ks, vs = _rand_case(rng, B, N, Hq, Hkv, D, prefix)
    out = _run(q, ks, vs, parents, prefix, Hkv)
    for b in range(B):
        L = prefix[b]
        mask = np.zeros((N, L + N), dtype=bool)
        for i in range(N):
            mask[i, :L] = True
            j = i
            while j >= 0:
                mask[i, L + j] = True
                j = parents[b][j]
        for h in range(Hq):
            ref = _sdpa(q[b, :, h], ks[b][:, h // 2], vs[b][:, h // 2], mask, 1 / math.sqrt(D))
            np.testing.assert_allclose(out[b, :, h], ref, rtol=1e-12, atol=1e-12)


def test_block_permutation_invariance():
    rng = np.random.default_rng(5)
    prefix = [45, 70]
    q, ks, vs = _rand_case(rng, 2, 5, 4, 2, 8, prefix)
    a = _run(q, ks, vs, [[-1, 0, 1, 0, 3]] * 2, prefix, 2)
    nb = contiguous_table(prefix, 5)[1]
    b = _run(q, ks, vs, [[-1, 0, 1, 0, 3]] * 2, prefix, 2, perm=rng.permutation(nb))
    np.testing.assert_array_equal(a, b)


def test_non_ancestor_values_do_not_matter():
    rng = np.random.default_rng(6)
    parent = [-1, 0, 1, 0, 3]
    L = 9
    q, ks, vs = _rand_case(rng, 1, 5, 2, 1, 8, [L])
    a = _run(q, ks, vs, parent, [L], 1)
    ks2 = [ks[0].copy()]
    vs2 = [vs[0].copy()]
    ks2[0][L + 3] += 5.0       # B1 is not an ancestor of A1 / A2
    vs2[0][L + 3] -= 7.0
    b = _run(q, ks2, vs2, parent, [L], 1)
    for i in (0, 1, 2):
        np.testing.assert_array_equal(a[0, i], b[0, i])
    assert np.abs(a[0, 3] - b[0, 3]).max() > 1e-3


def test_gqa_equals_repeated_kv_heads():
    rng = np.random.default_rng(8)
    G, Hkv = 4, 2
    q, ks, vs = _rand_case(rng, 1, 4, G * Hkv, Hkv, 8, [20])
    gqa = _run(q, ks, vs, [-1, 0, 0, 1], [20], Hkv)
    ks_rep = [np.repeat(ks[0], G, axis=1)]
    vs_rep = [np.repeat(vs[0], G, axis=1)]
    mha = _run(q, ks_rep, vs_rep, [-1, 0, 0, 1], [20], G * Hkv)
    np.testing.assert_array_equal(gqa, mha)


def test_bf16_input_path_widens_exactly():
    rng = np.random.default_rng(9)
    q, ks, vs = _rand_case(rng, 1, 3, 2, 1, 8, [10])
    to_bits = lambda a: (a.view(np.uint32) >> 16).astype(np.uint16)      # truncate to bf16
    widen = lambda a: (a.astype(np.uint32) << 16).view(np.float32)
    qb, kb, vb = to_bits(q), [to_bits(ks[0])], [to_bits(vs[0])]
    out_b = _run(qb, kb, vb, [-1, 0, 1], [10], 1, dtype="bf16")
    out_f = _run(widen(qb), [widen(kb[0])], [widen(vb[0])], [-1, 0, 1], [10], 1)
    np.testing.assert_array_equal(out_b, out_f)


def test_selected_rows_match_full_output():
    rng = np.random.default_rng(10)
    prefix = [33, 8]
    q, ks, vs = _rand_case(rng, 2, 4, 4, 2, 8, prefix)
    full = _run(q, ks, vs, [[-1, 0, 0, 2]] * 2, prefix, 2)
    bt, _ = contiguous_table(prefix, 4)
    rows = np.array([[1, 3, 2], [0, 0, 0], [1, 1, 3]], dtype=np.int32)
    sel = oracle.tree_attention(q, dense_kv_to_paged(ks, bt), dense_kv_to_paged(vs, bt), bt,
                                np.array(prefix, np.int32), np.array([[-1, 0, 0, 2]] * 2, np.int32), 2, "f32",
                                rows=rows)
    for r, (b, i, h) in enumerate(rows):
        np.testing.assert_array_equal(sel[r], full[b, i, h])

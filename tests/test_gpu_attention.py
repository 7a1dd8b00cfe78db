"""Tree-attention parity on the GPU: the library (through its C ABI) against
the fp64 oracle on the same seeded inputs, for every workload shape, plus
invariances and edge cases."""
import numpy as np
import pytest
import torch

import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import Attn, random_attn, sample_rows, dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_tiny_fp32_full_parity():
    a = Attn.from_workload(synth.make("tiny", need_tokens=False))
    err = a.compare(a.run_gpu())
    print("tiny fp32 row-relative error", err)


@pytest.mark.parametrize("unit", [False, True], ids=["default_scale", "unit_kv"])
def test_l8b_full_parity(unit):
    """Every row of the Llama-3-8B shape (9 KV splits, 2 row tiles, both mask
    words); unit_kv makes the outputs of order one (see synth.make)."""
    a = Attn.from_workload(synth.make("l8b", need_tokens=False, unit_kv=unit))
    err = a.compare(a.run_gpu())
    print("l8b", "unit" if unit else "default", err)


def _must_nodes(N):
    # the first and last node of every 32-bit word of the ancestor mask
    return tuple(sorted({n for w in range((N + 31) // 32) for n in (32 * w, min(N, 32 * w + 32) - 1)}))


@pytest.mark.parametrize("unit", [False, True], ids=["default_scale", "unit_kv"])
@pytest.mark.parametrize("name,count", [("l70b", 384), ("mix", 384), ("long", 256)])
def test_full_size_sampled_parity(name, count, unit):
    wl = synth.make(name, need_tokens=False, unit_kv=unit)
    a = Attn.from_workload(wl)
    out = a.run_gpu()
    assert np.isfinite(out).all()
    rows = sample_rows(wl.batch, wl.num_nodes, wl.num_q_heads, count, seed=7,
                       must_nodes=_must_nodes(wl.num_nodes) if wl.batch <= 8 else ())
    err = a.compare(out, rows)
    print(name, "unit" if unit else "default", len(rows), "rows", err)


@pytest.mark.parametrize("unit", [False, True], ids=["default_scale", "unit_kv"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,Hq,Hkv,D,prefix", [
    (1, 1, 8, 8, 128, [0]),              # plain decode of the root only, empty prefix
    (2, 5, 8, 2, 64, [0, 37]),           # empty prefix, ragged prefix
    (1, 65, 32, 8, 128, [1000]),         # node count just above 64
    (1, 128, 16, 8, 128, [513]),         # maximum node count, two 128-row tiles
    (3, 7, 4, 4, 128, [17, 300, 4096]),  # MHA (G = 1), prefixes not multiples of 16
    (2, 16, 64, 8, 128, [2500, 3]),      # G = 8
])
def test_edge_shapes(dtype, B, N, Hq, Hkv, D, prefix, unit):
    a = random_attn(11 + N, B, N, Hq, Hkv, D, prefix, dtype=dtype, kv_std=1.0 if unit else None,
                    tree_k_scale=synth.UNIT_TREE_K_SCALE if unit else 1.0)
    a.compare(a.run_gpu())


@pytest.mark.parametrize("unit", [False, True], ids=["default_scale", "unit_kv"])
@pytest.mark.parametrize("N", [40, 128])
def test_chain_tree_matches_oracle(unit, N):
    # A chain given by its parent array: its ancestor sets come from a bounded walk plus
    # pointer jumping (128 nodes: depth 127, every jumping round).  The same chain without
    # a parent array gets its sets in closed form and must give the same bits.
    parents = np.array([[-1] + list(range(N - 1))], np.int32)
    a = random_attn(5, 1, N, 32, 8, 128, [2000], parents=parents, kv_std=1.0 if unit else None,
                    tree_k_scale=synth.UNIT_TREE_K_SCALE if unit else 1.0)
    out = a.run_gpu()
    a.compare(out)
    a.dpar = None
    np.testing.assert_array_equal(a.run_gpu(), out)


@pytest.mark.parametrize("unit", [False, True], ids=["default_scale", "unit_kv"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_deep_trees_match_oracle(unit, dtype):
    # caterpillars: each node's parent is the previous node four times in five, else one two
    # to four places back, so 128-node trees of depth 92-97 with a branch every few levels
    rng = np.random.default_rng(9)
    B, N = 3, 128
    parents = np.array([[-1] + [i - 1 if (i < 2 or rng.random() < 0.8) else i - int(rng.integers(2, min(i, 4) + 1))
                                for i in range(1, N)] for _ in range(B)], np.int32)
    a = random_attn(6, B, N, 16, 8, 128, [300, 1500, 4000], dtype=dtype, parents=parents,
                    kv_std=1.0 if unit else None, tree_k_scale=synth.UNIT_TREE_K_SCALE if unit else 1.0)
    a.compare(a.run_gpu())


def test_block_permutation_gives_identical_output():
    a = random_attn(3, 4, 24, 32, 8, 128, [700, 1500, 33, 2048], permute=False)
    base = a.run_gpu()
    # move every logical block to a new physical slot
    rng = np.random.default_rng(0)
    nb = a.k.shape[0]
    perm = rng.permutation(nb)
    k2 = np.empty_like(a.k); v2 = np.empty_like(a.v)
    k2[perm] = a.k; v2[perm] = a.v
    bt2 = np.where(a.block_table >= 0, perm[np.maximum(a.block_table, 0)], -1).astype(np.int32)
    b = Attn(a.q, k2, v2, bt2, a.prefix_lens, a.parent_idx, "bf16", 8)
    np.testing.assert_array_equal(base, b.run_gpu())


def test_non_ancestor_kv_does_not_change_output():
    parents = np.array([[-1, 0, 1, 0, 3, 4, 1]], np.int32)
    a = random_attn(9, 1, 7, 32, 8, 128, [300], parents=parents, permute=False)
    base = a.run_gpu()
    L = 300
    k2, v2 = a.k.copy(), a.v.copy()
    # node 3 (position L + 3) is not an ancestor of nodes 1, 2, 6
    blk, slot = a.block_table[0, (L + 3) // 16], (L + 3) % 16
    k2[blk, slot] = synth.normals(k2[blk, slot].size, 99, 1, bf16=True).reshape(k2[blk, slot].shape)
    v2[blk, slot] = synth.normals(v2[blk, slot].size, 99, 2, bf16=True).reshape(v2[blk, slot].shape)
    b = Attn(a.q, k2, v2, a.block_table, a.prefix_lens, parents, "bf16", 8).run_gpu()
    for i in (0, 1, 2, 6):
        np.testing.assert_array_equal(base[0, i], b[0, i])
    assert np.abs(base[0, 3] - b[0, 3]).max() > 0


def test_deterministic():
    a = random_attn(4, 2, 32, 32, 8, 128, [5000, 12000])
    np.testing.assert_array_equal(a.run_gpu(), a.run_gpu())


def test_bad_tree_and_block_table_are_reported():
    a = random_attn(2, 2, 6, 8, 2, 128, [40, 50])
    a.parent_idx[1, 4] = 5           # parent after child
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = a.run_gpu(status)
    assert int(status.item()) == tv.TV_ERR_TREE
    assert np.isnan(out[1]).all()
    a2 = random_attn(2, 2, 6, 8, 2, 128, [40, 50])
    good = a2.run_gpu()
    a2.block_table[0, 1] = 10 ** 6    # out of range block id
    a2.to_device()
    status.zero_()
    out2 = a2.run_gpu(status)
    assert int(status.item()) == tv.TV_ERR_BLOCK_TABLE
    np.testing.assert_array_equal(out2[1], good[1])   # the other sequence is untouched


def test_output_buffer_tail_untouched():
    a = random_attn(6, 1, 20, 32, 8, 128, [900]).to_device()
    n = a.dq.numel()
    buf = torch.full((n + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[:n].view(a.dq.shape)
    tv.tree_attention(a.dq, a.dk, a.dv, a.dbt, a.dpl, a.dpar, out=out)
    torch.cuda.synchronize()
    assert (buf[n:] == 7.0).all()
    a.compare(out.float().cpu().numpy())

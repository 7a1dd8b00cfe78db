"""GPU parity for tv_commit_path against the oracle's or_commit_path.

The commit is pure data movement (accepted path rows move to L + 1 + k, the
new length is L + 1 + len), so caches and lengths must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import Attn, attention_errors, attention_ok, dev, random_attn, run_sampler_gpu

pytestmark = pytest.mark.gpu


def _host(t: torch.Tensor, like: np.ndarray) -> np.ndarray:
    if like.dtype == np.uint16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def _path_to(parent, node):
    out = []
    while node > 0:
        out.append(int(node))
        node = parent[node]
    return out[::-1]


def _random_paths(parents, rng, flagged=()):
    B, N = parents.shape
    path = np.full((B, N), -1, np.int32)
    alen = np.zeros(B, np.int32)
    for b in range(B):
        if b in flagged:
            alen[b] = -1
            continue
        nodes = _path_to(parents[b], int(rng.integers(0, N)))
        path[b, :len(nodes)] = nodes
        alen[b] = len(nodes)
    return path, alen


def _gpu_commit(a: Attn, path, alen, status=None):
    dk, dv = dev(a.k), dev(a.v)
    new = tv.commit_path(dk, dv, dev(a.block_table), dev(a.prefix_lens), dev(path), dev(alen), dev_status=status)
    torch.cuda.synchronize()
    return _host(dk, a.k), _host(dv, a.v), new.cpu().numpy()


def _check(a: Attn, path, alen):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k, v, new = _gpu_commit(a, path, alen, status)
    rk, rv, rnew, rst = oracle.commit_path(a.k, a.v, a.block_table, a.prefix_lens, path, alen)
    assert rst == 0 and int(status.item()) == 0
    np.testing.assert_array_equal(new, rnew)
    np.testing.assert_array_equal(k, rk)
    np.testing.assert_array_equal(v, rv)


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 128), ("f32", 64)])
def test_random_paths_match_oracle(dtype, D):
    a = random_attn(31, 6, 24, 4, 2, D, [0, 15, 16, 100, 1000, 333], dtype=dtype)
    rng = np.random.default_rng(7)
    path, alen = _random_paths(a.parent_idx, rng, flagged=(5,))
    alen[4] = 0  # the root alone
    path[4] = -1
    _check(a, path, alen)


def test_path_already_in_place_and_overlapping_moves():
    parents = np.array([[-1, 0, 1, 2, 3, 0, 5, 2],        # chain 1-2-3-4: already in place
                        [-1, 0, 0, 2, 0, 2, 5, 6]], np.int32)  # path [2, 5, 6]: 5 lands where 2 was
    a = random_attn(32, 2, 8, 8, 4, 128, [40, 17], parents=parents)
    path = np.array([[1, 2, 3, 4, -1, -1, -1, -1], [2, 5, 6, -1, -1, -1, -1, -1]], np.int32)
    _check(a, path, np.array([4, 3], np.int32))


def test_paths_from_the_walk_on_the_70b_shape():
    wl = synth.make("l70b")
    a = Attn.from_workload(wl)
    p, q = wl.pq()
    walk = run_sampler_gpu(p, q, wl.tree_tokens, wl.parent_idx, wl.uniforms())
    assert (walk["accepted_len"] >= 0).all()
    _check(a, walk["accepted_path"], walk["accepted_len"])


def test_malformed_inputs_leave_the_cache_and_report():
    a = random_attn(33, 3, 8, 4, 2, 64, [20, 20, 20], dtype="f32")
    path = np.array([[2, 2, -1, -1, -1, -1, -1, -1],   # not strictly increasing
                     [1, 9, -1, -1, -1, -1, -1, -1],   # past the tree
                     [1, 2, -1, -1, -1, -1, -1, -1]], np.int32)
    alen = np.array([2, 2, 2], np.int32)
    a.block_table[2, 1] = 10_000  # a block id out of range inside sequence 2's tree span
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k, v, new = _gpu_commit(a, path, alen, status)
    assert int(status.item()) in (tv.TV_ERR_TREE, tv.TV_ERR_BLOCK_TABLE)
    np.testing.assert_array_equal(new, a.prefix_lens)
    np.testing.assert_array_equal(k, a.k)
    np.testing.assert_array_equal(v, a.v)


def test_attention_after_commit_is_causal_attention():
    """Each accepted node's tree attention before the commit equals, after the
    commit, the attention of the same query as a one-node tree at its new
    position (both on the GPU)."""
    parents = np.array([[-1, 0, 1, 1, 0, 3, 5, 6, 2, 7, 9, 4]], np.int32)
    # unit-variance K/V with scaled tree keys: outputs of order one, so the
    # comparison below can tell a wrong key set from rounding
    a = random_attn(34, 1, 12, 8, 2, 128, [300], parents=parents, kv_std=1.0, tree_k_scale=4.0)
    before = a.run_gpu()
    nodes = _path_to(parents[0], 10)
    path = np.full((1, 12), -1, np.int32)
    path[0, :len(nodes)] = nodes
    k, v, new = _gpu_commit(a, path, np.array([len(nodes)], np.int32))
    assert new[0] == 300 + 1 + len(nodes)
    for kk, c in enumerate(nodes, start=1):
        one = Attn(a.q[:, c:c + 1], k, v, a.block_table, np.array([300 + kk], np.int32), np.array([[-1]], np.int32),
                   "bf16", 2)
        after = one.run_gpu()
        e = attention_errors(after[0, 0], before[0, c].astype(np.float64), np.arange(8) // 4, "bf16")
        assert attention_ok(e, "bf16"), (c, e)

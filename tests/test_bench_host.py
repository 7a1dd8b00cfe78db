"""Host-side bookkeeping of bench.py: the count of vocabulary rows an
acceptance walk reads in full, which the roofline's algorithmic bytes use,
matches the count the oracle logs while it walks."""
import numpy as np

import bench
import oracle
import synth


def test_walk_rows_matches_the_oracle_log():
    rng = np.random.default_rng(4)
    B, N, V = 300, 12, 64
    parent = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    lp = rng.normal(0, 2, (B, N, V))
    p = oracle.softmax_rows(lp)
    q = oracle.softmax_rows(lp + rng.normal(0, 1.5, (B, N, V)))
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    r = oracle.verify_sample(p, q, tok, parent, u)
    assert bench.walk_rows(parent, r["accepted_path"], r["accepted_len"]) == int(r["rows"].sum())
    # every visited row: one per accepted node plus the last one
    assert bench.walk_rows(parent, r["accepted_path"], r["accepted_len"], every_visited=True) == \
        int((r["accepted_len"] + 1).sum())


def test_walk_rows_on_the_small_workload():
    wl = synth.make("tiny")
    p, q = wl.pq()
    r = oracle.verify_sample(p, q, wl.tree_tokens, wl.parent_idx, wl.uniforms())
    assert bench.walk_rows(wl.parent_idx, r["accepted_path"], r["accepted_len"]) == int(r["rows"].sum())


def test_deepest_paths_respect_node_counts():
    par = np.array([[-1, 0, 1, 2, -1, -1], [-1, 0, 0, 2, 3, 4]], np.int32)
    path, plen = bench.deepest_paths(par, np.array([4, 3]))
    # sequence 1 keeps nodes 0, 1 <- 0, 2 <- 0: depth 1 at best, first deepest node 1
    assert plen.tolist() == [3, 1]
    assert path[0, :3].tolist() == [1, 2, 3] and path[1, :1].tolist() == [1]


def test_rotation_copies_exceed_twice_l2():
    l2 = 126 << 20
    # the 8B shape reads ~20 MB per step: one pass over the copies must read >= 2 x L2
    n = bench.rotation_copies(20 << 20, 90 << 20, l2)
    assert n >= 4 and n * (20 << 20) >= 2 * l2
    # a step that reads more than L2 by itself still rotates over 4 copies
    assert bench.rotation_copies(4 << 30, 6 << 30, l2) == 4


def test_tensor_flops_counts_every_key_of_every_row():
    wl = synth.make("l8b", need_tokens=False)
    # 4 * D * (L + N) * (G * N) per KV head
    assert bench.tensor_flops(wl) == 4 * 128 * (4096 + 64) * (4 * 64) * 8

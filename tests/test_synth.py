"""The seeded input generator: Philox4x32-10 known answers, determinism and
the workload shapes."""
import collections

import numpy as np

import synth
from helpers import golden_lines


def test_philox_known_answers():
    for row in golden_lines("philox4x32_10_kat.txt"):
        vals = [int(x, 16) for x in row]
        out = synth.philox4x32_10(vals[:4], vals[4:6])
        assert [int(x) for x in out] == vals[6:10]


def test_streams_are_counter_based():
    a = synth.uniforms(1000, 7, 3)
    b = synth.uniforms(10, 7, 3, offset=500)
    np.testing.assert_array_equal(a[500:510], b)
    assert (a >= 0).all() and (a < 1).all()
    n = synth.normals(200_000, 1, 2)
    assert abs(n.mean()) < 0.01 and abs(n.std() - 1) < 0.01


def test_workload_shapes():
    wl = synth.make("tiny")
    assert wl.parent_idx.tolist() == [[-1, 0, 1, 0, 3]]
    p, q = wl.pq()
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-5)
    np.testing.assert_allclose(q.sum(-1), 1.0, rtol=1e-5)
    wl = synth.make("l8b", need_tokens=False)
    par = wl.parent_idx[0]
    depth = [0] * 64
    for i in range(1, 64):
        assert 0 <= par[i] < i
        depth[i] = depth[par[i]] + 1
    assert collections.Counter(depth) == {0: 1, 1: 4, 2: 9, 3: 11, 4: 13, 5: 13, 6: 13}
    assert wl.block_table[0].tolist() == list(range(260))
    wl = synth.make("l70b", need_tokens=False)
    assert wl.parent_idx.shape == (8, 32)
    assert sorted(wl.block_table.reshape(-1).tolist()) == list(range(wl.num_blocks))
    wl = synth.make("mix", need_tokens=False)
    assert wl.batch == 64 and (wl.prefix_lens >= 512).all() and (wl.prefix_lens <= 32768).all()
    for b in range(64):
        par = wl.parent_idx[b]
        d = [0] * 16
        for i in range(1, 16):
            d[i] = d[par[i]] + 1
        assert 2 <= max(d) <= 6


def test_bf16_cache_is_rounded_normal():
    wl = synth.make("tiny")
    k = wl.k_cache()
    assert k.dtype == np.float32
    bt = wl.block_table[0]
    # logical position 0, head 0 equals element 0 of the K stream
    ref = synth.normals(4, wl.seed, synth.STREAM_K)[0]
    assert k[bt[0], 0, 0, 0] == ref


def test_logits_are_the_distributions_before_softmax():
    # the row softmax of the generated logits is the generated p, q
    for name in ("tiny", "l8b"):
        wl = synth.make(name)
        p, q = wl.pq()
        lp, lq = wl.logits()
        assert lp.shape == p.shape and lp.dtype == np.float32
        for l, d in ((lp, p), (lq, q)):
            x = l[0, :3].astype(np.float64)
            e = np.exp(x - x.max(axis=-1, keepdims=True))
            np.testing.assert_allclose(e / e.sum(axis=-1, keepdims=True), d[0, :3], rtol=2e-6, atol=1e-30)

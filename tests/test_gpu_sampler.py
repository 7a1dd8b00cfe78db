"""Acceptance-walk parity on the GPU: bit-exact with the fp64 oracle except
where the oracle flags a uniform within 1e-6 of a threshold, for every
workload shape; losslessness (chi-square) of the GPU kernel itself; edge
cases."""
import numpy as np
import pytest
import torch

import oracle
import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import compare_sampler, run_sampler_gpu
from test_oracle_sampler import lossless_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("name", list(synth.CONFIG_NAMES))
def test_workload_parity(name):
    wl = synth.make(name)
    p, q = wl.pq()
    u = wl.uniforms()
    ref = oracle.verify_sample(p, q, wl.tree_tokens, wl.parent_idx, u)
    tight = oracle.verify_sample(p, q, wl.tree_tokens, wl.parent_idx, u, eps=1e-9)
    gpu = run_sampler_gpu(p, q, wl.tree_tokens, wl.parent_idx, u)
    mism, flagged = compare_sampler(gpu, ref, tight)
    print(name, "mean accepted", ref["accepted_len"].mean(), "mismatches", mism, "flagged", flagged)


def test_many_uniform_draws_parity():
    # the same l8b tree and distributions under 512 independent uniform sets
    wl = synth.make("l8b")
    p, q = wl.pq()
    R = 512
    u = synth.uniforms(R * wl.num_nodes, 77, synth.STREAM_UNIFORM).reshape(R, wl.num_nodes)
    P = np.broadcast_to(p, (R,) + p.shape[1:])
    Q = np.broadcast_to(q, (R,) + q.shape[1:])
    tok = np.repeat(wl.tree_tokens, R, axis=0)
    par = np.repeat(wl.parent_idx, R, axis=0)
    ref = oracle.verify_sample(P, Q, tok, par, u)
    tight = oracle.verify_sample(P, Q, tok, par, u, eps=1e-9)
    gpu = run_sampler_gpu(P, Q, tok, par, u)
    mism, flagged = compare_sampler(gpu, ref, tight)
    print("l8b x512: mean accepted", ref["accepted_len"].mean(), "mismatches", mism, "flagged", flagged)


def test_gpu_kernel_is_lossless():
    ok1, ok2 = lossless_check(lambda p, q, t, par, u: run_sampler_gpu(p, q, t, par, u))
    assert ok1 and ok2


# 151,936 (a Qwen2-sized vocabulary) gives each warp more than four 128-entry steps, the
# shape whose residual passes read shared memory every time instead of registers
@pytest.mark.parametrize("V", [1, 3, 8, 1001, 4097, 65537, 128259, 151936])
def test_ragged_vocab_sizes(V):
    rng = np.random.default_rng(V)
    B, parent = 16, [-1, 0, 0, 1, 1, 2, 0, 6]
    N = len(parent)
    logits = rng.standard_normal((B, N, V)) * 2
    p = np.exp(logits); p /= p.sum(-1, keepdims=True)
    q = np.exp(logits + rng.standard_normal((B, N, V))); q /= q.sum(-1, keepdims=True)
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    args = (p.astype(np.float32), q.astype(np.float32), tok, np.array([parent] * B, np.int32), u)
    ref = oracle.verify_sample(*args)
    compare_sampler(run_sampler_gpu(*args), ref, oracle.verify_sample(*args, eps=1e-9))


def test_single_node_and_deep_chain():
    rng = np.random.default_rng(1)
    V = 5000
    for parent in ([-1], [-1] + list(range(299))):
        N = len(parent)
        p = rng.dirichlet(np.ones(V), size=(2, N)).astype(np.float32)
        tok = rng.integers(0, V, (2, N)).astype(np.int32)
        u = (rng.random((2, N)) * 0.01).astype(np.float32)    # mostly accepting
        args = (p, p, tok, np.array([parent] * 2, np.int32), u)
        compare_sampler(run_sampler_gpu(*args), oracle.verify_sample(*args))


def test_degenerate_distributions():
    V = 64
    p = np.zeros((3, 3, V), np.float32); q = np.zeros((3, 3, V), np.float32)
    p[:, :, :] = 1.0 / V; q[:, :, :] = 1.0 / V
    q[0, 0] = 0; q[0, 0, 5] = 1.0; p[0, 0, 5] = 0.0; p[0, 0] /= p[0, 0].sum()   # one-hot draft on p = 0
    p[1, 0] = 0; p[1, 0, 7] = 1.0                                            # zero residual after rejection
    q[2, 0, 9] = 0; q[2, 0] /= q[2, 0].sum()                                 # q(x) = 0 draft
    tok = np.array([[0, 5, 5], [0, 3, 4], [0, 9, 1]], np.int32)
    u = np.full((3, 3), 0.5, np.float32)
    args = (p, q, tok, np.array([[-1, 0, 0]] * 3, np.int32), u)
    compare_sampler(run_sampler_gpu(*args), oracle.verify_sample(*args))


def test_bad_tree_is_reported():
    V = 100
    p = np.full((2, 4, V), 0.01, np.float32)
    tok = np.array([[0, 1, 2, 3], [0, 1, 2, 300]], np.int32)     # token out of range in sequence 1
    par = np.array([[-1, 0, 0, 1], [-1, 0, 0, 1]], np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = run_sampler_gpu(p, p, tok, par, np.full((2, 4), 0.5, np.float32), status)
    assert int(status.item()) == tv.TV_ERR_TREE
    assert res["accepted_len"][1] == -1 and res["bonus_token"][1] == -1
    assert res["accepted_len"][0] >= 0


@pytest.mark.parametrize("V", [128256, 128259, 151936])
def test_bonus_draw_finds_the_owner_anywhere_in_the_vocabulary(V):
    # The root's only child has p(x) = 0, so it is always rejected, and the bonus token comes
    # from the residual max(0, p - q).  The residual is zero everywhere except a few chosen
    # entries, placed at the two ends of a 128,256-entry vocabulary and inside slices far from
    # the first (the walk spreads the vocabulary over up to 16 CTAs), so the owner of the draw
    # is found at the edges of the CTA and warp scans.  u0 = 0 takes the first entry with mass.
    # At 128,259 the last slice ends inside a lane's four-entry step (summed entry by entry);
    # at 151,936 each warp's segment is longer than the registers hold.
    spots = [[0], [V - 1], [3 * V // 16 + 5, 12 * V // 16 + 7], [3 * V // 16 + 5, 12 * V // 16 + 7],
             [V // 2 - 1, V // 2, V // 2 + 1], [7, V - 2]]
    u0 = [0.5, 0.5, 0.25, 0.75, 0.0, 0.3]
    B, x = len(spots), 11  # x: the child's draft token
    q = np.full((B, 2, V), 1.0 / V, np.float32)
    p = np.full((B, 2, V), 0.5 / V, np.float32)  # below q: no residual mass
    for s, ks in enumerate(spots):
        p[s, 0, x] = 0.0
        for k in ks:
            p[s, 0, k] = 2.0 / V  # above q: residual mass 1 / V each
        p[s, 0] /= p[s, 0].sum()
        p[s, 1] = p[s, 0]
    tok = np.array([[0, x]] * B, np.int32)
    par = np.array([[-1, 0]] * B, np.int32)
    u = np.array([[u0[s], 0.5] for s in range(B)], np.float32)
    ref = oracle.verify_sample(p, q, tok, par, u)
    gpu = run_sampler_gpu(p, q, tok, par, u)
    compare_sampler(gpu, ref, oracle.verify_sample(p, q, tok, par, u, eps=1e-9))
    want = [0, V - 1, spots[2][0], spots[3][1], spots[4][0], 7]
    assert list(gpu["bonus_token"]) == want
    assert (gpu["accepted_len"] == 0).all()


@pytest.mark.parametrize("V", [128256, 128259, 151936])
def test_bonus_draw_with_u0_just_below_one_takes_the_last_entry_with_mass(V):
    # target = u0 * Z sits within rounding of the total: whichever way the sums round, the
    # draw must be the last entry with residual mass (the oracle's fallback reading)
    B, x = 3, 11
    last = [V - 1, 9 * V // 16 + 3, 5]
    q = np.full((B, 2, V), 1.0 / V, np.float32)
    p = np.full((B, 2, V), 0.5 / V, np.float32)
    for s in range(B):
        p[s, 0, x] = 0.0
        for k in (2, 4 * V // 16 + 1, last[s]):
            if k <= last[s]:
                p[s, 0, k] = 2.0 / V
        p[s, 0] /= p[s, 0].sum()
        p[s, 1] = p[s, 0]
    tok = np.array([[0, x]] * B, np.int32)
    par = np.array([[-1, 0]] * B, np.int32)
    u = np.array([[np.nextafter(np.float32(1), np.float32(0)), 0.5]] * B, np.float32)
    gpu = run_sampler_gpu(p, q, tok, par, u)
    assert list(gpu["bonus_token"]) == last
    assert (gpu["accepted_len"] == 0).all()

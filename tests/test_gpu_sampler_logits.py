"""The fused-logits acceptance walk (tv_verify_sample_logits) on the GPU.

p and q are the target and draft models' output distributions (blog
"Speculative decoding x tree attention", section 2; glossary "Tree-based
speculative decoding", section "SpecInfer"); this entry point takes the logits
and forms each visited row's softmax itself.  Parity is against the oracle's
verify_sample_logits (fp64 softmax rounded to fp32, then the fp64 walk): equal
except where the oracle flags a uniform within 1e-6 of a threshold, the band
the kernel's fp32 exponentials need.  Also: the chi-square losslessness of the
kernel itself, masked (-inf) logits, ragged vocabularies and a bad tree."""
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


def _run(lp, lq, tok, par, u, status=None):
    return run_sampler_gpu(lp, lq, tok, par, u, status=status, logits=True)


@pytest.mark.parametrize("name", list(synth.CONFIG_NAMES))
def test_workload_parity(name):
    wl = synth.make(name)
    lp, lq = wl.logits()
    u = wl.uniforms()
    ref = oracle.verify_sample_logits(lp, lq, wl.tree_tokens, wl.parent_idx, u)
    mism, flagged = compare_sampler(_run(lp, lq, wl.tree_tokens, wl.parent_idx, u), ref)
    print(name, "mean accepted", ref["accepted_len"].mean(), "mismatches", mism, "flagged", flagged)


def test_many_uniform_draws_parity():
    # the l8b tree and logits under 96 independent uniform sets
    wl = synth.make("l8b")
    lp, lq = wl.logits()
    R = 96
    u = synth.uniforms(R * wl.num_nodes, 78, synth.STREAM_UNIFORM).reshape(R, wl.num_nodes)
    LP = np.broadcast_to(lp, (R,) + lp.shape[1:])
    LQ = np.broadcast_to(lq, (R,) + lq.shape[1:])
    tok = np.repeat(wl.tree_tokens, R, axis=0)
    par = np.repeat(wl.parent_idx, R, axis=0)
    ref = oracle.verify_sample_logits(LP, LQ, tok, par, u)
    mism, flagged = compare_sampler(_run(LP, LQ, tok, par, u), ref)
    assert flagged <= R // 8
    print("l8b x96: mean accepted", ref["accepted_len"].mean(), "mismatches", mism, "flagged", flagged)


def test_gpu_kernel_is_lossless_on_logits():
    # the walk on log p, log q draws from p exactly as the walk on p, q does
    def walk(p, q, t, par, u):
        with np.errstate(divide="ignore"):
            return _run(np.log(p.astype(np.float64)), np.log(q.astype(np.float64)), t, par, u)
    ok1, ok2 = lossless_check(walk)
    assert ok1 and ok2


def test_masked_logits_have_probability_zero():
    """Tokens whose logit is -inf are never accepted and never drawn as the
    bonus: with every token but a few masked in p, the emitted tokens stay in
    the unmasked set."""
    rng = np.random.default_rng(11)
    B, V = 64, 3000
    parent = np.array([[-1, 0, 0, 1, 2, 0]] * B, np.int32)
    N = parent.shape[1]
    lp = rng.normal(0, 2, (B, N, V)).astype(np.float32)
    lq = (lp + rng.normal(0, 1, (B, N, V))).astype(np.float32)
    keep = rng.random((B, N, V)) < 0.01
    keep[..., 0] = True
    lp[~keep] = -np.inf
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    ref = oracle.verify_sample_logits(lp, lq, tok, parent, u)
    gpu = _run(lp, lq, tok, parent, u)
    compare_sampler(gpu, ref)
    for b in range(B):
        n = int(gpu["accepted_len"][b])
        nodes = [0] + list(gpu["accepted_path"][b, :n])
        for k in range(n):
            assert keep[b, nodes[k], tok[b, nodes[k + 1]]]
        assert keep[b, nodes[n], gpu["bonus_token"][b]]


@pytest.mark.parametrize("V", [1, 3, 8, 1001, 4097, 65537, 128259])
def test_ragged_vocab_sizes(V):
    rng = np.random.default_rng(V + 5)
    B, parent = 16, [-1, 0, 0, 1, 1, 2, 0, 6]
    N = len(parent)
    lp = (rng.standard_normal((B, N, V)) * 2).astype(np.float32)
    lq = (lp + rng.standard_normal((B, N, V))).astype(np.float32)
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    args = (lp, lq, tok, np.array([parent] * B, np.int32), u)
    compare_sampler(_run(*args), oracle.verify_sample_logits(*args))


def test_large_logit_offsets():
    """Logits far from zero (the row max near 80) still give the softmax: the
    row maximum is subtracted before the exponentials."""
    rng = np.random.default_rng(3)
    B, V = 8, 20000
    parent = np.array([[-1, 0, 1, 2, 0]] * B, np.int32)
    N = parent.shape[1]
    lp = (rng.normal(0, 3, (B, N, V)) + 70.0).astype(np.float32)
    lq = (lp + rng.normal(0, 1, (B, N, V))).astype(np.float32)
    tok = rng.integers(0, V, (B, N)).astype(np.int32)
    u = rng.random((B, N)).astype(np.float32)
    compare_sampler(_run(lp, lq, tok, parent, u), oracle.verify_sample_logits(lp, lq, tok, parent, u))


def test_bad_tree_is_reported():
    V = 100
    lp = np.zeros((2, 4, V), np.float32)
    tok = np.array([[0, 1, 2, 3], [0, 1, 2, 300]], np.int32)     # token out of range in sequence 1
    par = np.array([[-1, 0, 0, 1], [-1, 0, 0, 1]], np.int32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = _run(lp, lp, tok, par, np.full((2, 4), 0.5, np.float32), status)
    assert int(status.item()) == tv.TV_ERR_TREE
    assert res["accepted_len"][1] == -1 and res["bonus_token"][1] == -1
    assert res["accepted_len"][0] >= 0

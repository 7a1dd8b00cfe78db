"""GPU-test plumbing: move seeded inputs to the device, call the library
through its C ABI, and call the oracle on the same host arrays.

Nothing here computes the method."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
import tree_speculative_decoding_07_b200 as tv

BF16_ATOL = 2e-2       # max-abs for bf16 storage (fp32 accumulation)
F32_RTOL = 1e-5        # fp32 path: max-abs error <= 1e-5 * max |oracle| of the row
# bf16 path, in addition to the max-abs bound: per (sequence, KV head) block,
# ||gpu - oracle||_2 <= REL_RMS * ||oracle||_2.  The rounding in the kernel
# (bf16 P and outputs, 2^-9 relative each) stays near 1e-3 of the block's
# norm; an all-zero output, a dropped ancestor or a wrong split weight moves
# the norm of the difference by a large fraction of the output's own norm,
# however small the outputs are.
REL_RMS = 1e-2


def attention_errors(got: np.ndarray, ref: np.ndarray, block: np.ndarray, dtype: str) -> dict:
    """Errors of attention rows got against the oracle's ref ([R][D] each);
    block[r] numbers the (sequence, KV head) block of row r."""
    got = got.astype(np.float64)
    err = got - ref
    out = {"finite": bool(np.isfinite(got).all())}
    if not out["finite"]:
        return out
    out["max_abs"] = float(np.abs(err).max()) if err.size else 0.0
    if dtype == "bf16":
        blocks = np.unique(block, return_inverse=True)[1]
        num = np.bincount(blocks, weights=(err ** 2).sum(axis=1))
        den = np.bincount(blocks, weights=(ref ** 2).sum(axis=1))
        out["rel_rms"] = float((np.sqrt(num) / np.maximum(np.sqrt(den), 1e-300)).max()) if num.size else 0.0
    else:
        scale = np.maximum(np.abs(ref).max(axis=1, keepdims=True), 1e-30)
        out["row_rel"] = float((np.abs(err) / scale).max()) if err.size else 0.0
    return out


def attention_ok(e: dict, dtype: str) -> bool:
    """The parity criterion: max-abs 2e-2 and relative rms 1e-2 per block for
    bf16, row-relative 1e-5 for fp32."""
    if not e["finite"]:
        return False
    if dtype == "bf16":
        return e["max_abs"] <= BF16_ATOL and e["rel_rms"] <= REL_RMS
    return e["row_rel"] <= F32_RTOL


def dev(arr: np.ndarray, dtype: str | None = None) -> torch.Tensor:
    """Host array -> contiguous CUDA tensor; uint16 arrays are bfloat16 bits."""
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr)).cuda()


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


class Attn:
    """One tree-attention problem: host arrays, device tensors, GPU and oracle runs."""

    def __init__(self, q, k, v, block_table, prefix_lens, parent_idx, dtype: str, num_kv_heads: int):
        self.q, self.k, self.v = q, k, v
        self.block_table = np.ascontiguousarray(block_table, np.int32)
        self.prefix_lens = np.ascontiguousarray(prefix_lens, np.int32)
        self.parent_idx = np.ascontiguousarray(parent_idx, np.int32)
        self.dtype = dtype
        self.num_kv_heads = num_kv_heads

    @classmethod
    def from_workload(cls, wl: synth.Workload) -> "Attn":
        return cls(wl.query(), wl.k_cache(), wl.v_cache(), wl.block_table, wl.prefix_lens, wl.parent_idx,
                   wl.dtype, wl.num_kv_heads)

    def to_device(self):
        self.dq, self.dk, self.dv = dev(self.q), dev(self.k), dev(self.v)
        self.dbt, self.dpl, self.dpar = dev(self.block_table), dev(self.prefix_lens), dev(self.parent_idx)
        return self

    def run_gpu(self, status: torch.Tensor | None = None) -> np.ndarray:
        if not hasattr(self, "dq"):
            self.to_device()
        out = tv.tree_attention(self.dq, self.dk, self.dv, self.dbt, self.dpl, self.dpar, dev_status=status)
        torch.cuda.synchronize()
        return host_f32(out)

    def oracle(self, rows=None) -> np.ndarray:
        return oracle.tree_attention(self.q, self.k, self.v, self.block_table, self.prefix_lens, self.parent_idx,
                                     self.num_kv_heads, self.dtype, rows=rows)

    def row_blocks(self, rows=None) -> np.ndarray:
        """(sequence, KV head) block number of every compared row."""
        B, N, Hq = self.q.shape[:3]
        G = Hq // self.num_kv_heads
        if rows is not None:
            rr = np.asarray(rows).reshape(-1, 3)
            return rr[:, 0] * self.num_kv_heads + rr[:, 2] // G
        b, _, h = np.meshgrid(np.arange(B), np.arange(N), np.arange(Hq), indexing="ij")
        return (b * self.num_kv_heads + h // G).reshape(-1)

    def compare(self, gpu: np.ndarray, rows=None) -> dict:
        """Check the GPU output against the oracle (rows: sampled (b, i, h)
        triples, else every row) and return the errors."""
        ref = self.oracle(rows)
        if rows is not None:
            rr = np.asarray(rows).reshape(-1, 3)
            got = gpu[rr[:, 0], rr[:, 1], rr[:, 2]]
        else:
            got = gpu.reshape(ref.shape)
        ref = ref.reshape(-1, ref.shape[-1])
        got = got.reshape(-1, got.shape[-1])
        e = attention_errors(got, ref, self.row_blocks(rows), self.dtype)
        assert attention_ok(e, self.dtype), f"attention parity failed: {e}"
        return e


def sample_rows(B, N, Hq, count, seed, must_nodes=()):
    """Deterministic (b, i, h) rows: every node in must_nodes for every b
    (head 0 and the last head), plus `count` random rows."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(B):
        for i in must_nodes:
            rows += [(b, i % N, 0), (b, i % N, Hq - 1)]
    rows += list(zip(rng.integers(0, B, count), rng.integers(0, N, count), rng.integers(0, Hq, count)))
    return np.array(rows, dtype=np.int32)


def random_attn(seed, B, N, Hq, Hkv, D, prefix_lens, dtype="bf16", permute=True, parents=None, kv_std=None,
                tree_k_scale=1.0):
    """Small seeded attention problem with random trees and a paged cache;
    tree_k_scale multiplies the keys of the tree block (positions L_b..L_b+N-1)."""
    rng = np.random.default_rng(seed)
    prefix_lens = np.asarray(prefix_lens, np.int32)
    if parents is None:
        parents = np.array([[-1] + [int(rng.integers(0, i)) for i in range(1, N)] for _ in range(B)], np.int32)
    nblk = [(int(L) + N + 15) // 16 for L in prefix_lens]
    total = sum(nblk)
    ids = rng.permutation(total) if permute else np.arange(total)
    mb = max(nblk) + 1
    bt = np.full((B, mb), -1, np.int32)
    off = 0
    for b in range(B):
        bt[b, :nblk[b]] = ids[off:off + nblk[b]]
        off += nblk[b]
    std = kv_std if kv_std is not None else (1.0 / np.sqrt(D) if dtype == "bf16" else 1.0)
    bf = dtype == "bf16"
    q = synth.normals(B * N * Hq * D, seed, synth.STREAM_QUERY, bf16=bf).reshape(B, N, Hq, D)
    k = synth.normals(total * 16 * Hkv * D, seed, synth.STREAM_K, std=std, bf16=bf).reshape(total, 16, Hkv, D)
    v = synth.normals(total * 16 * Hkv * D, seed, synth.STREAM_V, std=std, bf16=bf).reshape(total, 16, Hkv, D)
    if tree_k_scale != 1.0:
        for b in range(B):
            for t in range(int(prefix_lens[b]), int(prefix_lens[b]) + N):
                blk, slot = bt[b, t // 16], t % 16
                row = (synth.bf16_to_f32(k[blk, slot]) if bf else k[blk, slot]) * np.float32(tree_k_scale)
                k[blk, slot] = (row.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16) if bf else row
    return Attn(q, k, v, bt, prefix_lens, parents, dtype, Hkv)


def run_sampler_gpu(p, q, tokens, parent, uniforms, status=None, logits=False):
    """The walk on the GPU; with logits=True p and q are the two models' logits."""
    path, alen, bonus = tv.verify_sample(dev(np.asarray(p, np.float32)), dev(np.asarray(q, np.float32)),
                                         dev(np.asarray(tokens, np.int32)), dev(np.asarray(parent, np.int32)),
                                         dev(np.asarray(uniforms, np.float32)), dev_status=status, logits=logits)
    torch.cuda.synchronize()
    return {"accepted_path": path.cpu().numpy(), "accepted_len": alen.cpu().numpy(),
            "bonus_token": bonus.cpu().numpy()}


def compare_sampler(gpu, ref, ref_tight=None):
    """Bit-exact except sequences the oracle flags as near a threshold
    (within 1e-6).  Returns (mismatches, flagged)."""
    same = ((gpu["accepted_len"] == ref["accepted_len"]) & (gpu["bonus_token"] == ref["bonus_token"])
            & (gpu["accepted_path"] == ref["accepted_path"]).all(axis=1))
    flagged = ref["near"] > 0
    bad = ~same & ~flagged
    assert not bad.any(), f"sampler mismatch on unflagged sequences {np.nonzero(bad)[0][:10]}"
    if ref_tight is not None:
        bad_tight = ~same & ~(ref_tight["near"] > 0)
        assert not bad_tight.any(), f"mismatch outside the 1e-9 band: {np.nonzero(bad_tight)[0][:10]}"
    return int((~same).sum()), int(flagged.sum())

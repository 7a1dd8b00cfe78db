#!/usr/bin/env python3
"""Benchmark of the tree-verification step: one tree-attention call (one
layer) plus one acceptance walk, on seeded synthetic inputs.

Default workload (one GPU): the Llama-3-8B attention shape -- batch 1,
prefix 4096 (contiguous blocks), 32 query / 8 KV heads, head_dim 128, bf16,
a 64-node top-k [4,3,2,2,1,1] tree, vocabulary 128256 with fp32 p/q.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU runs (launched with torch.distributed.run) give every rank its own
independent sequences (weak scaling, no data-path collective); time is the
maximum over ranks.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "tree nodes verified/s and µs per verify step; achieved HBM GB/s vs B200 peak"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_SUSTAINED = 1400.0  # TFLOP/s, the profiling recipe's sustained figure
NOMINAL_HBM_GBS = 8000.0  # the "~8 TB/s" spec figure, reported beside the measured copy bandwidth
L2_FLUSH_BYTES = 512 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured", d
    except Exception:
        return FALLBACK_HBM_GBS, "fallback", {}


# the sources each kernel's code and launch configuration come from
KERNEL_SOURCES = {
    "attn_tc": ("api.cu", "attn_tc.cu", "kernels.h", "tc_device.cuh", "tv_common.cuh"),
    "attn_simt": ("api.cu", "attn_simt.cu", "kernels.h", "tv_common.cuh"),
    "verify_sample": ("api.cu", "sample.cu", "kernels.h", "tv_common.cuh"),
}


def kernel_source_hash(kernel_key: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "tree_speculative_decoding_07_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[kernel_key][workload]
        if e.get("source_hash") != kernel_source_hash(kernel_key):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """SM clock and throttle-reason samples during the timed region, read
    through NVML (a polling thread every few ms, plus sample_now(), which the
    timing loop calls while the GPU still works through the queued steps, so a
    region of a few ms still gets samples).  Falls back to nvidia-smi."""

    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    BITS = (0x8, 0x40, 0x20, 0x4)  # NVML clocks-event reason bits, in NAMES order

    def __init__(self, index: int):
        self.index = index
        self.handle = None
        self.nvml = None
        self.samples = []   # (sm_mhz, reason mask)
        self.smax = None
        self.thread = None
        self.stop_flag = None
        self.proc = None

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        h = None
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
        self.nvml, self.handle = pynvml, h
        self.smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))

    def sample_now(self):
        if self.handle is None:
            return
        n = self.nvml
        try:
            self.samples.append((float(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM)),
                                 int(n.nvmlDeviceGetCurrentClocksEventReasons(self.handle))))
        except Exception:
            pass

    def start(self):
        import threading
        try:
            self._open()
        except Exception:
            self.handle = None
        if self.handle is None:
            try:
                fields = ("index,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                          "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                          "clocks_event_reasons.sw_power_cap")
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                     "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
            return
        self.stop_flag = threading.Event()

        def poll():
            while not self.stop_flag.is_set():
                self.sample_now()
                self.stop_flag.wait(0.002)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join()
        elif self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            for line in out.strip().splitlines():
                parts = [x.strip() for x in line.split(",")]
                try:
                    mask = sum(b for b, v in zip(self.BITS, parts[3:7]) if v.lower().startswith("active"))
                    self.samples.append((float(parts[1]), mask))
                    self.smax = float(parts[2])
                except (ValueError, IndexError):
                    continue
        else:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock readout unavailable"], "samples": 0}
        reasons = sorted({n for _, m in self.samples for n, b in zip(self.NAMES, self.BITS) if m & b})
        sm = [c for c, _ in self.samples]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.smax, "reasons": reasons,
                "samples": len(sm), "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ------------------------------------------------------------------ inputs

def make_inputs(workload: str, seed: int):
    import synth
    wl = synth.make(workload, seed=seed)
    p, q = wl.pq()
    return wl, {
        "query": wl.query(), "k": wl.k_cache(), "v": wl.v_cache(), "block_table": wl.block_table,
        "prefix_lens": wl.prefix_lens, "parent_idx": wl.parent_idx, "p": p, "q": q,
        "tokens": wl.tree_tokens, "uniforms": wl.uniforms(),
        **({} if wl.node_counts is None else {"node_counts": wl.node_counts}),
    }


def attention_bytes(wl) -> int:
    """Algorithmic HBM bytes of one tree-attention call: every cached K and V
    row the call must read (prefix plus tree block, per KV head), the queries
    and the outputs."""
    el = 2 if wl.dtype == "bf16" else 4
    kv = 2 * int((wl.prefix_lens.astype(np.int64) + wl.counts).sum()) * wl.num_kv_heads * wl.head_dim * el
    qo = 2 * int(wl.counts.sum()) * wl.num_q_heads * wl.head_dim * el
    return kv + qo


def walk_rows(parent_idx, path, alen, every_visited: bool = False) -> int:
    """Vocabulary rows an acceptance walk reads in full, from its result: at a
    visited node the walk reads the whole row once a child is rejected (the
    residual), and the last visited node's row for the bonus draw.  Children
    are tested in ascending index order, so a rejection happened at node u iff
    u has a child below the accepted one.  With every_visited, each visited
    node's row counts (the logits walk needs every visited row's softmax)."""
    rows = 0
    for b in range(parent_idx.shape[0]):
        n = int(alen[b])
        if n < 0:
            continue
        nodes = [0] + [int(x) for x in path[b, :n]]
        for k in range(n):
            u, c = nodes[k], nodes[k + 1]
            if every_visited or bool((parent_idx[b, 1:c] == u).any()):
                rows += 1
        rows += 1
    return rows


def sampler_bytes(wl, h, path, alen, every_visited: bool = False) -> int:
    """Algorithmic bytes of the acceptance walk: both rows (p and q, 4 bytes
    each) of every row it reads in full, 12 bytes per tested child (p(x),
    q(x), its uniform) and the tree metadata (token, parent)."""
    rows = walk_rows(h["parent_idx"], path, alen, every_visited)
    counts = wl.counts
    tested = int((counts - 1).clip(min=0).sum())  # every node but the roots is a child
    return rows * 8 * wl.vocab + tested * 12 + int(counts.sum()) * 8


# ------------------------------------------------------------------ multi-rank plumbing

def reduce_max(values, world: int, device="cpu"):
    """Element-wise maximum over ranks (timing is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(world: int, nodes_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job nodes/s: every rank verifies its own sequences (weak scaling)."""
    return world * nodes_per_step * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ our arm

def workload_config(name: str, wl, world: int) -> dict:
    """The workload both arms of the bench report (same dict for each)."""
    N = wl.num_nodes
    tree = (f"{N}-node tree" if wl.node_counts is None else
            f"ragged trees of 1..{N} nodes ({int(wl.counts.sum())} in all; every fourth a chain)")
    return {"workload": f"{name}: batch {wl.batch}, prefix {int(wl.prefix_lens[0])}, "
                        f"Hq {wl.num_q_heads}/Hkv {wl.num_kv_heads}, D {wl.head_dim}, {wl.dtype}, "
                        f"{tree}, vocab {wl.vocab}",
            "global_batch": world * wl.batch, "tree_nodes": N, "seq_len": int(wl.prefix_lens.max()) + N,
            "parallelism": f"replicas x{world} (independent sequences per GPU)",
            "l2": f"flushed before every step ({L2_FLUSH_BYTES >> 20} MB write, outside the step events)"}


def deepest_paths(parent_idx: np.ndarray, counts=None):
    """Each tree's deepest root-to-leaf path (root excluded), as a walk that
    accepts every node on it would return it; counts[b] limits sequence b's
    tree to its first counts[b] nodes."""
    B, N = parent_idx.shape
    path = np.full((B, N), -1, np.int32)
    plen = np.zeros(B, np.int32)
    for b in range(B):
        n = N if counts is None else int(counts[b])
        depth = np.zeros(N, np.int64)
        for i in range(1, n):
            depth[i] = depth[parent_idx[b, i]] + 1
        node, nodes = int(np.argmax(depth)), []
        while node > 0:
            nodes.append(node)
            node = int(parent_idx[b, node])
        nodes.reverse()
        path[b, :len(nodes)] = nodes
        plen[b] = len(nodes)
    return path, plen


def time_commit(tv, wl, d, flush, stream, W, K):
    """tv_commit_path (the step after verification) on copies of the caches,
    every tree's deepest path accepted; CUDA events, L2 flushed per call."""
    import torch
    path, plen = deepest_paths(wl.parent_idx, wl.node_counts)
    kc, vc = d["k"].clone(), d["v"].clone()
    dpath = torch.from_numpy(path).cuda()
    dlen = torch.from_numpy(plen).cuda()
    new_pl = torch.empty_like(d["prefix_lens"])
    call = lambda: tv.commit_path(kc, vc, d["block_table"], d["prefix_lens"], dpath, dlen, new_pl, stream=stream,
                                  node_counts=d.get("node_counts"))
    for _ in range(W):
        flush.zero_()
        call()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    us = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3
    moved = int(sum(sum(1 for k in range(plen[b]) if path[b, k] != k + 1) for b in range(wl.batch)))
    row_bytes = wl.head_dim * (2 if wl.dtype == "bf16" else 4)
    nbytes = moved * wl.num_kv_heads * row_bytes * 2 * 2  # K and V, read and written
    del kc, vc
    return {"us": us, "accepted_nodes": int(plen.sum()), "moved_rows": moved, "bytes": nbytes,
            "achieved_gbs": nbytes / (us * 1e-6) / 1e9 if us > 0 else None,
            "note": "tv_commit_path, the step after verification (not part of the step timed above): every tree's "
                    "deepest root-to-leaf path accepted; mean over calls, L2 flushed before each"}


def time_logits_walk(tv, wl, d, flush, stream, W, K, ref):
    """tv_verify_sample_logits (the walk on the two models' logits) timed alone
    from its own graph, L2 flushed before each launch; also how many sequences
    end exactly as the walk on p, q (ref) does."""
    import torch
    lp, lq = wl.logits()
    dlp, dlq = torch.from_numpy(lp).cuda(), torch.from_numpy(lq).cuda()
    B, N = wl.batch, wl.num_nodes
    path = torch.empty((B, N), dtype=torch.int32, device="cuda")
    alen = torch.empty((B,), dtype=torch.int32, device="cuda")
    bonus = torch.empty((B,), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sdesc = tv.TvSampleDesc(B, N, wl.vocab, tv._ptr(d.get("node_counts")))

    def call(st):
        s = tv.tv_verify_sample_logits(sdesc, dlp, dlq, d["tokens"], d["parent_idx"], d["uniforms"], path, alen,
                                       bonus, None, 0, status, st)
        if s:
            raise tv.TreeVerifyError(s, "tv_verify_sample_logits")

    call(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    for _ in range(W):
        flush.zero_()
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} from the logits walk")
    us = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3
    p_np, a_np, b_np = path.cpu().numpy(), alen.cpu().numpy(), bonus.cpu().numpy()
    nbytes = sampler_bytes(wl, {"parent_idx": wl.parent_idx}, p_np, a_np, every_visited=True)
    same = ((a_np == ref["alen"]) & (b_np == ref["bonus"]) & (p_np == ref["path"]).all(axis=1))
    del g, dlp, dlq
    return {"us": us, "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9 if us > 0 else None,
            "same_as_pq_walk": int(same.sum()), "sequences": B,
            "note": "tv_verify_sample_logits on fp32 logits (softmax formed per visited row inside the walk); bytes: "
                    "both logit rows of every visited node plus per-child gathers; mean over launches, L2 flushed "
                    "before each"}


def time_fill_topk(tv, wl, d, flush, stream, W, K):
    """tv_tree_fill_topk (top-k branching: every child's token from its parent's
    draft row, ranks = sibling order) on the workload's own tree and q rows,
    timed alone from its own graph with L2 flushed before each launch."""
    import torch
    B, N = wl.batch, wl.num_nodes
    tokens = torch.empty((B, N), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    desc = tv.TvSampleDesc(B, N, wl.vocab, tv._ptr(d.get("node_counts")))

    def call(st):
        s = tv.tv_tree_fill_topk(desc, d["q"], d["parent_idx"], None, tokens, status, st)
        if s:
            raise tv.TreeVerifyError(s, "tv_tree_fill_topk")

    call(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    for _ in range(W):
        flush.zero_()
        g.replay()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} from the top-k fill")
    us = float(np.mean([e0.elapsed_time(e1) for e0, e1 in evs])) * 1e3
    internal = 0
    for b in range(B):
        n = int(wl.counts[b])
        internal += len({int(x) for x in wl.parent_idx[b, 1:n]})
    nbytes = internal * wl.vocab * 4 + int(wl.counts.sum()) * 8
    del g
    return {"us": us, "rows": internal, "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9 if us else None,
            "note": "tv_tree_fill_topk on the workload's tree (each internal node's q row read once); mean over "
                    "launches, L2 flushed before each"}


def to_device(h: dict) -> dict:
    import torch

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a)).cuda()

    return {k: dev(v) for k, v in h.items()}


class Step:
    """One verification step of a workload on the device: the tree-attention
    call and the acceptance walk, over `copies` independent copies of every
    input (for back-to-back timing with a working set larger than L2)."""

    def __init__(self, tv, wl, h, copies: int = 1):
        import torch
        self.tv, self.wl = tv, wl
        base = to_device(h)
        self.inputs = [base] + [{k: t.clone() for k, t in base.items()} for _ in range(copies - 1)]
        d = base
        B, N = wl.batch, wl.num_nodes
        self.out = torch.empty_like(d["query"])
        self.path = torch.empty((B, N), dtype=torch.int32, device="cuda")
        self.alen = torch.empty((B,), dtype=torch.int32, device="cuda")
        self.bonus = torch.empty((B,), dtype=torch.int32, device="cuda")
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.adesc = tv.attn_desc(d["query"], d["k"], d["block_table"], node_counts=d.get("node_counts"))
        self.aplan = tv.tv_tree_attention_plan(self.adesc)
        self.ws_bytes = self.aplan.workspace_bytes
        self.ws = torch.zeros(max(self.ws_bytes, 256), dtype=torch.uint8, device="cuda")
        self.sdescs = [tv.TvSampleDesc(B, N, wl.vocab, tv._ptr(x.get("node_counts"))) for x in self.inputs]
        self.splan = tv.tv_verify_sample_plan(self.sdescs[0])
        self.adescs = [tv.attn_desc(x["query"], x["k"], x["block_table"], node_counts=x.get("node_counts"))
                       for x in self.inputs]

    def attn(self, st, i: int = 0):
        d = self.inputs[i]
        s = self.tv.tv_tree_attention(self.adescs[i], d["query"], d["k"], d["v"], d["block_table"], d["prefix_lens"],
                                      d["parent_idx"], self.out, self.ws, self.ws_bytes, self.status, st)
        if s:
            raise self.tv.TreeVerifyError(s, "tv_tree_attention")

    def sample(self, st, i: int = 0):
        d = self.inputs[i]
        s = self.tv.tv_verify_sample(self.sdescs[i], d["p"], d["q"], d["tokens"], d["parent_idx"], d["uniforms"],
                                     self.path, self.alen, self.bonus, None, 0, self.status, st)
        if s:
            raise self.tv.TreeVerifyError(s, "tv_verify_sample")

    def graph(self, fn):
        """Capture fn(stream) into a CUDA graph."""
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(torch.cuda.current_stream())
        torch.cuda.synchronize()
        return g

    def check_status(self, what: str):
        if int(self.status.item()) != 0:
            raise RuntimeError(f"device status {int(self.status.item())} after {what}")

    def walk(self) -> dict:
        return {"path": self.path.cpu().numpy(), "alen": self.alen.cpu().numpy(), "bonus": self.bonus.cpu().numpy()}


def timed_replays(graph, flush, stream, W: int, K: int):
    """Device time of each of K replays of graph (ms), L2 flushed before each."""
    import torch
    for _ in range(W):
        flush.zero_()
        graph.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return [e0.elapsed_time(e1) for e0, e1 in ev]


def back_to_back_us(graph, per_graph: int, stream, W: int, reps: int) -> float:
    """Device time per unit (µs) of `reps` replays of a graph holding
    `per_graph` units launched back to back (no flush, no gap)."""
    import torch
    for _ in range(W):
        graph.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * per_graph)


def rotation_copies(read_bytes: int, input_bytes: int, l2_bytes: int, mem_cap: int = 24 << 30) -> int:
    """Input copies for back-to-back timing: at least 4, and enough that one
    pass over them reads at least twice the L2 size, within a memory cap."""
    want = max(4, -(-2 * l2_bytes // max(read_bytes, 1)))
    return int(max(4, min(want, mem_cap // max(input_bytes, 1))))


def tensor_flops(wl) -> int:
    """Attention FLOPs of one call: 2 * 2 * D per (query row, visible key), with
    every query row of a sequence's KV head reading the whole prefix plus the
    tree block (the MMA tile computes the masked entries too)."""
    G = wl.num_q_heads // wl.num_kv_heads
    tok = (wl.prefix_lens.astype(np.int64) + wl.counts).astype(np.int64)
    return int(4 * wl.head_dim * (tok * wl.counts * G).sum() * wl.num_kv_heads)


def measure_config(tv, name: str, seed: int, W: int, K: int, flush, stream, peaks: dict, full: bool):
    """GPU-only figures of one workload: the attention call and the walk, each
    timed alone with L2 flushed before every launch, and back to back over
    rotating input copies."""
    import torch
    wl, h = make_inputs(name, seed=seed)
    a_bytes = attention_bytes(wl)
    in_bytes = int(sum(v.nbytes for v in h.values()))
    l2 = int(getattr(torch.cuda.get_device_properties(torch.cuda.current_device()), "L2_cache_size", 126 << 20))
    copies = rotation_copies(a_bytes + 8 * wl.vocab * 3, in_bytes, l2)
    st = Step(tv, wl, h, copies)
    st.attn(stream)
    st.sample(stream)
    torch.cuda.synchronize()
    st.check_status(name)
    walk = st.walk()
    s_bytes = sampler_bytes(wl, h, walk["path"], walk["alen"])
    g_a = st.graph(lambda s: st.attn(s))
    g_s = st.graph(lambda s: st.sample(s))
    attn_ms = timed_replays(g_a, flush, stream, W, K)
    samp_ms = timed_replays(g_s, flush, stream, W, K)
    g_ab = st.graph(lambda s: [st.attn(s, i) for i in range(copies)])
    g_sb = st.graph(lambda s: [st.sample(s, i) for i in range(copies)])
    g_tb = st.graph(lambda s: [(st.attn(s, i), st.sample(s, i)) for i in range(copies)])
    reps = max(3, min(200, K // copies + 1))
    a_b2b = back_to_back_us(g_ab, copies, stream, 2, reps)
    s_b2b = back_to_back_us(g_sb, copies, stream, 2, reps)
    t_b2b = back_to_back_us(g_tb, copies, stream, 2, reps)
    st.check_status(name)
    hbm = peaks["hbm"]
    a_us = float(np.mean(attn_ms)) * 1e3
    res = {
        "workload": workload_config(name, wl, 1)["workload"],
        "attention_us": a_us, "sample_us": float(np.mean(samp_ms)) * 1e3,
        "attention_hbm_frac": a_bytes / (a_us * 1e-6) / 1e9 / hbm,
        "back_to_back": {"copies": copies, "step_us": t_b2b, "attention_us": a_b2b, "sample_us": s_b2b,
                         "attention_hbm_frac": a_bytes / (a_b2b * 1e-6) / 1e9 / hbm,
                         "step_hbm_frac": (a_bytes + s_bytes) / (t_b2b * 1e-6) / 1e9 / hbm,
                         "nodes_per_s": int(wl.counts.sum()) / (t_b2b * 1e-6)},
        "attention_bytes": a_bytes, "sampler_bytes": s_bytes,
        "kernel": "attn_tc" if st.aplan.kernel == 0 else "attn_simt", "splits": st.aplan.num_splits,
    }
    if wl.dtype == "bf16":
        fl = tensor_flops(wl)
        res["attention_tflops"] = fl / (a_us * 1e-6) / 1e12
        res["attention_tensor_frac_sustained"] = res["attention_tflops"] / peaks["bf16_sustained"]
        res["back_to_back"]["attention_tensor_frac_sustained"] = fl / (a_b2b * 1e-6) / 1e12 / peaks["bf16_sustained"]
    del g_a, g_s, g_ab, g_sb, g_tb
    return res, (wl, h, st, walk, attn_ms, samp_ms)


def time_select(tv, flush, stream, W, K, batch=64, per_seq=512, width=8, budget=64):
    """tv_tree_select_device (the dynamic tree, EAGLE-2) on grown candidate sets:
    `batch` sequences of `per_seq` candidates, trees of `budget` nodes; its own
    graph, L2 flushed before each launch."""
    import torch
    import synth
    off, par, tok, prob = synth.grown_candidates(batch, per_seq, width, seed=5)
    d = to_device({"off": off, "par": par, "tok": tok, "prob": prob})
    B = batch
    parent = torch.empty((B, budget), dtype=torch.int32, device="cuda")
    tokens = torch.empty_like(parent)
    index = torch.empty_like(parent)
    counts = torch.empty((B,), dtype=torch.int32, device="cuda")
    val = torch.empty((B,), dtype=torch.float64, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def call(st):
        s = tv.tv_tree_select_device(B, per_seq, d["off"], d["par"], d["tok"], d["prob"], budget, parent, tokens,
                                     index, counts, val, status, st)
        if s:
            raise tv.TreeVerifyError(s, "tv_tree_select_device")

    call(stream)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call(torch.cuda.current_stream())
    ms = timed_replays(g, flush, stream, W, K)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} from the tree selection")
    del g
    return {"us": float(np.mean(ms)) * 1e3, "sequences": B, "candidates_per_sequence": per_seq, "budget": budget,
            "note": "tv_tree_select_device on level-by-level grown candidates (width 8, best third expanded); "
                    "mean over launches, L2 flushed before each"}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import tree_speculative_decoding_07_b200 as tv

    torch.cuda.set_device(local_rank)
    wl, h = make_inputs(args.workload, seed=1 + 1000 * rank)
    st = Step(tv, wl, h)
    d = st.inputs[0]
    B, N = wl.batch, wl.num_nodes
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        st.attn(stream)
        st.sample(stream)

    # ---- device-resident timing (L2 flushed before every step).  The step is
    # replayed from one CUDA graph (attention, then the walk, launched with a
    # programmatic dependency so the walk's set-up overlaps attention's tail), so
    # host launch work stays out of the events.  Each kernel is then timed alone
    # from its own graph for the per-kernel figures and the roofline.
    W, K = args.warmup, args.steps
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    g_step = st.graph(lambda s: (st.attn(s), st.sample(s)))
    g_attn = st.graph(lambda s: st.attn(s))
    g_samp = st.graph(lambda s: st.sample(s))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for _ in range(W):
        flush.zero_()
        g_step.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_wall = time.perf_counter()
    for k in range(K):
        flush.zero_()
        e0, e1 = ev[k]
        e0.record(stream)
        g_step.replay()
        e1.record(stream)
    clocks.sample_now()  # the queued steps are still running
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    st.check_status("the timed steps")

    attn_ms = timed_replays(g_attn, flush, stream, W, K)
    samp_ms = timed_replays(g_samp, flush, stream, W, K)
    walk = st.walk()
    commit = time_commit(tv, wl, d, flush, stream, W, min(K, 200))
    logits_walk = time_logits_walk(tv, wl, d, flush, stream, W, min(K, 200), walk)
    fill = time_fill_topk(tv, wl, d, flush, stream, W, min(K, 200))
    select = time_select(tv, flush, stream, W, min(K, 200))
    total_ms = float(sum(step_ms))

    # ---- end to end: host (pinned) inputs -> device -> results back, every step
    pin = {k: torch.from_numpy(np.ascontiguousarray(v).view(np.int16) if v.dtype == np.uint16
                               else np.ascontiguousarray(v)).pin_memory() for k, v in h.items()}
    h2d = int(sum(v.numel() * v.element_size() for v in pin.values()))
    out_h = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    path_h = torch.empty(st.path.shape, dtype=torch.int32).pin_memory()
    alen_h = torch.empty(st.alen.shape, dtype=torch.int32).pin_memory()
    bonus_h = torch.empty(st.bonus.shape, dtype=torch.int32).pin_memory()
    d2h = sum(t.numel() * t.element_size() for t in (out_h, path_h, alen_h, bonus_h))
    K2 = max(3, min(K, 50))

    def e2e_step():
        for key, t in pin.items():
            dst = d[key]
            (dst.view(torch.int16) if dst.dtype == torch.bfloat16 else dst).copy_(t, non_blocking=True)
        step()
        out_h.copy_(st.out, non_blocking=True)
        path_h.copy_(st.path, non_blocking=True)
        alen_h.copy_(st.alen, non_blocking=True)
        bonus_h.copy_(st.bonus, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(K2):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a0.elapsed_time(a1)
    st.check_status("the end-to-end steps")

    # ---- every workload, GPU only (back-to-back figures beside the flushed ones)
    peak, peak_kind, pk = load_peaks()
    peaks = {"hbm": peak, "bf16_sustained": float(pk.get("bf16_tflops_sustained", FALLBACK_BF16_SUSTAINED))}
    configs = {}
    # every workload, at one GPU only (under torchrun each rank would repeat them)
    if not args.no_configs and world == 1:
        for name in ("tiny", "l8b", "l70b", "mix", "long", "ragged"):
            try:
                r, _ = measure_config(tv, name, 1 + 1000 * rank if name == args.workload else None, W,
                                      min(K, 200), flush, stream, peaks, full=False)
                configs[name] = r
            except Exception as e:  # a failure is reported, not hidden
                configs[name] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()

    total_ms, e2e_ms = reduce_max([total_ms, e2e_ms], world, "cuda")
    if rank != 0:
        return None

    nodes = int(wl.counts.sum())
    ms_step = total_ms / K
    value = job_throughput(world, nodes, K, total_ms)
    e2e_value = job_throughput(world, nodes, K2, e2e_ms)
    a_bytes = attention_bytes(wl)
    s_bytes = sampler_bytes(wl, h, walk["path"], walk["alen"])
    attn_avg_s = (sum(attn_ms) / K) / 1e3
    achieved = a_bytes / attn_avg_s / 1e9
    kernel_key = "attn_tc" if st.aplan.kernel == 0 else "attn_simt"
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "nodes/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_step,
        "us_per_step": ms_step * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic (Philox4x32-10 seeded; no dataset)",
        "config": workload_config(args.workload, wl, world),
        "attention_us": attn_avg_s * 1e6,
        "sample_us": (sum(samp_ms) / K) * 1e3,
        "per_kernel_timing": "each kernel replayed alone from its own graph, L2 flushed before each launch",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "frac_vs_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": ncu_traffic(kernel_key, args.workload), "kernel": kernel_key,
                     "algorithmic_bytes": a_bytes, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s"},
        "step_roofline": {"bytes": a_bytes + s_bytes, "sampler_bytes": s_bytes,
                          "frac": (a_bytes + s_bytes) / (ms_step / 1e3) / 1e9 / peak,
                          "frac_vs_nominal_8tbs": (a_bytes + s_bytes) / (ms_step / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                          "sampler_bytes_literal": 2 * 4 * B * N * wl.vocab,
                          "note": "sampler bytes: rows the walk reads (algorithmic); literal = all of p and q"},
        "median_us_per_step": float(np.median(step_ms)) * 1e3,
        "commit": commit,
        "sample_logits": logits_walk,
        "tree_fill_topk": fill,
        "tree_select_device": select,
        "e2e": {"value": e2e_value, "unit": "nodes/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": K2},
        "gpu_launches": K * (st.aplan.launches + st.splan.launches),
        "clocks": clk,
        "wall_s": t_wall,
    }
    if args.workload in configs and "back_to_back" in configs[args.workload]:
        line["back_to_back"] = dict(configs[args.workload]["back_to_back"],
                                    note="steps replayed back to back from one graph over rotating input copies "
                                         "(one pass over the copies reads at least twice the L2 size); no flush, "
                                         "so launch gaps overlap with the previous kernel's tail")
    if configs:
        line["configs"] = configs
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, h, budget_s=args.cpu_budget)
        ref = line["cpu_baseline"].pop("walk")
        same = ((walk["alen"] == ref["accepted_len"]) & (walk["bonus"] == ref["bonus_token"])
                & (walk["path"] == ref["accepted_path"]).all(axis=1))
        line["walk_check"] = {
            "near_threshold": int((ref["near"] > 0).sum()),
            "matches_oracle": bool(same.all()),
            "mismatches_outside_band": int((~same & ~(ref["near"] > 0)).sum()),
            "sequences": int(B),
            "note": "the timed inputs' walk against the oracle's (from the cpu_baseline leg); near_threshold counts "
                    "sequences with a uniform within 1e-6 of an acceptance or CDF threshold"}
    return line


# ------------------------------------------------------------------ oracle timing

def oracle_step_times(wl, h, rows_frac: float):
    """Time the oracle on one step: attention over a deterministic fraction of
    the query rows (extrapolated to all rows) plus the full acceptance walk."""
    import oracle
    B, N, Hq = wl.batch, wl.num_nodes, wl.num_q_heads
    if wl.node_counts is not None:
        # ragged trees: each sequence is its own oracle problem over its own nodes
        total_rows = int(wl.counts.sum()) * Hq
        done = 0
        t0 = time.perf_counter()
        for b in range(B):
            nb = int(wl.counts[b])
            m = max(1, int(round(nb * Hq * rows_frac)))
            sel = np.linspace(0, nb * Hq - 1, m).astype(np.int64)
            rows = np.stack([np.zeros_like(sel), sel // Hq, sel % Hq], axis=1).astype(np.int32)
            oracle.tree_attention(h["query"][b:b + 1, :nb], h["k"], h["v"], h["block_table"][b:b + 1],
                                  h["prefix_lens"][b:b + 1], h["parent_idx"][b:b + 1, :nb], wl.num_kv_heads,
                                  wl.dtype, rows=rows)
            done += m
        t_attn = (time.perf_counter() - t0) * total_rows / done
        t0 = time.perf_counter()
        walk = oracle.verify_sample_ragged(h["p"], h["q"], h["tokens"], h["parent_idx"], h["uniforms"], wl.counts)
        return t_attn + time.perf_counter() - t0, done, total_rows, walk
    total_rows = B * N * Hq
    n = max(1, int(round(total_rows * rows_frac)))
    sel = np.linspace(0, total_rows - 1, n).astype(np.int64)
    rows = np.stack([sel // (N * Hq), (sel // Hq) % N, sel % Hq], axis=1).astype(np.int32)
    t0 = time.perf_counter()
    oracle.tree_attention(h["query"], h["k"], h["v"], h["block_table"], h["prefix_lens"], h["parent_idx"],
                          wl.num_kv_heads, wl.dtype, rows=rows)
    t_attn = (time.perf_counter() - t0) * total_rows / n
    t0 = time.perf_counter()
    walk = oracle.verify_sample(h["p"], h["q"], h["tokens"], h["parent_idx"], h["uniforms"])
    t_walk = time.perf_counter() - t0
    return t_attn + t_walk, n, total_rows, walk


def cpu_baseline(wl, h, budget_s: float = 20.0):
    import oracle
    cores = oracle.max_threads()
    # calibrate with a small fraction, then size the sample to the budget
    t_est, n, total, walk = oracle_step_times(wl, h, 1.0 / 64)
    frac = min(1.0, max(1.0 / 64, budget_s / max(t_est, 1e-9)))
    steps, t_sum, rows_done = 0, 0.0, 0
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s or steps == 0:
        t, n, total, walk = oracle_step_times(wl, h, frac)
        t_sum += t
        rows_done += n
        steps += 1
        if frac >= 1.0 and time.perf_counter() - t_start > budget_s / 2:
            break
    per_step = t_sum / steps
    # the same step on one core, on a smaller attention sample (a few seconds at most)
    oracle.set_threads(1)
    try:
        t1, n1, _, _ = oracle_step_times(wl, h, 1.0 / 256)
    finally:
        oracle.set_threads(cores)
    return {"value": int(wl.counts.sum()) / per_step, "unit": "nodes/s", "cores": cores, "kind": "oracle",
            "sample": f"{steps} oracle step(s): attention on {rows_done // steps} of {total} query rows "
                      f"(time scaled to all rows) plus the full fp64 acceptance walk; "
                      f"{per_step * 1e3:.1f} ms per full step",
            "single_thread": {"value": int(wl.counts.sum()) / t1, "unit": "nodes/s", "cores": 1,
                              "sample": f"one step: attention on {n1} of {total} query rows (time scaled to all "
                                        f"rows) plus the full acceptance walk; {t1 * 1e3:.1f} ms per full step"},
            "walk": walk}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import oracle
    wl, h = make_inputs(args.workload, seed=1)
    K, W = args.steps, args.warmup
    budget = 150.0
    t_est, _, _, _ = oracle_step_times(wl, h, 1.0 / 64)
    frac = min(1.0, max(1.0 / 1024, budget / max(1, K + W) / max(t_est, 1e-9)))
    for _ in range(W):
        oracle_step_times(wl, h, frac)
    times = []
    n_rows = 0
    for _ in range(K):
        t, n_rows, total, _ = oracle_step_times(wl, h, frac)
        times.append(t)
    per_step = sum(times) / K
    value = int(wl.counts.sum()) / per_step
    cores = oracle.max_threads()
    sample = (f"each step: oracle attention on {n_rows} of {total} query rows (time scaled to all rows) "
              f"plus the full fp64 acceptance walk")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "nodes/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": per_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (Philox4x32-10 seeded; no dataset)",
            "config": workload_config(args.workload, wl, world), "cpu_baseline": {"value": value, "unit": "nodes/s",
                                                                  "cores": cores, "kind": "oracle",
                                                                  "sample": sample},
            "e2e": {"value": value, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="l8b", choices=("tiny", "l8b", "l70b", "mix", "long", "ragged"))
    ap.add_argument("--cpu-budget", type=float, default=20.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload GPU figures")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        import datetime

        import torch.distributed as dist
        if world > 1:
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=None)
        try:
            line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()

"""The C-ABI library loads, exports every symbol ``include/*.h`` declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

import tree_speculative_decoding_07_b200 as tv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"TV_API\s+[\w\s\*]*?\b(tv_\w+)\s*\(", text)
    return sorted(set(names))


def test_library_exports_every_declared_symbol():
    L = tv.lib()
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_version_and_status_strings():
    assert tv.tv_version() >= 100
    for s in range(8):
        assert tv.tv_status_string(s)
    assert "unknown" in tv.tv_status_string(99)


def _desc(**kw):
    base = dict(batch=1, num_nodes=5, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=16,
                max_blocks_per_seq=9, num_blocks=9, dtype=tv.TV_F32, softmax_scale=0.0)
    base.update(kw)
    return tv.TvAttnDesc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0), tv.TV_ERR_INVALID_ARG),
    (dict(num_q_heads=6, num_kv_heads=4), tv.TV_ERR_INVALID_ARG),
    (dict(num_nodes=129), tv.TV_ERR_UNSUPPORTED),
    (dict(head_dim=96), tv.TV_ERR_UNSUPPORTED),
    (dict(block_size=32), tv.TV_ERR_UNSUPPORTED),
    (dict(dtype=7), tv.TV_ERR_INVALID_ARG),
    (dict(softmax_scale=-1.0), tv.TV_ERR_INVALID_ARG),
    (dict(max_blocks_per_seq=0), tv.TV_ERR_INVALID_ARG),
])
def test_attention_rejects_bad_descriptors(kw, status):
    d = _desc(**kw)
    plan = tv.TvAttnPlan()
    assert tv.lib().tv_tree_attention_plan(ctypes.byref(d), ctypes.byref(plan)) == status
    dummy = 256
    assert tv.tv_tree_attention(d, dummy, dummy, dummy, dummy, dummy, dummy, dummy, stream=0) == status


def test_attention_rejects_null_pointers_and_small_workspace():
    d = _desc()
    assert tv.tv_tree_attention(d, None, 256, 256, 256, 256, 256, 256, stream=0) == tv.TV_ERR_INVALID_ARG
    d = _desc(batch=1, num_nodes=64, num_q_heads=32, num_kv_heads=8, head_dim=128, max_blocks_per_seq=4096,
              num_blocks=4096, dtype=tv.TV_F32)
    need = tv.tv_tree_attention_workspace_size(d)
    plan = tv.tv_tree_attention_plan(d)
    assert plan.workspace_bytes == need
    if need:
        assert tv.tv_tree_attention(d, 256, 256, 256, 256, 256, 256, 256, 256, need - 1, stream=0) == tv.TV_ERR_WORKSPACE
        assert tv.tv_tree_attention(d, 256, 256, 256, 256, 256, 256, 256, None, need, stream=0) == tv.TV_ERR_WORKSPACE


def test_static_attention_refuses_oversize_scratch_on_the_host():
    # fp32, head_dim 128: 96 query rows x 49 KV splits of partials need more than the fixed array
    d = _desc(batch=1, num_nodes=32, num_q_heads=3, num_kv_heads=1, head_dim=128, max_blocks_per_seq=800,
              num_blocks=800, dtype=tv.TV_F32)
    assert tv.tv_tree_attention_plan(d).workspace_bytes > tv.TV_STATIC_SCRATCH_BYTES
    a = 256
    assert tv.tv_tree_attention_static(d, a, a, a, a, a, a, a, None, stream=0) == tv.TV_ERR_WORKSPACE
    # the tensor-core path (bf16, head_dim 128) needs no scratch at all
    d = _desc(num_nodes=64, num_q_heads=32, num_kv_heads=8, head_dim=128, max_blocks_per_seq=260,
              num_blocks=260, dtype=tv.TV_BF16)
    assert tv.tv_tree_attention_plan(d).workspace_bytes == 0


def test_attention_plans():
    # bf16 head_dim 128 runs on the tensor-core kernel, fp32 on the CUDA-core kernel
    d = _desc(num_nodes=64, num_q_heads=32, num_kv_heads=8, head_dim=128, max_blocks_per_seq=260,
              num_blocks=260, dtype=tv.TV_BF16)
    p = tv.tv_tree_attention_plan(d)
    assert p.num_splits >= 1 and p.grid_ctas >= 1 and p.launches >= 1
    d = _desc()
    p = tv.tv_tree_attention_plan(d)
    assert p.kernel == 1 and p.row_tiles == 1


@pytest.mark.parametrize("kw,status", [
    (dict(batch=0, num_nodes=4, vocab=10), tv.TV_ERR_INVALID_ARG),
    (dict(batch=1, num_nodes=0, vocab=10), tv.TV_ERR_INVALID_ARG),
    (dict(batch=1, num_nodes=1025, vocab=10), tv.TV_ERR_UNSUPPORTED),
    (dict(batch=1, num_nodes=4, vocab=16 * 13824 + 1), tv.TV_ERR_UNSUPPORTED),
])
def test_sampler_rejects_bad_descriptors(kw, status):
    d = tv.TvSampleDesc(**kw)
    dummy = 256
    assert tv.tv_verify_sample(d, *([dummy] * 8), stream=0) == status
    assert tv.tv_verify_sample_logits(d, *([dummy] * 8), stream=0) == status


def test_sampler_rejects_null_pointers():
    d = tv.TvSampleDesc(2, 8, 1000)
    for i in (0, 1, 2, 4, 5, 6, 7):  # parent_idx (3) may be NULL: chains
        args = [256] * 8
        args[i] = 0
        assert tv.tv_verify_sample(d, *args, stream=0) == tv.TV_ERR_INVALID_ARG
        assert tv.tv_verify_sample_logits(d, *args, stream=0) == tv.TV_ERR_INVALID_ARG


def test_sampler_plan_covers_vocab():
    for V in (8, 1000, 128256, 151936):
        p = tv.tv_verify_sample_plan(tv.TvSampleDesc(1, 64, V))
        assert p.cluster_ctas * p.slice >= V and p.slice % 4 == 0
        assert 32 <= p.threads <= 512 and p.threads % 32 == 0
        # two row buffers of p and q, then (when they fit) the gathered child values,
        # 16 bytes per node; small vocabularies always leave room
        assert p.smem_bytes in (16 * p.slice, 16 * p.slice + 16 * 64)
        if V <= 1000:
            assert p.smem_bytes == 16 * p.slice + 16 * 64
    # the largest vocabulary leaves no room for the gathered values with 1024 nodes
    big = tv.tv_verify_sample_plan(tv.TvSampleDesc(1, 1024, 16 * 13824))
    assert big.smem_bytes == 16 * big.slice
    assert tv.tv_verify_sample_workspace_size(tv.TvSampleDesc(1, 64, 1000)) == 0


def test_commit_rejects_bad_arguments_before_launch():
    d = _desc(num_nodes=8, num_q_heads=4, num_kv_heads=2, head_dim=64, max_blocks_per_seq=4, num_blocks=8)
    a = 256  # a non-null, 16-byte aligned dummy address: nothing is launched on these paths
    assert tv.tv_commit_path(d, None, a, a, a, a, a, a + 64, stream=0) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_commit_path(d, a, a, a, a, a, a, None, stream=0) == tv.TV_ERR_INVALID_ARG
    # the new lengths may not overwrite the lengths still being read
    assert tv.tv_commit_path(d, a, a, a, 512, a, a, 512, stream=0) == tv.TV_ERR_INVALID_ARG
    # rows move as 16-byte pieces
    assert tv.tv_commit_path(d, a + 8, a, a, a, a, a, a + 64, stream=0) == tv.TV_ERR_INVALID_ARG
    bad = _desc(head_dim=96)
    assert tv.tv_commit_path(bad, a, a, a, a, a, a, a + 64, stream=0) == tv.TV_ERR_UNSUPPORTED


def test_fill_topk_rejects_bad_arguments_before_launch():
    assert tv.tv_tree_fill_topk(tv.TvSampleDesc(0, 4, 10), 256, 256, 256, 256, stream=0) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_fill_topk(tv.TvSampleDesc(1, 4, 10), None, 256, 256, 256, stream=0) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_fill_topk(tv.TvSampleDesc(1, 4, 10), 256, 256, 256, None, stream=0) == tv.TV_ERR_INVALID_ARG
    assert tv.tv_tree_fill_topk(tv.TvSampleDesc(1, 1025, 10), 256, 256, 256, 256, stream=0) == tv.TV_ERR_UNSUPPORTED


def test_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes structs have the C header's sizes and field offsets
    (compiled with the host C compiler against include/treeverify.h)."""
    import subprocess
    structs = {"tv_attn_desc": tv.TvAttnDesc, "tv_attn_plan": tv.TvAttnPlan, "tv_sample_desc": tv.TvSampleDesc,
               "tv_sample_plan": tv.TvSamplePlan}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "treeverify.h"', "int main(void) {"]
    for cname, cls in structs.items():
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in cls._fields_:
            lines.append(f'printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    include = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.check_call(["gcc", "-std=c11", "-I", include, "-o", str(exe), str(src)])
    got = dict(((l.split()[0], l.split()[1]), int(l.split()[2])) for l in subprocess.check_output([str(exe)], text=True)
               .splitlines())
    for cname, cls in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(cls), cname
        for fname, _ in cls._fields_:
            assert got[(cname, fname)] == getattr(cls, fname).offset, (cname, fname)

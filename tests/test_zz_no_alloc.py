"""tv_tree_attention_static: the attention call for callers that cannot
allocate device memory (a fixed memory pool, an allocator-free hot path, work
recorded into a CUDA graph).  It must give the same results as
tv_tree_attention with a caller workspace, bit for bit and call after call,
although every call reuses the library's one fixed scratch array: the calls
below alternate between problems with different launch plans, so a call
that read what the previous one left in the array would show here."""
import numpy as np
import pytest
import torch

import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import Attn, random_attn

pytestmark = pytest.mark.gpu


def _case(a):
    a.to_device()
    desc = tv.attn_desc(a.dq, a.dk, a.dbt)
    plan = tv.tv_tree_attention_plan(desc)
    ref = tv.tree_attention(a.dq, a.dk, a.dv, a.dbt, a.dpl, a.dpar)
    torch.cuda.synchronize()
    return a, desc, plan, ref


def _static(a, desc, status):
    out = torch.full_like(a.dq, float("nan"))
    rc = tv.tv_tree_attention_static(desc, a.dq, a.dk, a.dv, a.dbt, a.dpl, a.dpar, out, status)
    torch.cuda.synchronize()
    assert rc == tv.TV_OK, tv.tv_status_string(rc)
    assert int(status.item()) == 0
    return out


def test_static_scratch_matches_workspace_path():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cases = [
        # the Llama-3-8B shape (bf16, tensor cores, several KV splits)
        _case(Attn.from_workload(synth.make("l8b", need_tokens=False))),
        # fp32 on the CUDA cores: 10 KV splits merged through scratch memory
        _case(random_attn(71, 1, 16, 8, 2, 128, [600], dtype="f32")),
        # bf16, head_dim 64 (CUDA cores), another split count and batch
        _case(random_attn(72, 3, 9, 16, 4, 64, [700, 2100, 64], dtype="bf16")),
    ]
    assert any(c[2].workspace_bytes > 0 for c in cases)
    assert len({(c[2].kernel, c[2].num_splits, c[2].grid_ctas) for c in cases}) == len(cases)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):   # every problem twice, each call after a call with another plan
        for a, desc, plan, ref in cases:
            out = _static(a, desc, status)
            assert torch.equal(out, ref), (plan.kernel, plan.num_splits)


def test_static_scratch_refuses_oversize_problems():
    """A CUDA-core problem whose split merge needs more than the fixed array
    (fp32, head_dim 128, 96 query rows x 49 KV splits) is refused before any
    launch, and the refusal leaves the next call working."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    d = tv.TvAttnDesc(batch=1, num_nodes=32, num_q_heads=3, num_kv_heads=1, head_dim=128, block_size=16,
                      max_blocks_per_seq=800, num_blocks=800, dtype=tv.TV_F32, softmax_scale=0.0)
    plan = tv.tv_tree_attention_plan(d)
    assert plan.workspace_bytes > tv.TV_STATIC_SCRATCH_BYTES
    buf = torch.zeros(1 << 20, dtype=torch.float32, device="cuda")
    p = buf.data_ptr()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert tv.tv_tree_attention_static(d, p, p, p, p, p, p, p, status) == tv.TV_ERR_WORKSPACE
    a = random_attn(73, 1, 16, 8, 2, 128, [600], dtype="f32")
    a, desc, plan, ref = _case(a)
    assert torch.equal(_static(a, desc, status), ref)

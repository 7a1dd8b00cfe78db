"""tv_tree_attention_static: the attention call for callers that cannot
allocate device memory (a fixed memory pool, an allocator-free hot path, work
recorded into a CUDA graph).  It must give the same results as
tv_tree_attention with a caller workspace, call after call, although every
call reuses the library's one fixed scratch array."""
import numpy as np
import pytest
import torch

import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import BF16_ATOL, Attn


@pytest.mark.gpu
def test_static_scratch_matches_workspace_path():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    # the Llama-3-8B shape: its KV splits merge through scratch memory
    a = Attn.from_workload(synth.make("l8b", need_tokens=False)).to_device()
    desc = tv.attn_desc(a.dq, a.dk, a.dbt)
    plan = tv.tv_tree_attention_plan(desc)
    assert plan.workspace_bytes > 0
    ref = tv.tree_attention(a.dq, a.dk, a.dv, a.dbt, a.dpl, a.dpar)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):   # two calls in a row share the scratch array
        out = torch.full_like(a.dq, float("nan"))
        rc = tv.tv_tree_attention_static(desc, a.dq, a.dk, a.dv, a.dbt, a.dpl, a.dpar, out, status)
        torch.cuda.synchronize()
        assert rc == tv.TV_OK
        assert int(status.item()) == 0
        diff = (out.float() - ref.float()).abs().max().item()
        assert np.isfinite(diff) and diff <= BF16_ATOL

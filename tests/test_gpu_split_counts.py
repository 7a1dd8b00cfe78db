"""Tensor-core attention parity across the KV split counts the plan picks.

The splits of a row tile form one thread-block cluster and merge in place through
distributed shared memory, with one combine routine per split count.  These shapes
vary the number of (sequence, KV head, row tile) groups and the prefix length so the
plan, which depends on how many clusters of each size the device holds at once,
picks many different counts.  Outputs are of order one (unit-variance K and V,
scaled tree keys), so a wrong owner share, a wrong peer address or a missed partial
moves them far beyond bf16 rounding."""
import pytest
import torch

import synth
import tree_speculative_decoding_07_b200 as tv
from gpu_cases import random_attn, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


# (B, N, Hq, Hkv, prefix): groups = B * Hkv * ceil(N * Hq / Hkv / 128)
SHAPES = [
    (1, 32, 4, 1, 8192),    # 1 group: as many splits as a cluster allows
    (1, 32, 32, 8, 8192),   # 8 groups
    (3, 32, 16, 4, 8192),   # 12 groups
    (1, 64, 32, 8, 4096),   # 16 groups (the Llama-3-8B shape)
    (13, 32, 8, 2, 2048),   # 26 groups
    (15, 32, 8, 2, 2048),   # 30 groups
    (20, 32, 8, 2, 2048),   # 40 groups
    (30, 32, 8, 2, 2048),   # 60 groups
]

_seen = set()


@pytest.mark.parametrize("B,N,Hq,Hkv,prefix", SHAPES)
def test_split_count_parity(B, N, Hq, Hkv, prefix):
    a = random_attn(100 + B * Hkv, B, N, Hq, Hkv, 128, [prefix] * B, kv_std=1.0,
                    tree_k_scale=synth.UNIT_TREE_K_SCALE)
    a.to_device()
    plan = tv.tv_tree_attention_plan(tv.attn_desc(a.dq, a.dk, a.dbt))
    assert plan.kernel == 0  # the tensor-core path
    _seen.add(int(plan.num_splits))
    out = a.run_gpu()
    # every third node of every sequence at two heads, plus random rows
    a.compare(out, sample_rows(B, N, Hq, 96, B * 7 + N, must_nodes=range(0, N, 3)))


def test_split_counts_covered():
    # runs after the parity cases above (same module, definition order)
    print("split counts exercised:", sorted(_seen))
    assert len(_seen) >= 6, f"split counts exercised: {sorted(_seen)}"
    assert max(_seen) >= 10 and min(_seen) <= 3, f"split counts exercised: {sorted(_seen)}"

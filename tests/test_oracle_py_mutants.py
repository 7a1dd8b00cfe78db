"""The pins of the oracle's Python-level functions must catch plausible mistakes.

Each case copies the oracle package (with its C library), the input generator
and the tests into a scratch directory, plants one mistake in the copy of
``oracle/__init__.py`` (on the CPU), and runs the relevant pin tests there; at
least one pin must fail.  The C-level mutants live in test_oracle_mutants.py."""
import os
import shutil
import subprocess
import sys

import pytest

import oracle
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

TREE = ["tests/test_oracle_treebuild.py"]
RAGGED = ["tests/test_oracle_ragged.py"]
LOGITS = ["tests/test_oracle_logits.py"]

MUTANTS = [
    # (name, original text, planted text, pin files)
    ("dp_child_not_counted", "v = accept[i] * (1.0 + F[d - 1][t]) + G[i + 1][s - t]",
     "v = accept[i] * F[d - 1][t] + G[i + 1][s - t]", TREE),
    ("dp_depth_off_by_one", "D = budget - 1 if max_depth is None else min(max_depth, budget - 1)",
     "D = budget - 1 if max_depth is None else min(max_depth + 1, budget - 1)", TREE),
    ("dp_ties_to_larger_t", "if v > best:", "if v >= best:", TREE),
    ("value_not_a_product", "reach[c] = reach[parent[c]] * accept[rank[c]]", "reach[c] = accept[rank[c]]", TREE),
    ("topk_ties_to_higher_id", 'idx[r] = np.argsort(-flat[r].astype(np.float64), kind="stable")[:k]',
     'idx[r] = np.argsort(flat[r].astype(np.float64), kind="stable")[::-1][:k]', TREE),
    ("fill_ignores_rank", "tokens[b, c] = idx[int(rk[b, c])]", "tokens[b, c] = idx[0]", TREE),
    ("chain_parent_is_root", "return np.tile(np.arange(-1, N - 1, dtype=np.int32), (B, 1))",
     "return np.tile(np.array([-1] + [0] * (N - 1), dtype=np.int32), (B, 1))", RAGGED),
    ("ragged_walk_ignores_counts", """    for b in range(B):
        n = int(node_counts[b])
        if n == 0:
            continue
        r = walk(""", """    for b in range(B):
        n = N
        if n == 0:
            continue
        r = walk(""", RAGGED),
    ("ragged_empty_draws_a_token", '"bonus_token": np.full(B, -1, np.int32)', '"bonus_token": np.full(B, 0, np.int32)',
     RAGGED),
    ("select_score_not_a_product", "score[c] = (score[par[c]] if par[c] >= 0 else 1.0) * prob[c]",
     "score[c] = prob[c]", TREE),
    ("select_ties_to_higher_index", "order = sorted(range(M), key=lambda c: (-score[c], c))",
     "order = sorted(range(M), key=lambda c: (-score[c], -c))", TREE),
    ("speedup_counts_the_root_as_a_draft", "return (1.0 + expected_accepted) / (draft_cost + 1.0 + alpha * (num_nodes - 1))",
     "return (1.0 + expected_accepted) / (draft_cost + 1.0 + alpha * num_nodes)", TREE),
    ("speedup_without_the_bonus", "return (1.0 + expected_accepted) / (draft_cost + 1.0 + alpha * (num_nodes - 1))",
     "return expected_accepted / (draft_cost + 1.0 + alpha * (num_nodes - 1))", TREE),
    ("merge_keys_on_token_only", "            key = (u, int(t))", "            key = (0, int(t))", TREE),
    ("softmax_wrong_axis", "return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)",
     "return (e / e.sum(axis=0, keepdims=True)).astype(np.float32)", LOGITS),
]


def _scratch_copy(tmp_path):
    root = tmp_path / "root"
    shutil.copytree(os.path.join(ROOT, "oracle"), root / "oracle", ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "synth"), root / "synth", ignore=shutil.ignore_patterns("__pycache__"))
    shutil.copytree(os.path.join(ROOT, "tests"), root / "tests", ignore=shutil.ignore_patterns("__pycache__"))
    return root


def _run(root, files):
    oracle.build()
    synth.build()
    env = dict(os.environ)
    env.pop("ORACLE_LIB", None)
    return subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *files], cwd=root,
                          env=env, capture_output=True, text=True, timeout=600)


@pytest.mark.parametrize("name,orig,planted,files", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, orig, planted, files):
    root = _scratch_copy(tmp_path)
    init = root / "oracle" / "__init__.py"
    src = init.read_text()
    assert src.count(orig) == 1, f"mutation anchor for {name} not unique"
    init.write_text(src.replace(orig, planted))
    r = _run(root, files)
    assert r.returncode != 0, f"no pin caught mutant {name}:\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same procedure without a planted mistake passes."""
    root = _scratch_copy(tmp_path)
    r = _run(root, TREE + RAGGED + LOGITS)
    assert r.returncode == 0, r.stdout[-2000:]

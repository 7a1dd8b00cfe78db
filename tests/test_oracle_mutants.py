"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/oracle.c`` (on the CPU),
builds it, and runs the relevant pin tests against that build through
``ORACLE_LIB``; at least one pin must fail."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

ATTN = ["tests/test_oracle_mask.py", "tests/test_oracle_attention.py"]
SAMP = ["tests/test_oracle_sampler.py"]
COMMIT = ["tests/test_oracle_commit.py"]

MUTANTS = [
    # (name, original text, planted text, pin files)
    ("mask_transposed", "mask[(size_t)i * n + j] = 1", "mask[(size_t)j * n + i] = 1", ATTN),
    ("mask_parent_only", "j >= 0; j = parent[j]) mask", "j >= 0 && j >= i - 1; j = parent[j]) mask", ATTN),
    ("gqa_modulo", "const int32_t kvh = h / G;", "const int32_t kvh = h % Hkv;", ATTN),
    ("scale_dropped", "s[t] = scale * dot;", "s[t] = dot;", ATTN),
    ("prefix_off_by_one", "for (int64_t t = 0; t < L; ++t) pos[nk++] = t;",
     "for (int64_t t = 0; t + 1 < L; ++t) pos[nk++] = t;", ATTN),
    ("softmax_no_max_weight", "double w = exp(s[t] - m);", "double w = exp(s[t] - m) * (t == 0 ? 2.0 : 1.0);", ATTN),
    ("residual_sign", "R[y] = fmax(0.0, P[y] - (double)Q[y]);", "R[y] = fmax(0.0, P[y] + (double)Q[y]);", SAMP),
    ("residual_not_renormalised", "P[y] = R[y] / z;", "P[y] = R[y];", SAMP),
    ("residual_from_original_p", "P[y] = R[y] / z;", "P[y] = P[y];", SAMP),
    ("non_strict_accept", "accept = r < alpha;", "accept = r <= alpha;", SAMP),
    ("ratio_inverted", "const double alpha = P[x] / qx;", "const double alpha = qx / P[x];", SAMP),
    ("child_keeps_residual", "for (int64_t x = 0; x < V; ++x) P[x] = (double)pc[x];",
     "(void)pc;", SAMP),
    ("siblings_descending", "for (int32_t c = u + 1; c < N; ++c) {", "for (int32_t c = N - 1; c > u; --c) {", SAMP),
    ("cdf_non_strict", "if (run > target) { k = x; break; }", "if (run >= target) { k = x; break; }", SAMP),
    ("commit_dest_off_by_one", "const int32_t t = L + 1 + k;", "const int32_t t = L + k;", COMMIT),
    ("commit_length_without_root", "new_prefix_lens[b] = L + 1 + n;", "new_prefix_lens[b] = L + n;", COMMIT),
    ("commit_path_reversed", "const int32_t t = L + pb[k];", "const int32_t t = L + pb[n - 1 - k];", COMMIT),
    ("commit_accepts_non_increasing", "if (pb[k] <= prev || pb[k] >= N) ok = 0;", "if (pb[k] >= N) ok = 0;",
     COMMIT),
]


@pytest.mark.parametrize("name,orig,planted,files", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, orig, planted, files):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation anchor for {name} not unique"
    mutant_c = tmp_path / "oracle_mutant.c"
    mutant_c.write_text(src.replace(orig, planted))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(so), str(mutant_c), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", *files], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught mutant {name}:\n{r.stdout[-2000:]}"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same procedure without a planted mistake passes."""
    so = tmp_path / "liboracle_copy.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-o", str(so), SRC, "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", *ATTN, *SAMP], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:]

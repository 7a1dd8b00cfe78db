"""The C ABI from a plain C client: a small program compiled against
include/treeverify.h and linked to libtreeverify.so calls the host-only
entry points (and the argument checks of a device entry point, which return
before any launch) and prints what it gets; the results must equal the
Python binding's and the oracle's."""
import os
import subprocess

import numpy as np

import oracle
import tree_speculative_decoding_07_b200 as tv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

PROGRAM = r"""
#include <stdio.h>
#include "treeverify.h"

int main(void) {
    const double accept[3] = {0.6, 0.25, 0.1};
    int32_t parent[40], rank[40], n = 0;
    double value = 0.0;
    if (tv_tree_shape(accept, 3, 40, 5, parent, rank, &n, &value) != TV_OK) return 1;
    printf("shape %d %.17g\n", n, value);
    for (int i = 0; i < n; ++i) printf("%d %d\n", parent[i], rank[i]);

    const int32_t cand_parent[6] = {-1, -1, 0, 0, 2, 1};
    const int32_t cand_token[6] = {11, 12, 13, 14, 15, 16};
    const double cand_prob[6] = {0.7, 0.2, 0.6, 0.3, 0.9, 0.5};
    int32_t sp[4], st[4], si[4], sn = 0;
    double sv = 0.0;
    if (tv_tree_select(cand_parent, cand_token, cand_prob, 6, 4, sp, st, si, &sn, &sv) != TV_OK) return 2;
    printf("select %d %.17g\n", sn, sv);
    for (int i = 0; i < sn; ++i) printf("%d %d %d\n", sp[i], st[i], si[i]);

    tv_attn_desc bad = {0};
    printf("status %d %s\n", (int)tv_tree_attention(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0),
           tv_status_string(TV_ERR_INVALID_ARG));
    printf("version %d\n", (int)tv_version());
    return 0;
}
"""


def test_c_program_links_and_agrees(tmp_path):
    libdir = os.path.dirname(tv.lib()._name)
    src = tmp_path / "client.c"
    src.write_text(PROGRAM)
    exe = tmp_path / "client"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src),
                           "-L", libdir, "-ltreeverify", f"-Wl,-rpath,{libdir}"])
    out = subprocess.check_output([str(exe)], text=True).splitlines()
    head = out[0].split()
    n = int(head[1])
    par = np.array([int(l.split()[0]) for l in out[1:1 + n]], np.int32)
    rk = np.array([int(l.split()[1]) for l in out[1:1 + n]], np.int32)
    rp, rr, rv = oracle.tree_shape_dp([0.6, 0.25, 0.1], 40, 5)
    np.testing.assert_array_equal(par, rp)
    np.testing.assert_array_equal(rk, rr)
    assert float(head[2]) == rv
    sel = out[1 + n].split()
    m = int(sel[1])
    rows = [list(map(int, l.split())) for l in out[2 + n:2 + n + m]]
    sp, st, si, sv = oracle.select_tree([-1, -1, 0, 0, 2, 1], [11, 12, 13, 14, 15, 16],
                                        [0.7, 0.2, 0.6, 0.3, 0.9, 0.5], 4)
    assert [r[0] for r in rows] == sp.tolist() and [r[1] for r in rows] == st.tolist()
    assert [r[2] for r in rows] == si.tolist() and float(sel[2]) == sv
    status = out[2 + n + m].split()
    assert int(status[1]) == tv.TV_ERR_INVALID_ARG and "invalid argument" in out[2 + n + m]
    assert out[-1] == f"version {tv.tv_version()}"

"""Shared test helpers: golden-file readers and small input builders.

Nothing here computes the method; expected values come from the pages
(tests/golden), closed forms, library routines or the oracle."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def contiguous_table(prefix_lens, n_nodes, bs=16):
    """Identity block table: sequence b's logical blocks are consecutive."""
    nblk = [(int(L) + n_nodes + bs - 1) // bs for L in prefix_lens]
    mb = max(nblk)
    bt = np.full((len(prefix_lens), mb), -1, dtype=np.int32)
    off = 0
    for b, n in enumerate(nblk):
        bt[b, :n] = np.arange(off, off + n)
        off += n
    return bt, off


def dense_kv_to_paged(kv, block_table, bs=16):
    """kv: list over b of [T_b][Hkv][D] arrays -> paged cache [nb][bs][Hkv][D]."""
    nb = int(block_table.max()) + 1
    Hkv, D = kv[0].shape[1:]
    cache = np.zeros((nb, bs, Hkv, D), dtype=kv[0].dtype)
    for b, x in enumerate(kv):
        for t in range(x.shape[0]):
            cache[block_table[b, t // bs], t % bs] = x[t]
    return cache

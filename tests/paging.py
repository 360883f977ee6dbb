"""Test helpers: lay a logical per-sequence K/V stream into a block pool.

Plain numpy indexing in the documented cache layout [num_blocks, block_size,
num_kv_heads, head_dim]: token t of sequence b goes to
pool[table[b][t // bs], t % bs].  Used to build inputs whose dense (logically
contiguous) attention is known independently of any paged gather.
"""
from __future__ import annotations

import numpy as np


def cdiv(a, b):
    return -(-a // b)


def page_logical(seqs, block_size, rng, num_blocks=None, fill=None, order=None):
    """seqs: list of arrays [ctx_b, Hkv, d] (same dtype).  Returns (tables int32
    [B, MB], pool [NB, bs, Hkv, d]).  Blocks are drawn from a random
    permutation of the pool (or ``order`` if given); unused rows and free
    blocks hold ``fill`` (default: random values of the same dtype)."""
    Hkv, d = seqs[0].shape[1:]
    dtype = seqs[0].dtype
    nblk = [cdiv(s.shape[0], block_size) for s in seqs]
    demand = sum(nblk)
    NB = num_blocks if num_blocks is not None else max(1, demand + 3)
    assert NB >= demand
    if fill is None:
        pool = rng.standard_normal((NB, block_size, Hkv, d)).astype(dtype) if dtype.kind == "f" else \
            rng.integers(0, 256, (NB, block_size, Hkv, d)).astype(dtype)
    else:
        pool = np.full((NB, block_size, Hkv, d), fill, dtype)
    ids = rng.permutation(NB) if order is None else np.asarray(order)
    MB = max(1, max(nblk))
    tables = np.zeros((len(seqs), MB), np.int32)
    pos = 0
    for b, s in enumerate(seqs):
        tables[b, :nblk[b]] = ids[pos:pos + nblk[b]]
        pos += nblk[b]
        for t in range(s.shape[0]):
            pool[tables[b, t // block_size], t % block_size] = s[t]
    return tables, pool

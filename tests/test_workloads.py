"""The seeded generators build the block-manager state the pages describe:
a shuffled pool, per-sequence tables of distinct blocks, slots consistent
with the tables, prefix sharing with copy-on-write pairs."""
import numpy as np
import torch

from paged_kv_cache_450_b200 import workloads as W


def _small(spec, **kw):
    return spec.with_(**kw)


def test_tables_are_distinct_blocks_within_the_pool():
    for spec, kw in ((W.TINY, {}), (W.LLAMA7B, dict(num_seqs=6, ctx=("uniform", 1, 300))),
                     (W.LLAMA13B, dict(num_seqs=8, num_q_heads=4, num_kv_heads=4)),
                     (W.GQA_BATCH, dict(num_seqs=3, ctx=("fixed", 100)))):
        w = W.make_decode_workload(_small(spec, **kw), seed=3)
        bs = w.spec.block_size
        used = []
        for b, c in enumerate(w.ctx_list):
            n = -(-c // bs)
            used += w.block_tables[b, :n].tolist()
        assert len(used) == len(set(used))
        assert all(0 <= u < w.num_blocks for u in used)
        assert w.key_cache.shape == (w.num_blocks, bs, w.spec.num_kv_heads, w.spec.head_dim)


def test_pool_recipes():
    w = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=10, num_q_heads=2, num_kv_heads=2), seed=0)
    assert w.num_blocks == int(np.ceil(1.2 * w.info["demand_blocks"]))
    w = W.make_decode_workload(W.LLAMA13B.with_(num_seqs=10, num_q_heads=2, num_kv_heads=2), seed=0)
    assert w.num_blocks == int(np.ceil(w.info["demand_blocks"] / 0.7))
    assert all(16 <= c <= 4096 for c in w.ctx_list)


def test_new_token_slot_is_last_logical_position():
    w = W.make_decode_workload(W.TINY, seed=0)
    bs = w.spec.block_size
    for b, c in enumerate(w.ctx_list):
        s = int(w.slot_mapping[b])
        assert s == int(w.block_tables[b, (c - 1) // bs]) * bs + (c - 1) % bs


def test_parallel_sampling_structure():
    spec = W.PARALLEL_SAMPLING.with_(num_seqs=8, num_q_heads=2, num_kv_heads=2, sampling=(2, 4, 40, 1, 20))
    w = W.make_decode_workload(spec, seed=1)
    pairs = w.copy_pairs.tolist()
    assert len(pairs) == 2 * 3
    t = w.block_tables
    for p in range(2):
        base = t[p * 4]
        for c in range(1, 4):
            row = t[p * 4 + c]
            assert torch.equal(row[:2], base[:2])          # shared full prompt blocks
            assert [int(base[2]), int(row[2])] in pairs     # CoW copy of the last prompt block
    dsts = [d for _, d in pairs]
    srcs = {s for s, _ in pairs}
    assert len(set(dsts)) == len(dsts) and not (set(dsts) & srcs)


def test_fp8_pool_scale_is_amax_over_448():
    w = W.make_decode_workload(W.GQA_LONG.with_(num_seqs=2, ctx=("fixed", 64)), seed=0)
    assert w.key_cache.dtype == torch.float8_e4m3fn
    codes = w.key_cache.view(torch.uint8)
    assert int(((codes & 0x7F) == 0x7F).sum()) == 0         # no NaN codes
    assert float(w.key_cache.float().abs().max()) == 448.0  # amax maps onto the largest code
    assert w.k_scale > 0 and w.v_scale > 0


def test_seeded_generation_is_reproducible():
    a = W.make_decode_workload(W.TINY, seed=5)
    b = W.make_decode_workload(W.TINY, seed=5)
    assert torch.equal(a.key_cache, b.key_cache) and torch.equal(a.block_tables, b.block_tables)
    c = W.make_decode_workload(W.TINY, seed=6)
    assert not torch.equal(a.key_cache, c.key_cache)

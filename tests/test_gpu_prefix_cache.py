"""Prefix caching feeding the kernels.

"vLLM KV Cache 实现机制", 4.2: requests whose prompts share a prefix reuse the
cached blocks of that prefix, found by a hash chain over whole blocks; 3.2:
reference counts protect shared blocks and unreferenced ones are evicted LRU.
"vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点: a shared block read by
several sequences gives the same attention as private copies.

Here the block tables of several requests are built through the library's
PrefixCache (match, then fresh blocks for the rest, then insert), with the K/V
of a full block a function of its chained hash (a block with the same prefix
holds the same K/V, as it would in a model).  Decode and multi-query attention
over those tables are checked against the CPU oracle on the same tables, and
against the same requests laid out in private copies (bit-identical: the
kernels' arithmetic does not depend on where a block sits).  A second wave
releases, evicts and reuses physical blocks.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_450_b200 as pk
from step_helpers import assert_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
BS, HQ, HKV, D = 16, 8, 2, 128
TOL_BF16 = (2e-3, 1e-2)
SCALE = 1.0 / np.sqrt(D)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


class Pool:
    """The caller's side: a free list of physical blocks, the two caches and a
    prefix cache from full token blocks to physical ids."""

    def __init__(self, num_blocks, capacity, seed):
        g = torch.Generator(device=DEV).manual_seed(seed)
        shape = (num_blocks, BS, HKV, D)
        self.kc = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
        self.vc = torch.randn(shape, generator=g, device=DEV).to(torch.bfloat16)
        self.free = [int(x) for x in np.random.default_rng(seed).permutation(num_blocks)]
        self.cache = pk.PrefixCache(BS, capacity)
        self.gen = g

    def _fill(self, pid, seed):
        g = torch.Generator(device=DEV).manual_seed(seed)
        self.kc[pid] = torch.randn((BS, HKV, D), generator=g, device=DEV).to(torch.bfloat16)
        self.vc[pid] = torch.randn((BS, HKV, D), generator=g, device=DEV).to(torch.bfloat16)

    def admit(self, tokens, extra=0):
        """Block ids of a request: its longest cached prefix, fresh blocks for the
        other full blocks (registered in the cache), a private tail block."""
        n_full = len(tokens) // BS
        ids = self.cache.match(tokens, extra)
        shared = len(ids)
        hashes = pk.prefix_block_hashes(tokens, BS, 0, extra)
        for i in range(shared, n_full):
            pid = self.free.pop()
            self._fill(pid, int(hashes[i]) & 0x7FFFFFFFFFFFFFFF)  # same chain, same K/V
            ids.append(pid)
        self.cache.insert(tokens, ids[:n_full], extra)
        tail = None
        if len(tokens) % BS:
            tail = self.free.pop()
            self._fill(tail, 7919 * len(tokens) + tail)
            ids.append(tail)
        return ids, shared, tail


def tables_of(reqs, mb):
    t = torch.zeros((len(reqs), mb), dtype=torch.int32)
    for b, ids in enumerate(reqs):
        t[b, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
    return t.to(DEV)


def private_copies(pool, reqs):
    """The same requests with every block a private copy (a fresh pool)."""
    n = sum(len(ids) for ids in reqs)
    src = torch.tensor([i for ids in reqs for i in ids], dtype=torch.int64, device=DEV)
    kc, vc = pool.kc[src].contiguous(), pool.vc[src].contiguous()
    tables, nxt = [], 0
    for ids in reqs:
        tables.append(list(range(nxt, nxt + len(ids))))
        nxt += len(ids)
    assert nxt == n
    return kc, vc, tables


def check_attention(pool, reqs, lens, seed):
    mb = max(len(ids) for ids in reqs)
    tables = tables_of(reqs, mb)
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    g = torch.Generator(device=DEV).manual_seed(seed)
    B = len(reqs)
    q = torch.randn((B, HQ, D), generator=g, device=DEV).to(torch.bfloat16)
    pkc, pvc, ptab = private_copies(pool, reqs)
    ptables = tables_of(ptab, mb)

    # decode: oracle on the shared tables, and the private layout bit for bit
    for pt in (0, 32):
        out = pk.paged_attention_decode(q, pool.kc, pool.vc, tables, ctx, SCALE, partition_tokens=pt, validate=True)
        priv = pk.paged_attention_decode(q, pkc, pvc, ptables, ctx, SCALE, partition_tokens=pt, validate=True)
        torch.cuda.synchronize()
        ref = oracle.paged_attention_decode(to_np(q), to_np(pool.kc), to_np(pool.vc), to_np(tables), to_np(ctx),
                                            scale=SCALE, q_dtype=oracle.BF16, cache_dtype=oracle.BF16)
        assert_close(f64(out), ref, *TOL_BF16, what=f"decode over prefix-cache tables pt={pt}")
        assert torch.equal(out, priv), "shared blocks and private copies differ"

    # multi-query: verification-sized (mma.sync) and prefill-sized (tcgen05) query counts
    for q_lens in ([3] * B, [min(n, 40 + 9 * b) for b, n in enumerate(lens)]):
        qsl = torch.tensor(np.concatenate([[0], np.cumsum(q_lens)]), dtype=torch.int32, device=DEV)
        T = int(qsl[-1])
        qm = torch.randn((T, HQ, D), generator=g, device=DEV).to(torch.bfloat16)
        out = pk.paged_attention_multiquery(qm, pool.kc, pool.vc, tables, ctx, qsl, SCALE, validate=True)
        priv = pk.paged_attention_multiquery(qm, pkc, pvc, ptables, ctx, qsl, SCALE, validate=True)
        torch.cuda.synchronize()
        ref = oracle.paged_attention_multiquery(to_np(qm), to_np(qsl), to_np(pool.kc), to_np(pool.vc), to_np(tables),
                                                to_np(ctx), scale=SCALE, q_dtype=oracle.BF16,
                                                cache_dtype=oracle.BF16)
        assert_close(f64(out), ref, *TOL_BF16, what=f"multi-query over prefix-cache tables q_lens={q_lens}")
        assert torch.equal(out, priv), "multi-query: shared blocks and private copies differ"
    assert pk.device_status(clear=True) == 0


def test_prefix_cache_tables_drive_decode_and_multiquery():
    rng = np.random.default_rng(5)
    pool = Pool(num_blocks=160, capacity=64, seed=5)
    sys_prompt = rng.integers(0, 32000, 5 * BS).tolist()      # a 5-block system prompt
    few_shot = rng.integers(0, 32000, 2 * BS).tolist()        # 2 more blocks shared by two requests
    own = lambda n: rng.integers(0, 32000, n).tolist()        # noqa: E731
    prompts = [
        (sys_prompt + own(37), 0),
        (sys_prompt + own(20), 0),
        (sys_prompt + few_shot + own(9), 0),
        (sys_prompt + few_shot + own(3 * BS + 8), 0),
        (sys_prompt + own(10), 77),                            # another extra hash (multimodal): no reuse
        (own(100), 0),
        (sys_prompt + few_shot, 0),                            # whole blocks only: no tail block
    ]
    reqs, shared = [], []
    for toks, extra in prompts:
        ids, n_shared, _ = pool.admit(toks, extra)
        reqs.append(ids)
        shared.append(n_shared)
    assert shared == [0, 5, 5, 7, 0, 0, 7]
    assert reqs[1][:5] == reqs[0][:5] == reqs[2][:5] and reqs[3][:7] == reqs[2][:7] == reqs[6][:7]
    assert not set(reqs[4]) & set(reqs[0])
    lens = [len(t) for t, _ in prompts]
    check_attention(pool, reqs, lens, seed=50)

    # second wave: the requests finish, LRU eviction frees blocks, new requests reuse the freed ids
    for (toks, extra), ids in zip(prompts, reqs):
        pool.cache.release(toks, len(toks) // BS, extra)
        if len(toks) % BS:
            pool.free.append(ids[-1])                          # private tail blocks go back at once
    evicted = pool.cache.evict(6)
    assert len(evicted) == 6
    pool.free.extend(evicted)                                  # reused first (the free list pops from the end)
    prompts2 = [(sys_prompt + few_shot + own(50), 0), (sys_prompt + own(130), 0), (own(70), 0),
                (sys_prompt + own(5), 77)]
    reqs2 = [pool.admit(toks, extra)[0] for toks, extra in prompts2]
    assert set(evicted) & {i for ids in reqs2 for i in ids}, "no evicted block was reused"
    check_attention(pool, reqs2, [len(t) for t, _ in prompts2], seed=51)
    pool.cache.close()

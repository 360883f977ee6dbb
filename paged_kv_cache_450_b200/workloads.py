"""Seeded synthetic inputs for the paged decode path.

This module builds inputs only.  It holds none of the path's arithmetic (no
attention, no cache indexing of K/V values, no fp8 encoding of its own): both
the CUDA library and the CPU oracle consume the tensors it returns.

What it models is the caller above the kernels -- the block manager of
"vLLM KV Cache 实现机制" section 3 and "vLLM 与 KV Cache" section 工作原理:
a pre-allocated pool of fixed-size physical blocks, a per-sequence block table
(logical block j -> physical block id, any order), on-demand allocation, and
reference-counted sharing with copy-on-write for parallel sampling
("vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 2).

Recipes (every draw seeded; structure from numpy PCG64(seed), tensor values
from a torch generator seeded with ``seed`` on the target device, drawn in the
fixed order q, key pool, value pool, new k, new v):

* q, K, V ~ N(0, 1) drawn in fp32, then cast to the stored dtype.  Free pool
  blocks hold random values too.
* fp8 caches: per-tensor scale = amax(|x_bf16|) / 448 in fp32 over the whole
  pool; the stored codes are torch's ``float8_e4m3fn`` cast of x * (1/scale).
* block tables: a random permutation of the pool's ids, handed out in order.
* one new token per sequence sits at logical position ctx - 1; its slot is
  ``table[(ctx-1) // bs] * bs + (ctx-1) % bs`` (the caller's flat slot id).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

FP8 = torch.float8_e4m3fn
E4M3_MAX = 448.0


@dataclass(frozen=True)
class DecodeSpec:
    """One decode workload shape.

    ctx: ("uniform", lo, hi) inclusive | ("fixed", n) |
         ("lognormal", median, sigma, lo, hi) | ("list", (c0, c1, ...))
    pool: ("fixed", NB) | ("slack", factor) -> NB = ceil(factor * demand) |
          ("prefreed", frac) -> NB = ceil(demand / (1 - frac))
    sampling: None or (num_prompts, n, prompt_len, tail_lo, tail_hi) for
          parallel sampling with a shared prompt (num_seqs = prompts * n).
    """
    name: str
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: torch.dtype
    cache_dtype: torch.dtype
    ctx: tuple
    pool: tuple = ("slack", 1.2)
    new_tokens: bool = True
    sampling: tuple | None = None

    def with_(self, **kw) -> "DecodeSpec":
        return replace(self, **kw)


# The five workload families (sizes as stated for this library's benchmarks).
TINY = DecodeSpec("tiny_mha_fp32_d64", 4, 4, 4, 64, 16, torch.float32, torch.float32,
                  ("uniform", 1, 100), ("fixed", 64))
LLAMA7B = DecodeSpec("llama7b_decode_b64_bf16", 64, 32, 32, 128, 16, torch.bfloat16, torch.bfloat16,
                     ("uniform", 128, 2048), ("slack", 1.2))
LLAMA13B = DecodeSpec("llama13b_decode_b256_bf16", 256, 40, 40, 128, 16, torch.bfloat16, torch.bfloat16,
                      ("lognormal", 600.0, 0.8, 16, 4096), ("prefreed", 0.30))
PARALLEL_SAMPLING = DecodeSpec("parallel_sampling_32x4_bf16", 128, 40, 40, 128, 16, torch.bfloat16,
                               torch.bfloat16, ("fixed", 0), ("slack", 1.2),
                               sampling=(32, 4, 1024, 1, 64))
GQA_LONG = DecodeSpec("gqa70b_fp8_b16_ctx32k", 16, 64, 8, 128, 16, torch.bfloat16, FP8,
                      ("fixed", 32768), ("slack", 1.0))
GQA_BATCH = DecodeSpec("gqa70b_fp8_b128_ctx8k", 128, 64, 8, 128, 16, torch.bfloat16, FP8,
                       ("fixed", 8192), ("slack", 1.0))

# Extra (not one of the five families): the 70B-GQA shape with a bf16 cache.
GQA_BATCH_BF16 = GQA_BATCH.with_(name="gqa70b_bf16_b128_ctx8k", cache_dtype=torch.bfloat16)

SPECS = {s.name: s for s in (TINY, LLAMA7B, LLAMA13B, LLAMA13B.with_(name="llama13b_decode_b256_bf16_bs32",
                                                                      block_size=32),
                             PARALLEL_SAMPLING, GQA_LONG, GQA_BATCH, GQA_BATCH_BF16)}


@dataclass
class DecodeWorkload:
    spec: DecodeSpec
    seed: int
    device: str
    context_lens: torch.Tensor      # int32 [B]
    block_tables: torch.Tensor      # int32 [B, MB]
    num_blocks: int
    q: torch.Tensor                 # [B, Hq, d]
    key_cache: torch.Tensor         # [NB, bs, Hkv, d]
    value_cache: torch.Tensor       # [NB, bs, Hkv, d]
    k_scale: float
    v_scale: float
    scale: float                    # softmax scale 1/sqrt(d), an fp32 value
    new_k: torch.Tensor | None      # [T, Hkv, d] in q's dtype
    new_v: torch.Tensor | None
    slot_mapping: torch.Tensor | None  # int64 [T]
    copy_pairs: torch.Tensor | None    # int64 [n, 2] (src, dst)
    info: dict = field(default_factory=dict)
    # parallel sampling: the n candidates of a prompt form a group of consecutive
    # sequences whose first shared_blocks[g] blocks are the same physical blocks
    group_start: torch.Tensor | None = None    # int32 [G + 1]
    shared_blocks: torch.Tensor | None = None  # int32 [G]

    @property
    def ctx_list(self) -> list[int]:
        return [int(c) for c in self.context_lens.cpu().tolist()]

    def kv_bytes(self) -> int:
        """Logical KV bytes one decode pass reads: sum_b ctx_b * Hkv * d * elem * 2 (K and V)."""
        s = self.spec
        return int(sum(self.ctx_list)) * s.num_kv_heads * s.head_dim * elem_size(s.cache_dtype) * 2


def elem_size(dtype: torch.dtype) -> int:
    return torch.empty((), dtype=dtype).element_size()


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, dtype: torch.dtype) -> int:
    """K and V bytes one token occupies across all layers: 2 x L x H x d x sizeof(dtype)."""
    return 2 * num_layers * num_kv_heads * head_dim * elem_size(dtype)


def block_bytes(block_size: int, num_kv_heads: int, head_dim: int, dtype: torch.dtype) -> int:
    """Bytes of one physical block of one cache (K or V) of one layer."""
    return block_size * num_kv_heads * head_dim * elem_size(dtype)


def _draw_context_lens(spec: DecodeSpec, rng: np.random.Generator) -> np.ndarray:
    kind = spec.ctx[0]
    B = spec.num_seqs
    if kind == "uniform":
        return rng.integers(spec.ctx[1], spec.ctx[2] + 1, size=B).astype(np.int64)
    if kind == "fixed":
        return np.full(B, spec.ctx[1], np.int64)
    if kind == "lognormal":
        median, sigma, lo, hi = spec.ctx[1:]
        z = rng.standard_normal(B)
        return np.clip(np.round(median * np.exp(sigma * z)), lo, hi).astype(np.int64)
    if kind == "list":
        c = np.asarray(spec.ctx[1], np.int64)
        assert c.shape == (B,)
        return c
    raise ValueError(f"unknown ctx recipe {spec.ctx}")


def _pool_size(spec: DecodeSpec, demand: int) -> int:
    kind = spec.pool[0]
    if kind == "fixed":
        nb = int(spec.pool[1])
        if nb < demand:
            raise ValueError(f"pool of {nb} blocks is smaller than the demand of {demand} blocks")
        return nb
    if kind == "slack":
        return max(demand, int(math.ceil(spec.pool[1] * demand)))
    if kind == "prefreed":
        return max(demand, int(math.ceil(demand / (1.0 - spec.pool[1]))))
    raise ValueError(f"unknown pool recipe {spec.pool}")


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def _layout_independent(spec, rng):
    """Block tables for independent sequences from a shuffled pool."""
    bs = spec.block_size
    ctx = _draw_context_lens(spec, rng)
    nblk = [_cdiv(int(c), bs) for c in ctx]
    demand = int(sum(nblk))
    NB = _pool_size(spec, demand)
    perm = rng.permutation(NB)
    MB = max(1, max(nblk) if nblk else 1)
    tables = np.zeros((spec.num_seqs, MB), np.int32)
    pos = 0
    for b, n in enumerate(nblk):
        tables[b, :n] = perm[pos:pos + n]
        pos += n
    return ctx, tables, NB, None, {"demand_blocks": demand}


def _layout_sampling(spec, rng):
    """Parallel sampling: n candidates share their prompt's blocks (ref_count n).

    Candidate 0 keeps the prompt's last block; candidates 1..n-1 get a private
    copy of it (the n-1 copy-on-write copies of the first sampling step), then
    private blocks for their own tail tokens.  The tail continues in the last
    prompt block when the prompt does not fill it.
    """
    P, n, plen, tlo, thi = spec.sampling
    bs = spec.block_size
    assert spec.num_seqs == P * n
    tails = rng.integers(tlo, thi + 1, size=P * n).astype(np.int64)
    ctx = plen + tails
    n_prompt_blk = _cdiv(plen, bs)
    nblk = [_cdiv(int(c), bs) for c in ctx]
    private_tail = [nb - n_prompt_blk for nb in nblk]
    demand = P * n_prompt_blk + P * (n - 1) + int(sum(private_tail))
    NB = _pool_size(spec, demand)
    perm = iter(rng.permutation(NB).tolist())
    MB = max(nblk)
    tables = np.zeros((P * n, MB), np.int32)
    pairs = []
    ref_count = {}
    for p in range(P):
        prompt = [next(perm) for _ in range(n_prompt_blk)]
        for blk in prompt:
            ref_count[blk] = n
        for c in range(n):
            b = p * n + c
            tables[b, :n_prompt_blk] = prompt
            if c > 0:  # copy-on-write of the last prompt block
                dst = next(perm)
                pairs.append((prompt[-1], dst))
                tables[b, n_prompt_blk - 1] = dst
                ref_count[prompt[-1]] -= 1
                ref_count[dst] = 1
            for j in range(n_prompt_blk, nblk[b]):
                tables[b, j] = next(perm)
    info = {"demand_blocks": demand, "shared_prompt_blocks": P * n_prompt_blk,
            "ref_count_prompt": n, "cow_pairs": len(pairs),
            "ref_count_last_prompt_block_after_cow": ref_count[int(tables[0, n_prompt_blk - 1])],
            # blocks every candidate of a prompt still shares: all but the copied-on-write last one (a
            # single candidate: the prompt's full blocks, before the one its new tokens go to)
            "groups": (np.arange(0, P * n + 1, n, dtype=np.int32),
                       np.full(P, n_prompt_blk - 1 if n > 1 else plen // bs, np.int32))}
    return ctx, tables, NB, np.asarray(pairs, np.int64).reshape(-1, 2), info


def _randn(shape, gen, device, dtype, chunk=1 << 26):
    """N(0,1) drawn in fp32 chunk by chunk (bounded temporaries), stored as dtype."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def _fp8_pool(shape, gen, device, chunk=1 << 26):
    """bf16 N(0,1) pool -> per-tensor scale amax/448 -> float8_e4m3fn codes of x * (1/scale)."""
    src = _randn(shape, gen, device, torch.bfloat16, chunk)
    amax = float(src.abs().max().float().item()) if src.numel() else 1.0
    scale = np.float32(amax / E4M3_MAX) if amax > 0 else np.float32(1.0)
    inv = torch.tensor(np.float32(1.0) / scale, dtype=torch.float32, device=device)
    out = torch.empty(shape, dtype=FP8, device=device)
    fs, fo = src.view(-1), out.view(-1)
    for s in range(0, fs.numel(), chunk):
        e = min(fs.numel(), s + chunk)
        fo[s:e] = (fs[s:e].float() * inv).to(FP8)
    del src
    return out, float(scale)


def make_decode_workload(spec: DecodeSpec, seed: int = 0, device: str | torch.device = "cpu") -> DecodeWorkload:
    device = str(device)
    rng = np.random.Generator(np.random.PCG64(seed))
    if spec.sampling is not None:
        ctx, tables, NB, pairs, info = _layout_sampling(spec, rng)
    else:
        ctx, tables, NB, pairs, info = _layout_independent(spec, rng)
    B, Hq, Hkv, d, bs = spec.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _randn((B, Hq, d), gen, device, spec.q_dtype)
    if spec.cache_dtype == FP8:
        key_cache, k_scale = _fp8_pool((NB, bs, Hkv, d), gen, device)
        value_cache, v_scale = _fp8_pool((NB, bs, Hkv, d), gen, device)
    else:
        key_cache = _randn((NB, bs, Hkv, d), gen, device, spec.cache_dtype)
        value_cache = _randn((NB, bs, Hkv, d), gen, device, spec.cache_dtype)
        k_scale = v_scale = 1.0
    new_k = new_v = slot = None
    if spec.new_tokens:
        T = B
        new_k = _randn((T, Hkv, d), gen, device, spec.q_dtype)
        new_v = _randn((T, Hkv, d), gen, device, spec.q_dtype)
        s = np.full(T, -1, np.int64)
        for b in range(B):
            c = int(ctx[b])
            if c > 0:
                s[b] = int(tables[b, (c - 1) // bs]) * bs + (c - 1) % bs
        slot = torch.from_numpy(s).to(device)
    groups = info.pop("groups", None)
    info.update({"num_blocks": NB, "max_blocks_per_seq": int(tables.shape[1]),
                 "total_tokens": int(ctx.sum())})
    return DecodeWorkload(
        spec=spec, seed=seed, device=device,
        context_lens=torch.from_numpy(ctx.astype(np.int32)).to(device),
        block_tables=torch.from_numpy(tables).to(device),
        num_blocks=NB, q=q, key_cache=key_cache, value_cache=value_cache,
        k_scale=float(k_scale), v_scale=float(v_scale),
        scale=float(np.float32(1.0 / math.sqrt(d))),
        new_k=new_k, new_v=new_v, slot_mapping=slot,
        copy_pairs=None if pairs is None else torch.from_numpy(pairs).to(device),
        info=info,
        group_start=None if groups is None else torch.from_numpy(groups[0]).to(device),
        shared_blocks=None if groups is None else torch.from_numpy(groups[1]).to(device))


@dataclass
class MultiQueryWorkload:
    """A decode-style pool plus several query tokens per sequence: the queries
    of sequence b are its last q_len_b positions (their K/V are already in the
    pool, as after a paged_kv_write of those tokens)."""
    base: DecodeWorkload
    q: torch.Tensor                 # [total_q, Hq, d]
    query_start_loc: torch.Tensor   # int32 [B + 1]
    q_lens: list

    def flops(self) -> int:
        """4 * d flops per (query, visible key, query head) pair."""
        s = self.base.spec
        ctx = self.base.ctx_list
        pairs = 0
        for c, n in zip(ctx, self.q_lens):
            for i in range(n):
                pairs += max(0, c - n + i + 1)
        return 4 * s.head_dim * s.num_q_heads * pairs


def make_multiquery_workload(spec: DecodeSpec, q_lens, seed: int = 0,
                             device: str | torch.device = "cpu") -> MultiQueryWorkload:
    """q_lens: one query count per sequence (each <= its context length).
    The q tensor is drawn after the decode workload's tensors (same seed)."""
    base = make_decode_workload(spec.with_(new_tokens=False), seed=seed, device=device)
    q_lens = [int(n) for n in q_lens]
    assert len(q_lens) == spec.num_seqs
    for c, n in zip(base.ctx_list, q_lens):
        if n > c:
            raise ValueError("a sequence cannot have more queries than context tokens")
    qsl = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    gen = torch.Generator(device=str(device))
    gen.manual_seed(seed + 7919)
    q = _randn((int(qsl[-1]), spec.num_q_heads, spec.head_dim), gen, str(device), spec.q_dtype)
    return MultiQueryWorkload(base=base, q=q, query_start_loc=torch.from_numpy(qsl).to(device), q_lens=q_lens)


# Multi-query workload families: draft verification (4 draft tokens + the
# accepted one per sequence) and chunked prefill (512-token chunks after a
# prefix), on the LLaMA-7B and 70B-GQA (bf16 and fp8 cache) shapes.
MQ_SPECS = {
    "llama7b_verify_b64_q5": (LLAMA7B.with_(name="llama7b_verify_b64_q5"), 5),
    "llama7b_prefill_b8_chunk512": (LLAMA7B.with_(name="llama7b_prefill_b8_chunk512", num_seqs=8,
                                                  ctx=("uniform", 512, 2048)), 512),
    "gqa70b_bf16_verify_b64_q5": (GQA_BATCH_BF16.with_(name="gqa70b_bf16_verify_b64_q5", num_seqs=64,
                                                        ctx=("uniform", 1024, 8192)), 5),
    "gqa70b_fp8_verify_b64_q5": (GQA_BATCH.with_(name="gqa70b_fp8_verify_b64_q5", num_seqs=64,
                                                 ctx=("uniform", 1024, 8192)), 5),
}

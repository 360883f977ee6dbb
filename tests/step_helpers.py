"""One decode step run twice: through libpagedkv on the GPU and through the
CPU oracle on host copies of the same seeded inputs.

Step order (both sides): copy-on-write block copies, then the new-token
write, then decode attention over context_lens (which include the new token).
The oracle's inputs are the generator's tensors only; nothing the GPU path
produced is fed to it.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_450_b200 as pk

# Tolerances: bf16 output |gpu - ref| <= 2e-3 + 1e-2 |ref|; fp8 KV 3e-2 relative;
# fp32 end to end 1e-4 (fp32 accumulation over <= 4096 terms, ex2.approx).
TOL = {"bf16": (2e-3, 1e-2), "fp8": (2e-3, 3e-2), "f32": (1e-4, 1e-4)}


def tol_for(w):
    if w.spec.cache_dtype == torch.float8_e4m3fn:
        return TOL["fp8"]
    return TOL["f32"] if w.spec.q_dtype == torch.float32 else TOL["bf16"]


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def ocode(dtype: torch.dtype) -> int:
    return {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float8_e4m3fn: oracle.E4M3}[dtype]


def oracle_step(w, rows=None, num_threads=None):
    """Returns (key_cache, value_cache, out) computed on the host in fp64."""
    s = w.spec
    kc, vc = to_np(w.key_cache).copy(), to_np(w.value_cache).copy()
    if w.copy_pairs is not None and len(w.copy_pairs):
        oracle.kv_block_copy(to_np(w.copy_pairs), kc, vc)
    if w.new_k is not None:
        oracle.paged_kv_write(to_np(w.new_k), to_np(w.new_v), to_np(w.slot_mapping), kc, vc,
                              in_dtype=ocode(s.q_dtype), cache_dtype=ocode(s.cache_dtype), k_scale=w.k_scale,
                              v_scale=w.v_scale)
    out = oracle.paged_attention_decode(to_np(w.q), kc, vc, to_np(w.block_tables), to_np(w.context_lens),
                                        scale=w.scale, q_dtype=ocode(s.q_dtype), cache_dtype=ocode(s.cache_dtype),
                                        k_scale=w.k_scale, v_scale=w.v_scale, rows=rows, num_threads=num_threads)
    return kc, vc, out


def gpu_step(w, partition_tokens=0, validate=True, workspace=None):
    """Runs the step through libpagedkv on clones of the caches."""
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    if w.copy_pairs is not None and len(w.copy_pairs):
        pk.kv_block_copy(w.copy_pairs, kc, vc, validate=validate)
    if w.new_k is not None:
        pk.paged_kv_write(w.new_k, w.new_v, w.slot_mapping, kc, vc, k_scale=w.k_scale, v_scale=w.v_scale,
                          validate=validate)
    out = pk.paged_attention_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale,
                                    w.spec.block_size, w.spec.num_kv_heads, k_scale=w.k_scale, v_scale=w.v_scale,
                                    partition_tokens=partition_tokens, validate=validate, workspace=workspace)
    torch.cuda.synchronize()
    return kc, vc, out


def assert_close(got: np.ndarray, ref: np.ndarray, atol: float, rtol: float, what: str = ""):
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance "
                             f"(atol {atol}, rtol {rtol}); worst at {i}: got {got[i]!r}, ref {ref[i]!r}, "
                             f"max abs err {err.max():.3e}")


def assert_cache_equal(gpu: torch.Tensor, host: np.ndarray, what: str):
    ref = torch.from_numpy(host).to(gpu.device)
    a = gpu.contiguous().view(torch.uint8).view(-1)
    b = ref.contiguous().view(torch.uint8).view(-1)
    assert a.numel() == b.numel()
    if not torch.equal(a, b):
        n = int((a != b).sum())
        raise AssertionError(f"{what}: {n} bytes differ from the oracle")


def sample_rows(w, n, seed=0):
    """Rows b * Hq + hq to check at full size: the longest and shortest
    sequences' every head, first/last heads, and a seeded random rest."""
    B, Hq = w.spec.num_seqs, w.spec.num_q_heads
    ctx = np.array(w.ctx_list)
    rng = np.random.default_rng(seed)
    rows = set()
    for b in (int(ctx.argmax()), int(ctx.argmin())):
        rows.update(b * Hq + h for h in range(Hq))
    rows.update({0, Hq - 1, (B - 1) * Hq, B * Hq - 1})
    rest = rng.choice(B * Hq, size=min(B * Hq, max(0, n - len(rows))), replace=False)
    rows.update(int(r) for r in rest)
    return np.array(sorted(rows)[: max(n, len(rows))], np.int64)

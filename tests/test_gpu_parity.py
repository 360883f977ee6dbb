"""GPU parity: libpagedkv (through its C ABI) against the CPU oracle.

Bit-exact for the cache write and the block copy; decode attention within
the stated tolerances (bf16 2e-3 + 1e-2|ref|, fp8 KV 3e-2 relative, fp32 1e-4).
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_450_b200 as pk
from paged_kv_cache_450_b200 import workloads as W
from step_helpers import (assert_cache_equal, assert_close, gpu_step, ocode, oracle_step, sample_rows, to_np,
                          tol_for)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
FP8 = torch.float8_e4m3fn


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_step(w, partition_tokens=0, rows=None, what=""):
    kc, vc, out = gpu_step(w, partition_tokens=partition_tokens)
    rk, rv, ref = oracle_step(w, rows=rows)
    assert_cache_equal(kc, rk, f"{what} key_cache")
    assert_cache_equal(vc, rv, f"{what} value_cache")
    got = f64(out)
    if rows is not None:
        got = got.reshape(-1, w.spec.head_dim)[rows]
    assert_close(got, ref, *tol_for(w), what=what)
    return out


def test_tiny_config_full_parity():
    w = W.make_decode_workload(W.TINY, seed=0, device=DEV)
    check_step(w, what="tiny")


DTYPES = [(torch.float32, torch.float32), (torch.bfloat16, torch.bfloat16), (torch.bfloat16, FP8),
          (torch.float32, FP8)]


@pytest.mark.parametrize("dtypes,d,bs,g", list(itertools.product(DTYPES, [64, 128], [8, 16, 32], [1, 2, 4, 8])),
                         ids=lambda x: str(x).replace("torch.", "").replace(" ", ""))
def test_every_kernel_instance_small(dtypes, d, bs, g):
    qd, cd = dtypes
    spec = W.DecodeSpec("small", 5, 2 * g, 2, d, bs, qd, cd, ("list", (1, 700, bs, 3 * bs + 1, 257)),
                        ("slack", 1.3))
    w = W.make_decode_workload(spec, seed=d + bs + g, device=DEV)
    # partition lengths: automatic, one block, three blocks
    for pt in (0, bs, 3 * bs):
        check_step(w, partition_tokens=pt, what=f"pt={pt}")


@pytest.mark.parametrize("cd,hq", [(torch.bfloat16, 8), (FP8, 8), (FP8, 16)], ids=["bf16-g4", "fp8-g4", "fp8-g8-mma"])
def test_partition_partials_match_oracle(cd, hq):
    spec = W.DecodeSpec("partials", 3, hq, 2, 128, 16, torch.bfloat16, cd, ("list", (300, 17, 64)), ("slack", 1.2),
                        new_tokens=False)
    w = W.make_decode_workload(spec, seed=11, device=DEV)
    pt = 64
    B, Hq, d = 3, hq, 128
    MB = w.block_tables.shape[1]
    P = pk.decode_max_partitions(B, Hq, 2, d, 16, MB, cd, pt)
    nbytes = pk.decode_workspace_bytes(B, Hq, 2, d, 16, MB, cd, pt)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=DEV)
    gpu_step(w, partition_tokens=pt, workspace=ws)
    rows = B * Hq * P
    ml_bytes = ((rows * 2 * 4 + 255) // 256) * 256
    ml = ws[: rows * 8].view(torch.float32).view(B, Hq, P, 2).cpu().numpy().astype(np.float64)
    o = ws[ml_bytes: ml_bytes + rows * d * 4].view(torch.float32).view(B, Hq, P, d).cpu().numpy()
    m_ref, l_ref, o_ref = oracle.decode_partials(
        to_np(w.q), to_np(w.key_cache), to_np(w.value_cache), to_np(w.block_tables), to_np(w.context_lens),
        scale=w.scale, partition_tokens=pt, max_partitions=P, q_dtype=oracle.BF16, cache_dtype=ocode(cd),
        k_scale=w.k_scale, v_scale=w.v_scale)
    atol, rtol = tol_for(w)
    for b, c in enumerate(w.ctx_list):
        n = -(-c // pt)
        if n <= 1:
            continue  # single-partition rows are written straight to the output
        # (m, l) may be stored relative to any reference logit m; the partition's
        # log-sum-exp m + ln l and its normalised output o are what is defined.
        lse = ml[b, :, :n, 0] + np.log(ml[b, :, :n, 1])
        lse_ref = m_ref[b, :, :n] + np.log(l_ref[b, :, :n])
        assert_close(lse, lse_ref, 1e-4, 1e-4, what="partition log-sum-exp")
        assert np.all(ml[b, :, :n, 0] <= m_ref[b, :, :n] + 1e-5)   # the reference never exceeds the max
        assert_close(o[b, :, :n], o_ref[b, :, :n], atol, rtol, what="partition output")


def test_edge_contexts_zero_one_and_max():
    bs = 16
    spec = W.DecodeSpec("edges", 6, 4, 4, 128, bs, torch.bfloat16, torch.bfloat16,
                        ("list", (0, 1, 16, 17, 64, 0)), ("slack", 1.5), new_tokens=False)
    w = W.make_decode_workload(spec, seed=2, device=DEV)
    out = check_step(w, what="edges")
    assert torch.count_nonzero(out[0]) == 0 and torch.count_nonzero(out[5]) == 0
    # ctx = max_blocks_per_seq * bs exactly, several partitions
    spec = W.DecodeSpec("max", 2, 4, 4, 128, bs, torch.bfloat16, torch.bfloat16, ("fixed", 1024))
    w = W.make_decode_workload(spec, seed=3, device=DEV)
    assert w.block_tables.shape[1] * bs == 1024
    for pt in (0, 16, 512, 1024):
        check_step(w, partition_tokens=pt, what=f"max ctx pt={pt}")


def test_empty_batch_is_a_no_op():
    q = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device=DEV)
    kc = torch.zeros((4, 16, 4, 128), dtype=torch.bfloat16, device=DEV)
    out = pk.paged_attention_decode(q, kc, kc, torch.zeros((0, 1), dtype=torch.int32, device=DEV),
                                    torch.zeros((0,), dtype=torch.int32, device=DEV), 0.1)
    assert out.shape == (0, 4, 128)


def test_placement_invariance_on_gpu():
    """Moving every physical block to another id (tables rewritten to match)
    leaves the output bit-identical."""
    spec = W.LLAMA7B.with_(num_seqs=6, num_q_heads=4, num_kv_heads=4, ctx=("uniform", 100, 900), new_tokens=False)
    w = W.make_decode_workload(spec, seed=4, device=DEV)
    out1 = pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.scale)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(9)).to(DEV)
    kc, vc = torch.empty_like(w.key_cache), torch.empty_like(w.value_cache)
    kc[perm] = w.key_cache
    vc[perm] = w.value_cache
    tables = perm[w.block_tables.long()].to(torch.int32)
    out2 = pk.paged_attention_decode(w.q, kc, vc, tables, w.context_lens, w.scale)
    assert torch.equal(out1, out2)


FULL = [W.LLAMA7B, W.LLAMA13B, W.SPECS["llama13b_decode_b256_bf16_bs32"], W.PARALLEL_SAMPLING, W.GQA_LONG,
        W.GQA_BATCH]


@pytest.mark.parametrize("spec", FULL, ids=lambda s: s.name)
def test_full_size_configs_sampled(spec):
    w = W.make_decode_workload(spec, seed=0, device=DEV)
    rows = sample_rows(w, 512)
    check_step(w, rows=rows, what=spec.name)


def test_parallel_sampling_cow_semantics_prompt_1020():
    """Prompt of 1020 tokens: the last prompt block is partial, so each
    candidate's first new token goes into its own copy of it (ref_count 4
    shared prompt, 3 copy-on-write copies, one candidate keeps the block)."""
    spec = W.PARALLEL_SAMPLING.with_(num_seqs=16, sampling=(4, 4, 1020, 1, 1))
    w = W.make_decode_workload(spec, seed=5, device=DEV)
    assert len(w.copy_pairs) == 4 * 3
    check_step(w, what="cow-1020")


def test_validate_rejects_bad_inputs_without_launching():
    w = W.make_decode_workload(W.TINY, seed=0, device=DEV)
    before = pk.launch_count()
    bad = w.block_tables.clone()
    bad[0, 0] = w.num_blocks
    with pytest.raises(pk.PagedKVError) as e:
        pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, bad, w.context_lens, w.scale, validate=True)
    assert e.value.code == -8
    pairs = torch.tensor([[1, 5], [2, 5]], dtype=torch.int64, device=DEV)
    with pytest.raises(pk.PagedKVError) as e:
        pk.kv_block_copy(pairs, w.key_cache.clone(), w.value_cache.clone(), validate=True)
    assert e.value.code == -9
    slots = w.slot_mapping.clone()
    slots[0] = w.num_blocks * 16
    with pytest.raises(pk.PagedKVError) as e:
        pk.paged_kv_write(w.new_k, w.new_v, slots, w.key_cache.clone(), w.value_cache.clone(), validate=True)
    assert e.value.code == -8
    assert pk.launch_count() == before


def test_kernel_guards_set_status_instead_of_reading_outside_the_pool():
    """Ids past the pool reach the kernels only without validate; the kernels
    skip them (no access outside the pool) and report through the status word."""
    w = W.make_decode_workload(W.TINY, seed=0, device=DEV)
    pk.device_status(clear=True)
    bad = w.block_tables.clone()
    bad[1, 0] = w.num_blocks + 5
    out = pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, bad, w.context_lens, w.scale)
    torch.cuda.synchronize()
    assert pk.device_status(clear=True) & pk.STATUS_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    slots = w.slot_mapping.clone()
    slots[2] = w.num_blocks * 16 + 3
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    pk.paged_kv_write(w.new_k, w.new_v, slots, kc, vc)
    assert pk.device_status(clear=True) & pk.STATUS_BAD_SLOT
    pairs = torch.tensor([[0, w.num_blocks]], dtype=torch.int64, device=DEV)
    pk.kv_block_copy(pairs, kc, vc)
    assert pk.device_status(clear=True) & pk.STATUS_BAD_COPY_PAIR
    assert pk.device_status(clear=True) == 0


def test_launch_count_counts_kernels():
    w = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=4, num_q_heads=4, num_kv_heads=4), seed=1, device=DEV)
    n0 = pk.launch_count()
    gpu_step(w, partition_tokens=128, validate=False)
    assert pk.launch_count() - n0 == 3   # write, partition pass, reduce


def _poison_unused_rows(w):
    """NaN bit patterns in every cache row no sequence reads: the tail rows of
    each last block and all free blocks (bf16 0x7FC0, fp8 0x7F, fp32 NaN)."""
    bs = w.spec.block_size
    used = torch.zeros(w.num_blocks, bs, dtype=torch.bool, device=w.key_cache.device)
    for b, c in enumerate(w.ctx_list):
        n = -(-c // bs)
        for j in range(n):
            blk = int(w.block_tables[b, j])
            used[blk, : min(bs, c - j * bs)] = True
    for cache in (w.key_cache, w.value_cache):
        if cache.dtype == torch.float8_e4m3fn:
            raw = cache.view(torch.uint8)
            raw[~used] = 0x7F
        elif cache.dtype == torch.bfloat16:
            raw = cache.view(torch.int16)
            raw[~used] = 0x7FC0
        else:
            cache[~used] = float("nan")


@pytest.mark.parametrize("spec", [W.TINY.with_(new_tokens=False),
                                  W.LLAMA7B.with_(num_seqs=5, num_q_heads=4, num_kv_heads=4, ctx=("list", (1, 17, 200, 513, 31)),
                                                  new_tokens=False),
                                  W.GQA_BATCH.with_(num_seqs=5, ctx=("list", (1, 17, 200, 513, 31)), new_tokens=False),
                                  W.GQA_BATCH.with_(num_seqs=3, block_size=32, ctx=("list", (5, 33, 70)),
                                                    new_tokens=False)],
                         ids=["fp32-mha", "bf16-mha", "fp8-gqa-mma", "fp8-gqa-mma-bs32"])
def test_rows_past_the_context_are_never_used(spec):
    w = W.make_decode_workload(spec, seed=12, device=DEV)
    _poison_unused_rows(w)
    for pt in (0, 2 * spec.block_size):
        out = check_step(w, partition_tokens=pt, what=f"poisoned pool pt={pt}")
        assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("hkv", [1, 2, 3, 6])
@pytest.mark.parametrize("bs", [16, 32])
def test_fp8_gqa8_kv_head_counts(hkv, bs):
    """fp8 cache, 8 query heads per KV head (the tensor-core kernel) with odd and even KV-head
    counts: the oracle's result, with the fused new-token write, at several partition lengths."""
    spec = W.GQA_BATCH.with_(num_seqs=4, num_q_heads=8 * hkv, num_kv_heads=hkv, block_size=bs,
                             ctx=("list", (1, 3 * bs + 5, 700, 2 * bs)))
    w = W.make_decode_workload(spec, seed=20 + hkv + bs, device=DEV)
    for pt in (0, bs, 4 * bs):
        check_step(w, partition_tokens=pt, what=f"hkv={hkv} bs={bs} pt={pt}")
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    out = pk.paged_decode_append(w.q, w.new_k, w.new_v, kc, vc, w.block_tables, w.context_lens, w.scale,
                                 k_scale=w.k_scale, v_scale=w.v_scale, partition_tokens=bs, validate=True)
    torch.cuda.synchronize()
    rk, rv, ref = oracle_step(w)
    assert_cache_equal(kc, rk, "append key_cache")
    assert_cache_equal(vc, rv, "append value_cache")
    assert_close(f64(out), ref, *tol_for(w), what=f"fused append hkv={hkv} bs={bs}")
    assert pk.device_status(clear=True) == 0


def test_tensor_core_kernel_guards_bad_block_ids():
    w = W.make_decode_workload(W.GQA_BATCH.with_(num_seqs=3, ctx=("list", (40, 300, 7)), new_tokens=False), seed=13,
                               device=DEV)
    pk.device_status(clear=True)
    bad = w.block_tables.clone()
    bad[1, 3] = -7
    bad[0, 0] = w.num_blocks
    out = pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, bad, w.context_lens, w.scale,
                                    k_scale=w.k_scale, v_scale=w.v_scale, partition_tokens=64)
    torch.cuda.synchronize()
    assert pk.device_status(clear=True) & pk.STATUS_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    # the sequence without bad ids is unaffected
    rows = np.arange(2 * 64, 3 * 64)
    _, _, ref = oracle_step(w, rows=rows)
    assert_close(f64(out).reshape(-1, 128)[rows], ref, *tol_for(w), what="unaffected sequence")


@pytest.mark.parametrize("spec", [W.PARALLEL_SAMPLING.with_(num_seqs=8, num_q_heads=8, num_kv_heads=8,
                                                            sampling=(2, 4, 100, 1, 30)),
                                  W.GQA_BATCH.with_(num_seqs=4, ctx=("list", (1, 100, 700, 33)))],
                         ids=["bf16-cow", "fp8-gqa"])
def test_host_buffer_step_matches_device_step_and_oracle(spec):
    """pkv_decode_step_host: host inputs, one call (copies in, block copy,
    write, decode, copy out) -- same bytes as the device-side step."""
    w = W.make_decode_workload(spec, seed=14, device=DEV)
    kc_d, vc_d, out_d = gpu_step(w, validate=False)
    kc_h, vc_h = w.key_cache.clone(), w.value_cache.clone()
    pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
    out_h = pk.decode_step(pin(w.q), pin(w.new_k), pin(w.new_v), pin(w.slot_mapping), pin(w.block_tables),
                           pin(w.context_lens), kc_h, vc_h, w.scale, copy_pairs=pin(w.copy_pairs),
                           k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    assert torch.equal(out_h, out_d.cpu())
    assert torch.equal(kc_h, kc_d) and torch.equal(vc_h, vc_d)
    rk, rv, ref = oracle_step(w)
    assert_cache_equal(kc_h, rk, "host-step key_cache")
    assert_close(out_h.float().numpy().astype(np.float64), ref, *tol_for(w), what="host step")


@pytest.mark.parametrize("depth", [1, 2, 3])
def test_host_step_pipeline_matches_device_steps(depth):
    """pkv_decode_step_host_async through HostStepPipeline: several steps in
    flight (copies in, kernels and copies out on three streams), each step's
    output equal to the device-side step on the same inputs."""
    spec = W.PARALLEL_SAMPLING.with_(num_seqs=8, num_q_heads=8, num_kv_heads=8, sampling=(2, 4, 100, 1, 30))
    w = W.make_decode_workload(spec, seed=16, device=DEV)
    pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
    steps = 7
    g = torch.Generator(device="cpu").manual_seed(16)
    qs = [torch.randn(w.q.shape, generator=g).to(w.q.dtype).pin_memory() for _ in range(steps)]
    host = {k: pin(getattr(w, k)) for k in ("new_k", "new_v", "slot_mapping", "block_tables", "context_lens",
                                            "copy_pairs")}
    kc_h, vc_h = w.key_cache.clone(), w.value_cache.clone()
    pipe = pk.HostStepPipeline(qs[0], host["new_k"], kc_h, host["block_tables"], host["copy_pairs"], depth=depth)
    got = []
    for i in range(steps):
        out, done = pipe.step(qs[i], host["new_k"], host["new_v"], host["slot_mapping"], host["block_tables"],
                              host["context_lens"], kc_h, vc_h, w.scale, copy_pairs=host["copy_pairs"])
        if i >= depth - 1:  # the oldest step in flight is complete once its event is
            j = i - depth + 1
            pipe.done[j % depth].synchronize()
            got.append(pipe.outs[j % depth].clone())
    pipe.synchronize()
    for j in range(steps - depth + 1, steps):
        got.append(pipe.outs[j % depth].clone())
    # the same steps on the device: the copies and the write are idempotent, only q changes
    kc_d, vc_d = w.key_cache.clone(), w.value_cache.clone()
    for i in range(steps):
        ref = pk.decode_step(qs[i].to(DEV), w.new_k, w.new_v, w.slot_mapping, w.block_tables, w.context_lens, kc_d,
                             vc_d, w.scale, copy_pairs=w.copy_pairs)
        torch.cuda.synchronize()
        assert torch.equal(got[i], ref.cpu()), f"step {i}"
    assert torch.equal(kc_h, kc_d) and torch.equal(vc_h, vc_d)


def test_full_size_bf16_gqa_sampled():
    w = W.make_decode_workload(W.SPECS["gqa70b_bf16_b128_ctx8k"], seed=0, device=DEV)
    check_step(w, rows=sample_rows(w, 512), what="gqa70b_bf16_b128_ctx8k")


APPEND_SPECS = [W.TINY, W.LLAMA7B.with_(num_seqs=6, num_q_heads=4, num_kv_heads=4, ctx=("list", (1, 16, 17, 700, 513, 0))),
                W.LLAMA7B.with_(num_seqs=4, num_q_heads=16, num_kv_heads=2, ctx=("list", (1, 33, 300, 64))),
                W.GQA_BATCH.with_(num_seqs=4, ctx=("list", (1, 100, 700, 33))),
                W.GQA_BATCH.with_(num_seqs=3, num_q_heads=16, num_kv_heads=4, ctx=("list", (5, 48, 200))),
                W.GQA_BATCH.with_(num_seqs=3, block_size=32, ctx=("list", (5, 33, 300)))]


@pytest.mark.parametrize("spec", APPEND_SPECS, ids=["fp32-mha", "bf16-mha", "bf16-gqa8-mma", "fp8-gqa8-mma",
                                                     "fp8-gqa4-cudacore", "fp8-gqa8-mma-bs32"])
def test_fused_append_equals_write_then_decode(spec):
    """pkv_paged_decode_append writes the same cache bytes as the separate
    write at slot (ctx-1) and gives the same attention output (bit-identical:
    the same kernels compute it), which the oracle confirms."""
    w = W.make_decode_workload(spec, seed=15, device=DEV)
    kc_ref, vc_ref, out_ref = gpu_step(w, partition_tokens=2 * spec.block_size)
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    # sequences with an empty context have no position to write: their k_new row is ignored
    out = pk.paged_decode_append(w.q, w.new_k, w.new_v, kc, vc, w.block_tables, w.context_lens, w.scale,
                                 k_scale=w.k_scale, v_scale=w.v_scale, partition_tokens=2 * spec.block_size,
                                 validate=True)
    torch.cuda.synchronize()
    assert torch.equal(kc.view(torch.uint8), kc_ref.view(torch.uint8))
    assert torch.equal(vc.view(torch.uint8), vc_ref.view(torch.uint8))
    assert torch.equal(out, out_ref)
    rk, rv, ref = oracle_step(w)
    assert_cache_equal(kc, rk, "append key_cache")
    assert_close(f64(out), ref, *tol_for(w), what="fused append")
    assert pk.device_status(clear=True) == 0


@pytest.mark.parametrize("dtype", [torch.bfloat16, FP8])
def test_swap_out_and_in_through_pinned_host_memory(dtype):
    """One launch moves blocks device -> pinned host (swap out) and back (swap
    in), byte-exact against the oracle's copies."""
    spec = W.LLAMA7B.with_(num_seqs=4, num_q_heads=8, num_kv_heads=8, cache_dtype=dtype,
                           ctx=("list", (40, 300, 17, 129)), new_tokens=False)
    w = W.make_decode_workload(spec, seed=16, device=DEV)
    NB = w.num_blocks
    host_k = torch.zeros((7,) + tuple(w.key_cache.shape[1:]), dtype=dtype).pin_memory()
    host_v = torch.zeros_like(host_k).pin_memory()
    out_pairs = torch.tensor([[NB - 1, 0], [3, 6], [0, 2], [5, 1]], dtype=torch.int64)
    pk.swap_blocks(out_pairs.to(DEV), w.key_cache, w.value_cache, host_k, host_v, validate=True)
    torch.cuda.synchronize()
    hk = to_np(torch.zeros_like(host_k)).copy()
    hv = hk.copy()
    oracle.swap_blocks(out_pairs.numpy(), to_np(w.key_cache), to_np(w.value_cache), hk, hv)
    assert np.array_equal(to_np(host_k), hk) and np.array_equal(to_np(host_v), hv)
    # swap back in to other device blocks
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    in_pairs = torch.tensor([[0, 8], [6, 9], [2, 3]], dtype=torch.int64)
    pk.swap_blocks(in_pairs.to(DEV), host_k, host_v, kc, vc, validate=True)
    torch.cuda.synchronize()
    ek, ev = to_np(w.key_cache).copy(), to_np(w.value_cache).copy()
    oracle.swap_blocks(in_pairs.numpy(), hk, hv, ek, ev)
    assert_cache_equal(kc, ek, "swap-in key_cache")
    assert_cache_equal(vc, ev, "swap-in value_cache")
    assert pk.device_status(clear=True) == 0


@pytest.mark.parametrize("dtype,n", [(torch.bfloat16, 1 << 20), (torch.bfloat16, 1003), (torch.float32, 77777),
                                     (torch.float32, 5)])
def test_fp8_scale_on_device_matches_oracle(dtype, n):
    g = torch.Generator(device=DEV).manual_seed(n)
    x = torch.randn(n, generator=g, device=DEV, dtype=torch.float32).to(dtype)
    x[n // 3] = -7.5
    s = pk.fp8_scale_from_amax(x)
    assert float(s.item()) == oracle.fp8_scale(to_np(x), ocode(dtype))
    assert float(pk.fp8_scale_from_amax(torch.zeros(64, dtype=dtype, device=DEV)).item()) == 1.0


def _mq_check(mw, partition_tokens=0, rows=None, what="", validate=True):
    """Multi-query attention through the C ABI against the oracle on the same stored bytes
    (bf16 caches: 2e-3 + 1e-2 |ref|; fp8 caches: 2e-3 + 3e-2 |ref|)."""
    w = mw.base
    s = w.spec
    out = pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                        mw.query_start_loc, w.scale, k_scale=w.k_scale, v_scale=w.v_scale,
                                        partition_tokens=partition_tokens, validate=validate)
    torch.cuda.synchronize()
    ref = oracle.paged_attention_multiquery(to_np(mw.q), to_np(mw.query_start_loc), to_np(w.key_cache),
                                            to_np(w.value_cache), to_np(w.block_tables), to_np(w.context_lens),
                                            scale=w.scale, q_dtype=oracle.BF16, cache_dtype=ocode(s.cache_dtype),
                                            k_scale=w.k_scale, v_scale=w.v_scale, rows=rows)
    got = f64(out)
    if rows is not None:
        got = got.reshape(-1, s.head_dim)[rows]
    assert_close(got, ref, *(TOL_FP8 if s.cache_dtype == FP8 else TOL_BF16), what=what)
    assert pk.device_status(clear=True) == 0
    return out


TOL_BF16 = (2e-3, 1e-2)
TOL_FP8 = (2e-3, 3e-2)


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 2)])
def test_multiquery_small(bs, hq, hkv):
    ctxs = (1, 20, 700, 129, 33, 64)
    q_lens = (1, 5, 8, 129, 0, 17)            # a full prefill from scratch (129 of 129), an empty query set
    spec = W.DecodeSpec("mq", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs + hq, device=DEV)
    for pt in (0, 2 * bs, 256):
        _mq_check(mw, partition_tokens=pt, what=f"bs={bs} hq={hq} hkv={hkv} pt={pt}")


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv,q_lens", [(4, 4, (1, 5, 16, 0, 3, 7)), (8, 4, (8, 1, 0, 5, 2, 8)),
                                           (16, 2, (2, 1, 0, 2, 1, 2))])
def test_multiquery_verify_sized(bs, hq, hkv, q_lens):
    # at most 16 rows per (sequence, KV head): the 16-row tile kernel
    ctxs = (9, 20, 700, 129, 2100, 64)
    spec = W.DecodeSpec("mqv", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs * hq, device=DEV)
    for pt in (0, bs, 512):
        _mq_check(mw, partition_tokens=pt, what=f"bs={bs} hq={hq} hkv={hkv} pt={pt}")


def test_multiquery_queries_before_the_context_get_zero_rows():
    # context_lens shortened below q_len (which validate rejects): the leading queries have no position
    ctxs = (40, 300, 20, 900)
    spec = W.DecodeSpec("mqneg", len(ctxs), 8, 2, 128, 16, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, (20, 5, 20, 100), seed=11, device=DEV)
    w = mw.base
    w.context_lens.copy_(torch.tensor([7, 300, 0, 60], dtype=torch.int32, device=DEV))
    for pt in (0, 16, 128):
        out = _mq_check(mw, partition_tokens=pt, what=f"negative positions pt={pt}", validate=False)
        qsl = mw.query_start_loc.tolist()
        assert torch.all(out[qsl[0]:qsl[0] + 13] == 0) and torch.all(out[qsl[2]:qsl[3]] == 0)
        assert torch.all(out[qsl[3]:qsl[3] + 40] == 0)


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv,q_lens", [(8, 4, (12, 3, 0, 7, 16, 1)), (8, 2, (12, 5, 1, 0, 9, 11)),
                                           (4, 4, (64, 33, 1, 17, 0, 50)), (16, 2, (6, 5, 1, 2, 0, 3)),
                                           (16, 2, (8, 7, 8, 1, 4, 2))])
def test_multiquery_mid_sized_tiles(bs, hq, hkv, q_lens):
    # 17 to 64 rows per (sequence, KV head): 2, 3 or 4 compute warps per mma.sync CTA
    ctxs = (300, 40, 700, 2050, 16, 129)
    spec = W.DecodeSpec("mqm", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs + hq + sum(q_lens), device=DEV)
    for pt in (0, bs, 256):
        _mq_check(mw, partition_tokens=pt, what=f"bs={bs} hq={hq} hkv={hkv} q_lens={q_lens} pt={pt}")


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 4), (8, 2), (16, 2)])
def test_multiquery_prefill_sized_tiles(bs, hq, hkv):
    # more than 64 rows per (sequence, KV head): the 128-row tcgen05 kernel for
    # partitions of a multiple of 128 tokens (0 = automatic), mma.sync otherwise
    ctxs = (70, 500, 30, 1000, 10, 300, 2049)
    q_lens = (70, 129, 1, 200, 0, 300, 77)
    spec = W.DecodeSpec("mqp", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs + 3 * hq + hkv, device=DEV)
    for pt in (0, 128, 384, 2 * bs):
        _mq_check(mw, partition_tokens=pt, what=f"bs={bs} hq={hq} hkv={hkv} pt={pt}")


@pytest.mark.parametrize("q_lens", [(5, 5, 5, 5), (12, 9, 12, 3), (200, 129, 64, 300)],
                         ids=["verify", "verify-stacked-tile", "prefill"])
def test_multiquery_rows_past_the_context_are_never_used(q_lens):
    ctxs = (300, 129, 100, 700)
    spec = W.DecodeSpec("mqnan", len(ctxs), 8, 4, 128, 16, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=21, device=DEV)
    _poison_unused_rows(mw.base)
    for pt in (0, 128, 32):
        out = _mq_check(mw, partition_tokens=pt, what=f"poisoned pool pt={pt}")
        assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("q_lens", [(5, 5, 5), (100, 200, 40)], ids=["verify", "prefill"])
def test_multiquery_guards_bad_block_ids(q_lens):
    ctxs = (300, 400, 200)
    spec = W.DecodeSpec("mqbad", len(ctxs), 8, 2, 128, 16, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=22, device=DEV)
    w = mw.base
    bad = w.block_tables.clone()
    bad[1, 3] = -7
    bad[0, 10] = w.num_blocks
    pk.device_status(clear=True)
    out = pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, bad, w.context_lens, mw.query_start_loc,
                                        w.scale)
    torch.cuda.synchronize()
    assert pk.device_status(clear=True) & pk.STATUS_BAD_BLOCK_ID
    assert torch.isfinite(out.float()).all()
    qsl = mw.query_start_loc.tolist()
    rows = np.arange(qsl[2] * 8, qsl[3] * 8)  # the sequence without bad ids is unaffected
    ref = oracle.paged_attention_multiquery(to_np(mw.q), to_np(mw.query_start_loc), to_np(w.key_cache),
                                            to_np(w.value_cache), to_np(w.block_tables), to_np(w.context_lens),
                                            scale=w.scale, q_dtype=oracle.BF16, cache_dtype=oracle.BF16, rows=rows)
    assert_close(f64(out).reshape(-1, 128)[rows], ref, *TOL_BF16, what="unaffected sequence")


def test_multiquery_long_context_largest_partition():
    # a 16384-token partition (1024 blocks of bs 16, their ids read tile by tile by the tcgen05 kernel's
    # producers) and a context split in two by it
    ctxs = (20000, 16384, 300)
    spec = W.DecodeSpec("mqlong", len(ctxs), 8, 2, 128, 16, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.05))
    mw = W.make_multiquery_workload(spec, (40, 17, 300), seed=23, device=DEV)
    T = int(mw.query_start_loc[-1])
    rows = np.unique(np.concatenate([np.arange(0, T * 8, 7), [T * 8 - 1]]))
    for pt in (16384, 0):
        _mq_check(mw, partition_tokens=pt, rows=rows, what=f"long context pt={pt}")


@pytest.mark.parametrize("seed", range(6))
def test_multiquery_random_shapes(seed):
    """Seeded random mixes: head grouping, block size, context and query lengths (zero, one, a few,
    a full prefill), partition length -- both multi-query kernels."""
    rng = np.random.default_rng(100 + seed)
    hkv = int(rng.choice([1, 2, 4]))
    g = int(rng.choice([1, 2, 4, 8]))
    bs = int(rng.choice([16, 32]))
    B = int(rng.integers(1, 7))
    ctxs = tuple(int(c) for c in rng.integers(1, 1500, B))
    q_lens = tuple(int(min(c, rng.choice([0, 1, 3, 9, 40, 200, c]))) for c in ctxs)
    spec = W.DecodeSpec("mqrand", B, hkv * g, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=200 + seed, device=DEV)
    pt = int(rng.choice([0, bs, 4 * bs, 512]))
    _mq_check(mw, partition_tokens=pt, what=f"seed={seed} g={g} hkv={hkv} bs={bs} ctxs={ctxs} q_lens={q_lens} pt={pt}")


@pytest.mark.parametrize("seed", range(4))
def test_multiquery_random_verify_shapes(seed):
    """Seeded random verification mixes with at most 16 rows per (sequence, KV head): the mma.sync kernel."""
    rng = np.random.default_rng(300 + seed)
    hkv = int(rng.choice([1, 2, 4]))
    g = int(rng.choice([1, 2, 4, 8]))
    bs = int(rng.choice([16, 32]))
    B = int(rng.integers(1, 9))
    ctxs = tuple(int(c) for c in rng.integers(1, 3000, B))
    q_lens = tuple(int(min(c, rng.integers(0, 16 // g + 1))) for c in ctxs)
    spec = W.DecodeSpec("mqrandv", B, hkv * g, hkv, 128, bs, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=400 + seed, device=DEV)
    pt = int(rng.choice([0, bs, 4 * bs, 512]))
    _mq_check(mw, partition_tokens=pt, what=f"seed={seed} g={g} hkv={hkv} bs={bs} ctxs={ctxs} q_lens={q_lens} pt={pt}")


def test_multiquery_prefill_chunk_after_prefix():
    spec = W.LLAMA7B.with_(num_seqs=3, num_q_heads=8, num_kv_heads=8, ctx=("list", (600, 300, 1030)))
    mw = W.make_multiquery_workload(spec, (300, 300, 512), seed=3, device=DEV)
    for pt in (0, 128):
        _mq_check(mw, partition_tokens=pt, what=f"prefill chunk pt={pt}")


@pytest.mark.parametrize("name", sorted(W.MQ_SPECS))
def test_multiquery_full_size_sampled(name):
    spec, n = W.MQ_SPECS[name]
    rng = np.random.default_rng(0)
    mw = W.make_multiquery_workload(spec, [n] * spec.num_seqs, seed=0, device=DEV)
    T = int(mw.query_start_loc[-1])
    rows = np.unique(np.concatenate([rng.choice(T * spec.num_q_heads, 400, replace=False),
                                     np.arange(spec.num_q_heads), T * spec.num_q_heads - 1 - np.arange(spec.num_q_heads)]))
    _mq_check(mw, rows=rows, what=name)


@pytest.mark.parametrize("case", ["rounds-ranked", "sequence-ranked", "over-1024-sequences", "over-64-rounds"])
def test_multiquery_persistent_many_units(case):
    """The tcgen05 kernel's persistent CTAs over many units: about 8 units per CTA with the
    longest-first ranking of (sequence, partition, query tile) triples; more than 1024 triples, where
    whole sequences are ranked; more than 1024 sequences and more than 64 units per CTA, where units
    keep the sequences' order; empty query sets and sequences whose rows span two 128-row units among
    them.  Sampled rows against the oracle."""
    rng = np.random.default_rng({"rounds-ranked": 31, "sequence-ranked": 34, "over-1024-sequences": 32,
                                 "over-64-rounds": 33}[case])
    if case in ("rounds-ranked", "sequence-ranked"):
        B, hq, hkv = (300 if case == "rounds-ranked" else 600), 8, 2
        q_lens = [int(x) if x > 3 else 0 for x in rng.integers(0, 41, B)]      # up to 160 rows: two units
        ctxs = [int(max(q, c)) for q, c in zip(q_lens, rng.integers(50, 601, B))]
    elif case == "over-1024-sequences":
        B, hq, hkv = 1100, 4, 4
        q_lens = [int(x) for x in rng.integers(17, 25, B)]                      # 17-24 rows: stacked tile
        ctxs = [int(max(q, c)) for q, c in zip(q_lens, rng.integers(30, 201, B))]
    else:
        B, hq, hkv = 1000, 32, 16
        q_lens = [int(x) for x in rng.integers(9, 11, B)]                       # 18-20 rows, 16000 units
        ctxs = [int(max(q, c)) for q, c in zip(q_lens, rng.integers(20, 81, B))]
    spec = W.DecodeSpec("mqpers", B, hq, hkv, 128, 16, torch.bfloat16, torch.bfloat16, ("list", tuple(ctxs)),
                        ("slack", 1.1))
    mw = W.make_multiquery_workload(spec, q_lens, seed=int(rng.integers(1 << 30)), device=DEV)
    T = int(mw.query_start_loc[-1])
    rows = np.unique(np.concatenate([rng.choice(T * hq, 600, replace=False), np.arange(hq),
                                     T * hq - 1 - np.arange(hq)]))
    _mq_check(mw, rows=rows, what=case)


def test_multiquery_one_query_per_sequence_matches_decode():
    spec = W.LLAMA7B.with_(num_seqs=5, num_q_heads=16, num_kv_heads=2, ctx=("list", (1, 40, 300, 17, 1000)))
    mw = W.make_multiquery_workload(spec, (1,) * 5, seed=4, device=DEV)
    w = mw.base
    mq = pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                       mw.query_start_loc, w.scale)
    dec = pk.paged_attention_decode(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.scale)
    torch.cuda.synchronize()
    assert_close(f64(mq), f64(dec), *TOL_BF16, what="multi-query vs decode")


@pytest.mark.parametrize("q_lens", [(4, 2, 3), (12, 5, 9), (100, 200, 40)], ids=["verify", "verify-stacked-tile", "prefill"])
@pytest.mark.parametrize("case", ["end_past_total", "negative_start", "q_len_above_max"])
def test_multiquery_guards_bad_query_start_loc(q_lens, case):
    """query_start_loc entries outside [0, total_q] (or a q_len above max_q_len) reach the kernels only
    without validate: the sequence is skipped -- no store outside `out`, its rows untouched -- and the
    status bit is set; the other sequences are computed as usual."""
    ctxs = (300, 400, 200)
    spec = W.DecodeSpec("mqqsl", len(ctxs), 8, 2, 128, 16, torch.bfloat16, torch.bfloat16, ("list", ctxs),
                        ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=24, device=DEV)
    w = mw.base
    good = mw.query_start_loc.tolist()
    T = good[-1]
    bad, max_q, skipped = list(good), max(q_lens), set()
    if case == "end_past_total":
        bad[2] = T + 8            # sequence 1 ends past total_q, sequence 2 then ends before it starts
        skipped = {1, 2}
    elif case == "negative_start":
        bad[0] = -3
        skipped = {0}
    else:
        max_q = min(q_lens)
        skipped = {b for b in range(3) if q_lens[b] > max_q}
        assert skipped
    qsl = torch.tensor(bad, dtype=torch.int32, device=DEV)
    sentinel = 1000.0
    ref = oracle.paged_attention_multiquery(to_np(mw.q), to_np(mw.query_start_loc), to_np(w.key_cache),
                                            to_np(w.value_cache), to_np(w.block_tables), to_np(w.context_lens),
                                            scale=w.scale, q_dtype=oracle.BF16, cache_dtype=oracle.BF16)
    ref = ref.reshape(T, 8, 128)
    for pt in (0, 64):
        buf = torch.full((T + 2, 8, 128), sentinel, dtype=torch.bfloat16, device=DEV)
        out = buf[1:T + 1]
        pk.device_status(clear=True)
        pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, qsl,
                                      w.scale, max_q_len=max_q, out=out, partition_tokens=pt)
        torch.cuda.synchronize()
        assert pk.device_status(clear=True) == pk.STATUS_BAD_QUERY_LOC, f"{case} pt={pt}"
        assert torch.all(buf[0] == sentinel) and torch.all(buf[T + 1] == sentinel), "store outside out"
        for b in range(3):
            rows = slice(good[b], good[b + 1])
            if b in skipped:
                assert torch.all(out[rows] == sentinel), f"skipped sequence {b} was written ({case} pt={pt})"
            else:
                assert_close(f64(out[rows]), ref[rows], *TOL_BF16, what=f"{case} sequence {b} pt={pt}")



# ---- multi-query attention over fp8 (E4M3) caches: the mma.sync kernel, codes widened to fp16 ----

@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (16, 4), (16, 2)])
def test_multiquery_fp8_small(bs, hq, hkv):
    # ragged query counts: one, verification-sized, a full prefill from scratch (129 of 129), none
    ctxs = (1, 20, 700, 129, 33, 64)
    q_lens = (1, 5, 8, 129, 0, 17)
    spec = W.DecodeSpec("mqf8", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, FP8, ("list", ctxs), ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs + hq + hkv, device=DEV)
    for pt in (0, 2 * bs, 256):
        _mq_check(mw, partition_tokens=pt, what=f"fp8 bs={bs} hq={hq} hkv={hkv} pt={pt}")


def test_multiquery_fp8_queries_before_the_context_get_zero_rows():
    ctxs = (40, 300, 20, 900)
    spec = W.DecodeSpec("mqf8neg", len(ctxs), 16, 2, 128, 16, torch.bfloat16, FP8, ("list", ctxs), ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, (20, 5, 20, 100), seed=31, device=DEV)
    w = mw.base
    w.context_lens.copy_(torch.tensor([7, 300, 0, 60], dtype=torch.int32, device=DEV))
    for pt in (0, 16, 128):
        out = _mq_check(mw, partition_tokens=pt, what=f"fp8 negative positions pt={pt}", validate=False)
        qsl = mw.query_start_loc.tolist()
        assert torch.all(out[qsl[0]:qsl[0] + 13] == 0) and torch.all(out[qsl[2]:qsl[3]] == 0)
        assert torch.all(out[qsl[3]:qsl[3] + 40] == 0)


@pytest.mark.parametrize("q_lens", [(5, 5, 5, 5), (200, 129, 64, 300)], ids=["verify", "prefill"])
def test_multiquery_fp8_rows_past_the_context_are_never_used(q_lens):
    ctxs = (300, 129, 100, 700)
    spec = W.DecodeSpec("mqf8nan", len(ctxs), 16, 2, 128, 16, torch.bfloat16, FP8, ("list", ctxs), ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=32, device=DEV)
    _poison_unused_rows(mw.base)
    for pt in (0, 128, 32):
        out = _mq_check(mw, partition_tokens=pt, what=f"fp8 poisoned pool pt={pt}")
        assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("seed", range(6))
def test_multiquery_fp8_random_shapes(seed):
    """Seeded random mixes over fp8 caches: grouping, block size, context and query lengths, partition."""
    rng = np.random.default_rng(500 + seed)
    hkv = int(rng.choice([1, 2, 4]))
    g = int(rng.choice([1, 2, 4, 8]))
    bs = int(rng.choice([16, 32]))
    B = int(rng.integers(1, 7))
    ctxs = tuple(int(c) for c in rng.integers(1, 1500, B))
    q_lens = tuple(int(min(c, rng.choice([0, 1, 3, 5, 9, 40, 200, c]))) for c in ctxs)
    spec = W.DecodeSpec("mqf8rand", B, hkv * g, hkv, 128, bs, torch.bfloat16, FP8, ("list", ctxs), ("slack", 1.3))
    mw = W.make_multiquery_workload(spec, q_lens, seed=600 + seed, device=DEV)
    pt = int(rng.choice([0, bs, 4 * bs, 512]))
    _mq_check(mw, partition_tokens=pt,
              what=f"fp8 seed={seed} g={g} hkv={hkv} bs={bs} ctxs={ctxs} q_lens={q_lens} pt={pt}")


def test_multiquery_fp8_one_query_per_sequence_matches_decode():
    spec = W.GQA_BATCH.with_(num_seqs=5, ctx=("list", (1, 40, 300, 17, 1000)))
    mw = W.make_multiquery_workload(spec, (1,) * 5, seed=33, device=DEV)
    w = mw.base
    mq = pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                       mw.query_start_loc, w.scale, k_scale=w.k_scale, v_scale=w.v_scale)
    dec = pk.paged_attention_decode(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.scale,
                                    k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    assert_close(f64(mq), f64(dec), *TOL_FP8, what="fp8 multi-query vs fp8 decode")


def test_multiquery_fp8_rejects_missing_scales():
    spec = W.GQA_BATCH.with_(num_seqs=2, ctx=("list", (40, 30)))
    mw = W.make_multiquery_workload(spec, (3, 3), seed=34, device=DEV)
    w = mw.base
    with pytest.raises(pk.PagedKVError):
        pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                      mw.query_start_loc, w.scale, k_scale=0.0, v_scale=w.v_scale)


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv,q_lens", [(4, 4, (1, 5, 16, 0, 3, 7)), (8, 4, (8, 1, 0, 5, 2, 8)),
                                           (16, 4, (4, 1, 0, 2, 3, 4)), (16, 2, (2, 1, 0, 2, 1, 2))])
def test_multiquery_fp8_verify_sized(bs, hq, hkv, q_lens):
    # at most 16 rows per (sequence, KV head): the mma.sync kernel with its widening producer warp
    ctxs = (9, 20, 700, 129, 2100, 64)
    spec = W.DecodeSpec("mqf8v", len(ctxs), hq, hkv, 128, bs, torch.bfloat16, FP8, ("list", ctxs), ("slack", 1.2))
    mw = W.make_multiquery_workload(spec, q_lens, seed=bs * hq + hkv, device=DEV)
    for pt in (0, bs, 512):
        _mq_check(mw, partition_tokens=pt, what=f"fp8 verify bs={bs} hq={hq} hkv={hkv} pt={pt}")

"""The allocation-free decode entry point (pkv_paged_attention_decode_static).

It serves callers that cannot give the library device scratch -- an engine
whose KV block pool already holds nearly all device memory, code that must not
call cudaMalloc mid-step because it can synchronise the device, bindings with
no device allocator -- by keeping the split-context partials in a fixed array
inside the library.  These tests call it through the C ABI and check it
against pkv_paged_attention_decode (which takes a caller workspace) on two
calls in a row with different inputs, so stale partials from the first call
would show up in the second.  Both entry points run the same kernels with the
same partition length, so their outputs must be bit-identical; one case is
also checked against the CPU oracle.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_450_b200 as pk
from paged_kv_cache_450_b200 import _lib
from paged_kv_cache_450_b200 import workloads as W
from step_helpers import TOL, assert_close, oracle_step

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
CODES = {torch.float32: 0, torch.bfloat16: 1, torch.float8_e4m3fn: 2}
STATIC_LIMIT = 16 << 20


def call_static(w, out, partition_tokens=0):
    s = w.spec
    lib = _lib.load()
    stream = torch.cuda.current_stream(DEV).cuda_stream
    return lib.pkv_paged_attention_decode_static(
        out.data_ptr(), w.q.data_ptr(), w.key_cache.data_ptr(), w.value_cache.data_ptr(),
        w.block_tables.data_ptr(), w.context_lens.data_ptr(), s.num_seqs, s.num_q_heads, s.num_kv_heads,
        s.head_dim, s.block_size, w.block_tables.shape[1], w.num_blocks, w.scale, w.k_scale, w.v_scale,
        CODES[s.q_dtype], CODES[s.cache_dtype], partition_tokens, ctypes.c_void_p(stream))


def reference(w, partition_tokens=0):
    return pk.paged_attention_decode(w.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens, w.scale,
                                     k_scale=w.k_scale, v_scale=w.v_scale, partition_tokens=partition_tokens)


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def test_static_scratch_matches_workspace_entry_point_two_calls():
    # call 1: 64 sequences of up to 2048 tokens (four 512-token partitions)
    w1 = W.make_decode_workload(W.LLAMA7B.with_(new_tokens=False), seed=21, device=DEV)
    # call 2: another batch with other lengths, GQA and 128-token partitions
    w2 = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=24, num_q_heads=32, num_kv_heads=8,
                                                ctx=("uniform", 1, 3000), new_tokens=False), seed=22, device=DEV)
    cases = [(w1, 0), (w2, 128)]
    for w, pt in cases:
        need = pk.decode_workspace_bytes(w.spec.num_seqs, w.spec.num_q_heads, w.spec.num_kv_heads,
                                         w.spec.head_dim, w.spec.block_size, w.block_tables.shape[1],
                                         w.spec.cache_dtype, pt)
        assert 0 < need <= STATIC_LIMIT       # the cases really use the split-context scratch
    refs = [reference(w, pt) for w, pt in cases]
    torch.cuda.synchronize()
    outs = []
    for w, pt in cases:
        out = torch.empty_like(w.q)
        assert call_static(w, out, pt) == 0
        outs.append(out)
    torch.cuda.synchronize()
    # the first call on the device made its set-up already; later calls
    # allocate nothing at all
    out_again = torch.empty_like(w1.q)
    torch.cuda.synchronize()
    free_mid = torch.cuda.mem_get_info(DEV)[0]
    assert call_static(w1, out_again, 0) == 0
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(DEV)[0] == free_mid
    for (w, pt), out, ref in zip(cases, outs, refs):
        assert torch.equal(out, ref), f"static scratch differs from the workspace call (partition_tokens={pt})"
    assert torch.equal(out_again, refs[0]), "static scratch, third call"
    # the second case against the oracle as well (every row)
    _, _, oref = oracle_step(w2)
    atol, rtol = TOL["bf16"]
    assert_close(f64(outs[1]).reshape(oref.shape), oref, atol, rtol, what="static scratch vs oracle")
    assert pk.device_status(clear=True) == 0


def test_static_scratch_rejects_calls_that_need_more_than_the_array():
    w = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=8, new_tokens=False), seed=23, device=DEV)
    s = w.spec
    MB = 4096  # a table wide enough that 128-token partitions need > 16 MiB of partials
    tables = torch.zeros((s.num_seqs, MB), dtype=torch.int32, device=DEV)
    tables[:, : w.block_tables.shape[1]] = w.block_tables
    need = pk.decode_workspace_bytes(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                     s.cache_dtype, 128)
    assert need > STATIC_LIMIT
    big = W.DecodeWorkload(**{**w.__dict__, "block_tables": tables})
    out = torch.zeros_like(w.q)
    n0 = pk.launch_count()
    assert call_static(big, out, 128) == -6        # PKV_ERR_WORKSPACE, nothing launched
    assert pk.launch_count() == n0
    assert torch.count_nonzero(out) == 0


def test_static_scratch_argument_errors_and_empty_batch_match_the_workspace_call():
    w = W.make_decode_workload(W.LLAMA7B.with_(num_seqs=4, new_tokens=False), seed=24, device=DEV)
    s = w.spec
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream)
    out = torch.zeros_like(w.q)
    MB = w.block_tables.shape[1]

    def both(num_seqs, head_dim, pt):
        a = lib.pkv_paged_attention_decode_static(
            out.data_ptr(), w.q.data_ptr(), w.key_cache.data_ptr(), w.value_cache.data_ptr(),
            w.block_tables.data_ptr(), w.context_lens.data_ptr(), num_seqs, s.num_q_heads, s.num_kv_heads, head_dim,
            s.block_size, MB, w.num_blocks, w.scale, 1.0, 1.0, 1, 1, pt, stream)
        b = lib.pkv_paged_attention_decode(
            out.data_ptr(), w.q.data_ptr(), w.key_cache.data_ptr(), w.value_cache.data_ptr(),
            w.block_tables.data_ptr(), w.context_lens.data_ptr(), num_seqs, s.num_q_heads, s.num_kv_heads, head_dim,
            s.block_size, MB, w.num_blocks, w.scale, 1.0, 1.0, 1, 1, pt, None, 0, 0, stream)
        return a, b

    n0 = pk.launch_count()
    assert both(0, 128, 0) == (0, 0)                   # empty batch: nothing to do, nothing launched
    assert both(s.num_seqs, 96, 0) == (-3, -3)         # PKV_ERR_HEAD_DIM before any workspace question
    assert both(s.num_seqs, 128, 17) == (-13, -13)     # PKV_ERR_PARTITION
    assert pk.launch_count() == n0
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0

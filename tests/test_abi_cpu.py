"""The C ABI library loads without a GPU, exports every function that
include/pagedkv.h declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

import paged_kv_cache_450_b200 as pk
from paged_kv_cache_450_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pagedkv.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), f"{n} declared in pagedkv.h but not exported"
    assert set(names) == set(_lib.SIGNATURES), "binding signatures and header disagree"


def test_header_constants_match_binding():
    text = open(HEADER).read()
    consts = dict(re.findall(r"#define (PKV_\w+) \(?(-?0x[0-9a-fA-F]+|-?\d+)u?\)?", text))
    assert int(consts["PKV_DTYPE_F32"]) == pk.DTYPE_F32
    assert int(consts["PKV_DTYPE_BF16"]) == pk.DTYPE_BF16
    assert int(consts["PKV_DTYPE_FP8_E4M3"]) == pk.DTYPE_FP8_E4M3
    assert int(consts["PKV_STATUS_BAD_BLOCK_ID"], 16) == pk.STATUS_BAD_BLOCK_ID
    assert int(consts["PKV_STATUS_WAIT_TIMEOUT"], 16) == pk.STATUS_WAIT_TIMEOUT


def test_status_strings():
    lib = _lib.load()
    assert lib.pkv_status_string(0) == b"ok"
    for code in range(-13, 0):
        assert lib.pkv_status_string(code) != b"unknown status"


P = None


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=96), -3), (dict(block_size=24), -4), (dict(num_q_heads=12, num_kv_heads=8), -5),
    (dict(num_q_heads=48, num_kv_heads=4), -5), (dict(q_dtype=2), -2), (dict(cache_dtype=7), -2),
    (dict(q_dtype=0, cache_dtype=1), -2), (dict(num_seqs=-1), -7), (dict(partition_tokens=24), -13),
    (dict(out=0), -1), (dict(out=0x1008), -10), (dict(workspace=0), -6),
])
def test_decode_argument_errors(kw, code):
    lib = _lib.load()
    a = dict(out=0x1000, q=0x2000, key_cache=0x3000, value_cache=0x4000, block_tables=0x5000, context_lens=0x6000,
             num_seqs=4, num_q_heads=8, num_kv_heads=8, head_dim=128, block_size=16, max_blocks_per_seq=256,
             num_blocks=100, scale=0.1, k_scale=1.0, v_scale=1.0, q_dtype=1, cache_dtype=1, partition_tokens=0,
             workspace=0x7000, workspace_bytes=1 << 30, validate=0, stream=None)
    a.update(kw)
    args = [a[k] for k in ("out", "q", "key_cache", "value_cache", "block_tables", "context_lens", "num_seqs",
                           "num_q_heads", "num_kv_heads", "head_dim", "block_size", "max_blocks_per_seq",
                           "num_blocks", "scale", "k_scale", "v_scale", "q_dtype", "cache_dtype",
                           "partition_tokens", "workspace", "workspace_bytes", "validate", "stream")]
    if a["workspace"] == 0:
        args[20] = 0
    assert lib.pkv_paged_attention_decode(*args) == code


def test_write_and_copy_argument_errors():
    lib = _lib.load()
    assert lib.pkv_paged_kv_write(0x10, 0x20, 0x30, 0, 0x40, 0x50, 10, 16, 4, 128, 1, 1, 1.0, 1.0, 0, None) == 0
    assert lib.pkv_paged_kv_write(None, 0x20, 0x30, 5, 0x40, 0x50, 10, 16, 4, 128, 1, 1, 1.0, 1.0, 0, None) == -1
    assert lib.pkv_paged_kv_write(0x10, 0x20, 0x30, 5, 0x40, 0x50, 10, 16, 4, 128, 1, 0, 1.0, 1.0, 0, None) == -2
    assert lib.pkv_paged_kv_write(0x10, 0x20, 0x30, 5, 0x40, 0x50, 10, 16, 4, 128, 1, 2, 0.0, 1.0, 0, None) == -7
    assert lib.pkv_paged_kv_write(0x18, 0x20, 0x30, 5, 0x40, 0x50, 10, 16, 4, 128, 1, 1, 1.0, 1.0, 0, None) == -10
    assert lib.pkv_kv_block_copy(0x10, 0, 0x20, 0x30, 10, 4096, 0, None) == 0
    assert lib.pkv_kv_block_copy(0x10, 3, 0x20, 0x30, 10, 4004, 0, None) == -7
    assert lib.pkv_kv_block_copy(None, 3, 0x20, 0x30, 10, 4096, 0, None) == -1


def test_partition_choice_and_workspace_size():
    bf16, fp8 = torch.bfloat16, torch.float8_e4m3fn
    # single partition when the longest context fits in 512 tokens: no workspace
    assert pk.decode_partition_tokens(4, 4, 4, 64, 16, 7, torch.float32) == 112
    assert pk.decode_workspace_bytes(4, 4, 4, 64, 16, 7, torch.float32) == 0
    # 64 sequences x 32 heads, up to 2048 tokens: 512 (at least 4 partitions per long sequence)
    assert pk.decode_partition_tokens(64, 32, 32, 128, 16, 128, bf16) == 512
    P = pk.decode_max_partitions(64, 32, 32, 128, 16, 128, bf16)
    assert P == 4
    rows = 64 * 32 * P
    assert pk.decode_workspace_bytes(64, 32, 32, 128, 16, 128, bf16) == \
        ((rows * 8 + 255) // 256) * 256 + rows * 128 * 4
    # 256 x 40 heads up to 4096 tokens: more pairs than four waves of CTAs -> up to 2048 tokens
    assert pk.decode_partition_tokens(256, 40, 40, 128, 16, 256, bf16) == 2048
    # parallel sampling, 128 x 40 heads up to 1088 tokens: a single partition, no workspace
    assert pk.decode_partition_tokens(128, 40, 40, 128, 16, 68, bf16) == 2048
    assert pk.decode_workspace_bytes(128, 40, 40, 128, 16, 68, bf16) == 0
    # fp8 GQA 64/8: 16 x 32k -> 2048 CTAs, at least three quarters of a wave (148 SMs assumed without a GPU)
    assert pk.decode_partition_tokens(16, 64, 8, 128, 16, 2048, fp8) == 2048
    assert pk.decode_partition_tokens(128, 64, 8, 128, 16, 512, fp8) == 2048
    # explicit partition lengths
    assert pk.decode_partition_tokens(1, 1, 1, 128, 16, 100, bf16, 48) == 48
    with pytest.raises(pk.PagedKVError):
        pk.decode_partition_tokens(1, 1, 1, 128, 16, 100, bf16, 40)


def test_shared_prefix_partition_and_workspace():
    # 32 groups x 40 heads over up to 1088 tokens: three partitions at least -> 512 tokens
    assert pk.decode_shared_prefix_partition_tokens(32, 40, 16, 68) == 512
    # the plain decode of the same batch (128 x 40 pairs) keeps one partition
    assert pk.decode_partition_tokens(128, 40, 40, 128, 16, 68, torch.bfloat16) == 2048
    assert pk.decode_shared_prefix_partition_tokens(32, 40, 16, 68, 256) == 256
    assert pk.decode_shared_prefix_partition_tokens(2, 2, 16, 20) == 320   # <= 512 tokens: one partition
    with pytest.raises(pk.PagedKVError):
        pk.decode_shared_prefix_partition_tokens(32, 40, 16, 68, 24)
    with pytest.raises(pk.PagedKVError):
        pk.decode_shared_prefix_partition_tokens(32, 40, 8, 68)
    # two slots (shared + own) per partition of the longest table, per (sequence, query head): m, l and 128 floats
    P = 2 * -(-68 * 16 // 512)
    rows = 128 * 40 * P
    assert pk.decode_shared_prefix_workspace_bytes(128, 32, 40, 40, 128, 16, 68) == \
        (rows * 8 + 255) // 256 * 256 + rows * 128 * 4
    assert pk.decode_shared_prefix_workspace_bytes(128, 32, 40, 40, 128, 16, 68, 512) == \
        pk.decode_shared_prefix_workspace_bytes(128, 32, 40, 40, 128, 16, 68)


def test_shared_prefix_host_step_staging_and_argument_errors():
    lib = _lib.load()
    BF = pk.DTYPE_BF16
    # 128 sequences in 32 groups, 40 heads, d 128, bs 16, 68 blocks, 96 copy pairs: the staged inputs
    # (each piece 256-byte aligned) followed by the shared-prefix workspace
    a = lambda x: (x + 255) // 256 * 256  # noqa: E731
    qb, kb = 128 * 40 * 128 * 2, 128 * 40 * 128 * 2
    pieces = [qb, qb, kb, kb, 128 * 68 * 4, 128 * 4, 33 * 4, 32 * 4, 96 * 16]
    ws = pk.decode_shared_prefix_workspace_bytes(128, 32, 40, 40, 128, 16, 68)
    want = a(sum(a(x) for x in pieces) + ws)
    assert lib.pkv_decode_step_shared_prefix_staging_bytes(128, 32, 40, 40, 128, 16, 68, BF, 0, 96) == want
    assert lib.pkv_decode_step_shared_prefix_staging_bytes(128, 32, 40, 40, 128, 8, 68, BF, 0, 96) == 0  # bs 8
    # argument errors come back before anything is enqueued (no GPU needed)
    buf = ctypes.create_string_buffer(1024)
    p = ctypes.addressof(buf)
    aligned = (p + 255) // 256 * 256
    call = lambda out, k, v, staging: lib.pkv_decode_step_host_shared_prefix_async(  # noqa: E731
        out, p, k, v, p, p, p, p, 1, 1, None, 0, p, p, 1, 8, 8, 128, 16, 4, 16, 0.1, BF, BF, 0, staging, 512,
        None, None, None, None, None)
    ERR_NULL_POINTER, ERR_WORKSPACE, ERR_MISALIGNED = -1, -6, -10
    assert call(None, None, None, aligned) == ERR_NULL_POINTER       # no output buffer
    assert call(p, p, None, aligned) == ERR_NULL_POINTER             # k_new without v_new
    assert call(p, None, None, aligned + 16) == ERR_MISALIGNED       # staging not 256-byte aligned
    assert call(p, None, None, aligned) == ERR_WORKSPACE             # staging too small
    assert lib.pkv_decode_step_host_shared_prefix_async(
        None, None, None, None, None, None, None, None, 0, 0, None, 0, p, p, 0, 8, 8, 128, 16, 4, 16, 0.1, BF, BF, 0,
        aligned, 512, None, None, None, None, None) == 0                     # nothing to do


def test_multiquery_partition_and_workspace():
    lib = _lib.load()
    BF, F8 = pk.DTYPE_BF16, pk.DTYPE_FP8_E4M3
    PT0, WS0 = lib.pkv_multiquery_partition_tokens, lib.pkv_multiquery_workspace_bytes

    def PT(B, ql, hq, hkv, bs, mb, pt, cd=BF):  # (num_seqs, max_q_len, Hq, Hkv, bs, max_blocks, cache dtype, pt)
        return PT0(B, ql, hq, hkv, bs, mb, cd, pt)

    def WS(B, T, ql, hq, hkv, d, bs, mb, pt, cd=BF):
        return WS0(B, T, ql, hq, hkv, d, bs, mb, cd, pt)

    # prefill-sized rows, 1024 tcgen05 CTAs >= two waves: one partition over the longest context
    assert PT(8, 512, 32, 32, 16, 128, 0) == 2048
    assert WS(8, 8 * 512, 512, 32, 32, 128, 16, 128, 0) == 0
    # GQA verification (40 rows per KV head, tcgen05): 64 x 8 = 512 CTAs already fill two waves of
    # one CTA per SM -> one partition; 8 sequences -> split in 256-token multiples
    assert PT(64, 5, 64, 8, 16, 512, 0) == 8192
    assert WS(64, 64 * 5, 5, 64, 8, 128, 16, 512, 0) == 0
    pt = PT(8, 5, 64, 8, 16, 512, 0)
    assert pt % 256 == 0 and 256 <= pt < 8192
    P = -(-512 * 16 // pt)
    rows = 8 * 5 * 64 * P
    assert WS(8, 8 * 5, 5, 64, 8, 128, 16, 512, 0) == ((rows * 8 + 255) // 256) * 256 + rows * 128 * 4
    # fp8 caches follow the same kernel split (40 rows: tcgen05), hence the same partitions
    assert PT(64, 5, 64, 8, 16, 512, 0, F8) == 8192
    assert WS(64, 64 * 5, 5, 64, 8, 128, 16, 512, 0, F8) == 0
    assert PT(8, 5, 64, 8, 16, 512, 0, F8) == pt
    # MHA verification (5 rows): 16-row CTAs, 6 per SM
    assert PT(64, 5, 32, 32, 16, 128, 0) > 0
    # explicit partition lengths: a multiple of the block size up to 16384 tokens
    assert PT(1, 4, 8, 8, 16, 100, 48) == 48
    ERR_HEAD_DIM, ERR_BAD_DTYPE, ERR_BLOCK_SIZE, ERR_HEAD_GROUPING, ERR_BAD_SHAPE, ERR_PARTITION = -3, -2, -4, -5, -7, -13
    assert PT(1, 4, 8, 8, 16, 100, 40) == ERR_PARTITION
    assert PT(1, 4, 8, 8, 16, 100, 16400) == ERR_PARTITION
    # argument errors
    assert PT(1, 4, 8, 8, 8, 100, 0) == ERR_BLOCK_SIZE
    assert PT(1, 4, 8, 3, 16, 100, 0) == ERR_HEAD_GROUPING
    assert PT(-1, 4, 8, 8, 16, 100, 0) == ERR_BAD_SHAPE
    assert PT(1, 4, 8, 8, 16, 100, 0, pk.DTYPE_F32) == ERR_BAD_DTYPE
    # a call with no work launches nothing and needs nothing
    assert lib.pkv_paged_attention_multiquery(None, None, None, None, None, None, None, 0, 0, 0, 8, 8, 128, 16, 10,
                                              100, 0.1, 1.0, 1.0, BF, BF, 0, None, 0, 0, None) == 0
    # unsupported shapes are refused before anything else happens
    args = [ctypes.c_void_p(16)] * 7 + [1, 4, 4, 8, 8]
    assert lib.pkv_paged_attention_multiquery(*args, 64, 16, 10, 100, 0.1, 1.0, 1.0, BF, BF, 0, None, 0,
                                              0, None) == ERR_HEAD_DIM
    assert lib.pkv_paged_attention_multiquery(*args, 128, 16, 10, 100, 0.1, 1.0, 1.0, pk.DTYPE_F32, BF, 0, None,
                                              0, 0, None) == ERR_BAD_DTYPE
    assert lib.pkv_paged_attention_multiquery(*args, 128, 16, 10, 100, 0.1, 1.0, 1.0, BF, pk.DTYPE_F32, 0, None,
                                              0, 0, None) == ERR_BAD_DTYPE
    # fp8 caches need positive dequantisation scales
    assert lib.pkv_paged_attention_multiquery(*args, 128, 16, 10, 100, 0.1, 0.0, 1.0, BF, F8, 0, None,
                                              0, 0, None) == ERR_BAD_SHAPE


def test_ops_refuse_cpu_tensors():
    import torch
    x = torch.zeros(2, 2, 128)
    with pytest.raises(ValueError):
        pk.paged_attention_decode(x, torch.zeros(4, 16, 2, 128), torch.zeros(4, 16, 2, 128),
                                  torch.zeros(2, 1, dtype=torch.int32), torch.zeros(2, dtype=torch.int32), 0.1)

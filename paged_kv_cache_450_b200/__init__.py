"""paged_kv_cache_450_b200 -- B200 (sm_100a) paged KV-cache decode path.

Python binding of libpagedkv (C ABI in include/pagedkv.h).  Each function
only checks and marshals torch tensors (pointers, sizes, the current CUDA
stream) and calls the library; every step of the path runs in the CUDA
kernels.  Torch provides device memory and streams.  There is no CPU path:
CPU tensors are rejected, and a missing library raises.

    paged_kv_write(k, v, slot_mapping, key_cache, value_cache, ...)
    paged_attention_decode(q, key_cache, value_cache, block_tables, context_lens, scale, ...)
    kv_block_copy(src_dst_pairs, key_cache, value_cache, ...)

Cache layout: key_cache / value_cache are [num_blocks, block_size,
num_kv_heads, head_dim] (float32, bfloat16 or float8_e4m3fn).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib

DTYPE_F32, DTYPE_BF16, DTYPE_FP8_E4M3 = 0, 1, 2
_DTYPES = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float8_e4m3fn: DTYPE_FP8_E4M3}

STATUS_BAD_BLOCK_ID = 0x1
STATUS_BAD_CONTEXT = 0x2
STATUS_BAD_SLOT = 0x4
STATUS_BAD_COPY_PAIR = 0x8
STATUS_WAIT_TIMEOUT = 0x10
STATUS_BAD_QUERY_LOC = 0x20
STATUS_BAD_GROUP = 0x40

__all__ = ["paged_kv_write", "paged_attention_decode", "paged_decode_append", "paged_attention_decode_shared_prefix",
           "decode_shared_prefix_workspace_bytes", "decode_shared_prefix_partition_tokens",
           "paged_attention_multiquery", "multiquery_workspace_bytes", "kv_block_copy", "swap_blocks", "fp8_scale_from_amax",
           "prefix_block_hashes", "PrefixCache", "decode_step", "decode_step_staging_bytes",
           "HostStepPipeline", "SharedPrefixHostStepPipeline", "decode_step_shared_prefix_staging_bytes",
           "decode_workspace_bytes",
           "decode_partition_tokens", "decode_max_partitions", "decode_table_scan", "device_status", "launch_count", "PagedKVError",
           "library_path"]


class PagedKVError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.load().pkv_status_string(code).decode()
        super().__init__(f"{where}: {msg} (status {code})")


def _check(code: int, where: str):
    if code != 0:
        raise PagedKVError(code, where)


def _dtype(t: torch.Tensor) -> int:
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}") from None


def _cuda(*ts: torch.Tensor):
    dev = ts[0].device
    for t in ts:
        if t.device.type != "cuda":
            raise ValueError("libpagedkv works on CUDA tensors only (there is no CPU path)")
        if t.device != dev:
            raise ValueError("all tensors must be on one device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")
    return dev


def _stream(dev, stream):
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    return ctypes.c_void_p(s.cuda_stream)


def library_path() -> str:
    return _lib.path()


def paged_kv_write(k, v, slot_mapping, key_cache, value_cache, *, k_scale: float = 1.0, v_scale: float = 1.0,
                   validate: bool = False, stream=None) -> None:
    """Write each token's K/V into its slot (block = slot // bs, row = slot % bs).

    k, v: [T, Hkv, d] float32 / bfloat16; slot_mapping: int64 [T] (negative =
    skip); caches [NB, bs, Hkv, d] of k's dtype or float8_e4m3fn (then the
    stored code is E4M3(x * (1/k_scale)), saturating)."""
    dev = _cuda(k, v, slot_mapping, key_cache, value_cache)
    if slot_mapping.dtype != torch.int64:
        raise TypeError("slot_mapping must be int64")
    NB, bs, Hkv, d = key_cache.shape
    if value_cache.shape != key_cache.shape or k.shape != v.shape or k.shape[1:] != (Hkv, d) \
            or slot_mapping.shape != (k.shape[0],):
        raise ValueError("shape mismatch")
    lib = _lib.load()
    with torch.cuda.device(dev):
        _check(lib.pkv_paged_kv_write(k.data_ptr(), v.data_ptr(), slot_mapping.data_ptr(), k.shape[0],
                                      key_cache.data_ptr(), value_cache.data_ptr(), NB, bs, Hkv, d, _dtype(k),
                                      _dtype(key_cache), float(k_scale), float(v_scale), int(validate),
                                      _stream(dev, stream)), "paged_kv_write")


def _cache_code(cache_dtype) -> int:
    return cache_dtype if isinstance(cache_dtype, int) else _DTYPES[cache_dtype]


def decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                            cache_dtype, partition_tokens=0) -> int:
    """Split-context partition length (tokens) the decode call will use."""
    r = _lib.load().pkv_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                max_blocks_per_seq, _cache_code(cache_dtype), partition_tokens)
    _check(min(r, 0), "decode_partition_tokens")
    return r


def decode_max_partitions(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                          cache_dtype, partition_tokens=0) -> int:
    r = _lib.load().pkv_decode_max_partitions(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                              max_blocks_per_seq, _cache_code(cache_dtype), partition_tokens)
    _check(min(r, 0), "decode_max_partitions")
    return r


def decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                           cache_dtype, partition_tokens=0) -> int:
    return int(_lib.load().pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                      max_blocks_per_seq, _cache_code(cache_dtype),
                                                      partition_tokens))


def paged_attention_decode(q, key_cache, value_cache, block_tables, context_lens, scale: float,
                           block_size: int | None = None, num_kv_heads: int | None = None, *,
                           k_scale: float = 1.0, v_scale: float = 1.0, out=None, workspace=None,
                           partition_tokens: int = 0, validate: bool = False, stream=None):
    """Single-query decode attention over the block-paged cache.

    q: [B, Hq, d]; caches: [NB, bs, Hkv, d]; block_tables int32 [B, MB];
    context_lens int32 [B].  Returns out [B, Hq, d] in q's dtype.  The
    split-context workspace is allocated with torch when not given."""
    dev = _cuda(q, key_cache, value_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, Hq, d = q.shape
    NB, bs, Hkv, d2 = key_cache.shape
    if block_size is not None and block_size != bs:
        raise ValueError(f"block_size {block_size} does not match the cache's {bs}")
    if num_kv_heads is not None and num_kv_heads != Hkv:
        raise ValueError(f"num_kv_heads {num_kv_heads} does not match the cache's {Hkv}")
    if d2 != d or value_cache.shape != key_cache.shape or block_tables.dim() != 2 or \
            block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("shape mismatch")
    MB = block_tables.shape[1]
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out)
        if out.shape != q.shape or out.dtype != q.dtype:
            raise ValueError("out must match q")
    need = decode_workspace_bytes(B, Hq, Hkv, d, bs, MB, key_cache.dtype, partition_tokens) if B else 0
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    lib = _lib.load()
    with torch.cuda.device(dev):
        _check(lib.pkv_paged_attention_decode(
            out.data_ptr(), q.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(), block_tables.data_ptr(),
            context_lens.data_ptr(), B, Hq, Hkv, d, bs, MB, NB, float(scale), float(k_scale), float(v_scale),
            _dtype(q), _dtype(key_cache), int(partition_tokens), ws_ptr, ws_bytes, int(validate),
            _stream(dev, stream)), "paged_attention_decode")
    return out


def paged_decode_append(q, k_new, v_new, key_cache, value_cache, block_tables, context_lens, scale: float, *,
                        k_scale: float = 1.0, v_scale: float = 1.0, out=None, workspace=None,
                        partition_tokens: int = 0, validate: bool = False, stream=None):
    """Append each sequence's new token (k_new/v_new [B, Hkv, d], q's dtype) at
    logical position context_lens[b] - 1, then run decode attention -- one
    fused launch.  Returns out [B, Hq, d]."""
    dev = _cuda(q, k_new, v_new, key_cache, value_cache, block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, Hq, d = q.shape
    NB, bs, Hkv, d2 = key_cache.shape
    if k_new.shape != (B, Hkv, d) or v_new.shape != k_new.shape or k_new.dtype != q.dtype or d2 != d:
        raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim] in q's dtype")
    if value_cache.shape != key_cache.shape or block_tables.dim() != 2 or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    MB = block_tables.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(B, Hq, Hkv, d, bs, MB, key_cache.dtype, partition_tokens) if B else 0
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_paged_decode_append(
            out.data_ptr(), q.data_ptr(), k_new.data_ptr(), v_new.data_ptr(), key_cache.data_ptr(),
            value_cache.data_ptr(), block_tables.data_ptr(), context_lens.data_ptr(), B, Hq, Hkv, d, bs, MB, NB,
            float(scale), float(k_scale), float(v_scale), _dtype(q), _dtype(key_cache), int(partition_tokens), ws_ptr,
            ws_bytes, int(validate), _stream(dev, stream)), "paged_decode_append")
    return out


def multiquery_workspace_bytes(num_seqs, total_q, max_q_len, num_q_heads, num_kv_heads, head_dim, block_size,
                               max_blocks_per_seq, cache_dtype, partition_tokens=0) -> int:
    """Workspace bytes paged_attention_multiquery needs (0 when no context is split)."""
    return int(_lib.load().pkv_multiquery_workspace_bytes(num_seqs, total_q, max_q_len, num_q_heads, num_kv_heads,
                                                          head_dim, block_size, max_blocks_per_seq,
                                                          _cache_code(cache_dtype), partition_tokens))


def decode_shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size, max_blocks_per_seq,
                                          partition_tokens=0) -> int:
    """Partition length paged_attention_decode_shared_prefix uses for these arguments."""
    r = _lib.load().pkv_decode_shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size,
                                                              max_blocks_per_seq, partition_tokens)
    _check(min(r, 0), "decode_shared_prefix_partition_tokens")
    return int(r)


def decode_shared_prefix_workspace_bytes(num_seqs, num_groups, num_q_heads, num_kv_heads, head_dim, block_size,
                                         max_blocks_per_seq, partition_tokens=0) -> int:
    """Workspace bytes of paged_attention_decode_shared_prefix."""
    return int(_lib.load().pkv_decode_shared_prefix_workspace_bytes(num_seqs, num_groups, num_q_heads, num_kv_heads,
                                                                    head_dim, block_size, max_blocks_per_seq,
                                                                    partition_tokens))


def paged_attention_decode_shared_prefix(q, key_cache, value_cache, block_tables, context_lens, group_start,
                                         shared_blocks, scale: float, *, k_new=None, v_new=None,
                                         max_group_size: int | None = None, out=None, workspace=None,
                                         partition_tokens: int = 0, validate: bool = False, stream=None):
    """Decode attention where groups of consecutive sequences share their first
    shared_blocks[g] physical blocks (parallel sampling): each shared block is
    read once for the whole group.  group_start int32 [G + 1], shared_blocks
    int32 [G].  Same result as paged_attention_decode (or paged_decode_append
    when k_new / v_new are given).  Returns out [B, Hq, d]."""
    dev = _cuda(q, key_cache, value_cache, block_tables, context_lens, group_start, shared_blocks)
    for t in (block_tables, context_lens, group_start, shared_blocks):
        if t.dtype != torch.int32:
            raise TypeError("block_tables, context_lens, group_start and shared_blocks must be int32")
    B, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    Gn = shared_blocks.shape[0]
    if group_start.shape != (Gn + 1,) or block_tables.shape[0] != B or context_lens.shape != (B,):
        raise ValueError("shape mismatch")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    if k_new is not None:
        _cuda(k_new, v_new)
        if k_new.shape != (B, Hkv, d) or v_new.shape != k_new.shape or k_new.dtype != q.dtype:
            raise ValueError("k_new / v_new must be [num_seqs, num_kv_heads, head_dim] in q's dtype")
    MB = block_tables.shape[1]
    if max_group_size is None:
        max_group_size = int((group_start[1:] - group_start[:-1]).max().item()) if Gn else 1
    if out is None:
        out = torch.empty_like(q)
    need = decode_shared_prefix_workspace_bytes(B, max(Gn, 1), Hq, Hkv, d, bs, MB, partition_tokens) if B else 0
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_paged_attention_decode_shared_prefix(
            out.data_ptr(), q.data_ptr(), ptr(k_new), ptr(v_new), key_cache.data_ptr(), value_cache.data_ptr(),
            block_tables.data_ptr(), context_lens.data_ptr(), group_start.data_ptr(), shared_blocks.data_ptr(), B, Gn,
            int(max_group_size), Hq, Hkv, d, bs, MB, NB, float(scale), _dtype(q), _dtype(key_cache),
            int(partition_tokens), ws_ptr, ws_bytes, int(validate), _stream(dev, stream)),
            "paged_attention_decode_shared_prefix")
    return out


def paged_attention_multiquery(q, key_cache, value_cache, block_tables, context_lens, query_start_loc,
                                scale: float, *, k_scale: float = 1.0, v_scale: float = 1.0,
                                max_q_len: int | None = None, out=None, workspace=None,
                                partition_tokens: int = 0, validate: bool = False, stream=None):
    """Causal attention of several new query tokens per sequence over the paged
    cache (chunked prefill, speculative verification).  q: [total_q, Hq, d]
    bf16; caches bf16 or float8_e4m3fn (then k_scale / v_scale dequantise);
    query_start_loc int32 [B + 1]; the queries of sequence b are its last
    q_len_b positions (their K/V already written).  Returns [total_q, Hq, d]."""
    dev = _cuda(q, key_cache, value_cache, block_tables, context_lens, query_start_loc)
    for t in (block_tables, context_lens, query_start_loc):
        if t.dtype != torch.int32:
            raise TypeError("block_tables, context_lens and query_start_loc must be int32")
    T, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    B = context_lens.shape[0]
    if query_start_loc.shape != (B + 1,) or block_tables.shape[0] != B:
        raise ValueError("shape mismatch")
    MB = block_tables.shape[1]
    if max_q_len is None:
        max_q_len = int((query_start_loc[1:] - query_start_loc[:-1]).max().item()) if B else 0
    if out is None:
        out = torch.empty_like(q)
    lib = _lib.load()
    need = multiquery_workspace_bytes(B, T, max_q_len, Hq, Hkv, d, bs, MB, key_cache.dtype, partition_tokens) if B else 0
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(dev):
        _check(lib.pkv_paged_attention_multiquery(
            out.data_ptr(), q.data_ptr(), key_cache.data_ptr(), value_cache.data_ptr(), block_tables.data_ptr(),
            context_lens.data_ptr(), query_start_loc.data_ptr(), B, T, max_q_len, Hq, Hkv, d, bs, MB, NB,
            float(scale), float(k_scale), float(v_scale), _dtype(q), _dtype(key_cache), int(partition_tokens), ws_ptr,
            ws_bytes, int(validate), _stream(dev, stream)), "paged_attention_multiquery")
    return out


def kv_block_copy(src_dst_pairs, key_cache, value_cache, *, validate: bool = False, stream=None) -> None:
    """Copy block src onto block dst in both caches for every (src, dst) row of
    src_dst_pairs (int64 [n, 2]); destinations distinct and never a source."""
    dev = _cuda(src_dst_pairs, key_cache, value_cache)
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be int64 [n, 2]")
    if value_cache.shape != key_cache.shape or value_cache.dtype != key_cache.dtype:
        raise ValueError("caches must match")
    NB = key_cache.shape[0]
    block_bytes = key_cache[0].numel() * key_cache.element_size()
    lib = _lib.load()
    with torch.cuda.device(dev):
        _check(lib.pkv_kv_block_copy(src_dst_pairs.data_ptr(), src_dst_pairs.shape[0], key_cache.data_ptr(),
                                     value_cache.data_ptr(), NB, block_bytes, int(validate),
                                     _stream(dev, stream)), "kv_block_copy")


def fp8_scale_from_amax(x, *, out=None, stream=None):
    """Per-tensor fp8 scale amax(|x|) / 448 computed on the device (float32
    tensor of one element; 1.0 for an all-zero x)."""
    dev = _cuda(x)
    if out is None:
        out = torch.empty((1,), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_fp8_scale_from_amax(x.data_ptr(), x.numel(), _dtype(x), out.data_ptr(),
                                                   _stream(dev, stream)), "fp8_scale_from_amax")
    return out


def swap_blocks(src_dst_pairs, src_key, src_value, dst_key, dst_value, *, validate: bool = False, stream=None):
    """Copy block src of (src_key, src_value) onto block dst of (dst_key,
    dst_value) for every row of src_dst_pairs (int64 [n, 2], on the device), in
    one kernel launch.  Either pool may be pinned host memory (a CPU tensor
    from pin_memory()); the other must be on the device."""
    pools = (src_key, src_value, dst_key, dst_value)
    devs = [t for t in pools if t.device.type == "cuda"]
    if not devs:
        raise ValueError("at least one pool must be on the device")
    for t in pools:
        if t.device.type == "cpu" and not t.is_pinned():
            raise ValueError("host pools must be page-locked (pin_memory())")
        if not t.is_contiguous():
            raise ValueError("pools must be contiguous")
    dev = _cuda(src_dst_pairs, *devs)
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be int64 [n, 2]")
    if src_key.shape[1:] != dst_key.shape[1:] or src_key.dtype != dst_key.dtype or \
            src_value.shape != src_key.shape or dst_value.shape != dst_key.shape:
        raise ValueError("pools must share the block shape and dtype")
    block_bytes = src_key[0].numel() * src_key.element_size()
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_swap_blocks(src_dst_pairs.data_ptr(), src_dst_pairs.shape[0], src_key.data_ptr(),
                                           src_value.data_ptr(), src_key.shape[0], dst_key.data_ptr(),
                                           dst_value.data_ptr(), dst_key.shape[0], block_bytes, int(validate),
                                           _stream(dev, stream)), "swap_blocks")


def decode_table_scan(block_tables, context_lens, num_kv_heads: int, block_size: int, num_blocks: int,
                      partition_tokens: int, *, sink=None, stream=None):
    """The decode grid's block-table reads alone (a measurement aid): one CTA per
    (kv head, partition, sequence) reads its partition's block ids and writes one
    word to ``sink`` (uint32-sized int32 [B * P * Hkv], allocated when not given)."""
    dev = _cuda(block_tables, context_lens)
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise TypeError("block_tables and context_lens must be int32")
    B, MB = block_tables.shape
    P = -(-MB * block_size // partition_tokens)
    if sink is None:
        sink = torch.empty(max(1, B * P * num_kv_heads), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_decode_table_scan(block_tables.data_ptr(), context_lens.data_ptr(), B, num_kv_heads,
                                                 block_size, MB, num_blocks, partition_tokens, sink.data_ptr(),
                                                 sink.numel(), _stream(dev, stream)), "decode_table_scan")
    return sink


def device_status(clear: bool = True, device=None, stream=None) -> int:
    """The library's device status word (STATUS_* bits) on `device`."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    v = ctypes.c_uint(0)
    with torch.cuda.device(dev):
        _check(_lib.load().pkv_device_status(ctypes.byref(v), int(clear), _stream(dev, stream)), "device_status")
    return int(v.value)


def launch_count() -> int:
    """Kernel launches the library has issued in this process."""
    return int(_lib.load().pkv_launch_count())


def decode_step_staging_bytes(q, new_k, key_cache, block_tables, copy_pairs=None, partition_tokens: int = 0) -> int:
    """Device staging bytes decode_step needs for host inputs of these shapes."""
    B, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    T = 0 if new_k is None else new_k.shape[0]
    n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
    return int(_lib.load().pkv_decode_step_staging_bytes(B, Hq, Hkv, d, bs, block_tables.shape[1], _dtype(q),
                                                         _dtype(key_cache), partition_tokens, T, n_pairs))


def decode_step(q, new_k, new_v, slot_mapping, block_tables, context_lens, key_cache, value_cache, scale: float, *,
                copy_pairs=None, k_scale: float = 1.0, v_scale: float = 1.0, out=None, workspace=None,
                staging=None, partition_tokens: int = 0, stream=None):
    """One decode step of one attention layer over a device-resident paged cache.

    Order: copy-on-write block copies (``copy_pairs``, if any), the new-token
    write (``new_k``/``new_v`` at ``slot_mapping``), then decode attention over
    ``context_lens`` (which include the new token).

    Host inputs (CPU tensors; pinned memory keeps the copies asynchronous): a
    single library call (pkv_decode_step_host) enqueues the copies in, the
    step and the copy of the output into ``out`` (a host tensor, allocated
    pinned when not given); ``staging`` is the device scratch it uses
    (allocated when not given, see decode_step_staging_bytes).  Synchronise
    the stream before reading ``out``.  Device inputs: everything stays on the
    device and the device output is returned."""
    dev = key_cache.device
    st = stream if stream is not None else torch.cuda.current_stream(dev)
    if q.device.type == "cpu":
        host = [t for t in (q, new_k, new_v, slot_mapping, block_tables, context_lens, copy_pairs) if t is not None]
        if any(t.device.type != "cpu" or not t.is_contiguous() for t in host):
            raise ValueError("host inputs must all be contiguous CPU tensors")
        _cuda(key_cache, value_cache)
        B, Hq, d = q.shape
        NB, bs, Hkv, _ = key_cache.shape
        T = 0 if new_k is None else new_k.shape[0]
        n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
        need = decode_step_staging_bytes(q, new_k, key_cache, block_tables, copy_pairs, partition_tokens)
        if staging is None:
            staging = torch.empty(need, dtype=torch.uint8, device=dev)
        if out is None:
            out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        with torch.cuda.device(dev):
            _check(_lib.load().pkv_decode_step_host(
                out.data_ptr(), q.data_ptr(), ptr(new_k), ptr(new_v), ptr(slot_mapping), T, block_tables.data_ptr(),
                context_lens.data_ptr(), ptr(copy_pairs), n_pairs, key_cache.data_ptr(), value_cache.data_ptr(), B, Hq,
                Hkv, d, bs, block_tables.shape[1], NB, float(scale), float(k_scale), float(v_scale), _dtype(q),
                _dtype(key_cache), int(partition_tokens), staging.data_ptr(),
                staging.numel() * staging.element_size(), ctypes.c_void_p(st.cuda_stream)), "decode_step")
        return out
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if copy_pairs is not None and copy_pairs.numel():
            kv_block_copy(copy_pairs, key_cache, value_cache, stream=st)
        if new_k is not None:
            paged_kv_write(new_k, new_v, slot_mapping, key_cache, value_cache, k_scale=k_scale, v_scale=v_scale,
                           stream=st)
        return paged_attention_decode(q, key_cache, value_cache, block_tables, context_lens, scale, k_scale=k_scale,
                                      v_scale=v_scale, out=out, workspace=workspace,
                                      partition_tokens=partition_tokens, stream=st)


class HostStepPipeline:
    """Decode steps with host inputs and outputs, ``depth`` of them in flight
    (pkv_decode_step_host_async): the copies in of step i+1 overlap the
    kernels of step i, which run in order on the compute stream.

    ``step(...)`` takes the same host tensors as :func:`decode_step` and
    returns ``(out, done)``: ``out`` is a pinned host tensor owned by the
    pipeline that holds the step's output once ``done`` (a CUDA event) has
    completed, and that is overwritten ``depth`` steps later."""

    def __init__(self, q, new_k, key_cache, block_tables, copy_pairs=None, partition_tokens: int = 0,
                 depth: int = 2, compute_stream=None):
        dev = key_cache.device
        self.depth = int(depth)
        self.partition_tokens = int(partition_tokens)
        need = decode_step_staging_bytes(q, new_k, key_cache, block_tables, copy_pairs, partition_tokens)
        self.staging = [torch.empty(max(need, 1), dtype=torch.uint8, device=dev) for _ in range(self.depth)]
        self.outs = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(self.depth)]
        self.compute = compute_stream if compute_stream is not None else torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.done = [torch.cuda.Event() for _ in range(self.depth)]
        for e in self.done:  # create the events (torch makes them on first record)
            e.record(self.compute)
        self.used = [False] * self.depth
        self.i = 0

    def step(self, q, new_k, new_v, slot_mapping, block_tables, context_lens, key_cache, value_cache, scale: float, *,
             copy_pairs=None, k_scale: float = 1.0, v_scale: float = 1.0):
        host = [t for t in (q, new_k, new_v, slot_mapping, block_tables, context_lens, copy_pairs) if t is not None]
        if any(t.device.type != "cpu" or not t.is_contiguous() for t in host):
            raise ValueError("host inputs must all be contiguous CPU tensors")
        _cuda(key_cache, value_cache)
        k = self.i % self.depth
        B, Hq, d = q.shape
        NB, bs, Hkv, _ = key_cache.shape
        T = 0 if new_k is None else new_k.shape[0]
        n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
        ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        out, st = self.outs[k], self.staging[k]
        with torch.cuda.device(key_cache.device):
            _check(_lib.load().pkv_decode_step_host_async(
                out.data_ptr(), q.data_ptr(), ptr(new_k), ptr(new_v), ptr(slot_mapping), T, block_tables.data_ptr(),
                context_lens.data_ptr(), ptr(copy_pairs), n_pairs, key_cache.data_ptr(), value_cache.data_ptr(), B, Hq,
                Hkv, d, bs, block_tables.shape[1], NB, float(scale), float(k_scale), float(v_scale), _dtype(q),
                _dtype(key_cache), self.partition_tokens, st.data_ptr(), st.numel(),
                ctypes.c_void_p(self.copy_in.cuda_stream), ctypes.c_void_p(self.compute.cuda_stream),
                ctypes.c_void_p(self.copy_out.cuda_stream),
                ctypes.c_void_p(self.done[k].cuda_event if self.used[k] else 0),
                ctypes.c_void_p(self.done[k].cuda_event)), "decode_step_pipelined")
        self.used[k] = True
        self.i += 1
        return out, self.done[k]

    def synchronize(self):
        for e in self.done:
            e.synchronize()


def decode_step_shared_prefix_staging_bytes(q, key_cache, block_tables, num_groups: int, copy_pairs=None,
                                            partition_tokens: int = 0) -> int:
    """Device staging bytes of a shared-prefix host step for inputs of these shapes."""
    B, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
    return int(_lib.load().pkv_decode_step_shared_prefix_staging_bytes(B, int(num_groups), Hq, Hkv, d, bs,
                                                                       block_tables.shape[1], _dtype(q),
                                                                       partition_tokens, n_pairs))


class SharedPrefixHostStepPipeline:
    """HostStepPipeline for groups of sequences sharing their prompt's blocks
    (pkv_decode_step_host_shared_prefix_async): per step the copy-on-write
    copies, then the shared-prefix decode with each sequence's new token
    (``new_k``/``new_v``, [num_seqs][num_kv_heads][head_dim], at position
    context_lens - 1) written inside it.  ``depth`` steps in flight, as
    HostStepPipeline; ``step(...)`` returns ``(out, done)`` the same way."""

    def __init__(self, q, key_cache, block_tables, group_start, copy_pairs=None, partition_tokens: int = 0,
                 depth: int = 2, compute_stream=None):
        dev = key_cache.device
        self.depth = int(depth)
        self.partition_tokens = int(partition_tokens)
        self.num_groups = int(group_start.shape[0]) - 1
        need = decode_step_shared_prefix_staging_bytes(q, key_cache, block_tables, self.num_groups, copy_pairs,
                                                       partition_tokens)
        if need == 0 and q.shape[0] > 0:
            raise ValueError("unsupported shapes or dtypes for the shared-prefix step")
        self.staging = [torch.empty(max(need, 1), dtype=torch.uint8, device=dev) for _ in range(self.depth)]
        self.outs = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(self.depth)]
        self.compute = compute_stream if compute_stream is not None else torch.cuda.current_stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.done = [torch.cuda.Event() for _ in range(self.depth)]
        for e in self.done:  # create the events (torch makes them on first record)
            e.record(self.compute)
        self.used = [False] * self.depth
        self.i = 0

    def step(self, q, new_k, new_v, block_tables, context_lens, group_start, shared_blocks, key_cache, value_cache,
             scale: float, *, max_group_size: int, copy_pairs=None):
        host = [t for t in (q, new_k, new_v, block_tables, context_lens, group_start, shared_blocks, copy_pairs)
                if t is not None]
        if any(t.device.type != "cpu" or not t.is_contiguous() for t in host):
            raise ValueError("host inputs must all be contiguous CPU tensors")
        if (new_k is None) != (new_v is None):
            raise ValueError("new_k and new_v: both or neither")
        _cuda(key_cache, value_cache)
        k = self.i % self.depth
        B, Hq, d = q.shape
        NB, bs, Hkv, _ = key_cache.shape
        n_groups = int(group_start.shape[0]) - 1
        n_pairs = 0 if copy_pairs is None else copy_pairs.shape[0]
        ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        out, st = self.outs[k], self.staging[k]
        with torch.cuda.device(key_cache.device):
            _check(_lib.load().pkv_decode_step_host_shared_prefix_async(
                out.data_ptr(), q.data_ptr(), ptr(new_k), ptr(new_v), block_tables.data_ptr(),
                context_lens.data_ptr(), group_start.data_ptr(), shared_blocks.data_ptr(), n_groups,
                int(max_group_size), ptr(copy_pairs), n_pairs, key_cache.data_ptr(), value_cache.data_ptr(), B, Hq,
                Hkv, d, bs, block_tables.shape[1], NB, float(scale), _dtype(q), _dtype(key_cache),
                self.partition_tokens, st.data_ptr(), st.numel(), ctypes.c_void_p(self.copy_in.cuda_stream),
                ctypes.c_void_p(self.compute.cuda_stream), ctypes.c_void_p(self.copy_out.cuda_stream),
                ctypes.c_void_p(self.done[k].cuda_event if self.used[k] else 0),
                ctypes.c_void_p(self.done[k].cuda_event)), "decode_step_shared_prefix")
        self.used[k] = True
        self.i += 1
        return out, self.done[k]

    def synchronize(self):
        for e in self.done:
            e.synchronize()


# --------------------------------------------------------------------------- #
# prefix caching by hash chain (host side)
# --------------------------------------------------------------------------- #

def _i32(tokens):
    import numpy as np
    return np.ascontiguousarray(tokens, dtype=np.int32)


def prefix_block_hashes(tokens, block_size: int, parent_hash: int = 0, extra_hash: int = 0):
    """Chained FNV-1a 64 hashes of the full blocks of `tokens` (numpy uint64)."""
    import numpy as np
    t = _i32(tokens)
    out = np.zeros(max(1, t.size // block_size), np.uint64)
    n = _lib.load().pkv_prefix_block_hashes(t.ctypes.data, t.size, block_size, parent_hash, extra_hash,
                                            out.ctypes.data)
    _check(min(n, 0), "prefix_block_hashes")
    return out[:n]


class PrefixCache:
    """Hash-chain prefix cache mapping full token blocks to physical block ids
    (reference counted, LRU eviction of unreferenced entries).  Host only."""

    def __init__(self, block_size: int, capacity_blocks: int):
        self.block_size = block_size
        self._lib = _lib.load()
        self._h = self._lib.pkv_prefix_cache_create(block_size, capacity_blocks)
        if not self._h:
            raise ValueError("bad prefix cache arguments")

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pkv_prefix_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        self.close()

    def __len__(self):
        return int(self._lib.pkv_prefix_cache_size(self._h))

    def match(self, tokens, extra_hash: int = 0, max_blocks: int | None = None) -> list:
        import numpy as np
        t = _i32(tokens)
        cap = t.size // self.block_size if max_blocks is None else max_blocks
        ids = np.zeros(max(1, cap), np.int32)
        n = self._lib.pkv_prefix_cache_match(self._h, t.ctypes.data, t.size, extra_hash, ids.ctypes.data, cap)
        _check(min(n, 0), "prefix_cache_match")
        return ids[:n].tolist()

    def insert(self, tokens, block_ids, extra_hash: int = 0) -> int:
        t, ids = _i32(tokens), _i32(block_ids)
        n = self._lib.pkv_prefix_cache_insert(self._h, t.ctypes.data, t.size, extra_hash, ids.ctypes.data, ids.size)
        _check(min(n, 0), "prefix_cache_insert")
        return int(n)

    def release(self, tokens, num_blocks: int, extra_hash: int = 0) -> int:
        t = _i32(tokens)
        n = self._lib.pkv_prefix_cache_release(self._h, t.ctypes.data, t.size, extra_hash, num_blocks)
        _check(min(n, 0), "prefix_cache_release")
        return int(n)

    def evict(self, max_evict: int) -> list:
        import numpy as np
        ids = np.zeros(max(1, max_evict), np.int32)
        n = self._lib.pkv_prefix_cache_evict(self._h, max_evict, ids.ctypes.data)
        _check(min(n, 0), "prefix_cache_evict")
        return ids[:n].tolist()

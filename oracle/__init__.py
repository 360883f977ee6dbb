"""CPU fp64 oracle for the paged KV-cache decode path (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product (``paged_kv_cache_450_b200``) never imports it, and it
imports nothing from the product.

The arithmetic lives in ``pagedkv_oracle.c`` (plain C, fp64, libm ``exp``);
that file's header states what is computed and which page and section each
function follows.  This wrapper only marshals numpy arrays:

* bf16 tensors are passed as ``uint16`` bit patterns, fp8 E4M3 as ``uint8``;
* dtype codes: ``F32 = 0``, ``BF16 = 1``, ``E4M3 = 2`` (the oracle's own).

Every function raises ``OracleError`` on a negative return code (bad shapes,
ids out of range) instead of reading out of bounds.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

F32, BF16, E4M3 = 0, 1, 2

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pagedkv_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


class OracleError(RuntimeError):
    pass


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc into ``oracle/liboracle.so``.

    ``-ffp-contract=off`` keeps every multiply-add as two rounded operations,
    so the fp32 product used by the fp8 encoding is a single binary32 multiply.
    """
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P, I, I64, F, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
    lib.orc_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_to_double.restype = D
    lib.orc_e4m3_from_float.argtypes = [F]
    lib.orc_e4m3_from_float.restype = ctypes.c_uint8
    lib.orc_paged_attention_decode.argtypes = [P, P, I, P, P, I, P, P, I64, I, I, I, I, I64, I64, F, F, F,
                                               P, I64, I]
    lib.orc_paged_attention_decode.restype = I
    lib.orc_decode_partials.argtypes = [P, P, P, P, I, P, P, I, P, P, I64, I, I, I, I, I64, I64, F, F, F,
                                        I64, I64, I]
    lib.orc_decode_partials.restype = I
    lib.orc_merge_partials.argtypes = [P, P, P, P, I64, I64, I]
    lib.orc_merge_partials.restype = None
    lib.orc_paged_kv_write.argtypes = [P, P, I, P, I64, P, P, I, I64, I, I, I, F, F]
    lib.orc_paged_kv_write.restype = I
    lib.orc_kv_block_copy.argtypes = [P, I64, P, P, I64, I64]
    lib.orc_kv_block_copy.restype = I
    lib.orc_swap_blocks.argtypes = [P, I64, P, P, I64, P, P, I64, I64]
    lib.orc_swap_blocks.restype = I
    lib.orc_paged_attention_multiquery.argtypes = [P, P, I, P, P, P, I, P, P, I64, I, I, I, I, I64, I64, F, F, F,
                                                   P, I64, I]
    lib.orc_paged_attention_multiquery.restype = I
    lib.orc_fp8_scale.argtypes = [P, I64, I]
    lib.orc_fp8_scale.restype = F
    lib.orc_e4m3_encode_array.argtypes = [P, P, I64]
    lib.orc_e4m3_encode_array.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle rejected the inputs (code {rc})")


def _dtype_code(a: np.ndarray, declared: int | None) -> int:
    if declared is not None:
        return declared
    if a.dtype == np.float32:
        return F32
    raise OracleError("pass dtype= for bf16 (uint16 bits) or E4M3 (uint8 codes) arrays")


def default_threads() -> int:
    return int(os.environ.get("ORACLE_THREADS", os.cpu_count() or 1))


def e4m3_to_double(code: int) -> float:
    return _load().orc_e4m3_to_double(code)


def e4m3_from_float(x: float) -> int:
    return _load().orc_e4m3_from_float(x)


def e4m3_encode_array(x) -> np.ndarray:
    """E4M3 codes (uint8) of an fp32 array: round to nearest even, saturate to +-448."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.zeros(x.shape, np.uint8)
    if x.size:
        _load().orc_e4m3_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def paged_attention_decode(q, key_cache, value_cache, block_tables, context_lens, *, scale, q_dtype=None,
                           cache_dtype=None, k_scale=1.0, v_scale=1.0, rows=None, num_threads=None):
    """Decode attention over the logically gathered K/V, fp64.

    q: [B, Hq, d]; caches: [NB, bs, Hkv, d]; block_tables int32 [B, MB];
    context_lens int32 [B].  ``rows`` selects flat rows b * Hq + hq (default:
    all).  Returns float64 [len(rows), d] (or [B, Hq, d] for all rows).
    """
    lib = _load()
    q = np.ascontiguousarray(q)
    key_cache = np.ascontiguousarray(key_cache)
    value_cache = np.ascontiguousarray(value_cache)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, d = q.shape
    NB, bs, Hkv, d2 = key_cache.shape
    assert d2 == d and value_cache.shape == key_cache.shape
    MB = block_tables.shape[1] if block_tables.ndim == 2 else 0
    if block_tables.size == 0:
        block_tables = np.zeros((max(B, 1), 1), np.int32)
        MB = 1 if B else 0
    sel = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = B * Hq if sel is None else sel.shape[0]
    out = np.zeros((max(n, 1), d), np.float64)
    rc = lib.orc_paged_attention_decode(
        _ptr(out), _ptr(q), _dtype_code(q, q_dtype), _ptr(key_cache), _ptr(value_cache),
        _dtype_code(key_cache, cache_dtype), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, d, bs, MB, NB,
        scale, k_scale, v_scale, _ptr(sel), n, num_threads or default_threads())
    _check(rc, "paged_attention_decode")
    out = out[:n]
    return out.reshape(B, Hq, d) if sel is None else out


def decode_partials(q, key_cache, value_cache, block_tables, context_lens, *, scale, partition_tokens,
                    max_partitions, q_dtype=None, cache_dtype=None, k_scale=1.0, v_scale=1.0,
                    num_threads=None):
    """Split-context partials (m, l, o) per (b, hq, partition), fp64.

    Returns m [B, Hq, P], l [B, Hq, P], o [B, Hq, P, d] where m is the
    partition's max logit (natural units), l = sum e^{s - m}, o = sum e^{s-m} V / l.
    """
    lib = _load()
    q = np.ascontiguousarray(q)
    key_cache = np.ascontiguousarray(key_cache)
    value_cache = np.ascontiguousarray(value_cache)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    MB = block_tables.shape[1]
    P = int(max_partitions)
    m = np.zeros((B, Hq, P), np.float64)
    l = np.zeros((B, Hq, P), np.float64)
    o = np.zeros((B, Hq, P, d), np.float64)
    rc = lib.orc_decode_partials(
        _ptr(m), _ptr(l), _ptr(o), _ptr(q), _dtype_code(q, q_dtype), _ptr(key_cache), _ptr(value_cache),
        _dtype_code(key_cache, cache_dtype), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, d, bs, MB, NB,
        scale, k_scale, v_scale, int(partition_tokens), P, num_threads or default_threads())
    _check(rc, "decode_partials")
    return m, l, o


def merge_partials(m, l, o):
    """Softmax-identity merge of partials: m, l [R, P]; o [R, P, d] -> [R, d]."""
    lib = _load()
    m = np.ascontiguousarray(m, dtype=np.float64)
    l = np.ascontiguousarray(l, dtype=np.float64)
    o = np.ascontiguousarray(o, dtype=np.float64)
    R, P = m.shape
    d = o.shape[-1]
    out = np.zeros((max(R, 1), d), np.float64)
    lib.orc_merge_partials(_ptr(out), _ptr(m), _ptr(l), _ptr(o), R, P, d)
    return out[:R]


def paged_kv_write(k, v, slot_mapping, key_cache, value_cache, *, in_dtype=None, cache_dtype=None,
                   k_scale=1.0, v_scale=1.0):
    """Scatter new tokens into the caches IN PLACE (numpy arrays)."""
    lib = _load()
    k = np.ascontiguousarray(k)
    v = np.ascontiguousarray(v)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert key_cache.flags["C_CONTIGUOUS"] and value_cache.flags["C_CONTIGUOUS"]
    T = slot_mapping.shape[0]
    NB, bs, Hkv, d = key_cache.shape
    rc = lib.orc_paged_kv_write(_ptr(k), _ptr(v), _dtype_code(k, in_dtype), _ptr(slot_mapping), T,
                                _ptr(key_cache), _ptr(value_cache), _dtype_code(key_cache, cache_dtype), NB, bs,
                                Hkv, d, k_scale, v_scale)
    _check(rc, "paged_kv_write")


def kv_block_copy(pairs, key_cache, value_cache):
    """Copy-on-write block copy IN PLACE: pairs int64 [n, 2] of (src, dst)."""
    lib = _load()
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    assert key_cache.flags["C_CONTIGUOUS"] and value_cache.flags["C_CONTIGUOUS"]
    NB = key_cache.shape[0]
    block_bytes = key_cache.nbytes // NB if NB else 1
    rc = lib.orc_kv_block_copy(_ptr(pairs), pairs.shape[0], _ptr(key_cache), _ptr(value_cache), NB,
                               block_bytes)
    _check(rc, "kv_block_copy")


def swap_blocks(pairs, src_key, src_value, dst_key, dst_value):
    """Copy block src of the source pool onto block dst of the destination pool IN PLACE."""
    lib = _load()
    pairs = np.ascontiguousarray(pairs, dtype=np.int64).reshape(-1, 2)
    for a in (src_key, src_value, dst_key, dst_value):
        assert a.flags["C_CONTIGUOUS"]
    assert src_key.shape[1:] == dst_key.shape[1:] and src_key.dtype == dst_key.dtype
    block_bytes = src_key[0].nbytes if src_key.shape[0] else 1
    rc = lib.orc_swap_blocks(_ptr(pairs), pairs.shape[0], _ptr(src_key), _ptr(src_value), src_key.shape[0],
                             _ptr(dst_key), _ptr(dst_value), dst_key.shape[0], block_bytes)
    _check(rc, "swap_blocks")


def fp8_scale(x, dtype=None) -> float:
    """amax(|x|) / 448 as an fp32 value (1.0 for all zeros)."""
    x = np.ascontiguousarray(x)
    return float(np.float32(_load().orc_fp8_scale(_ptr(x), x.size, _dtype_code(x, dtype))))


def paged_attention_multiquery(q, query_start_loc, key_cache, value_cache, block_tables, context_lens, *, scale,
                               q_dtype=None, cache_dtype=None, k_scale=1.0, v_scale=1.0, rows=None,
                               num_threads=None):
    """Causal multi-query attention over the paged cache, fp64.

    q: [total_q, Hq, d]; query_start_loc int32 [B + 1]; the queries of sequence
    b are its last q_len_b positions.  Returns float64 [total_q, Hq, d] (or
    [len(rows), d] for selected flat rows token * Hq + hq)."""
    lib = _load()
    q = np.ascontiguousarray(q)
    qsl = np.ascontiguousarray(query_start_loc, dtype=np.int32)
    key_cache = np.ascontiguousarray(key_cache)
    value_cache = np.ascontiguousarray(value_cache)
    block_tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    context_lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    T, Hq, d = q.shape
    NB, bs, Hkv, _ = key_cache.shape
    B = context_lens.shape[0]
    MB = block_tables.shape[1]
    sel = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n = T * Hq if sel is None else sel.shape[0]
    out = np.zeros((max(n, 1), d), np.float64)
    rc = lib.orc_paged_attention_multiquery(
        _ptr(out), _ptr(q), _dtype_code(q, q_dtype), _ptr(qsl), _ptr(key_cache), _ptr(value_cache),
        _dtype_code(key_cache, cache_dtype), _ptr(block_tables), _ptr(context_lens), B, Hq, Hkv, d, bs, MB, NB, scale,
        k_scale, v_scale, _ptr(sel), n, num_threads or default_threads())
    _check(rc, "paged_attention_multiquery")
    out = out[:n]
    return out.reshape(T, Hq, d) if sel is None else out

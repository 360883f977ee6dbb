"""Loads libpagedkv.so (building it in-tree first if it is missing or older
than its sources) and declares the C signatures of include/pagedkv.h.

There is no fallback: if the library cannot be built or loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

P, I, I64, F, U64, SZ = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64,
                         ctypes.c_size_t)

# name -> (restype, argtypes), exactly the declarations in include/pagedkv.h
SIGNATURES = {
    "pkv_status_string": (ctypes.c_char_p, [I]),
    "pkv_paged_kv_write": (I, [P, P, P, I64, P, P, I64, I, I, I, I, I, F, F, I, P]),
    "pkv_paged_attention_decode": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I64, F, F, F, I, I, I, P, SZ, I, P]),
    "pkv_paged_decode_append": (I, [P, P, P, P, P, P, P, P, I, I, I, I, I, I, I64, F, F, F, I, I, I, P, SZ, I, P]),
    "pkv_paged_attention_decode_shared_prefix": (I, [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I64, F, I,
                                                     I, I, P, SZ, I, P]),
    "pkv_decode_shared_prefix_partition_tokens": (I, [I, I, I, I, I]),
    "pkv_decode_shared_prefix_workspace_bytes": (SZ, [I, I, I, I, I, I, I, I]),
    "pkv_paged_attention_decode_static": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I64, F, F, F, I, I, I, P]),
    "pkv_decode_step_host": (I, [P, P, P, P, P, I64, P, P, P, I64, P, P, I, I, I, I, I, I, I64, F, F, F, I, I, I,
                                 P, SZ, P]),
    "pkv_decode_step_staging_bytes": (SZ, [I, I, I, I, I, I, I, I, I, I64, I64]),
    "pkv_decode_step_host_async": (I, [P, P, P, P, P, I64, P, P, P, I64, P, P, I, I, I, I, I, I, I64, F, F, F, I, I,
                                       I, P, SZ, P, P, P, P, P]),
    "pkv_decode_step_host_shared_prefix_async": (I, [P, P, P, P, P, P, P, P, I, I, P, I64, P, P, I, I, I, I, I, I, I64,
                                                     F, I, I, I, P, SZ, P, P, P, P, P]),
    "pkv_decode_step_shared_prefix_staging_bytes": (SZ, [I, I, I, I, I, I, I, I, I, I64]),
    "pkv_decode_partition_tokens": (I, [I, I, I, I, I, I, I, I]),
    "pkv_decode_max_partitions": (I, [I, I, I, I, I, I, I, I]),
    "pkv_decode_workspace_bytes": (SZ, [I, I, I, I, I, I, I, I]),
    "pkv_kv_block_copy": (I, [P, I64, P, P, I64, I64, I, P]),
    "pkv_paged_attention_multiquery": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I64, F, F, F, I, I, I, P, SZ,
                                           I, P]),
    "pkv_multiquery_partition_tokens": (I, [I, I, I, I, I, I, I, I]),
    "pkv_multiquery_workspace_bytes": (SZ, [I, I, I, I, I, I, I, I, I, I]),
    "pkv_fp8_scale_from_amax": (I, [P, I64, I, P, P]),
    "pkv_swap_blocks": (I, [P, I64, P, P, I64, P, P, I64, I64, I, P]),
    "pkv_prefix_block_hashes": (I64, [P, I64, I, U64, U64, P]),
    "pkv_prefix_cache_create": (P, [I, I64]),
    "pkv_prefix_cache_destroy": (None, [P]),
    "pkv_prefix_cache_size": (I64, [P]),
    "pkv_prefix_cache_match": (I64, [P, P, I64, U64, P, I64]),
    "pkv_prefix_cache_insert": (I64, [P, P, I64, U64, P, I64]),
    "pkv_prefix_cache_release": (I64, [P, P, I64, U64, I64]),
    "pkv_prefix_cache_evict": (I64, [P, I64, P]),
    "pkv_selftest_wait_timeout": (I, [I64, P, P]),
    "pkv_decode_table_scan": (I, [P, P, I, I, I, I, I64, I, P, SZ, P]),
    "pkv_device_status": (I, [ctypes.POINTER(ctypes.c_uint), I, P]),
    "pkv_launch_count": (U64, []),
}


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def path() -> str:
    return _build.LIB

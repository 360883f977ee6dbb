"""Prefix caching by hash chain: the reference (oracle/prefix.py) pinned to
the chain's defining properties, then the library's native implementation
checked against it operation by operation (host only, no GPU)."""
import numpy as np
import pytest

import paged_kv_cache_450_b200 as pk
from oracle import prefix as ref


def test_fnv1a_definition_cases():
    assert ref.fnv1a(b"") == ref.FNV_OFFSET                                   # no input: the offset basis
    assert ref.fnv1a(b"\x00") == (ref.FNV_OFFSET * ref.FNV_PRIME) % 2 ** 64   # xor with 0 leaves h
    assert ref.fnv1a(b"\x01") != ref.fnv1a(b"\x00")
    # published FNV-1a 64 test vectors
    assert ref.fnv1a(b"a") == 0xaf63dc4c8601ec8c
    assert ref.fnv1a(b"foobar") == 0x85944171f73967e8


def test_chain_properties():
    rng = np.random.default_rng(0)
    toks = rng.integers(0, 50000, 16 * 6).tolist()
    h = ref.block_hashes(toks, 16)
    assert len(h) == 6 and len(set(h)) == 6
    assert ref.block_hashes(toks + [1, 2, 3], 16) == h                        # partial blocks are not hashed
    for i in range(6):                                                        # a token change in block i
        t2 = list(toks)
        t2[16 * i + 5] += 1
        h2 = ref.block_hashes(t2, 16)
        assert h2[:i] == h[:i] and all(a != b for a, b in zip(h2[i:], h[i:]))
    assert all(a != b for a, b in zip(ref.block_hashes(toks, 16, extra=7), h))   # the extra hash
    assert all(a != b for a, b in zip(ref.block_hashes(toks, 16, parent=1), h))  # the parent


def test_reference_cache_semantics():
    c = ref.RefPrefixCache(4, capacity=6)
    sys_prompt = [9, 8, 7, 6, 5, 4, 3, 2]
    a = sys_prompt + [1, 1, 1, 1]
    b = sys_prompt + [2, 2, 2, 2, 0]
    assert c.match(a) == []
    assert c.insert(a, [10, 11, 12]) == 3
    assert c.match(b) == [10, 11]                 # the shared prefix, whole blocks only
    assert c.match(a, extra=5) == []              # another multimodal extra hash: no reuse
    assert c.insert(b, [10, 11, 13]) == 1         # two blocks already cached
    assert c.evict(10) == []                      # everything is referenced
    assert c.release(a, 3) == 3 and c.release(b, 3) == 3
    assert c.evict(1) == [12]                     # least recently used unreferenced entry first
    assert c.insert([0] * 16, [20, 21, 22, 23]) is None   # 4 new > capacity 6 - 4: nothing inserted


def test_native_hashes_match_reference():
    rng = np.random.default_rng(1)
    for bs in (8, 16, 32):
        toks = rng.integers(-5, 2 ** 31 - 1, bs * 9 + 3).astype(np.int32)
        for parent, extra in ((0, 0), (12345, 0), (0, 2 ** 63 + 7)):
            got = pk.prefix_block_hashes(toks, bs, parent, extra)
            assert [int(x) for x in got] == ref.block_hashes(toks.tolist(), bs, parent, extra)


@pytest.mark.parametrize("seed,bs,capacity", [(2, 4, 24), (3, 4, 8), (4, 2, 64), (5, 8, 12), (6, 1, 40)])
def test_native_cache_matches_reference_on_random_operations(seed, bs, capacity):
    rng = np.random.default_rng(seed)
    native, oracle_cache = pk.PrefixCache(bs, capacity), ref.RefPrefixCache(bs, capacity)
    prompts = [rng.integers(0, 6, bs * rng.integers(1, 7)).tolist() for _ in range(12)]
    for p in prompts[6:]:                      # share prefixes between some prompts
        p[:bs * 2] = prompts[0][:bs * 2] if len(prompts[0]) >= 2 * bs else p[:bs * 2]
    next_id = 100
    for step in range(400):
        op = rng.integers(0, 4)
        p = prompts[rng.integers(len(prompts))]
        extra = int(rng.integers(0, 2))
        if op == 0:
            assert native.match(p, extra) == oracle_cache.match(p, extra), step
        elif op == 1:
            n = len(p) // bs
            ids = list(range(next_id, next_id + n))
            next_id += n
            r = oracle_cache.insert(p, ids, extra)
            if r is None:
                with pytest.raises(pk.PagedKVError):
                    native.insert(p, ids, extra)
            else:
                assert native.insert(p, ids, extra) == r, step
        elif op == 2:
            n = int(rng.integers(0, len(p) // bs + 1))
            assert native.release(p, n, extra) == oracle_cache.release(p, n, extra), step
        else:
            k = int(rng.integers(0, 4))
            assert native.evict(k) == oracle_cache.evict(k), step
        assert len(native) == len(oracle_cache)
    native.close()



@pytest.mark.parametrize("impl", ["reference", "native"])
def test_eviction_follows_last_use_not_release_order(impl):
    """The reading of "LRU" ("vLLM KV Cache 实现机制", 3.1: a block keeps a last-accessed time for
    LRU; 3.2: LRU eviction, reference counts protect shared blocks): a block is accessed when a
    request matches or inserts it; dropping a reference is not an access.  So among the
    unreferenced entries the one whose last match or insert is oldest goes first, whatever order
    they were released in."""
    c = ref.RefPrefixCache(2, 8) if impl == "reference" else pk.PrefixCache(2, 8)
    A, B, C = [1, 1], [2, 2], [3, 3]
    assert c.insert(A, [10]) == 1 and c.insert(B, [20]) == 1 and c.insert(C, [30]) == 1  # accessed A, B, C
    assert c.match(A) == [10]                                                             # accessed B, C, A
    # released A first (both references), then C; B keeps its reference
    assert c.release(A, 1) == 1 and c.release(A, 1) == 1 and c.release(C, 1) == 1
    assert c.evict(3) == [30, 10]     # C was accessed before A; least-recently-released would give [10, 30]
    assert c.evict(3) == []           # B is referenced
    assert c.release(B, 1) == 1 and c.evict(3) == [20]
    # a released entry that is matched again moves behind the others
    assert c.insert(A, [11]) == 1 and c.insert(B, [21]) == 1
    assert c.release(A, 1) == 1 and c.release(B, 1) == 1
    assert c.match(A) == [11] and c.release(A, 1) == 1
    assert c.evict(1) == [21] and c.evict(1) == [11]
    if impl == "native":
        c.close()

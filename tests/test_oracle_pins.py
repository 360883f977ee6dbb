"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's formula: the references are a library
routine (torch's fp64 scaled_dot_product_attention over the logically
contiguous K/V, torch's float8_e4m3fn / bfloat16 casts), closed forms,
invariances the pages state, and byte-level facts.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from paging import page_logical

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)


def bf16_value(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def fp8_value(codes, scale=1.0):
    return torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy() * scale


def sdpa(qv, K, V, scale):
    """Library reference: torch fp64 SDPA for one query over contiguous K/V."""
    q = torch.from_numpy(np.asarray(qv, np.float64))[None, None, None, :]
    k = torch.from_numpy(np.asarray(K, np.float64))[None, None]
    v = torch.from_numpy(np.asarray(V, np.float64))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)[0, 0, 0].numpy()


def logical_seqs(rng, ctxs, Hkv, d):
    return [rng.standard_normal((c, Hkv, d)).astype(np.float32) for c in ctxs]


# --------------------------------------------------------------------------- #
# paged decode attention == dense attention over the logical K/V
# --------------------------------------------------------------------------- #

def test_decode_equals_python_double_loop_brute_force():
    """Tiny cases against plain Python: every score, the max, math.exp and the
    weighted sum written out element by element over explicitly gathered
    rows (no library routine at all)."""
    rng = np.random.default_rng(30)
    for trial in range(6):
        B, Hkv, g, d, bs = int(rng.integers(1, 5)), int(rng.integers(1, 3)), int(rng.choice([1, 2])), 8, 4
        Hq = Hkv * g
        ctxs = [int(c) for c in rng.integers(1, 41, B)]
        ks, vs = logical_seqs(rng, ctxs, Hkv, d), logical_seqs(rng, ctxs, Hkv, d)
        nb = sum(-(-c // bs) for c in ctxs) + 3
        order = rng.permutation(nb)
        tk, kp = page_logical(ks, bs, rng, num_blocks=nb, order=order)
        _, vp = page_logical(vs, bs, rng, num_blocks=nb, order=order)
        q = rng.standard_normal((B, Hq, d)).astype(np.float32)
        scale = float(np.float32(0.3))  # the scale crosses the C interface as a float
        out = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=scale)
        for b in range(B):
            for h in range(Hq):
                kh = h // g
                rows_k, rows_v = [], []
                for t in range(ctxs[b]):  # gather through the block table, by hand
                    blk = int(tk[b, t // bs])
                    rows_k.append([float(x) for x in kp[blk, t % bs, kh]])
                    rows_v.append([float(x) for x in vp[blk, t % bs, kh]])
                sc = [scale * sum(float(q[b, h, i]) * kr[i] for i in range(d)) for kr in rows_k]
                mx = max(sc)
                w = [math.exp(x - mx) for x in sc]
                den = sum(w)
                ref = [sum(w[t] * rows_v[t][i] for t in range(len(w))) / den for i in range(d)]
                assert np.allclose(out[b, h], ref, rtol=1e-12, atol=1e-12), (trial, b, h)


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_decode_equals_dense_sdpa_fp32(bs):
    rng = np.random.default_rng(1)
    ctxs = [1, 16, 17, 100, 33]
    Hq = Hkv = 4
    d = 64
    ks, vs = logical_seqs(rng, ctxs, Hkv, d), logical_seqs(rng, ctxs, Hkv, d)
    order = rng.permutation(64)
    tk, kp = page_logical(ks, bs, rng, num_blocks=64, order=order)
    tv, vp = page_logical(vs, bs, rng, num_blocks=64, order=order)
    assert np.array_equal(tk, tv)
    q = rng.standard_normal((len(ctxs), Hq, d)).astype(np.float32)
    scale = float(np.float32(1 / math.sqrt(d)))
    out = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=scale)
    for b, c in enumerate(ctxs):
        for h in range(Hq):
            ref = sdpa(q[b, h], ks[b][:, h], vs[b][:, h], scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


def test_decode_gqa_bf16_equals_sdpa_with_repeated_heads():
    """Query head hq reads KV head hq // g: contiguous groups (repeat_interleave)."""
    rng = np.random.default_rng(2)
    ctxs = [5, 40, 64, 77]
    Hq, Hkv, d, bs = 8, 2, 128, 16
    g = Hq // Hkv
    ks = [bf16_bits(x) for x in logical_seqs(rng, ctxs, Hkv, d)]
    vs = [bf16_bits(x) for x in logical_seqs(rng, ctxs, Hkv, d)]
    order = rng.permutation(40)
    tk, kp = page_logical(ks, bs, rng, num_blocks=40, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=40, order=order)
    q = bf16_bits(rng.standard_normal((len(ctxs), Hq, d)))
    scale = float(np.float32(1 / math.sqrt(d)))
    out = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=scale,
                                        q_dtype=oracle.BF16, cache_dtype=oracle.BF16)
    for b, c in enumerate(ctxs):
        K = torch.from_numpy(bf16_value(ks[b])).repeat_interleave(g, dim=1).numpy()
        V = torch.from_numpy(bf16_value(vs[b])).repeat_interleave(g, dim=1).numpy()
        for h in range(Hq):
            ref = sdpa(bf16_value(q[b, h]), K[:, h], V[:, h], scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


def test_decode_fp8_cache_equals_sdpa_on_scaled_codes():
    rng = np.random.default_rng(3)
    ctxs = [3, 31, 48]
    Hq, Hkv, d, bs = 16, 2, 128, 16
    codes = lambda c: rng.integers(0, 256, (c, Hkv, d)).astype(np.uint8)
    ks, vs = [codes(c) for c in ctxs], [codes(c) for c in ctxs]
    for arr in ks + vs:                       # no NaN codes (S.1111.111)
        arr[(arr & 0x7F) == 0x7F] = 0x3F
    order = rng.permutation(12)
    tk, kp = page_logical(ks, bs, rng, num_blocks=12, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=12, order=order)
    kp[(kp & 0x7F) == 0x7F] = 0
    vp[(vp & 0x7F) == 0x7F] = 0
    q = bf16_bits(rng.standard_normal((len(ctxs), Hq, d)))
    k_scale, v_scale = float(np.float32(0.0123)), float(np.float32(0.0456))
    scale = float(np.float32(1 / math.sqrt(d)))
    out = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=scale, q_dtype=oracle.BF16,
                                        cache_dtype=oracle.E4M3, k_scale=k_scale, v_scale=v_scale)
    g = Hq // Hkv
    for b in range(len(ctxs)):
        for h in range(Hq):
            ref = sdpa(bf16_value(q[b, h]), fp8_value(ks[b][:, h // g], k_scale),
                       fp8_value(vs[b][:, h // g], v_scale), scale)
            np.testing.assert_allclose(out[b, h], ref, rtol=1e-12, atol=1e-12)


def test_row_selection_matches_full():
    rng = np.random.default_rng(4)
    ctxs = [9, 50]
    ks, vs = logical_seqs(rng, ctxs, 2, 64), logical_seqs(rng, ctxs, 2, 64)
    order = rng.permutation(10)
    tk, kp = page_logical(ks, 16, rng, num_blocks=10, order=order)
    _, vp = page_logical(vs, 16, rng, num_blocks=10, order=order)
    q = rng.standard_normal((2, 4, 64)).astype(np.float32)
    full = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125)
    rows = np.array([7, 0, 3, 5])
    part = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125, rows=rows)
    assert np.array_equal(part, full.reshape(8, 64)[rows])


# --------------------------------------------------------------------------- #
# closed forms
# --------------------------------------------------------------------------- #

def _single(q, K, V, scale=0.125):
    """Run the oracle on one sequence whose logical K/V are K, V [ctx, 1, d]."""
    rng = np.random.default_rng(0)
    tk, kp = page_logical([K], 16, rng, num_blocks=8)
    vp = np.zeros_like(kp)                       # same placement for V
    for t in range(K.shape[0]):
        vp[tk[0, t // 16], t % 16] = V[t]
    return oracle.paged_attention_decode(q[None, None, :], kp, vp, tk, np.array([K.shape[0]], np.int32),
                                         scale=scale)[0, 0]


def test_ctx1_returns_v0_exactly():
    rng = np.random.default_rng(5)
    K = rng.standard_normal((1, 1, 64)).astype(np.float32)
    V = rng.standard_normal((1, 1, 64)).astype(np.float32)
    out = _single(rng.standard_normal(64).astype(np.float32), K, V)
    assert np.array_equal(out, V[0, 0].astype(np.float64))


def test_zero_query_gives_mean_of_v():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((37, 1, 64)).astype(np.float32)
    V = rng.standard_normal((37, 1, 64)).astype(np.float32)
    out = _single(np.zeros(64, np.float32), K, V)
    np.testing.assert_allclose(out, V[:, 0].astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)


def test_equal_keys_give_mean_of_v():
    rng = np.random.default_rng(7)
    K = np.repeat(rng.standard_normal((1, 1, 64)).astype(np.float32), 23, axis=0)
    V = rng.standard_normal((23, 1, 64)).astype(np.float32)
    out = _single(rng.standard_normal(64).astype(np.float32), K, V)
    np.testing.assert_allclose(out, V[:, 0].astype(np.float64).mean(0), rtol=1e-13, atol=1e-14)


def test_dominant_logit_selects_its_value_row():
    rng = np.random.default_rng(8)
    d = 64
    q = np.zeros(d, np.float32)
    q[0] = 1.0
    K = np.zeros((30, 1, d), np.float32)
    K[17, 0, 0] = 1000.0          # logit 0.125 * 1000 = 125 above every other (0)
    V = rng.standard_normal((30, 1, d)).astype(np.float32)
    out = _single(q, K, V)
    np.testing.assert_allclose(out, V[17, 0].astype(np.float64), rtol=0, atol=1e-12)  # others weigh e^-125


def test_empty_context_gives_zeros():
    kp = np.ones((2, 16, 1, 64), np.float32)
    out = oracle.paged_attention_decode(np.ones((1, 1, 64), np.float32), kp, kp, np.zeros((1, 1), np.int32),
                                        np.array([0], np.int32), scale=0.125)
    assert np.array_equal(out, np.zeros((1, 1, 64)))


# --------------------------------------------------------------------------- #
# invariances the pages state
# --------------------------------------------------------------------------- #

def test_physical_placement_invariance():
    """Physical blocks may sit anywhere in the pool, in any order
    (分页搬进 GPU KV cache, 核心要点 间接寻址)."""
    rng = np.random.default_rng(9)
    ctxs = [70, 3, 128, 45]
    ks, vs = logical_seqs(rng, ctxs, 2, 64), logical_seqs(rng, ctxs, 2, 64)
    q = rng.standard_normal((4, 2, 64)).astype(np.float32)
    outs = []
    for trial in range(3):
        order = rng.permutation(30)
        tk, kp = page_logical(ks, 16, rng, num_blocks=30, order=order)
        _, vp = page_logical(vs, 16, rng, num_blocks=30, order=order)
        outs.append(oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_block_size_invariance():
    """block_size is a free parameter (16 default, 8 / 32 alternatives)."""
    rng = np.random.default_rng(10)
    ctxs = [70, 3, 128, 45, 16, 17]
    ks, vs = logical_seqs(rng, ctxs, 2, 64), logical_seqs(rng, ctxs, 2, 64)
    q = rng.standard_normal((len(ctxs), 4, 64)).astype(np.float32)
    outs = []
    for bs in (8, 16, 32):
        nb = sum(-(-c // bs) for c in ctxs) + 5
        order = rng.permutation(nb)
        tk, kp = page_logical(ks, bs, rng, num_blocks=nb, order=order)
        _, vp = page_logical(vs, bs, rng, num_blocks=nb, order=order)
        outs.append(oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125))
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])


def test_shared_blocks_equal_private_copies():
    """n candidates sharing a prompt's blocks (ref_count n) read the same
    values as n private copies (分页搬进 GPU KV cache, 实践案例 2)."""
    rng = np.random.default_rng(11)
    n, plen, bs, Hkv, d = 4, 40, 16, 2, 64
    prompt_k = rng.standard_normal((plen, Hkv, d)).astype(np.float32)
    prompt_v = rng.standard_normal((plen, Hkv, d)).astype(np.float32)
    tails = [rng.integers(1, 20) for _ in range(n)]
    # private: every candidate owns a full copy
    ks = [np.concatenate([prompt_k, rng.standard_normal((t, Hkv, d)).astype(np.float32)]) for t in tails]
    vs = [np.concatenate([prompt_v, rng.standard_normal((t, Hkv, d)).astype(np.float32)]) for t in tails]
    ctxs = [plen + t for t in tails]
    q = rng.standard_normal((n, Hkv, d)).astype(np.float32)
    order = rng.permutation(40)
    tk, kp = page_logical(ks, bs, rng, num_blocks=40, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=40, order=order)
    private = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125)
    # shared: the two full prompt blocks of candidates 1..n-1 point at candidate 0's
    shared_t = tk.copy()
    full = plen // bs
    for c in range(1, n):
        shared_t[c, :full] = tk[0, :full]
    shared = oracle.paged_attention_decode(q, kp, vp, shared_t, np.array(ctxs, np.int32), scale=0.125)
    assert np.array_equal(private, shared)


def test_gqa_equals_mha_with_repeated_kv_heads():
    rng = np.random.default_rng(12)
    ctxs = [19, 64, 5]
    Hq, Hkv, d, bs = 8, 2, 64, 16
    ks, vs = logical_seqs(rng, ctxs, Hkv, d), logical_seqs(rng, ctxs, Hkv, d)
    q = rng.standard_normal((3, Hq, d)).astype(np.float32)
    order = rng.permutation(12)
    tk, kp = page_logical(ks, bs, rng, num_blocks=12, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=12, order=order)
    gqa = oracle.paged_attention_decode(q, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125)
    kr = np.repeat(kp, Hq // Hkv, axis=2)
    vr = np.repeat(vp, Hq // Hkv, axis=2)
    mha = oracle.paged_attention_decode(q, kr, vr, tk, np.array(ctxs, np.int32), scale=0.125)
    assert np.array_equal(gqa, mha)


# --------------------------------------------------------------------------- #
# split-context partials and their merge
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("ptok,nparts", [(640, 1), (320, 2), (96, 7), (10, 64)])
def test_partition_merge_reproduces_single_pass(ptok, nparts):
    rng = np.random.default_rng(13)
    ctxs = [640, 1, 333]
    ks, vs = logical_seqs(rng, ctxs, 2, 64), logical_seqs(rng, ctxs, 2, 64)
    order = rng.permutation(70)
    tk, kp = page_logical(ks, 16, rng, num_blocks=70, order=order)
    _, vp = page_logical(vs, 16, rng, num_blocks=70, order=order)
    q = (3 * rng.standard_normal((3, 4, 64))).astype(np.float32)
    cl = np.array(ctxs, np.int32)
    single = oracle.paged_attention_decode(q, kp, vp, tk, cl, scale=0.125)
    m, l, o = oracle.decode_partials(q, kp, vp, tk, cl, scale=0.125, partition_tokens=ptok, max_partitions=nparts)
    assert -(-640 // ptok) == nparts
    merged = oracle.merge_partials(m.reshape(12, nparts), l.reshape(12, nparts), o.reshape(12, nparts, 64))
    np.testing.assert_allclose(merged.reshape(3, 4, 64), single, rtol=1e-12, atol=1e-12)
    # each partial is dense attention over its own token range
    g = 2
    for p in range(nparts):
        t0, t1 = p * ptok, min((p + 1) * ptok, ctxs[0])
        ref = sdpa(q[0, 3], ks[0][t0:t1, 3 // g], vs[0][t0:t1, 3 // g], 0.125)
        np.testing.assert_allclose(o[0, 3, p], ref, rtol=1e-12, atol=1e-12)


def test_partials_past_context_are_empty():
    rng = np.random.default_rng(14)
    ks, vs = logical_seqs(rng, [20], 1, 64), logical_seqs(rng, [20], 1, 64)
    tk, kp = page_logical(ks, 16, rng, num_blocks=4, order=np.arange(4))
    _, vp = page_logical(vs, 16, rng, num_blocks=4, order=np.arange(4))
    q = rng.standard_normal((1, 1, 64)).astype(np.float32)
    m, l, o = oracle.decode_partials(q, kp, vp, tk, np.array([20], np.int32), scale=0.125, partition_tokens=16,
                                     max_partitions=4)
    assert np.all(l[0, 0, 2:] == 0) and np.all(np.isneginf(m[0, 0, 2:])) and np.all(o[0, 0, 2:] == 0)
    assert np.all(l[0, 0, :2] >= 1.0)      # the max term contributes e^0 = 1


# --------------------------------------------------------------------------- #
# bf16 / fp8 element formats
# --------------------------------------------------------------------------- #

def test_e4m3_decode_all_codes_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = fp8_value(codes)
    mine = np.array([oracle.e4m3_to_double(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert nan.sum() == 2                         # S.1111.111 only
    assert np.array_equal(mine[~nan], ref[~nan])
    assert mine[0x7E] == 448.0 and mine[0x01] == 2.0 ** -9


def test_e4m3_roundtrip_every_code():
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        assert oracle.e4m3_from_float(np.float32(oracle.e4m3_to_double(c))) == c


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(15)
    parts = [rng.standard_normal(400_000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)]
    codes = np.arange(256, dtype=np.uint8)
    vals = np.sort(np.unique(fp8_value(codes)[~np.isnan(fp8_value(codes))]))
    mids = (vals[1:] + vals[:-1]) / 2        # exact ties: must go to the even code
    ulp = np.float32(1e-6)
    x = np.concatenate(parts + [mids, mids * (1 + ulp), mids * (1 - ulp), vals]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    mine = oracle.e4m3_encode_array(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)
    # ties really land on even mantissas
    tie_codes = oracle.e4m3_encode_array(mids.astype(np.float32))
    assert np.all((tie_codes & 1) == 0)


def _e4m3_nearest_lib():
    """tests/native/e4m3_nearest.c, built against the oracle library."""
    import ctypes
    import os
    import subprocess
    import tempfile
    here = os.path.dirname(os.path.abspath(__file__))
    lib = oracle.build()
    out = os.path.join(tempfile.mkdtemp(prefix="e4m3_"), "libe4m3_nearest.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", out,
                    os.path.join(here, "native", "e4m3_nearest.c"), lib, "-Wl,-rpath," + os.path.dirname(lib), "-lm"],
                   check=True)
    so = ctypes.CDLL(out)
    so.e4m3_mismatches.restype = ctypes.c_int64
    so.e4m3_mismatches.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint32)]
    return so


def test_e4m3_encoder_matches_nearest_code_search_on_every_fp32_pattern():
    """All 2^32 fp32 bit patterns: the oracle's arithmetic RNE-satfinite
    encoder equals a nearest-representable search over the 127 finite
    magnitudes built from the format definition (ties to the even code)."""
    import ctypes
    so = _e4m3_nearest_lib()
    first = ctypes.c_uint32(0)
    bad = so.e4m3_mismatches(0, 1 << 32, ctypes.byref(first))
    assert bad == 0, f"{bad} mismatches, first at bit pattern {first.value:#010x}"


def test_e4m3_saturates_instead_of_nan():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, np.inf, -np.inf, -1000.0], np.float32)
    assert list(oracle.e4m3_encode_array(x)) == [0x7E] * 7 + [0xFE, 0xFE]


# --------------------------------------------------------------------------- #
# new-token KV write and copy-on-write block copy (byte level)
# --------------------------------------------------------------------------- #

def test_kv_write_scatter_is_bit_exact_and_touches_nothing_else():
    rng = np.random.default_rng(16)
    NB, bs, Hkv, d, T = 9, 16, 3, 64, 12
    kc = bf16_bits(rng.standard_normal((NB, bs, Hkv, d)))
    vc = bf16_bits(rng.standard_normal((NB, bs, Hkv, d)))
    k = bf16_bits(rng.standard_normal((T, Hkv, d)))
    v = bf16_bits(rng.standard_normal((T, Hkv, d)))
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    slots[3] = -1                                # padding token: skipped
    k0, v0 = kc.copy(), vc.copy()
    oracle.paged_kv_write(k, v, slots, kc, vc, in_dtype=oracle.BF16, cache_dtype=oracle.BF16)
    ek, ev = k0.copy(), v0.copy()
    for t, s in enumerate(slots):
        if s >= 0:
            ek[s // bs, s % bs] = k[t]
            ev[s // bs, s % bs] = v[t]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


def test_kv_write_fp8_codes_match_torch_cast_of_scaled_values():
    rng = np.random.default_rng(17)
    NB, bs, Hkv, d, T = 4, 16, 2, 128, 10
    k = bf16_bits(rng.standard_normal((T, Hkv, d)) * 3)
    v = bf16_bits(rng.standard_normal((T, Hkv, d)))
    kc = np.zeros((NB, bs, Hkv, d), np.uint8)
    vc = np.zeros((NB, bs, Hkv, d), np.uint8)
    slots = rng.choice(NB * bs, T, replace=False).astype(np.int64)
    k_scale, v_scale = np.float32(0.037), np.float32(0.011)
    oracle.paged_kv_write(k, v, slots, kc, vc, in_dtype=oracle.BF16, cache_dtype=oracle.E4M3,
                          k_scale=float(k_scale), v_scale=float(v_scale))
    for src, cache, sc in ((k, kc, k_scale), (v, vc, v_scale)):
        x = torch.from_numpy(src.view(np.int16)).view(torch.bfloat16).float()
        prod = (x * torch.tensor(np.float32(1.0) / sc)).numpy()        # one fp32 multiply
        # torch's cast gives NaN past 448 where the stored format saturates; clip first
        ref = torch.from_numpy(np.clip(prod, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        for t, s in enumerate(slots):
            assert np.array_equal(cache[s // bs, s % bs], ref[t])


def test_kv_write_rejects_slot_past_pool_and_writes_nothing():
    kc = np.zeros((2, 16, 1, 64), np.float32)
    vc = np.zeros_like(kc)
    k = np.ones((2, 1, 64), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.paged_kv_write(k, k, np.array([0, 32], np.int64), kc, vc)
    assert not kc.any() and not vc.any()


def test_block_copy_bytes_and_untouched_blocks():
    rng = np.random.default_rng(18)
    kc = rng.integers(0, 256, (10, 16, 2, 64)).astype(np.uint8)
    vc = rng.integers(0, 256, (10, 16, 2, 64)).astype(np.uint8)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 7], [1, 8], [4, 2]], np.int64)
    oracle.kv_block_copy(pairs, kc, vc)
    ek, ev = k0.copy(), v0.copy()
    for s, d in pairs:
        ek[d], ev[d] = k0[s], v0[s]
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


@pytest.mark.parametrize("pairs", [[[1, 7], [2, 7]], [[1, 7], [7, 3]], [[3, 3]], [[0, 10]], [[-1, 2]]])
def test_block_copy_rejects_order_dependent_or_out_of_range_pairs(pairs):
    kc = np.zeros((10, 16, 1, 64), np.uint8)
    with pytest.raises(oracle.OracleError):
        oracle.kv_block_copy(np.array(pairs, np.int64), kc, kc.copy())


def test_decode_rejects_out_of_range_block_id_and_context():
    kp = np.zeros((4, 16, 1, 64), np.float32)
    q = np.zeros((1, 1, 64), np.float32)
    with pytest.raises(oracle.OracleError):
        oracle.paged_attention_decode(q, kp, kp, np.array([[4]], np.int32), np.array([3], np.int32), scale=1.0)
    with pytest.raises(oracle.OracleError):
        oracle.paged_attention_decode(q, kp, kp, np.array([[0]], np.int32), np.array([17], np.int32), scale=1.0)


# --------------------------------------------------------------------------- #
# the pages' printed numbers
# --------------------------------------------------------------------------- #

def test_kv_size_formula_golden():
    from paged_kv_cache_450_b200 import workloads as W
    g = json.load(open(os.path.join(GOLDEN, "kv_size_formula.json")))
    per_tok = W.kv_bytes_per_token(g["num_layers"], g["num_heads"], g["head_dim"], torch.bfloat16)
    assert per_tok == g["bytes_per_token"] == 819200
    assert per_tok * g["tokens_per_sequence"] == g["mib_per_1024_token_sequence"] * 2 ** 20
    # one layer's pool accounting: cache bytes / (blocks x block_size) x layers
    kc = torch.empty((7, 16, 40, 128), dtype=torch.bfloat16)
    assert 2 * kc.nbytes // (7 * 16) * g["num_layers"] == 819200


def test_block_bytes_golden():
    from paged_kv_cache_450_b200 import workloads as W
    g = json.load(open(os.path.join(GOLDEN, "block_bytes.json")))
    dt = {"bf16": torch.bfloat16, "fp8": torch.float8_e4m3fn}
    for c in g["cases"]:
        assert W.block_bytes(c["block_size"], c["num_kv_heads"], c["head_dim"], dt[c["dtype"]]) == c["bytes"]


def test_parallel_sampling_first_step_copies_golden():
    from paged_kv_cache_450_b200 import workloads as W
    g = json.load(open(os.path.join(GOLDEN, "parallel_sampling_cow.json")))
    spec = W.PARALLEL_SAMPLING
    ctx, tables, NB, pairs, info = W._layout_sampling(spec, np.random.default_rng(0))
    prompts = spec.sampling[0]
    assert spec.sampling[1] == g["n"]
    assert info["ref_count_prompt"] == g["prompt_ref_count"]
    assert len(pairs) == prompts * g["copies_per_prompt_first_step"] == 96


def test_swap_blocks_between_pools_byte_exact():
    rng = np.random.default_rng(19)
    dev_k = rng.integers(0, 256, (12, 16, 2, 64)).astype(np.uint8)
    dev_v = rng.integers(0, 256, (12, 16, 2, 64)).astype(np.uint8)
    host_k = rng.integers(0, 256, (5, 16, 2, 64)).astype(np.uint8)
    host_v = rng.integers(0, 256, (5, 16, 2, 64)).astype(np.uint8)
    hk0, hv0 = host_k.copy(), host_v.copy()
    pairs = np.array([[11, 0], [3, 4], [3, 2]], np.int64)     # a source may be copied twice
    oracle.swap_blocks(pairs, dev_k, dev_v, host_k, host_v)
    ek, ev = hk0.copy(), hv0.copy()
    for s_, d_ in pairs:
        ek[d_], ev[d_] = dev_k[s_], dev_v[s_]
    assert np.array_equal(host_k, ek) and np.array_equal(host_v, ev)
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(np.array([[0, 5]]), dev_k, dev_v, host_k, host_v)       # dst past the host pool
    with pytest.raises(oracle.OracleError):
        oracle.swap_blocks(np.array([[0, 1], [2, 1]]), dev_k, dev_v, host_k, host_v)  # repeated destination


def test_fp8_scale_is_amax_over_448():
    rng = np.random.default_rng(20)
    x = rng.standard_normal(1001).astype(np.float32)
    x[417] = -9.75                                   # the largest magnitude is negative
    assert oracle.fp8_scale(x) == np.float32(np.float32(9.75) / np.float32(448.0))
    assert oracle.fp8_scale(np.zeros(10, np.float32)) == 1.0
    b = bf16_bits(x)
    assert oracle.fp8_scale(b, oracle.BF16) == np.float32(np.abs(bf16_value(b)).max().astype(np.float32) / np.float32(448))
    # the scale maps the amax onto the largest finite code
    s = oracle.fp8_scale(x)
    assert oracle.e4m3_from_float(np.float32(np.float32(9.75) * (np.float32(1) / np.float32(s)))) in (0x7E, 0xFE)


# --------------------------------------------------------------------------- #
# multi-query (chunked prefill / verification) attention
# --------------------------------------------------------------------------- #

def test_multiquery_equals_sdpa_with_bottom_right_causal_mask():
    rng = np.random.default_rng(21)
    ctxs, qlens = [9, 40, 100, 17], [3, 40, 7, 1]
    Hq, Hkv, d, bs = 4, 2, 64, 16
    ks, vs = logical_seqs(rng, ctxs, Hkv, d), logical_seqs(rng, ctxs, Hkv, d)
    order = rng.permutation(20)
    tk, kp = page_logical(ks, bs, rng, num_blocks=20, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=20, order=order)
    qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = rng.standard_normal((int(qsl[-1]), Hq, d)).astype(np.float32)
    out = oracle.paged_attention_multiquery(q, qsl, kp, vp, tk, np.array(ctxs, np.int32), scale=0.125)
    g = Hq // Hkv
    for b, (c, n) in enumerate(zip(ctxs, qlens)):
        qb = torch.from_numpy(q[qsl[b]:qsl[b + 1]].astype(np.float64)).permute(1, 0, 2)        # [Hq, n, d]
        kb = torch.from_numpy(ks[b].astype(np.float64)).repeat_interleave(g, 1).permute(1, 0, 2)  # [Hq, c, d]
        vb = torch.from_numpy(vs[b].astype(np.float64)).repeat_interleave(g, 1).permute(1, 0, 2)
        # query i (position c - n + i) sees keys 0 .. c - n + i: a bottom-right aligned causal mask
        mask = torch.arange(c)[None, :] <= (c - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=0.125)
        np.testing.assert_allclose(out[qsl[b]:qsl[b + 1]], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


def test_multiquery_queries_before_the_context_get_zero_rows():
    """More queries than context tokens: the first q_len - ctx queries sit at
    negative positions, see no key and give zero rows; the rest equal a pass
    over only the queries with a position."""
    rng = np.random.default_rng(24)
    ks, vs = logical_seqs(rng, [3], 1, 64), logical_seqs(rng, [3], 1, 64)
    tk, kp = page_logical(ks, 16, rng, num_blocks=2, order=np.array([1, 0]))
    vp = np.zeros_like(kp)
    vp[tk[0, 0], :3] = vs[0]
    q = rng.standard_normal((5, 2, 64)).astype(np.float32)
    cl = np.array([3], np.int32)
    out = oracle.paged_attention_multiquery(q, np.array([0, 5], np.int32), kp, vp, tk, cl, scale=0.125)
    assert np.all(out[:2] == 0.0)
    tail = oracle.paged_attention_multiquery(q[2:], np.array([0, 3], np.int32), kp, vp, tk, cl, scale=0.125)
    assert np.array_equal(out[2:], tail)


def test_multiquery_equals_python_double_loop_brute_force():
    """Tiny causal cases against plain Python: for query i of a sequence with
    q_len queries and context c, the keys 0 .. c - q_len + i, scores, max,
    math.exp and the weighted sum written out element by element."""
    rng = np.random.default_rng(31)
    for trial in range(5):
        B, Hkv, g, d, bs = int(rng.integers(1, 4)), int(rng.integers(1, 3)), int(rng.choice([1, 2])), 8, 4
        Hq = Hkv * g
        ctxs = [int(c) for c in rng.integers(1, 30, B)]
        qlens = [int(rng.integers(0, c + 1)) for c in ctxs]
        ks, vs = logical_seqs(rng, ctxs, Hkv, d), logical_seqs(rng, ctxs, Hkv, d)
        nb = sum(-(-c // bs) for c in ctxs) + 2
        order = rng.permutation(nb)
        tk, kp = page_logical(ks, bs, rng, num_blocks=nb, order=order)
        _, vp = page_logical(vs, bs, rng, num_blocks=nb, order=order)
        qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
        q = rng.standard_normal((int(qsl[-1]), Hq, d)).astype(np.float32)
        scale = float(np.float32(0.25))
        out = oracle.paged_attention_multiquery(q, qsl, kp, vp, tk, np.array(ctxs, np.int32), scale=scale)
        for b in range(B):
            for i in range(qlens[b]):
                pos = ctxs[b] - qlens[b] + i
                for h in range(Hq):
                    rows_k, rows_v = [], []
                    for t in range(pos + 1):
                        blk = int(tk[b, t // bs])
                        rows_k.append([float(x) for x in kp[blk, t % bs, h // g]])
                        rows_v.append([float(x) for x in vp[blk, t % bs, h // g]])
                    qv = [float(x) for x in q[qsl[b] + i, h]]
                    sc = [scale * sum(qv[e] * kr[e] for e in range(d)) for kr in rows_k]
                    mx = max(sc)
                    w = [math.exp(x - mx) for x in sc]
                    ref = [sum(w[t] * rows_v[t][e] for t in range(len(w))) / sum(w) for e in range(d)]
                    assert np.allclose(out[qsl[b] + i, h], ref, rtol=1e-12, atol=1e-12), (trial, b, i, h)


def test_multiquery_with_one_query_per_sequence_is_decode():
    rng = np.random.default_rng(22)
    ctxs = [1, 33, 70]
    ks, vs = logical_seqs(rng, ctxs, 2, 64), logical_seqs(rng, ctxs, 2, 64)
    order = rng.permutation(12)
    tk, kp = page_logical(ks, 16, rng, num_blocks=12, order=order)
    _, vp = page_logical(vs, 16, rng, num_blocks=12, order=order)
    q = rng.standard_normal((3, 8, 64)).astype(np.float32)
    cl = np.array(ctxs, np.int32)
    mq = oracle.paged_attention_multiquery(q, np.arange(4, dtype=np.int32), kp, vp, tk, cl, scale=0.2)
    dec = oracle.paged_attention_decode(q, kp, vp, tk, cl, scale=0.2)
    assert np.array_equal(mq, dec)


def test_multiquery_chunked_prefill_is_consistent():
    """Prefilling a prompt in two chunks (the second chunk's queries see the
    first chunk's keys) gives the same rows as one causal pass."""
    rng = np.random.default_rng(23)
    n = 50
    ks, vs = logical_seqs(rng, [n], 1, 64), logical_seqs(rng, [n], 1, 64)
    tk, kp = page_logical(ks, 16, rng, num_blocks=5, order=rng.permutation(5))
    vp = np.zeros_like(kp)
    for t in range(n):
        vp[tk[0, t // 16], t % 16] = vs[0][t]
    q = rng.standard_normal((n, 1, 64)).astype(np.float32)
    whole = oracle.paged_attention_multiquery(q, np.array([0, n], np.int32), kp, vp, tk, np.array([n], np.int32),
                                              scale=0.125)
    first = oracle.paged_attention_multiquery(q[:30], np.array([0, 30], np.int32), kp, vp, tk,
                                              np.array([30], np.int32), scale=0.125)
    second = oracle.paged_attention_multiquery(q[30:], np.array([0, 20], np.int32), kp, vp, tk,
                                               np.array([n], np.int32), scale=0.125)
    np.testing.assert_allclose(np.concatenate([first, second]), whole, rtol=1e-13, atol=1e-14)


def test_multiquery_fp8_cache_bf16_q_equals_sdpa_on_scaled_codes():
    """Multi-query over E4M3 caches with per-tensor scales and bf16 queries (grouped heads): torch's
    fp64 SDPA, with a bottom-right causal mask, on the codes decoded by torch's own float8_e4m3fn and
    multiplied by their scales, and on the bf16 queries decoded by torch."""
    rng = np.random.default_rng(25)
    ctxs, qlens = [5, 40, 70], [5, 3, 17]
    Hq, Hkv, d, bs = 8, 2, 128, 16
    codes = lambda c: rng.integers(0, 256, (c, Hkv, d)).astype(np.uint8)  # noqa: E731
    ks, vs = [codes(c) for c in ctxs], [codes(c) for c in ctxs]
    for arr in ks + vs:                       # no NaN codes (S.1111.111)
        arr[(arr & 0x7F) == 0x7F] = 0x3F
    order = rng.permutation(12)
    tk, kp = page_logical(ks, bs, rng, num_blocks=12, order=order)
    _, vp = page_logical(vs, bs, rng, num_blocks=12, order=order)
    kp[(kp & 0x7F) == 0x7F] = 0
    vp[(vp & 0x7F) == 0x7F] = 0
    qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = bf16_bits(rng.standard_normal((int(qsl[-1]), Hq, d)))
    k_scale, v_scale = float(np.float32(0.0173)), float(np.float32(0.0391))
    scale = float(np.float32(1 / math.sqrt(d)))
    out = oracle.paged_attention_multiquery(q, qsl, kp, vp, tk, np.array(ctxs, np.int32), scale=scale,
                                            q_dtype=oracle.BF16, cache_dtype=oracle.E4M3, k_scale=k_scale,
                                            v_scale=v_scale)
    g = Hq // Hkv
    for b, (c, n) in enumerate(zip(ctxs, qlens)):
        qb = torch.from_numpy(bf16_value(q[qsl[b]:qsl[b + 1]])).permute(1, 0, 2)                       # [Hq, n, d]
        kb = torch.from_numpy(fp8_value(ks[b], k_scale)).repeat_interleave(g, 1).permute(1, 0, 2)   # [Hq, c, d]
        vb = torch.from_numpy(fp8_value(vs[b], v_scale)).repeat_interleave(g, 1).permute(1, 0, 2)
        mask = torch.arange(c)[None, :] <= (c - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=scale)
        np.testing.assert_allclose(out[qsl[b]:qsl[b + 1]], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)

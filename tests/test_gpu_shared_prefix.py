"""Shared-prefix decode (pkv_paged_attention_decode_shared_prefix) against the oracle.

"vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 2: the candidates of parallel
sampling share their prompt's blocks.  The call reads each shared block once
for the whole group; every output row must still equal plain attention over the
sequence's own table (the oracle knows nothing of groups), and the caches after
the fused new-token write must equal the oracle's byte for byte.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_450_b200 as pk
from paged_kv_cache_450_b200 import workloads as W
from step_helpers import assert_cache_equal, assert_close, oracle_step, sample_rows, to_np, tol_for

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def shared_step(w, partition_tokens=0, validate=True, append=True):
    """Copy-on-write copies, then the shared-prefix decode with the new tokens fused in."""
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    if w.copy_pairs is not None and len(w.copy_pairs):
        pk.kv_block_copy(w.copy_pairs, kc, vc, validate=validate)
    out = pk.paged_attention_decode_shared_prefix(
        w.q, kc, vc, w.block_tables, w.context_lens, w.group_start, w.shared_blocks, w.scale,
        k_new=w.new_k if append else None, v_new=w.new_v if append else None, partition_tokens=partition_tokens,
        validate=validate)
    torch.cuda.synchronize()
    assert pk.device_status(clear=True) == 0
    return kc, vc, out


@pytest.mark.parametrize("bs", [16, 32])
@pytest.mark.parametrize("hq,hkv,n", [(8, 8, 4), (8, 4, 4), (8, 2, 2), (16, 2, 1), (4, 4, 8)],
                         ids=["mha-n4", "g2-n4", "g4-n2", "g8-n1", "mha-n8"])
def test_parallel_sampling_small(bs, hq, hkv, n):
    spec = W.PARALLEL_SAMPLING.with_(name="sp", num_seqs=3 * n, num_q_heads=hq, num_kv_heads=hkv, block_size=bs,
                                     sampling=(3, n, 150, 1, 70))
    w = W.make_decode_workload(spec, seed=bs + hq + n, device=DEV)
    rk, rv, ref = oracle_step(w)
    for pt in (0, bs, 2 * bs, 256):
        kc, vc, out = shared_step(w, partition_tokens=pt)
        assert_cache_equal(kc, rk, f"key_cache pt={pt}")
        assert_cache_equal(vc, rv, f"value_cache pt={pt}")
        assert_close(f64(out), ref, *tol_for(w), what=f"shared-prefix decode bs={bs} pt={pt}")


def test_parallel_sampling_1020_token_prompt_and_no_append():
    # a partial last prompt block: the copy holds the candidates' tails; and the call without the write
    spec = W.PARALLEL_SAMPLING.with_(name="sp1020", num_seqs=16, num_q_heads=8, num_kv_heads=8,
                                     sampling=(4, 4, 1020, 1, 64))
    w = W.make_decode_workload(spec, seed=5, device=DEV)
    rk, rv, ref = oracle_step(w)
    kc, vc, out = shared_step(w)
    assert_cache_equal(kc, rk, "key_cache")
    assert_close(f64(out), ref, *tol_for(w), what="1020-token prompt")
    # without the new tokens: attention over the cache as it is
    w2 = W.make_decode_workload(spec.with_(new_tokens=False), seed=6, device=DEV)
    _, _, ref2 = oracle_step(w2)
    _, _, out2 = shared_step(w2, append=False)
    assert_close(f64(out2), ref2, *tol_for(w2), what="no append")


def _grouped_tables(rng, group_sizes, bs, num_blocks):
    """Tables where the members of each group share their first S_g blocks (S_g random,
    possibly 0) and then own private blocks; returns (tables, ctxs, group_start, shared)."""
    perm = iter(rng.permutation(num_blocks).tolist())
    rows, ctxs, gs, sh = [], [], [0], []
    for n in group_sizes:
        S = int(rng.integers(0, 9))
        shared_ids = [next(perm) for _ in range(S)]
        for _ in range(n):
            tail = int(rng.integers(0 if S else 1, 3 * bs))
            ctx = S * bs + tail
            own = [next(perm) for _ in range(-(-tail // bs))]
            rows.append(shared_ids + own)
            ctxs.append(ctx)
        gs.append(gs[-1] + n)
        sh.append(S)
    MB = max(1, max(len(r) for r in rows))
    tables = np.zeros((len(rows), MB), np.int32)
    for b, r in enumerate(rows):
        tables[b, :len(r)] = r
    return tables, np.array(ctxs, np.int32), np.array(gs, np.int32), np.array(sh, np.int32)


@pytest.mark.parametrize("seed", range(8))
def test_random_group_structures(seed):
    """Seeded random groupings: group sizes up to 8 / G members (singletons included), 0 to 8 shared
    blocks, empty tails, block size 16 / 32, several partition lengths."""
    rng = np.random.default_rng(700 + seed)
    g = int(rng.choice([1, 2, 4, 8]))
    hkv = int(rng.choice([1, 2, 4]))
    bs = int(rng.choice([16, 32]))
    sizes = [int(x) for x in rng.integers(1, 8 // g + 1, int(rng.integers(1, 7)))]
    B = sum(sizes)
    tables, ctxs, gs, sh = _grouped_tables(rng, sizes, bs, num_blocks=B * 12 + 16)
    spec = W.DecodeSpec("grp", B, hkv * g, hkv, 128, bs, torch.bfloat16, torch.bfloat16,
                        ("list", tuple(int(c) for c in ctxs)), ("fixed", B * 12 + 16), new_tokens=False)
    w = W.make_decode_workload(spec, seed=800 + seed, device=DEV)
    w.block_tables = torch.from_numpy(tables).to(DEV)
    w.group_start = torch.from_numpy(gs).to(DEV)
    w.shared_blocks = torch.from_numpy(sh).to(DEV)
    _, _, ref = oracle_step(w)
    for pt in (0, bs, 4 * bs):
        out = pk.paged_attention_decode_shared_prefix(w.q, w.key_cache, w.value_cache, w.block_tables,
                                                      w.context_lens, w.group_start, w.shared_blocks, w.scale,
                                                      partition_tokens=pt, validate=True)
        torch.cuda.synchronize()
        assert pk.device_status(clear=True) == 0
        assert_close(f64(out), ref, *tol_for(w), what=f"seed={seed} g={g} bs={bs} sizes={sizes} pt={pt}")


def test_full_size_parallel_sampling_sampled():
    w = W.make_decode_workload(W.PARALLEL_SAMPLING, seed=0, device=DEV)
    rows = sample_rows(w, 512, seed=0)
    rk, rv, ref = oracle_step(w, rows=rows)
    kc, vc, out = shared_step(w)
    assert_cache_equal(kc, rk, "key_cache")
    assert_cache_equal(vc, rv, "value_cache")
    assert_close(f64(out).reshape(-1, 128)[rows], ref, *tol_for(w), what="parallel sampling, full size")
    # and the plain decode over the same bytes agrees within the same bound
    plain = pk.paged_attention_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
    torch.cuda.synchronize()
    assert_close(f64(out), f64(plain), *tol_for(w), what="shared-prefix vs plain decode")


def test_validate_rejects_wrong_groupings():
    spec = W.PARALLEL_SAMPLING.with_(name="spbad", num_seqs=8, num_q_heads=8, num_kv_heads=8,
                                     sampling=(2, 4, 150, 1, 40))
    w = W.make_decode_workload(spec, seed=9, device=DEV)

    def call(tables=None, gs=None, sh=None, max_group=None, append=True):
        return pk.paged_attention_decode_shared_prefix(
            w.q, w.key_cache.clone(), w.value_cache.clone(), tables if tables is not None else w.block_tables,
            w.context_lens, gs if gs is not None else w.group_start, sh if sh is not None else w.shared_blocks,
            w.scale, k_new=w.new_k if append else None, v_new=w.new_v if append else None,
            max_group_size=max_group, validate=True)

    n0 = pk.launch_count()
    bad = w.block_tables.clone()
    bad[1, 2] = bad[0, 2] + 1 if int(bad[0, 2]) + 1 < w.num_blocks else 0   # a member disagrees in the prefix
    with pytest.raises(pk.PagedKVError):
        call(tables=bad)
    with pytest.raises(pk.PagedKVError):                    # groups do not cover every sequence
        call(gs=torch.tensor([0, 4, 7], dtype=torch.int32, device=DEV))
    too_far = w.shared_blocks.clone()
    too_far[0] = int(w.context_lens[:4].min()) // 16 + 1      # past a member's context
    with pytest.raises(pk.PagedKVError):
        call(sh=too_far)
    with pytest.raises(pk.PagedKVError):                    # 4 members x 8 heads > 8 columns: refused outright
        pk.paged_attention_decode_shared_prefix(
            torch.zeros(8, 32, 128, dtype=torch.bfloat16, device=DEV), w.key_cache, w.value_cache, w.block_tables,
            w.context_lens, w.group_start, w.shared_blocks, w.scale, max_group_size=4)
    assert pk.launch_count() == n0


def test_kernel_skips_a_group_past_the_batch():
    """Without validate, a group whose members run past num_seqs reaches the kernel: its shared unit
    reads and writes nothing and sets the status bit; the other group is computed as usual."""
    spec = W.PARALLEL_SAMPLING.with_(name="spguard", num_seqs=8, num_q_heads=8, num_kv_heads=8,
                                     sampling=(2, 4, 150, 1, 40), new_tokens=False)
    w = W.make_decode_workload(spec, seed=10, device=DEV)
    _, _, ref = oracle_step(w)
    kc, vc = w.key_cache.clone(), w.value_cache.clone()
    pk.kv_block_copy(w.copy_pairs, kc, vc)   # the copy-on-write copies the oracle applies too
    bad = torch.tensor([0, 4, 9], dtype=torch.int32, device=DEV)
    pk.device_status(clear=True)
    out = pk.paged_attention_decode_shared_prefix(w.q, kc, vc, w.block_tables, w.context_lens, bad, w.shared_blocks,
                                                  w.scale, max_group_size=4)
    torch.cuda.synchronize()
    assert pk.device_status(clear=True) & pk.STATUS_BAD_GROUP
    assert_close(f64(out)[:4], ref[:4], *tol_for(w), what="the well-formed group")


@pytest.mark.parametrize("depth", [1, 2])
def test_shared_prefix_host_step_pipeline(depth):
    """pkv_decode_step_host_shared_prefix_async through SharedPrefixHostStepPipeline: host inputs
    copied in, the copy-on-write copies, the shared-prefix decode with the new tokens fused in, the
    output copied out -- every step equal to the device-side calls on the same inputs; one step's
    caches equal to the oracle's and its output within tolerance of it."""
    spec = W.PARALLEL_SAMPLING.with_(name="sph", num_seqs=12, num_q_heads=8, num_kv_heads=4,
                                     sampling=(3, 4, 150, 1, 70))
    w = W.make_decode_workload(spec, seed=23, device=DEV)
    pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
    host = {k: pin(getattr(w, k)) for k in ("new_k", "new_v", "block_tables", "context_lens", "group_start",
                                            "shared_blocks", "copy_pairs")}
    max_group = int((w.group_start[1:] - w.group_start[:-1]).max().item())
    steps = 4
    g = torch.Generator(device="cpu").manual_seed(23)
    qs = [torch.randn(w.q.shape, generator=g).to(w.q.dtype).pin_memory() for _ in range(steps)]
    kc_h, vc_h = w.key_cache.clone(), w.value_cache.clone()
    pipe = pk.SharedPrefixHostStepPipeline(qs[0], kc_h, host["block_tables"], host["group_start"],
                                           host["copy_pairs"], depth=depth)
    got = []
    for i in range(steps):
        pipe.step(qs[i], host["new_k"], host["new_v"], host["block_tables"], host["context_lens"],
                  host["group_start"], host["shared_blocks"], kc_h, vc_h, w.scale, max_group_size=max_group,
                  copy_pairs=host["copy_pairs"])
        if i >= depth - 1:
            j = i - depth + 1
            pipe.done[j % depth].synchronize()
            got.append(pipe.outs[j % depth].clone())
    pipe.synchronize()
    for j in range(steps - depth + 1, steps):
        got.append(pipe.outs[j % depth].clone())
    assert pk.device_status(clear=True) == 0
    # the same steps on the device (the copies and the write are idempotent, only q changes)
    kc_d, vc_d = w.key_cache.clone(), w.value_cache.clone()
    for i in range(steps):
        pk.kv_block_copy(w.copy_pairs, kc_d, vc_d)
        ref = pk.paged_attention_decode_shared_prefix(qs[i].to(DEV), kc_d, vc_d, w.block_tables, w.context_lens,
                                                      w.group_start, w.shared_blocks, w.scale, k_new=w.new_k,
                                                      v_new=w.new_v, max_group_size=max_group)
        torch.cuda.synchronize()
        assert torch.equal(got[i], ref.cpu()), f"step {i}"
    assert torch.equal(kc_h, kc_d) and torch.equal(vc_h, vc_d)
    # one step on fresh caches against the oracle (repeated steps are not idempotent: a candidate that
    # writes into the block the others copy changes what the next step's copies carry)
    kc1, vc1 = w.key_cache.clone(), w.value_cache.clone()
    out1, done1 = pipe.step(qs[0], host["new_k"], host["new_v"], host["block_tables"], host["context_lens"],
                            host["group_start"], host["shared_blocks"], kc1, vc1, w.scale,
                            max_group_size=max_group, copy_pairs=host["copy_pairs"])
    done1.synchronize()
    w.q = qs[0].to(DEV)
    rk, rv, oref = oracle_step(w)
    assert_cache_equal(kc1, rk, "host-step key_cache")
    assert_cache_equal(vc1, rv, "host-step value_cache")
    assert_close(f64(out1), oref, *tol_for(w), what="shared-prefix host step")

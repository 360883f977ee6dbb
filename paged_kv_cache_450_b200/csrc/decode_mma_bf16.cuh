// decode_mma_bf16.cuh -- paged decode attention on the tensor cores for bf16
// caches (head_dim 128, 1/2/4/8 query heads per KV head).
//
// Same structure as the fp8 kernel (decode_mma.cuh): one warp per CTA, a
// pipeline of TMA stages, software-pipelined 16-token tiles, reference-max
// online softmax, epilogue from registers.  Per tile:
//
//   S = K_tile . Q^T  : M = 16 tokens, N = 8 heads (G real, the rest zero), 8 MMAs
//   O^T += V^T . P^T  : M = 128 dims (8 tiles), N = 8 heads, K = 16 tokens, 16 MMAs
//
// bf16 needs no conversion: the A operands come straight from shared memory
// with ldmatrix (K rows as stored; V through ldmatrix.trans, which delivers
// V^T), and q is the B operand of S as stored.  The tiles arrive through TMA
// as two 128-byte half rows (dims 0..63 and 64..127) with the 128-byte
// swizzle, which makes every ldmatrix phase bank-conflict free.  The
// probabilities are split into bf16 hi + lo parts (two MMAs per output tile)
// so P.V keeps ~16 bits of each weight, like an fp16 operand would.
//
// For MHA the N = 8 columns carry one real head: the tensor pipe does 8x the
// needed multiply-adds, which costs nothing here (the kernel is bound by
// HBM and the pipe is otherwise idle) and removes the shuffles and the
// per-element widening of the CUDA-core kernel.
//
// Shared-prefix mode (GROUPED, pkv_paged_attention_decode_shared_prefix):
// sequences come in groups of consecutive members whose first
// shared_blocks[g] logical blocks are the same physical blocks (the n
// candidates of parallel sampling share their prompt's blocks, ref_count n:
// "vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 2).  Grid z < num_groups
// is a shared unit: the queries of all members (members x G <= 8 columns) over
// the group's shared blocks, read once; grid z >= num_groups is sequence
// z - num_groups over its own blocks past the shared prefix (the fused append
// included).  Every unit writes partials; the merge combines a sequence's
// shared and own partials by the softmax identity.
#pragma once

#include "decode.cuh"
#include "decode_mma.cuh"

namespace pkv {

template <int BS, int NS_ = 0>
struct MmaBf16Traits {
  static constexpr int D = 128;
  static constexpr int HALF_BYTES = BS * 128;        // BS rows x 64 bf16 (one TMA box)
  static constexpr int TILE_BYTES = 2 * HALF_BYTES;  // a K or V tile: two half rows
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NS_ > 0 ? NS_ : 3;
  static constexpr int NT = BS / 16;
  static constexpr int STAGE_AREA = NS * STAGE_BYTES;
  static constexpr int BAR_BYTES = NS * 8;
  static constexpr int MIN_BLOCKS = 8;
  static_assert(BS == 16 || BS == 32, "16-token MMA tiles");
  static constexpr size_t smem_bytes(int pb) {
    return 1024 + STAGE_AREA + BAR_BYTES + static_cast<size_t>(pb) * 4;
  }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D(16x8, f32) += A(16x16, bf16, row) . B(16x8, bf16, col)
__device__ __forceinline__ void mma_16816_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16x2 {lo, hi} of two floats (round to nearest even), and the residuals
// x - bf16(x) as a second bf16x2: hi + lo carries ~16 significant bits.
__device__ __forceinline__ void bf16x2_split(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int BS, int G, bool GROUPED = false, int NS = 0, int MINB = MmaBf16Traits<BS, NS>::MIN_BLOCKS>
__global__ void __launch_bounds__(32, MINB)
    paged_decode_mma_bf16_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                                 const DecodeParams p) {
  using T = MmaBf16Traits<BS, NS>;
  constexpr int D = T::D;
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "query heads per KV head");
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(data + T::STAGE_AREA);
  int* ids = reinterpret_cast<int*>(data + T::STAGE_AREA + T::BAR_BYTES);

  const int hk = blockIdx.x, part = blockIdx.y;
  const int lane = threadIdx.x;
  const int r = lane >> 2, c = lane & 3;
  const int max_ctx = p.max_blocks_per_seq * BS;
  const int pb = p.partition_blocks;
  const int Hq = p.num_q_heads;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  // This CTA's unit: table row b, blocks [blk0, blk0 + nb) of it, `cols` real
  // MMA columns (query rows), column j being q / out row row_of(j), partial
  // slot slot0 + part; ctx_eff = the tokens of the table row that count.
  int b, ctx, ctx_eff, nparts, blk0, nb, cols, slot0 = 0;
  int64_t row_first, member_stride = 0;  // row_of(j) = row_first + (j / G) * member_stride + j % G
  bool append;
  if constexpr (GROUPED) {
    const int z = blockIdx.z;
    if (z < p.num_groups) {  // the group's shared prefix, all members at once
      const int b0 = p.group_start[z], n = p.group_start[z + 1] - b0;
      if (b0 < 0 || n < 1 || n * G > 8 || b0 + n > p.num_seqs) {  // before any load or store
        if (lane == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_GROUP);
        return;
      }
      b = b0;
      const int sh = shared_blocks_of(p, z, p.max_blocks_per_seq);
      cols = n * G;
      ctx = ctx_eff = sh * BS;
      nparts = (sh + pb - 1) / pb;
      if (part >= nparts) return;
      blk0 = part * pb;
      nb = min(pb, sh - blk0);
      row_first = static_cast<int64_t>(b0) * Hq + hk * G;
      member_stride = Hq;
      append = false;
    } else {  // the sequence's own blocks past its group's shared prefix
      b = z - p.num_groups;
      ctx = p.context_lens[b];
      if (ctx < 0 || ctx > max_ctx) {
        if (lane == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
        ctx = ctx < 0 ? 0 : max_ctx;
      }
      ctx_eff = ctx;
      const int nblk = (ctx + BS - 1) / BS;
      const int sh = shared_blocks_of(p, group_of_sequence(p, b), nblk);
      nparts = (nblk - sh + pb - 1) / pb;
      if (part >= nparts) return;
      blk0 = sh + part * pb;
      nb = min(pb, nblk - blk0);
      cols = G;
      row_first = static_cast<int64_t>(b) * Hq + hk * G;
      slot0 = p.shared_partitions;
      append = p.new_k != nullptr && part == nparts - 1;
    }
  } else {
    b = blockIdx.z;
    ctx = p.context_lens[b];
    if (ctx < 0 || ctx > max_ctx) {
      if (lane == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
      ctx = ctx < 0 ? 0 : max_ctx;
    }
    ctx_eff = ctx;
    const int nblk = (ctx + BS - 1) / BS;
    nparts = (nblk + pb - 1) / pb;
    row_first = static_cast<int64_t>(b) * Hq + hk * G;
    cols = G;
    if (nparts == 0) {
      if (part == 0)
        for (int i = lane; i < G * D; i += 32) out[row_first * D + i] = __float2bfloat16_rn(0.f);
      return;
    }
    if (part >= nparts) return;
    blk0 = part * pb;
    nb = min(pb, nblk - blk0);
    append = p.new_k != nullptr && part == nparts - 1;
  }
  auto row_of = [&](int j) -> int64_t { return row_first + (j / G) * member_stride + j % G; };

  for (int i = lane; i < nb; i += 32) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + blk0 + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  if (append) append_new_token<__nv_bfloat16, __nv_bfloat16, D, BS>(p, b, hk, ctx, lane, 32);
  const uint32_t bar0 = smem_u32(bars);
  if (lane == 0) {
    for (int s = 0; s < T::NS; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
    if (append) fence_proxy_async_global();
  }
  __syncwarp();

  const uint32_t stage0 = smem_u32(data);
  const uint64_t policy = l2_policy_evict_first();
  int n_issued = 0;
  auto issue = [&](int ib) {
    n_issued = ib + 1;
    const int s = ib % T::NS;
    const uint32_t bar = bar0 + 8 * s;
    const int id = ids[ib];
    if (id >= 0) {
      mbar_arrive_expect_tx(bar, T::STAGE_BYTES);
      const uint32_t dst = stage0 + s * T::STAGE_BYTES;  // [K dims 0-63][K 64-127][V 0-63][V 64-127]
      tma_load_4d(dst, &kmap, bar, 0, hk, 0, id, policy);
      tma_load_4d(dst + T::HALF_BYTES, &kmap, bar, 64, hk, 0, id, policy);
      tma_load_4d(dst + T::TILE_BYTES, &vmap, bar, 0, hk, 0, id, policy);
      tma_load_4d(dst + T::TILE_BYTES + T::HALF_BYTES, &vmap, bar, 64, hk, 0, id, policy);
    } else {
      mbar_arrive(bar);
    }
  };
  if (lane == 0) {
    const int pre = nb < T::NS ? nb : T::NS;
    for (int i = 0; i < pre; ++i) issue(i);
  }

  // q (B operand of S) as stored: chunk j, lane (r, c): dims 16j + 2c (+1) and +8 (+9).
  // Columns r >= cols are padding (zero).
  uint32_t qf[8][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) +
                                                             (r < cols ? row_of(r) : 0) * D);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      qf[j][0] = r < cols ? qrow[8 * j + c] : 0u;
      qf[j][1] = r < cols ? qrow[8 * j + c + 4] : 0u;
    }
  }
  const float qk = p.q_scale;

  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[8][4];  // m-tile i: {O[2c][16i+r], O[2c+1][16i+r], O[2c][16i+r+8], O[2c+1][16i+r+8]}
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[i][k] = 0.f;

  // ldmatrix row addresses (byte offsets inside a 16-row half tile), fixed per lane.
  // K (A operand of S, chunk jj of a half): matrix i = lane/8 covers rows 8(i&1).., cols 8(i>>1)..
  // V (A operand of O^T via .trans, m-tile mm of a half): rows (tokens) 8(i>>1).., dims 8(i&1)..
  int koff[4], voff[4];
  {
    const int i = lane >> 3, row_k = (lane & 7) + 8 * (i & 1), tok_v = (lane & 7) + 8 * (i >> 1);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      koff[jj] = row_k * 128 + ((((2 * jj + (i >> 1)) ^ (row_k & 7))) << 4);
      voff[jj] = tok_v * 128 + ((((2 * jj + (i & 1)) ^ (tok_v & 7))) << 4);
    }
  }

  const int n_tiles = nb * T::NT;
  auto tile_k = [&](int u) -> uint32_t {  // K half 0 of tile u (half 1 is HALF_BYTES further)
    return stage0 + ((u / T::NT) % T::NS) * T::STAGE_BYTES + (u % T::NT) * 16 * 128;
  };
  auto tile_valid = [&](int u) -> int {
    const int j = u / T::NT;
    if (ids[j] < 0) return 0;
    const int v = ctx_eff - (blk0 + j) * BS - 16 * (u % T::NT);
    return v < 0 ? 0 : (v > 16 ? 16 : v);
  };
  auto compute_s = [&](int u, float (&sacc)[4]) {
    const uint32_t kt = tile_k(u);
    float s2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 4; ++k) sacc[k] = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(kt + (j >> 2) * T::HALF_BYTES + koff[j & 3], a0, a1, a2, a3);
      mma_16816_bf16((j & 1) ? s2 : sacc, a0, a1, a2, a3, qf[j][0], qf[j][1]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sacc[k] += s2[k];
  };
  int waited = 0;
  bool ok = true;
  auto wait_block = [&](int ib) -> bool {
    if (!mbar_wait_bounded(bar0 + 8 * (ib % T::NS), (ib / T::NS) & 1, p.status)) return false;
    waited = ib + 1;
    return true;
  };

  float sc[4] = {0.f, 0.f, 0.f, 0.f};
  if (n_tiles > 0) {
    if (wait_block(0))
      compute_s(0, sc);
    else
      ok = false;
  }
  for (int u = 0; ok && u < n_tiles; ++u) {
    float sn[4] = {0.f, 0.f, 0.f, 0.f};
    if (u + 1 < n_tiles) {
      if ((u + 1) % T::NT == 0 && !wait_block((u + 1) / T::NT)) {
        ok = false;
        break;
      }
      compute_s(u + 1, sn);
    }
    const int valid = tile_valid(u);
    if (valid > 0) {
      const bool full = valid == 16;
      // S rows r (token r) and r+8 (token r+8), columns heads 2c, 2c+1.
      float s0 = sc[0] * qk, s1 = sc[1] * qk, s2 = sc[2] * qk, s3 = sc[3] * qk;
      if (!full) {
        const bool va = r < valid, vb = r + 8 < valid;
        s0 = va ? s0 : -INFINITY;
        s1 = va ? s1 : -INFINITY;
        s2 = vb ? s2 : -INFINITY;
        s3 = vb ? s3 : -INFINITY;
      }
      const bool over = fmaxf(s0, s2) > m0 + 8.f || fmaxf(s1, s3) > m1 + 8.f;
      if (__any_sync(kFullMask, over)) {
        float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          bm0 = fmaxf(bm0, __shfl_xor_sync(kFullMask, bm0, off));
          bm1 = fmaxf(bm1, __shfl_xor_sync(kFullMask, bm1, off));
        }
        const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
        const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int i3 = 0; i3 < 8; ++i3) {
          o[i3][0] *= al0;
          o[i3][1] *= al1;
          o[i3][2] *= al0;
          o[i3][3] *= al1;
        }
        m0 = mn0;
        m1 = mn1;
      }
      const float p0 = fast_exp2(s0 - m0), p1 = fast_exp2(s1 - m1);
      const float p2 = fast_exp2(s2 - m0), p3 = fast_exp2(s3 - m1);
      l0 += p0 + p2;
      l1 += p1 + p3;
      uint32_t h01, l01, h23, l23;
      bf16x2_split(p0, p1, h01, l01);
      bf16x2_split(p2, p3, h23, l23);
      const uint32_t pbh0 = movmatrix_trans(h01), pbh1 = movmatrix_trans(h23);
      const uint32_t pbl0 = movmatrix_trans(l01), pbl1 = movmatrix_trans(l23);
      // V^T fragments: regs {tokens 2c,2c+1 at dim 16i+r, same at 16i+r+8, tokens 2c+8,2c+9 ...}
      uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;  // zero rows past the context (never NaN)
      if (!full) {
        mlo = (2 * c < valid ? 0x0000ffffu : 0u) | (2 * c + 1 < valid ? 0xffff0000u : 0u);
        mhi = (2 * c + 8 < valid ? 0x0000ffffu : 0u) | (2 * c + 9 < valid ? 0xffff0000u : 0u);
      }
      const uint32_t vt = tile_k(u) + T::TILE_BYTES;
#pragma unroll
      for (int mi = 0; mi < 8; ++mi) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4_trans(vt + (mi >> 2) * T::HALF_BYTES + voff[mi & 3], a0, a1, a2, a3);
        a0 &= mlo;
        a1 &= mlo;
        a2 &= mhi;
        a3 &= mhi;
        mma_16816_bf16(o[mi], a0, a1, a2, a3, pbh0, pbh1);
        mma_16816_bf16(o[mi], a0, a1, a2, a3, pbl0, pbl1);
      }
    }
    if ((u + 1) % T::NT == 0) {
      const int ib = u / T::NT;
      __syncwarp();
      if (lane == 0 && ib + T::NS < nb) {
        fence_proxy_async_smem();
        issue(ib + T::NS);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sc[k] = sn[k];
  }
  if (!ok) {
    const int issued = __shfl_sync(kFullMask, n_issued, 0);
    for (int i = waited; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % T::NS), (i / T::NS) & 1, p.status);
  }

#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(kFullMask, l0, off);
    l1 += __shfl_xor_sync(kFullMask, l1, off);
  }
  const float f0 = l0 > 0.f ? p.out_scale / l0 : 0.f;
  const float f1 = l1 > 0.f ? p.out_scale / l1 : 0.f;
  const int ha = 2 * c, hb = 2 * c + 1;  // this lane's columns (real if < cols)
  if (!GROUPED && nparts == 1) {
#pragma unroll
    for (int mi = 0; mi < 8; ++mi) {
      const int d0 = 16 * mi + r, d1 = d0 + 8;
      if (ha < cols) {
        out[row_of(ha) * D + d0] = __float2bfloat16_rn(o[mi][0] * f0);
        out[row_of(ha) * D + d1] = __float2bfloat16_rn(o[mi][2] * f0);
      }
      if (hb < cols) {
        out[row_of(hb) * D + d0] = __float2bfloat16_rn(o[mi][1] * f1);
        out[row_of(hb) * D + d1] = __float2bfloat16_rn(o[mi][3] * f1);
      }
    }
  } else {
    const int64_t slot_a = (ha < cols ? row_of(ha) : 0) * p.max_partitions + slot0 + part;
    const int64_t slot_b = (hb < cols ? row_of(hb) : 0) * p.max_partitions + slot0 + part;
    const uint64_t keep = l2_policy_evict_last();
#pragma unroll
    for (int mi = 0; mi < 8; ++mi) {
      const int d0 = 16 * mi + r, d1 = d0 + 8;
      if (ha < cols) {
        st_global_hint(p.ws_o + slot_a * D + d0, o[mi][0] * f0, keep);
        st_global_hint(p.ws_o + slot_a * D + d1, o[mi][2] * f0, keep);
      }
      if (hb < cols) {
        st_global_hint(p.ws_o + slot_b * D + d0, o[mi][1] * f1, keep);
        st_global_hint(p.ws_o + slot_b * D + d1, o[mi][3] * f1, keep);
      }
    }
    if (r == 0) {
      if (ha < cols) {
        st_global_hint(p.ws_ml + slot_a * 2, m0 * kLn2, keep);
        st_global_hint(p.ws_ml + slot_a * 2 + 1, l0, keep);
      }
      if (hb < cols) {
        st_global_hint(p.ws_ml + slot_b * 2, m1 * kLn2, keep);
        st_global_hint(p.ws_ml + slot_b * 2 + 1, l1, keep);
      }
    }
  }
}

}  // namespace pkv

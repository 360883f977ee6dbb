// decode_mma.cuh -- paged decode attention on the tensor cores for grouped-query
// attention with an fp8 (E4M3) cache: 8 query heads per KV head, head_dim 128.
//
// With 8 query heads sharing each KV head and one byte per cached element the
// step does 16 flops per byte of KV (2 x 8 heads x (q.K + p.V)); at HBM speed
// that is ~110 TFLOP/s, beyond what fp32 FMAs deliver, so both contractions
// run as mma.sync m16n8k16 (fp16 operands, fp32 accumulation):
//
//   S = K_tile . Q^T  : M = 16 tokens, N = 8 heads, K = 128 dims (8 MMAs)
//   O^T += V^T . P^T  : M = 128 dims (8 tiles), N = 8 heads, K = 16 tokens (8 MMAs)
//
// E4M3 codes are exact in fp16, so K and V are widened in registers with
// cvt.f16x2.e4m3x2 straight into the operand fragments (no dequantisation
// pass, no extra shared-memory traffic); the per-tensor scales are applied to
// the fp32 logits and to the output.  q is rounded once to fp16 (exact for
// bf16 values of magnitude 2^-14 .. 65504, the range of real queries).
//
// Layout tricks (all fixed permutations, checked exhaustively):
// - The K/V tiles arrive through TMA with the 128-byte swizzle: 16-byte chunk
//   q of smem row t sits at chunk q ^ (t & 7).
// - The contraction order over head_dim is permuted so that each thread's
//   four K bytes per MMA are contiguous: k-chunk j, fragment columns
//   {2c, 2c+1, 2c+8, 2c+9} <-> dims 64(j>>2) + 16c + 4(j&3) + {0,1,2,3}.
// - Fragment token row tau reads physical row rho(tau) = tau ^ ((tau & 1) << 2)
//   (and +8), and the P.V output dims are d = 8m + i for m-tile i, row m.
//   With the swizzle these make every K (128-bit) and V (64-bit) shared load
//   bank-conflict free.
// - S comes out as [token][head] pairs; movmatrix.trans turns the fp16
//   probabilities into the [token][head]^T operand of P.V in registers.
// Softmax is online per KV block in base 2, as in the CUDA-core kernel; the
// CTA-level merge and the output epilogue are shared with it.
#pragma once

#include "decode.cuh"

namespace pkv {

// One warp per CTA with a pipeline of NS stages.  The warp's softmax state
// and O fragments never leave registers: no shared-memory merge, no CTA
// barrier, and the epilogue is a handful of 16-byte stores.  Many such small
// CTAs (16 per SM at 128 registers) hide the per-tile dependency chains.
template <int BS, int NS_ = 0>
struct MmaTraits {
  static constexpr int D = 128, G = 8;
  static constexpr int ROW_BYTES = 128;  // one fp8 token row of one kv head
  static constexpr int TILE_BYTES = BS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NS_ > 0 ? NS_ : (12288 / STAGE_BYTES >= 2 ? 12288 / STAGE_BYTES : 2);
  static constexpr int NT = BS / 16;              // 16-token MMA tiles per block
  static constexpr int STAGE_AREA = NS * STAGE_BYTES;
  static constexpr int BAR_BYTES = NS * 8;
  static constexpr int MIN_BLOCKS = 16;
  static_assert(BS == 16 || BS == 32, "16-token MMA tiles");
  static_assert(NS >= 2, "stages");
  static constexpr size_t smem_bytes(int pb) {
    return 1024 + STAGE_AREA + BAR_BYTES + static_cast<size_t>(pb) * 4;
  }
};

__device__ __forceinline__ uint32_t f16x2_pack(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D(16x8, f32) += A(16x16, f16, row) . B(16x8, f16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Stores 8 consecutive outputs (one 16-byte store for bf16, two for fp32).
__device__ __forceinline__ void store8(__nv_bfloat16* dst, const float (&v)[8]) {
  uint4 w;
  w.x = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[0])) | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[1])) << 16);
  w.y = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[2])) | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[3])) << 16);
  w.z = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[4])) | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[5])) << 16);
  w.w = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[6])) | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v[7])) << 16);
  *reinterpret_cast<uint4*>(dst) = w;
}
__device__ __forceinline__ void store8(float* dst, const float (&v)[8]) {
  reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
// (split-context partials: with an L2 policy)
__device__ __forceinline__ void store8(float* dst, const float (&v)[8], uint64_t policy) {
  st_global_hint(dst, make_float4(v[0], v[1], v[2], v[3]), policy);
  st_global_hint(dst + 4, make_float4(v[4], v[5], v[6], v[7]), policy);
}

// Byte offset of logical 16-byte chunk q of row t in a 128-byte-swizzled tile.
__device__ __forceinline__ int swz(int t, int q) { return t * 128 + ((q ^ (t & 7)) << 4); }

template <typename TQ, int BS, int NS = 0, int MINB = MmaTraits<BS, NS>::MIN_BLOCKS>
__global__ void __launch_bounds__(32, MINB)
    paged_decode_gqa8_fp8_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                                     const DecodeParams p) {
  using T = MmaTraits<BS, NS>;
  constexpr int D = T::D, G = T::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(data + T::STAGE_AREA);
  int* ids = reinterpret_cast<int*>(data + T::STAGE_AREA + T::BAR_BYTES);

  pdl_wait_and_release();
  const int hk = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x;
  const int r = lane >> 2, c = lane & 3;  // fragment row / column-pair of this lane
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[b];
  if (ctx < 0 || ctx > max_ctx) {
    if (lane == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int pb = p.partition_blocks;
  const int nparts = (nblk + pb - 1) / pb;
  const int64_t out_row0 = static_cast<int64_t>(b) * p.num_q_heads + hk * G;
  if (nparts == 0) {
    if (part == 0) {
      TQ* out = static_cast<TQ*>(p.out);
      for (int i = lane; i < G * D; i += 32) out[out_row0 * D + i] = Elem<TQ>::from_float(0.f);
    }
    return;
  }
  if (part >= nparts) return;
  const int blk0 = part * pb;
  const int nb = min(pb, nblk - blk0);

  for (int i = lane; i < nb; i += 32) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + blk0 + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  const bool append = p.new_k != nullptr && part == nparts - 1;
  if (append) append_new_token<TQ, __nv_fp8_e4m3, D, BS>(p, b, hk, ctx, lane, 32);
  const uint32_t bar0 = smem_u32(bars);
  if (lane == 0) {
    for (int s = 0; s < T::NS; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
    if (append) fence_proxy_async_global();
  }
  __syncwarp();

  const uint32_t stage0 = smem_u32(data);
  const uint64_t policy = l2_policy_evict_first();
  int n_issued = 0;  // blocks whose loads lane 0 has started
  auto issue = [&](int ib) {
    n_issued = ib + 1;
    const int s = ib % T::NS;
    const uint32_t bar = bar0 + 8 * s;
    const int id = ids[ib];
    if (id >= 0) {
      mbar_arrive_expect_tx(bar, T::STAGE_BYTES);
      const uint32_t dst = stage0 + s * T::STAGE_BYTES;
      tma_load_4d(dst, &kmap, bar, 0, hk, 0, id, policy);
      tma_load_4d(dst + T::TILE_BYTES, &vmap, bar, 0, hk, 0, id, policy);
    } else {
      mbar_arrive(bar);
    }
  };
  if (lane == 0) {
    const int pre = nb < T::NS ? nb : T::NS;
    for (int i = 0; i < pre; ++i) issue(i);
  }

  // q fragments (B operand of S), fp16, in the permuted contraction order:
  // chunk j holds dims 64(j>>2) + 16c + 4(j&3) + {0..3} -> one 8-byte load each.
  uint32_t qf[8][2];
  {
    const TQ* qrow = static_cast<const TQ*>(p.q) + (out_row0 + r) * D;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int base = 64 * (j >> 2) + 16 * c + 4 * (j & 3);
      float x[4];
      if constexpr (sizeof(TQ) == 2) {
        const uint2 w = *reinterpret_cast<const uint2*>(qrow + base);
        x[0] = __uint_as_float(w.x << 16);
        x[1] = __uint_as_float(w.x & 0xffff0000u);
        x[2] = __uint_as_float(w.y << 16);
        x[3] = __uint_as_float(w.y & 0xffff0000u);
      } else {
        const float4 w = *reinterpret_cast<const float4*>(qrow + base);
        x[0] = w.x;
        x[1] = w.y;
        x[2] = w.z;
        x[3] = w.w;
      }
      qf[j][0] = f16x2_pack(x[0], x[1]);
      qf[j][1] = f16x2_pack(x[2], x[3]);
    }
  }
  const float qk = p.q_scale;  // scale * log2(e) * k_scale, applied to the fp32 logits

  // Online-softmax state of heads 2c and 2c+1 and the O^T fragments:
  // o[i] = {O[2c][8r+i], O[2c+1][8r+i], O[2c][8r+64+i], O[2c+1][8r+64+i]}.
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[i][k] = 0.f;

  // Shared-memory byte offsets (within a 16-token tile) of this lane's loads,
  // fixed for the whole kernel: K rows rho(r), rho(r)+8 at chunks c, 4+c;
  // V rows 2c, (2c+1)^4, and +8, at the chunks holding dims 8r.. and 8r+64..
  const int rho_r = r ^ ((r & 1) << 2);
  const int vrow[4] = {2 * c, (2 * c + 1) ^ 4, 2 * c + 8, ((2 * c + 1) ^ 4) + 8};
  int koff[2][2], voff[4][2];
#pragma unroll
  for (int i2 = 0; i2 < 2; ++i2) {
    koff[0][i2] = swz(rho_r, 4 * i2 + c);
    koff[1][i2] = swz(rho_r + 8, 4 * i2 + c);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int h = 0; h < 2; ++h) voff[k][h] = swz(vrow[k], (r >> 1) + 4 * h) + 8 * (r & 1);

  // The loop runs over 16-token tiles u = 0 .. nb * NT - 1 (tile u % NT of
  // block u / NT) and is software-pipelined: S of tile u+1 is computed before
  // the softmax and P.V of tile u, so the two dependency chains overlap.
  const int n_tiles = nb * T::NT;
  auto tile_base = [&](int u) -> const uint8_t* {
    return data + ((u / T::NT) % T::NS) * T::STAGE_BYTES + (u % T::NT) * 16 * 128;
  };
  auto tile_valid = [&](int u) -> int {  // valid tokens of tile u (0 for a skipped block)
    const int j = u / T::NT;
    if (ids[j] < 0) return 0;
    const int v = ctx - (blk0 + j) * BS - 16 * (u % T::NT);
    return v < 0 ? 0 : (v > 16 ? 16 : v);
  };
  auto compute_s = [&](int u, float (&sacc)[4]) {
    const uint8_t* kt = tile_base(u);
    float s2[4] = {0.f, 0.f, 0.f, 0.f};  // odd k-chunks: two independent MMA chains
#pragma unroll
    for (int k = 0; k < 4; ++k) sacc[k] = 0.f;
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2) {
      const uint4 ka = *reinterpret_cast<const uint4*>(kt + koff[0][i2]);
      const uint4 kb = *reinterpret_cast<const uint4*>(kt + koff[1][i2]);
      const uint32_t kaw[4] = {ka.x, ka.y, ka.z, ka.w};
      const uint32_t kbw[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t a0, a1, a2, a3;
        e4m3x4_to_f16x2x2(kaw[q], a0, a2);
        e4m3x4_to_f16x2x2(kbw[q], a1, a3);
        mma_16816((q & 1) ? s2 : sacc, a0, a1, a2, a3, qf[4 * i2 + q][0], qf[4 * i2 + q][1]);
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) sacc[k] += s2[k];
  };
  int waited = 0;  // blocks whose stage has been waited for
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
      const uint8_t* vt = tile_base(u) + T::TILE_BYTES;
      const bool full = valid == 16;  // warp-uniform: no masking needed
      // ---- online softmax (base 2), heads 2c and 2c+1 -----------------------------
      // m0/m1 is a reference max: probabilities are 2^(s - m) and may exceed 1 by
      // up to 2^8 (fine in fp16 and fp32).  Only when a score passes m + 8 is the
      // exact max over the tile's tokens taken (three xor-shuffle levels) and the
      // state rescaled, so the common case needs one warp vote, no shuffles.
      float s0 = sc[0] * qk, s1 = sc[1] * qk, s2 = sc[2] * qk, s3 = sc[3] * qk;
      if (!full) {
        const bool va = rho_r < valid, vb = rho_r + 8 < valid;
        s0 = va ? s0 : -INFINITY;
        s1 = va ? s1 : -INFINITY;
        s2 = vb ? s2 : -INFINITY;
        s3 = vb ? s3 : -INFINITY;
      }
      const bool over = fmaxf(s0, s2) > m0 + 8.f || fmaxf(s1, s3) > m1 + 8.f;  // m = -inf: any finite s
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
      const uint32_t pb0 = movmatrix_trans(f16x2_pack(p0, p1));
      const uint32_t pb1 = movmatrix_trans(f16x2_pack(p2, p3));
      // ---- O^T += V^T . P^T ---------------------------------------------------------
      uint2 w[4][2];  // [row: 2c, (2c+1)^4, +8, +8][dims 8r.. / 8r+64..]
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int h = 0; h < 2; ++h) w[k][h] = *reinterpret_cast<const uint2*>(vt + voff[k][h]);
      if (!full) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (vrow[k] >= valid) w[k][0] = w[k][1] = make_uint2(0u, 0u);  // never feed NaN codes
      }
#pragma unroll
      for (int wi = 0; wi < 2; ++wi) {
        uint32_t f[2][2][4];  // [row pair 01 / 23][h][dim byte e] fp16x2 (token pair)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t x0 = wi ? w[0][h].y : w[0][h].x, x1 = wi ? w[1][h].y : w[1][h].x;
          const uint32_t x2 = wi ? w[2][h].y : w[2][h].x, x3 = wi ? w[3][h].y : w[3][h].x;
          e4m3x4_to_f16x2x2(__byte_perm(x0, x1, 0x5140), f[0][h][0], f[0][h][1]);
          e4m3x4_to_f16x2x2(__byte_perm(x0, x1, 0x7362), f[0][h][2], f[0][h][3]);
          e4m3x4_to_f16x2x2(__byte_perm(x2, x3, 0x5140), f[1][h][0], f[1][h][1]);
          e4m3x4_to_f16x2x2(__byte_perm(x2, x3, 0x7362), f[1][h][2], f[1][h][3]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)  // m-tile 4wi+e: output dims 8r + 4wi + e and 8r + 64 + 4wi + e
          mma_16816(o[4 * wi + e], f[0][0][e], f[0][1][e], f[1][0][e], f[1][1][e], pb0, pb1);
      }
    }
    if ((u + 1) % T::NT == 0) {  // last tile of block u / NT: its stage is free again
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
    // Drain (bounded): the loads lane 0 started must land before the CTA's
    // shared memory is released.
    const int issued = __shfl_sync(kFullMask, n_issued, 0);
    for (int i = waited; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % T::NS), (i / T::NS) & 1, p.status);
  }

  // ---- epilogue straight from registers ------------------------------------------
  // Row sums over the 8 lanes sharing c (they hold different tokens of the same heads).
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(kFullMask, l0, off);
    l1 += __shfl_xor_sync(kFullMask, l1, off);
  }
  const float f0 = l0 > 0.f ? p.out_scale / l0 : 0.f;
  const float f1 = l1 > 0.f ? p.out_scale / l1 : 0.f;
  const int64_t row_a = out_row0 + 2 * c, row_b = row_a + 1;  // query heads 2c, 2c+1
  if (nparts == 1) {
    TQ* out = static_cast<TQ*>(p.out);
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // dims 8r + 64h + 0..7: one 8-element vector per head
      float va[8], vb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        va[i] = o[i][2 * h] * f0;
        vb[i] = o[i][2 * h + 1] * f1;
      }
      store8(out + row_a * D + 8 * r + 64 * h, va);
      store8(out + row_b * D + 8 * r + 64 * h, vb);
    }
  } else {
    const int64_t slot_a = row_a * p.max_partitions + part, slot_b = row_b * p.max_partitions + part;
    const uint64_t keep = l2_policy_evict_last();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float va[8], vb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        va[i] = o[i][2 * h] * f0;
        vb[i] = o[i][2 * h + 1] * f1;
      }
      store8(p.ws_o + slot_a * D + 8 * r + 64 * h, va, keep);
      store8(p.ws_o + slot_b * D + 8 * r + 64 * h, vb, keep);
    }
    if (r == 0) {
      st_global_hint(p.ws_ml + slot_a * 2, m0 * kLn2, keep);
      st_global_hint(p.ws_ml + slot_a * 2 + 1, l0, keep);
      st_global_hint(p.ws_ml + slot_b * 2, m1 * kLn2, keep);
      st_global_hint(p.ws_ml + slot_b * 2 + 1, l1, keep);
    }
  }
}

}  // namespace pkv

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

// NW warps per CTA, each with a private pipeline of NS stages.  Defaults from
// a sweep on B200: 2 warps x 12 KB of stages and at least 8 resident CTAs per
// SM (registers capped at 128) -- many small CTAs hide the dependent
// convert -> MMA -> softmax chains better than deep per-warp pipelines.
template <int BS, int NW_ = 2, int NS_ = 0>
struct MmaTraits {
  static constexpr int D = 128, G = 8, NW = NW_;
  static constexpr int ROW_BYTES = 128;  // one fp8 token row of one kv head
  static constexpr int TILE_BYTES = BS * ROW_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NS_ > 0 ? NS_ : (12288 / STAGE_BYTES >= 1 ? 12288 / STAGE_BYTES : 1);
  static constexpr int MIN_BLOCKS = 8;
  static constexpr int NT = BS / 16;              // 16-token MMA tiles per block
  static constexpr int STAGE_AREA = NW * NS * STAGE_BYTES;
  static constexpr int COMBINE_BYTES = NW * G * (D + 2) * 4;
  static constexpr int DATA_BYTES = STAGE_AREA > COMBINE_BYTES ? STAGE_AREA : COMBINE_BYTES;
  static constexpr int BAR_BYTES = NW * NS * 8;
  static_assert(BS == 16 || BS == 32, "16-token MMA tiles");
  static_assert(NS >= 1, "stages");
  static constexpr size_t smem_bytes(int pb) {
    return 1024 + DATA_BYTES + BAR_BYTES + static_cast<size_t>(pb) * 4;
  }
};

// Four E4M3 codes (bytes 0..3 of w) -> two fp16x2 words: lo = bytes {0,1}, hi = bytes {2,3}
// (the lower byte of each pair lands in the lower half).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

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

// Byte offset of logical 16-byte chunk q of row t in a 128-byte-swizzled tile.
__device__ __forceinline__ int swz(int t, int q) { return t * 128 + ((q ^ (t & 7)) << 4); }

template <typename TQ, int BS, int NW = 2, int NS = 0, int MINB = 8>
__global__ void __launch_bounds__(NW * 32, MINB)
    paged_decode_gqa8_fp8_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                                     const DecodeParams p) {
  using T = MmaTraits<BS, NW, NS>;
  constexpr int D = T::D, G = T::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(data + T::DATA_BYTES);
  int* ids = reinterpret_cast<int*>(data + T::DATA_BYTES + T::BAR_BYTES);

  const int hk = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane >> 2, c = lane & 3;  // fragment row / column-pair of this lane
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[b];
  if (ctx < 0 || ctx > max_ctx) {
    if (threadIdx.x == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int pb = p.partition_blocks;
  const int nparts = (nblk + pb - 1) / pb;
  const int64_t out_row0 = static_cast<int64_t>(b) * p.num_q_heads + hk * G;
  if (nparts == 0) {
    if (part == 0) {
      TQ* out = static_cast<TQ*>(p.out);
      for (int i = threadIdx.x; i < G * D; i += blockDim.x) out[out_row0 * D + i] = Elem<TQ>::from_float(0.f);
    }
    return;
  }
  if (part >= nparts) return;
  const int blk0 = part * pb;
  const int nb = min(pb, nblk - blk0);

  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + blk0 + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  const uint32_t bar0 = smem_u32(bars) + warp * T::NS * 8;
  if (lane == 0) {
    for (int s = 0; s < T::NS; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
  }
  __syncthreads();

  const int n_w = nb > warp ? (nb - warp + T::NW - 1) / T::NW : 0;
  const uint32_t stage0 = smem_u32(data) + warp * T::NS * T::STAGE_BYTES;
  const uint64_t policy = l2_policy_evict_first();
  auto issue = [&](int i) {
    const int s = i % T::NS;
    const uint32_t bar = bar0 + 8 * s;
    const int id = ids[warp + i * T::NW];
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
    const int pre = n_w < T::NS ? n_w : T::NS;
    for (int i = 0; i < pre; ++i) issue(i);
  }

  // q fragments (B operand of S), fp16, in the permuted contraction order.
  uint32_t qf[8][2];
  {
    const TQ* qrow = static_cast<const TQ*>(p.q) + (out_row0 + r) * D;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int base = 64 * (j >> 2) + 16 * c + 4 * (j & 3);
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) x[e] = Elem<TQ>::to_float(qrow[base + e]);
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

  int waited = 0;
  bool ok = true;
  for (int i = 0; i < n_w; ++i) {
    const int s = i % T::NS;
    if (!mbar_wait_bounded(bar0 + 8 * s, (i / T::NS) & 1, p.status)) {
      ok = false;
      break;
    }
    waited = i + 1;
    const int j = warp + i * T::NW;
    if (ids[j] >= 0) {
      const uint8_t* kt0 = data + warp * T::NS * T::STAGE_BYTES + s * T::STAGE_BYTES;
      const int valid = min(BS, ctx - (blk0 + j) * BS);
#pragma unroll
      for (int t = 0; t < T::NT; ++t) {
        const int t0 = 16 * t;
        if (t0 >= valid) break;
        const uint8_t* kt = kt0 + t0 * T::ROW_BYTES;  // 16-row tiles start at 2 KB multiples: same swizzle
        const uint8_t* vt = kt + T::TILE_BYTES;
        const bool full = t0 + 16 <= valid;            // warp-uniform: no masking needed
        // ---- S = K . Q^T -------------------------------------------------------
        float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sacc2[4] = {0.f, 0.f, 0.f, 0.f};  // even / odd k-chunks
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
            mma_16816((q & 1) ? sacc2 : sacc, a0, a1, a2, a3, qf[4 * i2 + q][0], qf[4 * i2 + q][1]);
          }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) sacc[k] += sacc2[k];
        // ---- online softmax (base 2), heads 2c and 2c+1 --------------------------
        float s0 = sacc[0] * qk, s1 = sacc[1] * qk, s2 = sacc[2] * qk, s3 = sacc[3] * qk;
        if (!full) {
          const bool va = t0 + rho_r < valid, vb = t0 + rho_r + 8 < valid;
          s0 = va ? s0 : -INFINITY;
          s1 = va ? s1 : -INFINITY;
          s2 = vb ? s2 : -INFINITY;
          s3 = vb ? s3 : -INFINITY;
        }
        float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          bm0 = fmaxf(bm0, __shfl_xor_sync(kFullMask, bm0, off));
          bm1 = fmaxf(bm1, __shfl_xor_sync(kFullMask, bm1, off));
        }
        const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
        // Rescale only when some head's running max moved (rare after the first blocks).
        if (__any_sync(kFullMask, mn0 != m0 || mn1 != m1)) {
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
        // ---- O^T += V^T . P^T ---------------------------------------------------
        uint2 w[4][2];  // [row: 2c, (2c+1)^4, +8, +8][dims 8r.. / 8r+64..]
#pragma unroll
        for (int k = 0; k < 4; ++k)
#pragma unroll
          for (int h = 0; h < 2; ++h) w[k][h] = *reinterpret_cast<const uint2*>(vt + voff[k][h]);
        if (!full) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            if (t0 + vrow[k] >= valid) w[k][0] = w[k][1] = make_uint2(0u, 0u);  // never feed NaN codes
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
    }
    __syncwarp();
    if (lane == 0 && i + T::NS < n_w) {
      fence_proxy_async_smem();
      issue(i + T::NS);
    }
  }
  if (!ok) {
    const int issued = min(n_w, waited + T::NS);
    for (int i = waited; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % T::NS), (i / T::NS) & 1, p.status);
  }
  // Row sums over the 8 lanes sharing c (they hold different tokens of the same heads).
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(kFullMask, l0, off);
    l1 += __shfl_xor_sync(kFullMask, l1, off);
  }
  __syncthreads();  // every warp is done with the stage area

  float* c_m = reinterpret_cast<float*>(data);
  float* c_l = c_m + T::NW * G;
  float* c_acc = c_l + T::NW * G;
  if (r == 0) {
    c_m[warp * G + 2 * c] = m0;
    c_m[warp * G + 2 * c + 1] = m1;
    c_l[warp * G + 2 * c] = l0;
    c_l[warp * G + 2 * c + 1] = l1;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float* a0 = c_acc + (warp * G + 2 * c) * D;
    float* a1 = a0 + D;
    a0[8 * r + i] = o[i][0];
    a1[8 * r + i] = o[i][1];
    a0[8 * r + 64 + i] = o[i][2];
    a1[8 * r + 64 + i] = o[i][3];
  }
  __syncthreads();
  finish_partition<TQ, D, G, T::NW>(c_m, c_l, c_acc, p, out_row0, part, nparts);
}

}  // namespace pkv

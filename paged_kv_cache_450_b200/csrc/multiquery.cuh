// multiquery.cuh -- paged attention for several new query tokens per sequence
// (chunked prefill, speculative-decoding verification), causal over the
// paged cache: the q_len queries of a sequence are its last q_len positions
// and query i (position p = ctx - q_len + i) attends the logical tokens 0..p.
//
// FlashAttention-2 style on the tensor cores (mma.sync m16n8k16, fp32
// accumulation).  One CTA = 16, 32, 48 or 64 query rows (the
// rows of a (sequence, KV head), rounded up to 16, at most 64) x one KV head x one
// split-context partition of one sequence; rows are (query i, query head g)
// with g fastest, so grouped-query heads share every K/V tile.  A producer
// warp streams the partition's blocks through a ring of TMA stages (K and V
// tiles as two 128-byte half rows with the 128-byte swizzle, as the decode
// kernels); the compute warps (16 rows each) holding at least one valid row
// consume every stage and release it through an "empty" mbarrier.  Per 16-token tile and warp:
//   S = Q . K^T   M = 16 rows, N = 16 tokens, K = 128  (16 MMAs; K via ldmatrix)
//   O += P . V    M = 16 rows, N = 128 dims,  K = 16   (2 x 16 MMAs; V via
//                 ldmatrix.trans; P as bf16 hi + lo, ~16 bits per weight)
// The online softmax per row keeps a reference max as in the decode kernels.
// Partitions write (m, l, o) partials merged by paged_multiquery_reduce_kernel.
//
// Caches of fp8 (E4M3, per-tensor scales; F8 = true): the producer warp
// TMA-loads each block's raw codes (128 bytes per token row) into a ring of
// its own and widens them to fp16 -- exactly: every E4M3 value is an fp16
// value -- into the stage, in the same swizzled layout a bf16 tile has, so
// the compute warps read it with the same ldmatrix offsets.  Q is rounded
// once to fp16, and both contractions run on fp16 operands with one fp16 P
// (11 significant bits).  The K scale is folded into the logit scale and the
// V scale into the output.
// The dispatch (launch.h) sends it up to 16 rows per (sequence, KV head), for
// either cache type; more rows go to the tcgen05 kernel (multiquery_tc.cuh).
#pragma once

#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_mma_bf16.cuh"
#include "multiquery_params.h"

namespace pkv {

// NWC_ compute warps of 16 rows each: as many as the rows of a (sequence, KV
// head) need, up to 4, so that CTAs are no larger than the work and more of
// them fit on an SM.
template <int BS, int NWC_ = 4, int NS_ = 0, bool F8 = false>
struct MqTraits {
  static constexpr int D = 128;
  static constexpr int NWC = NWC_;                   // compute warps (16 rows each)
  static constexpr int ROWS = 16 * NWC;              // query rows per CTA
  static constexpr int THREADS = 32 * (NWC + 1);     // + one producer warp
  static constexpr int HALF_BYTES = BS * 128;
  static constexpr int TILE_BYTES = 2 * HALF_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NS_ > 0 ? NS_ : (NWC_ == 1 ? 3 : 4);
  // resident CTAs per SM (registers: ~170 per thread at these counts)
  static constexpr int MIN_BLOCKS = NWC_ == 1 ? 6 : (NWC_ == 2 ? 4 : (NWC_ == 3 ? 3 : 2));
  static constexpr int NT = BS / 16;
  static constexpr int STAGE_AREA = NS * STAGE_BYTES;
  // fp8 caches: a ring of raw blocks (K then V codes, 128 bytes per token row)
  static constexpr int RAW_HALF = BS * 128;
  static constexpr int RAW_BYTES = 2 * RAW_HALF;
  static constexpr int NR = F8 ? 3 : 0;
  static constexpr int RAW_AREA = NR * RAW_BYTES;
  static constexpr int BAR_BYTES = (2 * NS + NR) * 8;  // full[NS], empty[NS], raw_full[NR]
  static constexpr size_t smem_bytes(int pb) {
    return 1024 + STAGE_AREA + RAW_AREA + BAR_BYTES + static_cast<size_t>(pb) * 4;
  }
};

// Widens one block of raw E4M3 codes (K and V: BS rows x 128 codes, 128-byte
// swizzle) into fp16 in the bf16 stage layout (two 64-dim halves of BS rows x
// 128 bytes, 128-byte swizzle).  Raw chunk q of row t (dims 16q .. 16q+15)
// becomes stage chunks 2(q % 4) and 2(q % 4) + 1 of half q / 4.  One warp.
template <int BS>
__device__ __forceinline__ void widen_e4m3_block(const uint8_t* raw, uint8_t* stage, int lane) {
  constexpr int RAW_HALF = BS * 128, TILE = BS * 256, HALF = BS * 128;
#pragma unroll
  for (int kv = 0; kv < 2; ++kv) {
#pragma unroll
    for (int i = lane; i < BS * 8; i += 32) {
      const int t = i >> 3, q = i & 7;
      const uint4 w = *reinterpret_cast<const uint4*>(raw + kv * RAW_HALF + t * 128 + ((q ^ (t & 7)) << 4));
      uint32_t f[8];
      e4m3x4_to_f16x2x2(w.x, f[0], f[1]);
      e4m3x4_to_f16x2x2(w.y, f[2], f[3]);
      e4m3x4_to_f16x2x2(w.z, f[4], f[5]);
      e4m3x4_to_f16x2x2(w.w, f[6], f[7]);
      uint8_t* dst = stage + kv * TILE + (q >> 2) * HALF + t * 128;
      const int c0 = 2 * (q & 3);
      *reinterpret_cast<uint4*>(dst + ((c0 ^ (t & 7)) << 4)) = make_uint4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<uint4*>(dst + (((c0 + 1) ^ (t & 7)) << 4)) = make_uint4(f[4], f[5], f[6], f[7]);
    }
  }
}

// D(16x8, f32) += A(16x16) . B(16x8): bf16 operands, or fp16 (F16 = true).
template <bool F16>
__device__ __forceinline__ void mma_16816_t(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    mma_16816(d, a0, a1, a2, a3, b0, b1);
  } else {
    mma_16816_bf16(d, a0, a1, a2, a3, b0, b1);
  }
}

template <int BS, int G, int NWC, bool F8>
__global__ void __launch_bounds__(MqTraits<BS, NWC, 0, F8>::THREADS, MqTraits<BS, NWC, 0, F8>::MIN_BLOCKS)
    paged_multiquery_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                                const MultiQueryParams p) {
  using T = MqTraits<BS, NWC, 0, F8>;
  constexpr int D = T::D;
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* raw = data + T::STAGE_AREA;  // fp8 caches: the raw ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(data + T::STAGE_AREA + T::RAW_AREA);  // full, empty, raw_full
  int* ids = reinterpret_cast<int*>(data + T::STAGE_AREA + T::RAW_AREA + T::BAR_BYTES);

  const int Hkv = p.num_kv_heads;
  const int hk = blockIdx.x % Hkv, qt = blockIdx.x / Hkv, part = blockIdx.y;
  // Longest work first: CTAs start in grid order, so grid row z takes the sequence with the z-th
  // longest context (ties by index: a permutation) and the CTAs that start last are the short ones.
  // The lengths are staged in the stage area, which no load has reached yet.  Each CTA's ranking
  // takes ~B^2 comparisons, so it runs only where it is cheap beside the CTA's work and the tail
  // matters: at most 64 sequences (more CTAs, more waves to even out) and a block table of at least
  // 1024 tokens.  (In the decode kernel, with 256 sequences and ~10000 short CTAs, the same ranking
  // measured 18% slower.)
  int b = blockIdx.z;
  if (p.num_seqs <= 64 && p.max_blocks_per_seq * BS >= 1024) {
    int* lens = reinterpret_cast<int*>(data);
    int* pick = lens + 64;
    for (int i = threadIdx.x; i < p.num_seqs; i += blockDim.x) lens[i] = p.context_lens[i];
    __syncthreads();
    for (int j = threadIdx.x; j < p.num_seqs; j += blockDim.x) {
      const int lj = lens[j];
      int r = 0;
      for (int i = 0; i < p.num_seqs; ++i) {
        const int li = lens[i];
        r += (li > lj) || (li == lj && i < j);
      }
      if (r == static_cast<int>(blockIdx.z)) *pick = j;
    }
    __syncthreads();
    b = *pick;
    fence_proxy_async_smem();  // these writes before the tile loads that later land there
    __syncthreads();
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int q0, q_len;
  if (!query_rows_ok(p, b, q0, q_len)) {  // before any load or store
    if (threadIdx.x == 0) set_status(p.status, PKV_STATUS_BAD_QUERY_LOC);
    return;
  }
  const int rows_total = q_len * G;
  if (q_len <= 0 || qt * T::ROWS >= rows_total) return;
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[b];
  if (ctx < 0 || ctx > max_ctx) {
    if (threadIdx.x == 0 && hk == 0 && part == 0 && qt == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int pb = p.partition_blocks;
  const int nparts = (nblk + pb - 1) / pb;
  const int Hq = p.num_q_heads;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  const int base_pos = ctx - q_len;  // position of query 0
  // rows of this CTA: row = qt*ROWS + m, query i = row / G, head g = row % G
  const int row_last = min(rows_total, (qt + 1) * T::ROWS) - 1;
  const int pos_last = base_pos + row_last / G;
  if (nparts == 0 || pos_last < 0) {  // nothing to attend: zero rows (partition 0 writes them)
    if (part == 0 && threadIdx.x < T::ROWS) {
      const int row = qt * T::ROWS + threadIdx.x;
      if (row < rows_total) {
        const int64_t orow = static_cast<int64_t>(q0 + row / G) * Hq + hk * G + row % G;
        for (int d = 0; d < D; ++d) out[orow * D + d] = __float2bfloat16_rn(0.f);
      }
    }
    return;
  }
  if (part >= nparts) return;
  const int blk0 = part * pb;
  // blocks of this partition the CTA's rows can see (causal): up to pos_last
  const int nb = max(0, min(min(pb, nblk - blk0), pos_last / BS + 1 - blk0));

  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + blk0 + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  // compute warps holding at least one row of this CTA (the others leave now)
  const int n_active = min(T::NWC, (min(rows_total - qt * T::ROWS, T::ROWS) + 15) / 16);
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * T::NS, rfull0 = empty0 + 8 * T::NS;
  if (threadIdx.x == 0) {
    for (int s = 0; s < T::NS; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, n_active);
    }
    for (int s = 0; s < T::NR; ++s) mbar_init(rfull0 + 8 * s, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp < T::NWC && warp >= n_active) return;
  const uint32_t stage0 = smem_u32(data);

  if (warp == T::NWC && F8) {  // ---------------- producer warp (fp8: loads and widens) ----------
    const uint64_t policy = l2_policy_evict_first();
    const uint32_t raw0 = smem_u32(raw);
    int issued = 0, landed = 0;
    auto issue_raw = [&](int j) {  // lane 0: block j's raw K and V codes into ring slot j % NR
      const int r = j % T::NR;
      const uint32_t bar = rfull0 + 8 * r;
      const int id = ids[j];
      if (id >= 0) {
        mbar_arrive_expect_tx(bar, T::RAW_BYTES);
        tma_load_4d(raw0 + r * T::RAW_BYTES, &kmap, bar, 0, hk, 0, id, policy);
        tma_load_4d(raw0 + r * T::RAW_BYTES + T::RAW_HALF, &vmap, bar, 0, hk, 0, id, policy);
      } else {
        mbar_arrive(bar);
      }
    };
    if (lane == 0)
      for (int j = 0; j < min(nb, T::NR); ++j) issue_raw(j);
    issued = min(nb, T::NR);
    for (int j = 0; j < nb; ++j) {
      const int r = j % T::NR, s = j % T::NS;
      if (!__all_sync(kFullMask, mbar_wait_bounded(rfull0 + 8 * r, (j / T::NR) & 1, p.status))) break;
      landed = j + 1;
      if (j >= T::NS && !__all_sync(kFullMask, mbar_wait_bounded(empty0 + 8 * s, ((j / T::NS) - 1) & 1, p.status)))
        break;
      if (ids[j] >= 0) widen_e4m3_block<BS>(raw + r * T::RAW_BYTES, data + s * T::STAGE_BYTES, lane);
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(full0 + 8 * s);  // (arrive releases the widened stage to the compute warps)
        if (j + T::NR < nb) {
          fence_proxy_async_smem();  // the raw slot's reads before the next TMA write into it
          issue_raw(j + T::NR);
        }
      }
      if (j + T::NR < nb) issued = j + T::NR + 1;
    }
    // Drain (bounded): every raw load started has landed before the CTA exits.
    if (lane == 0)
      for (int j = landed; j < issued; ++j) mbar_wait_bounded(rfull0 + 8 * (j % T::NR), (j / T::NR) & 1, p.status);
    return;
  }
  if (warp == T::NWC) {  // ---------------- producer warp ----------------------
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      for (int j = 0; j < nb; ++j) {
        const int s = j % T::NS;
        if (j >= T::NS && !mbar_wait_bounded(empty0 + 8 * s, ((j / T::NS) - 1) & 1, p.status)) break;
        const uint32_t bar = full0 + 8 * s;
        const int id = ids[j];
        if (id >= 0) {
          mbar_arrive_expect_tx(bar, T::STAGE_BYTES);
          const uint32_t dst = stage0 + s * T::STAGE_BYTES;
          tma_load_4d(dst, &kmap, bar, 0, hk, 0, id, policy);
          tma_load_4d(dst + T::HALF_BYTES, &kmap, bar, 64, hk, 0, id, policy);
          tma_load_4d(dst + T::TILE_BYTES, &vmap, bar, 0, hk, 0, id, policy);
          tma_load_4d(dst + T::TILE_BYTES + T::HALF_BYTES, &vmap, bar, 64, hk, 0, id, policy);
        } else {
          mbar_arrive(bar);
        }
      }
      // Drain (bounded): every stage must be released before the CTA exits.
      for (int j = (nb > T::NS ? nb - T::NS : 0); j < nb; ++j)
        mbar_wait_bounded(empty0 + 8 * (j % T::NS), (j / T::NS) & 1, p.status);
    }
    return;
  }

  // ---------------- compute warps --------------------------------------------
  const int r = lane >> 2, c = lane & 3;
  const int wrow0 = qt * T::ROWS + 16 * warp;            // first row of this warp
  const int ra = wrow0 + r, rb = wrow0 + r + 8;          // this lane's two rows
  const bool va_row = ra < rows_total, vb_row = rb < rows_total;
  const int pos_a = base_pos + ra / G, pos_b = base_pos + rb / G;
  const int64_t orow_a = static_cast<int64_t>(q0 + ra / G) * Hq + hk * G + ra % G;
  const int64_t orow_b = static_cast<int64_t>(q0 + rb / G) * Hq + hk * G + rb % G;
  const int warp_min_pos = base_pos + wrow0 / G;

  // Q fragments (A operand of S): rows ra / rb, dims 16j + 2c (+1) and +8 (+9).
  uint32_t qf[8][4];
  {
    const uint32_t* qa = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) + orow_a * D);
    const uint32_t* qb = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) + orow_b * D);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      qf[j][0] = va_row ? qa[8 * j + c] : 0u;
      qf[j][1] = vb_row ? qb[8 * j + c] : 0u;
      qf[j][2] = va_row ? qa[8 * j + c + 4] : 0u;
      qf[j][3] = vb_row ? qb[8 * j + c + 4] : 0u;
      if constexpr (F8) {  // fp16 operands (exact for |q| in [2^-14, 65504])
#pragma unroll
        for (int e = 0; e < 4; ++e) qf[j][e] = bf16x2_to_f16x2(qf[j][e]);
      }
    }
  }
  const float qk = p.q_scale;
  float ma = -INFINITY, mb = -INFINITY, la = 0.f, lb = 0.f;
  float o[16][4];  // d n-tile nt: {O[ra][8nt+2c], O[ra][8nt+2c+1], O[rb][8nt+2c], O[rb][8nt+2c+1]}
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) o[i][k] = 0.f;

  // ldmatrix offsets: K (B operand of S, non-trans): matrix i covers tokens
  // 8(i>>1).. and dims 8(i&1).. of a 16x16 chunk; V (B operand of P.V, trans):
  // tokens 8(i&1).., dims 8(i>>1)..
  int koff[4], voff[4];
  {
    const int i = lane >> 3;
    const int tk = (lane & 7) + 8 * (i >> 1), tv = (lane & 7) + 8 * (i & 1);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      koff[jj] = tk * 128 + (((2 * jj + (i & 1)) ^ (tk & 7)) << 4);
      voff[jj] = tv * 128 + (((2 * jj + (i >> 1)) ^ (tv & 7)) << 4);
    }
  }

  bool ok = true;
  for (int j = 0; j < nb; ++j) {
    const int s = j % T::NS;
    if (!mbar_wait_bounded(full0 + 8 * s, (j / T::NS) & 1, p.status)) {
      ok = false;
      break;
    }
    if (ids[j] >= 0) {
      const uint32_t kt0 = stage0 + s * T::STAGE_BYTES;
#pragma unroll
      for (int t = 0; t < T::NT; ++t) {
        const int tok0 = (blk0 + j) * BS + 16 * t;  // absolute position of the tile's first token
        if (tok0 >= ctx || tok0 > pos_last) break;
        const uint32_t kt = kt0 + 16 * t * 128;
        const uint32_t vt = kt + T::TILE_BYTES;
        // ---- S = Q . K^T: two n-tiles of 8 tokens ----------------------------
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kt + (jj >> 2) * T::HALF_BYTES + koff[jj & 3], b0, b1, b2, b3);
          mma_16816_t<F8>(s0, qf[jj][0], qf[jj][1], qf[jj][2], qf[jj][3], b0, b1);
          mma_16816_t<F8>(s1, qf[jj][0], qf[jj][1], qf[jj][2], qf[jj][3], b2, b3);
        }
        // values: row ra: s0[0..1] (tokens 2c, 2c+1), s1[0..1] (8+2c, 8+2c+1); row rb: s0[2..3], s1[2..3]
        float sa[4] = {s0[0] * qk, s0[1] * qk, s1[0] * qk, s1[1] * qk};
        float sb[4] = {s0[2] * qk, s0[3] * qk, s1[2] * qk, s1[3] * qk};
        const bool need_mask = tok0 + 15 > warp_min_pos || tok0 + 16 > ctx;  // warp-uniform
        if (need_mask) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = tok0 + (e >> 1) * 8 + 2 * c + (e & 1);
            if (tok > pos_a || tok >= ctx) sa[e] = -INFINITY;
            if (tok > pos_b || tok >= ctx) sb[e] = -INFINITY;
          }
        }
        float ta = fmaxf(fmaxf(sa[0], sa[1]), fmaxf(sa[2], sa[3]));
        float tb = fmaxf(fmaxf(sb[0], sb[1]), fmaxf(sb[2], sb[3]));
        const bool over = ta > ma + 8.f || tb > mb + 8.f;
        if (__any_sync(kFullMask, over)) {
#pragma unroll
          for (int off = 1; off < 4; off <<= 1) {
            ta = fmaxf(ta, __shfl_xor_sync(kFullMask, ta, off));
            tb = fmaxf(tb, __shfl_xor_sync(kFullMask, tb, off));
          }
          const float na = fmaxf(ma, ta), nb2 = fmaxf(mb, tb);
          // rows whose every score so far is masked keep m = -inf (alpha 1, p 0)
          const float aa = na == -INFINITY ? 1.f : fast_exp2(ma - na);
          const float ab = nb2 == -INFINITY ? 1.f : fast_exp2(mb - nb2);
          la *= aa;
          lb *= ab;
#pragma unroll
          for (int i3 = 0; i3 < 16; ++i3) {
            o[i3][0] *= aa;
            o[i3][1] *= aa;
            o[i3][2] *= ab;
            o[i3][3] *= ab;
          }
          ma = na;
          mb = nb2;
        }
        float pa[4], pbv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pa[e] = ma == -INFINITY ? 0.f : fast_exp2(sa[e] - ma);
          pbv[e] = mb == -INFINITY ? 0.f : fast_exp2(sb[e] - mb);
        }
        la += (pa[0] + pa[1]) + (pa[2] + pa[3]);
        lb += (pbv[0] + pbv[1]) + (pbv[2] + pbv[3]);
        // P (A operand of P.V): {row ra tok 2c.., row rb tok 2c.., row ra tok 8+2c.., row rb tok 8+2c..};
        // bf16: a high part and a residual (~16 bits); fp16 (fp8 caches): one fp16 value (11 bits)
        uint32_t ah[4], al[4];
        if constexpr (F8) {
          ah[0] = f16x2_pack(pa[0], pa[1]);
          ah[1] = f16x2_pack(pbv[0], pbv[1]);
          ah[2] = f16x2_pack(pa[2], pa[3]);
          ah[3] = f16x2_pack(pbv[2], pbv[3]);
        } else {
          bf16x2_split(pa[0], pa[1], ah[0], al[0]);
          bf16x2_split(pbv[0], pbv[1], ah[1], al[1]);
          bf16x2_split(pa[2], pa[3], ah[2], al[2]);
          bf16x2_split(pbv[2], pbv[3], ah[3], al[3]);
        }
        // V rows past the context must not feed NaN bits into the products
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (tok0 + 16 > ctx) {
          mlo = (tok0 + 2 * c < ctx ? 0x0000ffffu : 0u) | (tok0 + 2 * c + 1 < ctx ? 0xffff0000u : 0u);
          mhi = (tok0 + 8 + 2 * c < ctx ? 0x0000ffffu : 0u) | (tok0 + 9 + 2 * c < ctx ? 0xffff0000u : 0u);
        }
        // ---- O += P . V: d n-tiles 2m, 2m+1 per ldmatrix.trans -----------------
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(vt + (m >> 2) * T::HALF_BYTES + voff[m & 3], b0, b1, b2, b3);
          b0 &= mlo;
          b1 &= mhi;
          b2 &= mlo;
          b3 &= mhi;
          mma_16816_t<F8>(o[2 * m], ah[0], ah[1], ah[2], ah[3], b0, b1);
          mma_16816_t<F8>(o[2 * m + 1], ah[0], ah[1], ah[2], ah[3], b2, b3);
          if constexpr (!F8) {
            mma_16816_bf16(o[2 * m], al[0], al[1], al[2], al[3], b0, b1);
            mma_16816_bf16(o[2 * m + 1], al[0], al[1], al[2], al[3], b2, b3);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);  // this warp is done with the stage
  }
  (void)ok;  // a timed-out wait leaves the status bit; the rows are still written

  // ---- epilogue --------------------------------------------------------------------
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    la += __shfl_xor_sync(kFullMask, la, off);
    lb += __shfl_xor_sync(kFullMask, lb, off);
  }
  const float fa = la > 0.f ? p.out_scale / la : 0.f, fb = lb > 0.f ? p.out_scale / lb : 0.f;
  if (nparts == 1) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 8 * nt + 2 * c;
      if (va_row)
        *reinterpret_cast<__nv_bfloat162*>(out + orow_a * D + d) = __floats2bfloat162_rn(o[nt][0] * fa, o[nt][1] * fa);
      if (vb_row)
        *reinterpret_cast<__nv_bfloat162*>(out + orow_b * D + d) = __floats2bfloat162_rn(o[nt][2] * fb, o[nt][3] * fb);
    }
  } else {
    const int64_t sa_ = orow_a * p.max_partitions + part, sb_ = orow_b * p.max_partitions + part;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int d = 8 * nt + 2 * c;
      if (va_row) *reinterpret_cast<float2*>(p.ws_o + sa_ * D + d) = make_float2(o[nt][0] * fa, o[nt][1] * fa);
      if (vb_row) *reinterpret_cast<float2*>(p.ws_o + sb_ * D + d) = make_float2(o[nt][2] * fb, o[nt][3] * fb);
    }
    if (c == 0) {
      if (va_row) {
        p.ws_ml[sa_ * 2] = la > 0.f ? ma * kLn2 : 0.f;
        p.ws_ml[sa_ * 2 + 1] = la;
      }
      if (vb_row) {
        p.ws_ml[sb_ * 2] = lb > 0.f ? mb * kLn2 : 0.f;
        p.ws_ml[sb_ * 2 + 1] = lb;
      }
    }
  }
}

}  // namespace pkv

// multiquery_tc.cuh -- multi-query paged attention on the tcgen05 tensor cores
// for prefill-sized query counts (more than 64 rows per sequence and KV head).
//
// Same operation as multiquery.cuh (causal over the paged cache, queries are
// the sequence's last q_len positions), written for the Blackwell MMA:
//
//   one CTA = 128 query rows (query i, head g; g fastest) x one KV head x one
//   split-context partition; KV tiles of 128 tokens (8 blocks of 16 or 4 of 32)
//   from the partition's start (a partition that is not a multiple of 128
//   tokens ends in a partial tile, masked like the context end).
//   S = Q . K^T      M = 128 rows, N = 128 tokens, K = 128 dims -> TMEM columns [0, 128)
//   O += P . V       M = 128 rows, N = 128 dims,   K = 128 tokens -> TMEM columns [128, 256)
//
// Q, K and V sit in shared memory in the 128-byte-swizzled layout (two
// 64-element halves of every 256-byte row) as TMA delivers them; Q and K are
// K-major operands, V (stored token-major, dims contiguous) is the N-major B
// operand of P . V, so no transpose is ever made.  P never touches shared
// memory: it is the TMEM A operand of P . V, split into a bf16 high part
// (columns [256, 320)) and a bf16 residual (columns [320, 384)) -- two MMAs
// per k-step -- so each probability keeps ~16 significant bits (a bf16 P
// alone costs up to ~3e-3 absolute on short contexts).  Six warps:
//   warps 0-3  softmax: thread t owns row t (TMEM lane t).  It reads its row
//              of S from TMEM, applies the causal / context mask, keeps a
//              reference max (the accumulator is rescaled only when a score
//              passes it by more than 2^8), writes its row of P into TMEM
//              and, at the end, reads its row of O, divides by the row sum
//              and stores it (or the split-context partial).
//   warp 4     TMA producer: Q once, then K and V tiles block by block through
//              two-stage rings (one 4-D box per block and 64-dim half).
//   warp 5     MMA issuer: one thread issues S_j as soon as the softmax has
//              taken S_{j-1} into registers, then P_{j-1} . V_{j-1}; completion
//              is signalled through tcgen05.commit on mbarriers.
// Every wait is bounded (2 s); on a timeout the status bit is set, the loops
// stop, in-flight work is drained with bounded waits and TMEM is freed.
#pragma once

#include "common.cuh"
#include "multiquery_params.h"
#include "tcgen05.cuh"

namespace pkv {

template <int BS>
struct MqTcTraits {
  static constexpr int D = 128;
  static constexpr int ROWS = 128;           // query rows per CTA (MMA M)
  static constexpr int TOK = 128;            // tokens per KV tile
  static constexpr int BPT = TOK / BS;       // blocks per KV tile
  static constexpr int HALF = 128 * 128;     // 128 rows x 128 bytes (64 bf16)
  static constexpr int TILE = 2 * HALF;      // 32 KB: 128 rows x 128 bf16
  static constexpr int NSTAGE = 2;           // K ring and V ring depth
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + NSTAGE * TILE;
  static constexpr int BAR_OFF = V_OFF + NSTAGE * TILE;
  // mbarriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full, s_free, p_full, pv_done, mma_done
  static constexpr int NBAR = 1 + 4 * NSTAGE + 5;
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;   // TMEM base address written by tcgen05.alloc
  static constexpr int IDS_OFF = SLOT_OFF + 16;
  static constexpr int THREADS = 192;
  static constexpr uint32_t TMEM_COLS = 512;  // S 128 | O 128 | P hi 64 | P lo 64 | unused
  static constexpr size_t smem_bytes(int pb) { return 1024 + IDS_OFF + static_cast<size_t>(pb) * 4; }
};

// 3-D tiled TMA load (coordinates innermost first; c0 is 0 or 64 elements).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Bounded wait taken by every lane of a warp; the result is the same on every
// lane (false if any lane gave up), so the warp stays converged for the
// .sync.aligned tensor-memory instructions that follow.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity, unsigned* status) {
  return __all_sync(kFullMask, mbar_wait_bounded(bar, parity, status));
}

template <int BS, int G>
__global__ void __launch_bounds__(MqTcTraits<BS>::THREADS, 1)
    paged_multiquery_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                               const __grid_constant__ CUtensorMap vmap, const MultiQueryParams p) {
  using T = MqTcTraits<BS>;
  constexpr int D = T::D;
  constexpr int QPT = T::ROWS / G;  // queries per CTA tile
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  int* ids = reinterpret_cast<int*>(data + T::IDS_OFF);

  const int Hkv = p.num_kv_heads;
  const int hk = blockIdx.x % Hkv, qt = blockIdx.x / Hkv, part = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = p.query_start_loc[b];
  const int q_len = p.query_start_loc[b + 1] - q0;
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
  const int base_pos = ctx - q_len;
  const int row_last = min(rows_total, (qt + 1) * T::ROWS) - 1;
  const int pos_last = base_pos + row_last / G;
  if (nparts == 0 || pos_last < 0) {  // nothing to attend: zero rows (partition 0 writes them)
    if (part == 0 && threadIdx.x < T::ROWS) {
      const int row = qt * T::ROWS + threadIdx.x;
      if (row < rows_total) {
        const int64_t orow = static_cast<int64_t>(q0 + row / G) * Hq + hk * G + row % G;
        for (int d = 0; d < D; d += 8)
          *reinterpret_cast<uint4*>(out + orow * D + d) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  if (part >= nparts) return;
  const int tok_begin = part * pb * BS;
  // tokens this CTA's rows can see in the partition: [tok_begin, tok_end)
  const int tok_end = min(min(ctx, tok_begin + pb * BS), pos_last + 1);
  if (tok_end <= tok_begin) return;  // every row sits before this partition (never merged)
  const int nt = (tok_end - tok_begin + T::TOK - 1) / T::TOK;
  const int nb = (tok_end - tok_begin + BS - 1) / BS;

  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + part * pb + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  const uint32_t base = smem_u32(data);
  const uint32_t bar0 = base + T::BAR_OFF;
  const uint32_t q_full = bar0;
  auto k_full = [&](int s) { return bar0 + 8 * (1 + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (3 + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (5 + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (7 + s); };
  const uint32_t s_full = bar0 + 8 * 9, s_free = bar0 + 8 * 10, p_full = bar0 + 8 * 11, pv_done = bar0 + 8 * 12,
                 mma_done = bar0 + 8 * 13;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < T::NSTAGE; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 4) {
    __syncwarp();
    tmem_alloc(base + T::SLOT_OFF, T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(data + T::SLOT_OFF);
  const uint32_t tmem_s = tmem, tmem_o = tmem + 128, tmem_phi = tmem + 256, tmem_plo = tmem + 320;

  if (warp == 4) {  // ---------------- TMA producer ------------------------------------
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      mbar_arrive_expect_tx(q_full, T::TILE);
      tma_load_3d(base + T::Q_OFF, &qmap, q_full, 0, hk * G, q0 + qt * QPT);
      tma_load_3d(base + T::Q_OFF + T::HALF, &qmap, q_full, 64, hk * G, q0 + qt * QPT);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1;
        const int i0 = j * T::BPT, i1 = min(nb, i0 + T::BPT);
        int nvalid = 0;
        for (int i = i0; i < i1; ++i) nvalid += ids[i] >= 0;
        const uint32_t bytes = static_cast<uint32_t>(nvalid) * 2u * BS * 128u;
        // K tile j
        if (j >= T::NSTAGE && !mbar_wait_bounded(k_empty(s), ((j >> 1) - 1) & 1, p.status)) break;
        if (bytes) mbar_arrive_expect_tx(k_full(s), bytes); else mbar_arrive(k_full(s));
        for (int i = i0; i < i1; ++i) {
          const int id = ids[i];
          if (id < 0) continue;
          const uint32_t dst = base + T::K_OFF + s * T::TILE + (i - i0) * BS * 128;
          tma_load_4d(dst, &kmap, k_full(s), 0, hk, 0, id, policy);
          tma_load_4d(dst + T::HALF, &kmap, k_full(s), 64, hk, 0, id, policy);
        }
        k_issued = j + 1;
        // V tile j
        if (j >= T::NSTAGE && !mbar_wait_bounded(v_empty(s), ((j >> 1) - 1) & 1, p.status)) break;
        if (bytes) mbar_arrive_expect_tx(v_full(s), bytes); else mbar_arrive(v_full(s));
        for (int i = i0; i < i1; ++i) {
          const int id = ids[i];
          if (id < 0) continue;
          const uint32_t dst = base + T::V_OFF + s * T::TILE + (i - i0) * BS * 128;
          tma_load_4d(dst, &vmap, v_full(s), 0, hk, 0, id, policy);
          tma_load_4d(dst + T::HALF, &vmap, v_full(s), 64, hk, 0, id, policy);
        }
        v_issued = j + 1;
      }
      // drain (bounded): the copies of the last stages have landed before exit
      mbar_wait_bounded(q_full, 0, p.status);
      for (int j = max(0, k_issued - T::NSTAGE); j < k_issued; ++j)
        mbar_wait_bounded(k_full(j & 1), (j >> 1) & 1, p.status);
      for (int j = max(0, v_issued - T::NSTAGE); j < v_issued; ++j)
        mbar_wait_bounded(v_full(j & 1), (j >> 1) & 1, p.status);
    }
  } else if (warp == 5) {  // ---------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, 1);
      bool ok = mbar_wait_bounded(q_full, 0, p.status);
      for (int j = 0; ok && j <= nt; ++j) {
        if (j < nt) {
          const int s = j & 1;
          if (!mbar_wait_bounded(k_full(s), (j >> 1) & 1, p.status)) break;
          if (j > 0 && !mbar_wait_bounded(s_free, (j - 1) & 1, p.status)) break;
          tc_fence_after();
          const uint32_t ka = base + T::K_OFF + s * T::TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * T::HALF + (kk & 3) * 32;
            tc_mma_bf16(tmem_s, smem_desc_sw128(base + T::Q_OFF + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024),
                        idesc_s, kk > 0 ? 1u : 0u);
          }
          tc_commit(s_full);
          tc_commit(k_empty(s));
        }
        if (j > 0) {
          const int jj = j - 1, s = jj & 1;
          if (!mbar_wait_bounded(v_full(s), (jj >> 1) & 1, p.status)) break;
          if (!mbar_wait_bounded(p_full, jj & 1, p.status)) break;
          tc_fence_after();
          const uint32_t va = base + T::V_OFF + s * T::TILE;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // 16 tokens = 8 packed TMEM columns of P per k-step
            const uint64_t vdesc = smem_desc_sw128(va + kk * 16 * 128, T::HALF, 1024);
            tc_mma_bf16_tmem_a(tmem_o, tmem_phi + 8 * kk, vdesc, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
            tc_mma_bf16_tmem_a(tmem_o, tmem_plo + 8 * kk, vdesc, idesc_pv, 1u);
          }
          tc_commit(pv_done);
          tc_commit(v_empty(s));
        }
      }
      // drain (bounded): no MMA may still read shared memory or write TMEM at exit
      tc_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, p.status);
    }
  } else {  // ---------------- softmax warps 0-3: thread t owns row t -------------------------
    const int r = threadIdx.x;
    const int row = qt * T::ROWS + r;
    const bool valid = row < rows_total;
    const int pos = valid ? base_pos + row / G : -1;  // an invalid row sees nothing
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float qk = p.q_scale;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int t0 = tok_begin + j * T::TOK;
      if (!warp_wait_bounded(s_full, j & 1, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t u[32];
        tmem_ld32(tmem_s + lane_off + 32 * c, u);
        tmem_ld_wait(u);
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[32 * c + e] = __uint_as_float(u[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);

      // blocks of this tile with a bad id (their tokens are masked, their V rows zeroed)
      bool bad_tile = false;
      {
        const int i0 = j * T::BPT, i1 = min(nb, i0 + T::BPT);
        for (int i = i0; i < i1; ++i) bad_tile |= ids[i] < 0;
      }
      const bool ragged = t0 + T::TOK > tok_end;  // tokens at or past tok_end in this tile
      float mx = -INFINITY;
      if (t0 + T::TOK - 1 > pos || ragged || bad_tile) {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int t = t0 + c;
          bool masked = t > pos || t >= tok_end;
          if (bad_tile) masked = masked || ids[(t - tok_begin) / BS] < 0;
          sv[c] = masked ? -INFINITY : sv[c] * qk;
          mx = fmaxf(mx, sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          sv[c] *= qk;
          mx = fmaxf(mx, sv[c]);
        }
      }
      // reference max: move it (and rescale) only when a score passes it by more than 8 (log2 units)
      float alpha = 1.f;
      if (mx > m + 8.f) {
        alpha = m == -INFINITY ? 0.f : fast_exp2(m - mx);
        l *= alpha;
        m = mx;
      }
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        sv[c] = m == -INFINITY ? 0.f : fast_exp2(sv[c] - m);
        sum += sv[c];
      }
      l += sum;
      // P_{j-1} . V_{j-1} must be complete before P and O are touched
      if (j > 0) {
        if (!warp_wait_bounded(pv_done, (j - 1) & 1, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(kFullMask, alpha != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t u[32];
            tmem_ld32(tmem_o + lane_off + 32 * c, u);
            tmem_ld_wait(u);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
            tmem_st32(tmem_o + lane_off + 32 * c, u);
          }
          tmem_st_wait();
        }
      }
      // V rows of tokens that must not contribute (past tok_end, bad blocks) are zeroed: 0 * NaN would poison O
      if (ragged || bad_tile) {
        if (!warp_wait_bounded(v_full(j & 1), (j >> 1) & 1, p.status)) {
          ok = false;
          break;
        }
        const int t = t0 + r;
        if (t >= tok_end || (bad_tile && ids[(t - tok_begin) / BS] < 0)) {
          uint8_t* vrow = data + T::V_OFF + (j & 1) * T::TILE + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            *reinterpret_cast<uint4*>(vrow + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
            *reinterpret_cast<uint4*>(vrow + T::HALF + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      // row r of P into TMEM lane r: tokens (2k, 2k+1) in column k, high part and residual
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float a = sv[32 * c + 2 * k], bb = sv[32 * c + 2 * k + 1];
          const __nv_bfloat162 h = __floats2bfloat162_rn(a, bb);
          const __nv_bfloat162 lw = __floats2bfloat162_rn(a - __low2float(h), bb - __high2float(h));
          hi[k] = *reinterpret_cast<const uint32_t*>(&h);
          lo[k] = *reinterpret_cast<const uint32_t*>(&lw);
        }
        tmem_st16(tmem_phi + lane_off + 16 * c, hi);
        tmem_st16(tmem_plo + lane_off + 16 * c, lo);
      }
      tmem_st_wait();
      fence_proxy_async_smem();  // zeroed V rows (if any) before the MMA reads them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok && !warp_wait_bounded(pv_done, (nt - 1) & 1, p.status)) ok = false;
    tc_fence_after();
    // ---- epilogue: row r of O / l ------------------------------------------------------
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int64_t orow = static_cast<int64_t>(q0 + row / G) * Hq + hk * G + row % G;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t u[32];
      tmem_ld32(tmem_o + lane_off + 32 * c, u);
      tmem_ld_wait(u);
      if (!valid || !ok) continue;
      if (nparts == 1) {
        __nv_bfloat16* dst = out + orow * D + 32 * c;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(u[e + 2 * k]) * inv,
                                                     __uint_as_float(u[e + 2 * k + 1]) * inv);
            w[k] = *reinterpret_cast<uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(dst + e) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
        float* dst = p.ws_o + (orow * p.max_partitions + part) * D + 32 * c;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) =
              make_float4(__uint_as_float(u[e]) * inv, __uint_as_float(u[e + 1]) * inv,
                          __uint_as_float(u[e + 2]) * inv, __uint_as_float(u[e + 3]) * inv);
      }
    }
    if (valid && ok && nparts > 1) {
      const int64_t srow = orow * p.max_partitions + part;
      p.ws_ml[srow * 2] = l > 0.f ? m * kLn2 : 0.f;
      p.ws_ml[srow * 2 + 1] = l;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

}  // namespace pkv

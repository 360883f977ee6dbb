// decode.cuh -- paged single-query decode attention: partition pass + reduce.
//
// What is computed ("vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点):
// for each sequence b and query head hq, attention of q[b,hq] over the
// sequence's K/V, where logical token t lives in row t % block_size of the
// physical block block_tables[b][t / block_size] -- one table load and one
// multiply per block, then the usual q.K^T, softmax and weighted sum of V.
//
// Grid: one CTA per (kv head, partition, sequence).  A partition is a run of
// partition_blocks logical blocks; with grouped-query attention the CTA serves
// all G query heads that share the KV head, so every K/V byte is read from
// HBM once per step.
//
// Inside a CTA four warps each own a private TMA pipeline of NS stages.  A
// stage holds one (block, kv head) tile of K and of V: block_size rows of
// head_dim contiguous elements at the pool's row stride, fetched by one 4-D
// tensor-map load each (box {head_dim, 1, block_size, 1}).  Warp w takes the
// partition's blocks w, w+4, w+8, ... and keeps its own online-softmax state
// (running max m, running sum l, unnormalised accumulator); the four states
// are merged in shared memory at the end.
//
// QK^T: a token row is split over TG = head_dim / 8 lanes, 8 elements each,
// so one warp instruction covers 32 / TG tokens; the partial dots are summed
// with xor shuffles.  Softmax works in base 2: q is pre-multiplied by
// scale * log2(e) (and by the fp8 K scale), so e^{s-m} = 2^{s2-m2}.
// P.V: lane l owns head_dim / 32 consecutive output elements and walks the
// block's valid rows; the probabilities come from a per-warp shared array.
//
// A sequence with a single partition gets its normalised output written
// directly.  Otherwise every partition writes (m, l, o = acc / l) to the
// workspace and paged_decode_reduce_kernel merges them:
//     out = sum_p l_p e^{m_p - M} o_p / sum_p l_p e^{m_p - M}.
#pragma once

#include "common.cuh"

namespace pkv {

struct DecodeParams {
  void* out;                    // [B][Hq][D] of TQ
  const void* q;                // [B][Hq][D] of TQ
  const int32_t* block_tables;  // [B][max_blocks_per_seq]
  const int32_t* context_lens;  // [B]
  float* ws_ml;                 // [B][Hq][P][2]: reference logit m (natural units), l = sum e^{s-m}
  float* ws_o;                  // [B][Hq][P][D]: normalised partial outputs
  unsigned* status;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int num_blocks;
  int block_size;
  int partition_blocks;
  int max_partitions;
  float q_scale;    // scale * log2(e) * (fp8 ? k_scale : 1)
  float out_scale;  // fp8 ? v_scale : 1
  // Fused append (pkv_paged_decode_append): new_k/new_v [B][Hkv][D] in q's
  // dtype, written to logical position context_lens[b] - 1 before it is read.
  // NULL for plain decode.
  const void* new_k;
  const void* new_v;
  void* key_cache;
  void* value_cache;
  float k_inv;  // fp8 caches: 1/k_scale and 1/v_scale rounded to fp32
  float v_inv;
  // Shared-prefix decode (pkv_paged_attention_decode_shared_prefix): groups of
  // consecutive sequences whose first shared_blocks[g] logical blocks are the
  // same physical blocks.  Partial slots [0, shared_partitions) of a
  // (sequence, head) hold its group's shared-prefix partials, the slots from
  // shared_partitions on its own blocks'.  group_start is NULL otherwise.
  const int32_t* group_start = nullptr;    // [num_groups + 1]
  const int32_t* shared_blocks = nullptr;  // [num_groups]
  int num_groups = 0;
  int shared_partitions = 0;
};

// The group holding sequence b (group_start is non-decreasing; the last g with
// group_start[g] <= b).
__device__ __forceinline__ int group_of_sequence(const DecodeParams& p, int b) {
  int lo = 0, hi = p.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (p.group_start[mid] <= b) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Shared blocks of group g, clamped to what the table and the context allow.
__device__ __forceinline__ int shared_blocks_of(const DecodeParams& p, int g, int nblk) {
  const int s = p.shared_blocks[g];
  return s < 0 ? 0 : (s > nblk ? nblk : s);
}

// Fused append: the CTA that reads the last block of sequence b writes that
// sequence's new token for its kv head (row (ctx-1) % BS of physical block
// block_tables[b][(ctx-1) / BS]) -- a copy, or for fp8 one fp32 multiply and
// a round-to-nearest saturating E4M3 encode, exactly as paged_kv_write_kernel
// -- and fences the generic writes against the TMA reads that follow.  An id
// outside the pool writes nothing (the partition pass reports it).
template <typename TQ, typename TC, int D, int BS>
__device__ __forceinline__ void append_new_token(const DecodeParams& p, int b, int hk, int ctx, int tid,
                                                 int nthreads) {
  const int t = ctx - 1;
  const int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + t / BS];
  if (id < 0 || id >= p.num_blocks) return;
  const int64_t dst = ((static_cast<int64_t>(id) * BS + t % BS) * p.num_kv_heads + hk) * D;
  const int64_t src = (static_cast<int64_t>(b) * p.num_kv_heads + hk) * D;
  const TQ* kin = static_cast<const TQ*>(p.new_k) + src;
  const TQ* vin = static_cast<const TQ*>(p.new_v) + src;
  for (int c8 = tid; c8 < D / 8; c8 += nthreads) {
    if constexpr (sizeof(TQ) == sizeof(TC)) {
      constexpr int kVec = 8 * sizeof(TQ) / 16;
      const uint4* ks = reinterpret_cast<const uint4*>(kin + 8 * c8);
      const uint4* vs = reinterpret_cast<const uint4*>(vin + 8 * c8);
      uint4* kd = reinterpret_cast<uint4*>(static_cast<TC*>(p.key_cache) + dst + 8 * c8);
      uint4* vd = reinterpret_cast<uint4*>(static_cast<TC*>(p.value_cache) + dst + 8 * c8);
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        kd[i] = ks[i];
        vd[i] = vs[i];
      }
    } else {
      uint8_t kb[8], vb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kb[e] = __nv_cvt_float_to_fp8(__fmul_rn(Elem<TQ>::to_float(kin[8 * c8 + e]), p.k_inv), __NV_SATFINITE,
                                      __NV_E4M3);
        vb[e] = __nv_cvt_float_to_fp8(__fmul_rn(Elem<TQ>::to_float(vin[8 * c8 + e]), p.v_inv), __NV_SATFINITE,
                                      __NV_E4M3);
      }
      uint2 kw, vw;
      kw.x = kb[0] | (kb[1] << 8) | (kb[2] << 16) | (uint32_t(kb[3]) << 24);
      kw.y = kb[4] | (kb[5] << 8) | (kb[6] << 16) | (uint32_t(kb[7]) << 24);
      vw.x = vb[0] | (vb[1] << 8) | (vb[2] << 16) | (uint32_t(vb[3]) << 24);
      vw.y = vb[4] | (vb[5] << 8) | (vb[6] << 16) | (uint32_t(vb[7]) << 24);
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.key_cache) + dst + 8 * c8) = kw;
      *reinterpret_cast<uint2*>(static_cast<uint8_t*>(p.value_cache) + dst + 8 * c8) = vw;
    }
  }
  fence_proxy_async_global();
}

// NW warps per CTA, each with a private pipeline of NS stages (0: about 8 KB of
// stages per warp).  Small CTAs win: with ~34 KB of shared memory per CTA six
// CTAs share an SM, and while one warp computes the others' loads stay in
// flight (a sweep on B200 put 4 warps x 1 stage of 8 KB at 96% of the
// streaming rate of the same TMA pattern without compute).
template <typename TQ, typename TC, int D, int BS, int G, int NW_ = 4, int NS_ = 0>
struct DecodeTraits {
  static constexpr int NW = NW_;
  static constexpr int ES = Elem<TC>::kBytes;
  static constexpr int ROW_BYTES = D * ES;          // one token of one kv head
  static constexpr int TILE_BYTES = BS * ROW_BYTES; // one (block, kv head) of K or V
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  static constexpr int NS = NS_ > 0 ? NS_ : ((8192 / STAGE_BYTES) >= 1 ? 8192 / STAGE_BYTES : 1);
  static constexpr int TG = D / 8;                  // lanes per token row in q.K
  static constexpr int TPI = 32 / TG;               // tokens per warp instruction
  static constexpr int NIT = BS / TPI;              // q.K steps per block
  static constexpr int PVV = D / 32;                // output elements per lane
  static constexpr int STAGE_AREA = NW * NS * STAGE_BYTES;
  static constexpr int COMBINE_BYTES = NW * G * (D + 2) * 4;
  static constexpr int DATA_BYTES = STAGE_AREA > COMBINE_BYTES ? STAGE_AREA : COMBINE_BYTES;
  static constexpr int BAR_BYTES = NW * NS * 8;
  static constexpr int Q_BYTES = G * D * 4;
  static constexpr int P_BYTES = NW * G * BS * 4;
  static_assert(32 % TG == 0 && BS % TPI == 0, "tile mapping");
  static_assert(TILE_BYTES % 16 == 0, "TMA boxes are multiples of 16 bytes");

  // Dynamic shared memory for a partition of pb blocks (1 KB alignment slack).
  static constexpr size_t smem_bytes(int pb) {
    return 1024 + DATA_BYTES + BAR_BYTES + Q_BYTES + P_BYTES + static_cast<size_t>(pb) * 4;
  }
};

// Reads N consecutive elements of T at p (N * sizeof(T) in {2, 4, 8, 16, 32}).
template <typename T, int N>
__device__ __forceinline__ void load_elems(const uint8_t* p, float* out) {
  constexpr int bytes = N * Elem<T>::kBytes;
  if constexpr (bytes == 2) {
    const uint32_t w = *reinterpret_cast<const uint16_t*>(p);
    float tmp[4];
    Elem<T>::unpack_word(w, tmp);
    out[0] = tmp[0];
    out[1] = tmp[1];
  } else if constexpr (bytes == 4) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    unpack<T, N>(&w, out);
  } else if constexpr (bytes == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    const uint32_t ws[2] = {w.x, w.y};
    unpack<T, N>(ws, out);
  } else if constexpr (bytes == 16) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    unpack<T, N>(ws, out);
  } else {
    static_assert(bytes == 32, "unsupported slice");
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint4 c = *reinterpret_cast<const uint4*>(p + 16);
    const uint32_t ws[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
    unpack<T, N>(ws, out);
  }
}

// Merges the NW warp states of one CTA (left in shared memory as c_m[w][g],
// c_l[w][g] in base-2 units and c_acc[w][g][D] unnormalised) and writes the
// normalised output row (single partition) or the partition's (m, l, o)
// partial.  Called by all threads of the CTA after a __syncthreads().
template <typename TQ, int D, int G, int NW>
__device__ __forceinline__ void finish_partition(const float* c_m, const float* c_l, const float* c_acc,
                                                 const DecodeParams& p, int64_t out_row0, int part, int nparts) {
  TQ* out = static_cast<TQ*>(p.out);
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, e = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, c_m[w * G + g]);
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float f = fast_exp2(c_m[w * G + g] - M);  // warps without blocks: 2^-inf = 0
      L = fmaf(c_l[w * G + g], f, L);
      O = fmaf(c_acc[(w * G + g) * D + e], f, O);
    }
    const float o = L > 0.f ? O / L * p.out_scale : 0.f;
    if (nparts == 1) {
      out[(out_row0 + g) * D + e] = Elem<TQ>::from_float(o);
    } else {
      const int64_t slot = (out_row0 + g) * p.max_partitions + part;
      const uint64_t keep = l2_policy_evict_last();
      st_global_hint(p.ws_o + slot * D + e, o, keep);
      if (e == 0) {
        st_global_hint(p.ws_ml + slot * 2, M * kLn2, keep);
        st_global_hint(p.ws_ml + slot * 2 + 1, L, keep);
      }
    }
  }
}

template <typename TQ, typename TC, int D, int BS, int G, int NW = 4, int NS = 0, int MINB = 1>
__global__ void __launch_bounds__(NW * 32, MINB)
    paged_decode_partition_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                                  const DecodeParams p) {
  using T = DecodeTraits<TQ, TC, D, BS, G, NW, NS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(data + T::DATA_BYTES);
  float* q_s = reinterpret_cast<float*>(data + T::DATA_BYTES + T::BAR_BYTES);
  float* p_s = q_s + G * D;
  int* ids = reinterpret_cast<int*>(p_s + T::NW * G * BS);

  pdl_wait_and_release();
  const int hk = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = p.num_q_heads;
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[b];
  if (ctx < 0 || ctx > max_ctx) {
    if (threadIdx.x == 0 && hk == 0 && part == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int pb = p.partition_blocks;
  const int nparts = (nblk + pb - 1) / pb;
  TQ* out = static_cast<TQ*>(p.out);
  const int64_t out_row0 = static_cast<int64_t>(b) * Hq + hk * G;  // first query head of the group
  if (nparts == 0) {  // empty context: a zero output row
    if (part == 0)
      for (int i = threadIdx.x; i < G * D; i += blockDim.x) out[out_row0 * D + i] = Elem<TQ>::from_float(0.f);
    return;
  }
  if (part >= nparts) return;
  const int blk0 = part * pb;
  const int nb = min(pb, nblk - blk0);

  // Block-table lookups for the whole partition, with the pool-range guard.
  for (int i = threadIdx.x; i < nb; i += blockDim.x) {
    int id = p.block_tables[static_cast<int64_t>(b) * p.max_blocks_per_seq + blk0 + i];
    if (id < 0 || id >= p.num_blocks) {
      set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
      id = -1;
    }
    ids[i] = id;
  }
  // q of the G heads, pre-scaled into the base-2 logit domain.
  for (int i = threadIdx.x; i < G * D; i += blockDim.x)
    q_s[i] = Elem<TQ>::to_float(static_cast<const TQ*>(p.q)[out_row0 * D + i]) * p.q_scale;
  const bool append = p.new_k != nullptr && part == nparts - 1;
  if (append) append_new_token<TQ, TC, D, BS>(p, b, hk, ctx, threadIdx.x, blockDim.x);
  const uint32_t bar0 = smem_u32(bars) + warp * T::NS * 8;
  if (lane == 0) {
    for (int s = 0; s < T::NS; ++s) mbar_init(bar0 + 8 * s, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (append && lane == 0) fence_proxy_async_global();

  const int n_w = nb > warp ? (nb - warp + T::NW - 1) / T::NW : 0;  // blocks of this warp
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
      mbar_arrive(bar);  // bad id: nothing to fetch, the block is skipped
    }
  };
  if (lane == 0) {
    const int pre = n_w < T::NS ? n_w : T::NS;
    for (int i = 0; i < pre; ++i) issue(i);
  }

  const int gi = lane / T::TG;  // token slot within a q.K instruction
  const int gl = lane % T::TG;  // 8-element slice of the row
  float m[G], l[G], acc[G][T::PVV];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < T::PVV; ++e) acc[g][e] = 0.f;
  }
  float* pw = p_s + warp * G * BS;

  int waited = 0;  // stages whose load this warp has waited for
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
      const uint8_t* kt = data + warp * T::NS * T::STAGE_BYTES + s * T::STAGE_BYTES;
      const uint8_t* vt = kt + T::TILE_BYTES;
      const int valid = min(BS, ctx - (blk0 + j) * BS);  // >= 1
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float qf[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[e] = q_s[g * D + gl * 8 + e];
        float sc[T::NIT];
#pragma unroll
        for (int it = 0; it < T::NIT; ++it) {
          const int t = it * T::TPI + gi;
          float kf[8];
          load_elems<TC, 8>(kt + t * T::ROW_BYTES + gl * 8 * T::ES, kf);
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qf[e], kf[e], a);
#pragma unroll
          for (int off = T::TG / 2; off > 0; off >>= 1) a += __shfl_xor_sync(kFullMask, a, off);
          sc[it] = t < valid ? a : -INFINITY;
        }
        float bm = -INFINITY;
#pragma unroll
        for (int it = 0; it < T::NIT; ++it) bm = fmaxf(bm, sc[it]);
#pragma unroll
        for (int off = T::TG; off < 32; off <<= 1) bm = fmaxf(bm, __shfl_xor_sync(kFullMask, bm, off));
        const float mn = fmaxf(m[g], bm);
        const float alpha = fast_exp2(m[g] - mn);
        float ps = 0.f;
#pragma unroll
        for (int it = 0; it < T::NIT; ++it) {
          sc[it] = fast_exp2(sc[it] - mn);
          ps += sc[it];
        }
#pragma unroll
        for (int off = T::TG; off < 32; off <<= 1) ps += __shfl_xor_sync(kFullMask, ps, off);
        l[g] = l[g] * alpha + ps;
#pragma unroll
        for (int e = 0; e < T::PVV; ++e) acc[g][e] *= alpha;
        m[g] = mn;
        if (gl == 0) {
#pragma unroll
          for (int it = 0; it < T::NIT; ++it) pw[g * BS + it * T::TPI + gi] = sc[it];
        }
      }
      __syncwarp();
      for (int t = 0; t < valid; ++t) {  // rows past the context are never read
        float vf[T::PVV];
        load_elems<TC, T::PVV>(vt + t * T::ROW_BYTES + lane * T::PVV * T::ES, vf);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pt = pw[g * BS + t];
#pragma unroll
          for (int e = 0; e < T::PVV; ++e) acc[g][e] = fmaf(pt, vf[e], acc[g][e]);
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
    // Drain: wait (bounded) for every load still in flight before the
    // shared memory is released.
    const int issued = min(n_w, waited + T::NS);
    for (int i = waited; i < issued; ++i) mbar_wait_bounded(bar0 + 8 * (i % T::NS), (i / T::NS) & 1, p.status);
  }
  __syncthreads();  // every warp is done with the stage area

  float* c_m = reinterpret_cast<float*>(data);
  float* c_l = c_m + T::NW * G;
  float* c_acc = c_l + T::NW * G;
  if (lane == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      c_m[warp * G + g] = m[g];
      c_l[warp * G + g] = l[g];
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < T::PVV; ++e) c_acc[(warp * G + g) * D + lane * T::PVV + e] = acc[g][e];
  __syncthreads();
  finish_partition<TQ, D, G, T::NW>(c_m, c_l, c_acc, p, out_row0, part, nparts);
}

// PVV consecutive floats of a partial output (16- or 8-byte aligned: offsets are multiples of PVV).
template <int PVV>
__device__ __forceinline__ void load_partial(const float* src, float (&v)[PVV]) {
  if constexpr (PVV == 4) {
    const float4 x = *reinterpret_cast<const float4*>(src);
    v[0] = x.x;
    v[1] = x.y;
    v[2] = x.z;
    v[3] = x.w;
  } else if constexpr (PVV == 2) {
    const float2 x = *reinterpret_cast<const float2*>(src);
    v[0] = x.x;
    v[1] = x.y;
  } else {
#pragma unroll
    for (int e = 0; e < PVV; ++e) v[e] = src[e];
  }
}

// Merge of split-context partials, one warp per (sequence, query head).  BATCH partial outputs are
// loaded at once (8 or 16: the registers they take set how many CTAs share an SM, so launches whose
// rows have at most 8 partitions use 8).
template <typename TQ, int D, int BATCH = 16>
__global__ void __launch_bounds__(128) paged_decode_reduce_kernel(const DecodeParams p) {
  constexpr int PVV = D / 32;
  pdl_wait_and_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  if (row >= static_cast<int64_t>(p.num_seqs) * p.num_q_heads) return;
  const int b = static_cast<int>(row / p.num_q_heads);
  const int BS = p.block_size;
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[b];
  ctx = ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx);
  const int nblk = (ctx + BS - 1) / BS;
  // slots [0, n0) and [s1, s1 + n1): one range for plain decode, the group's
  // shared-prefix partials and the sequence's own for shared-prefix decode
  int n0, s1 = 0, n1 = 0;
  if (p.group_start) {  // every partial is merged here, even a single one
    const int sh = shared_blocks_of(p, group_of_sequence(p, b), nblk);
    n0 = (sh + p.partition_blocks - 1) / p.partition_blocks;
    s1 = p.shared_partitions;
    n1 = (nblk - sh + p.partition_blocks - 1) / p.partition_blocks;
  } else {
    n0 = (nblk + p.partition_blocks - 1) / p.partition_blocks;
    if (n0 <= 1) return;  // written by the partition pass
  }
  const int nparts = n0 + n1;
  auto slot = [&](int i) { return i < n0 ? i : s1 + (i - n0); };
  const float* ml = p.ws_ml + row * p.max_partitions * 2;
  const float* o = p.ws_o + row * p.max_partitions * D;
  TQ* out = static_cast<TQ*>(p.out) + row * D + lane * PVV;
  if (nparts <= 64) {
    // Lane i holds (m, l) of partitions i and i + 32; the partial outputs are read BATCH partitions
    // at a time, every load of a batch in flight at once, the first batch beside the (m, l) loads.
    // The arithmetic and its order are those of the general loop below (the same results).
    float m0 = -INFINITY, l0 = 0.f, m1 = -INFINITY, l1 = 0.f;
    if (lane < nparts) {
      const float2 x = *reinterpret_cast<const float2*>(ml + 2 * slot(lane));
      m0 = x.x;
      l0 = x.y;
    }
    if (lane + 32 < nparts) {
      const float2 x = *reinterpret_cast<const float2*>(ml + 2 * slot(lane + 32));
      m1 = x.x;
      l1 = x.y;
    }
    float v[BATCH][PVV];
    auto load_batch = [&](int c) {
#pragma unroll
      for (int q = 0; q < BATCH; ++q)
        if (c + q < nparts) load_partial<PVV>(o + static_cast<int64_t>(slot(c + q)) * D + lane * PVV, v[q]);
    };
    load_batch(0);
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
    const float w0 = l0 > 0.f ? l0 * fast_exp2((m0 - M) * kLog2e) : 0.f;
    const float w1 = l1 > 0.f ? l1 * fast_exp2((m1 - M) * kLog2e) : 0.f;
    float acc[PVV];
#pragma unroll
    for (int e = 0; e < PVV; ++e) acc[e] = 0.f;
    for (int c = 0; c < nparts; c += BATCH) {
      if (c > 0) load_batch(c);
      const float wsrc = c < 32 ? w0 : w1;  // (a batch never straddles partition 32)
#pragma unroll
      for (int q = 0; q < BATCH; ++q) {
        if (c + q < nparts) {
          const float w = __shfl_sync(kFullMask, wsrc, (c + q) & 31);
#pragma unroll
          for (int e = 0; e < PVV; ++e) acc[e] = fmaf(w, v[q][e], acc[e]);
        }
      }
    }
    float W = w0 + w1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(kFullMask, W, off);
#pragma unroll
    for (int e = 0; e < PVV; ++e) out[e] = Elem<TQ>::from_float(W > 0.f ? acc[e] / W : 0.f);
    return;
  }
  // Partitions are taken 32 at a time: lane i loads (m, l) of partition c + i at once, the weights
  // l e^{m - M} go to the other lanes by shuffle, and the partial outputs are read four at a time,
  // so the loads of a row overlap instead of following one another.
  float M = -INFINITY;
  for (int i = lane; i < nparts; i += 32) M = fmaxf(M, ml[2 * slot(i)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
  float acc[PVV];
#pragma unroll
  for (int e = 0; e < PVV; ++e) acc[e] = 0.f;
  float W = 0.f;
  for (int c = 0; c < nparts; c += 32) {
    const int n = min(32, nparts - c);
    float wl = 0.f;  // this lane's partition c + lane
    if (lane < n) {
      const int i = slot(c + lane);
      const float li = ml[2 * i + 1];
      wl = li > 0.f ? li * fast_exp2((ml[2 * i] - M) * kLog2e) : 0.f;
    }
    W += wl;
    int k = 0;
    for (; k + 4 <= n; k += 4) {
      float w4[4], v[4][PVV];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        w4[q] = __shfl_sync(kFullMask, wl, k + q);
        const float* oi = o + static_cast<int64_t>(slot(c + k + q)) * D + lane * PVV;
#pragma unroll
        for (int e = 0; e < PVV; ++e) v[q][e] = oi[e];
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int e = 0; e < PVV; ++e) acc[e] = fmaf(w4[q], v[q][e], acc[e]);
    }
    for (; k < n; ++k) {
      const float w = __shfl_sync(kFullMask, wl, k);
      const float* oi = o + static_cast<int64_t>(slot(c + k)) * D + lane * PVV;
#pragma unroll
      for (int e = 0; e < PVV; ++e) acc[e] = fmaf(w, oi[e], acc[e]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) W += __shfl_xor_sync(kFullMask, W, off);
#pragma unroll
  for (int e = 0; e < PVV; ++e) out[e] = Elem<TQ>::from_float(W > 0.f ? acc[e] / W : 0.f);
}

}  // namespace pkv

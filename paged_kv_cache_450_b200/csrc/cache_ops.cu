// cache_ops.cu -- the two data-movement companions of paged decode.
//
// paged_kv_write_kernel: the new-token KV write ("vLLM 与 KV Cache",
// KV Cache：为什么需要缓存 -- each step computes the new token's K,V only and
// appends them).  Token t goes to row slot % block_size of block
// slot / block_size; with the [block][row][kv head][dim] layout a token's
// K (and V) row of num_kv_heads * head_dim elements is contiguous both in the
// input and in the cache, so the write is a row copy (or an fp8 encode).
//
// kv_block_copy_kernel: copy-on-write copies ("vLLM — 把操作系统的分页搬进
// GPU KV cache", 核心要点 引用计数 + copy-on-write): one physical block of
// both caches copied onto another, 16 bytes per thread access.
#include "common.cuh"
#include "launch.h"

namespace pkv {

// One CTA per token; each thread handles 8-element chunks of the K and V rows.
template <typename TI, typename TC>
__global__ void __launch_bounds__(256)
    paged_kv_write_kernel(const TI* __restrict__ k, const TI* __restrict__ v, const int64_t* __restrict__ slots,
                          TC* __restrict__ kc, TC* __restrict__ vc, int64_t num_blocks, int block_size,
                          int row_elems, float k_inv, float v_inv, unsigned* status) {
  pdl_wait_and_release();
  const int64_t t = blockIdx.x;
  const int64_t slot = slots[t];
  if (slot < 0) return;  // padding token
  if (slot >= num_blocks * block_size) {
    if (threadIdx.x == 0) set_status(status, PKV_STATUS_BAD_SLOT);
    return;
  }
  // (block, row) = (slot / bs, slot % bs); the row starts at element
  // (block * bs + row) * row_elems == slot * row_elems.
  const int64_t dst0 = slot * row_elems;
  const int64_t src0 = t * row_elems;
  const int chunks = row_elems / 8;
  for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
    const int64_t si = src0 + c * 8, di = dst0 + c * 8;
    if constexpr (sizeof(TI) == sizeof(TC)) {
      // same type: copy the bytes
      constexpr int kVec = 8 * sizeof(TI) / 16;  // uint4 per chunk
      const uint4* ks = reinterpret_cast<const uint4*>(k + si);
      const uint4* vs = reinterpret_cast<const uint4*>(v + si);
      uint4* kd = reinterpret_cast<uint4*>(kc + di);
      uint4* vd = reinterpret_cast<uint4*>(vc + di);
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        kd[i] = ks[i];
        vd[i] = vs[i];
      }
    } else {
      // fp8 cache: code = E4M3_satfinite_rn(x * (1/scale)), one fp32 multiply.
      float kx[8], vx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kx[e] = Elem<TI>::to_float(k[si + e]);
        vx[e] = Elem<TI>::to_float(v[si + e]);
      }
      uint8_t kb[8], vb[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        kb[e] = __nv_cvt_float_to_fp8(__fmul_rn(kx[e], k_inv), __NV_SATFINITE, __NV_E4M3);
        vb[e] = __nv_cvt_float_to_fp8(__fmul_rn(vx[e], v_inv), __NV_SATFINITE, __NV_E4M3);
      }
      uint2 kw, vw;
      kw.x = kb[0] | (kb[1] << 8) | (kb[2] << 16) | (uint32_t(kb[3]) << 24);
      kw.y = kb[4] | (kb[5] << 8) | (kb[6] << 16) | (uint32_t(kb[7]) << 24);
      vw.x = vb[0] | (vb[1] << 8) | (vb[2] << 16) | (uint32_t(vb[3]) << 24);
      vw.y = vb[4] | (vb[5] << 8) | (vb[6] << 16) | (uint32_t(vb[7]) << 24);
      *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(kc) + di) = kw;
      *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(vc) + di) = vw;
    }
  }
}

// grid.x: chunks of one block, grid.y: pairs (strided).  4 x 16 B per thread.
__global__ void __launch_bounds__(256)
    kv_block_copy_kernel(const int64_t* __restrict__ pairs, int64_t num_pairs, uint8_t* kc, uint8_t* vc,
                         int64_t num_blocks, int64_t block_bytes, unsigned* status) {
  constexpr int kIlp = 4;
  pdl_wait_and_release();
  const int64_t vecs = block_bytes / 16;
  for (int64_t pi = blockIdx.y; pi < num_pairs; pi += gridDim.y) {
    const int64_t src = pairs[2 * pi], dst = pairs[2 * pi + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, PKV_STATUS_BAD_COPY_PAIR);
      continue;
    }
    const uint4* ks = reinterpret_cast<const uint4*>(kc + src * block_bytes);
    const uint4* vs = reinterpret_cast<const uint4*>(vc + src * block_bytes);
    uint4* kd = reinterpret_cast<uint4*>(kc + dst * block_bytes);
    uint4* vd = reinterpret_cast<uint4*>(vc + dst * block_bytes);
    const int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x * kIlp + threadIdx.x;
    uint4 a[kIlp], c[kIlp];
#pragma unroll
    for (int i = 0; i < kIlp; ++i) {
      const int64_t x = base + i * blockDim.x;
      if (x < vecs) {
        a[i] = ks[x];
        c[i] = vs[x];
      }
    }
#pragma unroll
    for (int i = 0; i < kIlp; ++i) {
      const int64_t x = base + i * blockDim.x;
      if (x < vecs) {
        kd[x] = a[i];
        vd[x] = c[i];
      }
    }
  }
}

template <typename TI, typename TC>
static cudaError_t launch_write(const KvWriteArgs& a, cudaStream_t st) {
  const int row_elems = a.num_kv_heads * a.head_dim;
  const int chunks = row_elems / 8;
  const int threads = chunks >= 256 ? 256 : ((chunks + 31) / 32) * 32;
  return launch_pdl(paged_kv_write_kernel<TI, TC>, dim3(static_cast<unsigned>(a.num_tokens)), dim3(threads), 0, st,
                    static_cast<const TI*>(a.k), static_cast<const TI*>(a.v), a.slot_mapping,
                    static_cast<TC*>(a.key_cache), static_cast<TC*>(a.value_cache), a.num_blocks, a.block_size,
                    row_elems, a.k_inv, a.v_inv, a.status);
}

cudaError_t launch_kv_write(const KvWriteArgs& a, cudaStream_t st) {
  if (a.in_dtype == PKV_DTYPE_F32 && a.cache_dtype == PKV_DTYPE_F32) return launch_write<float, float>(a, st);
  if (a.in_dtype == PKV_DTYPE_BF16 && a.cache_dtype == PKV_DTYPE_BF16)
    return launch_write<__nv_bfloat16, __nv_bfloat16>(a, st);
  if (a.in_dtype == PKV_DTYPE_F32 && a.cache_dtype == PKV_DTYPE_FP8_E4M3)
    return launch_write<float, __nv_fp8_e4m3>(a, st);
  if (a.in_dtype == PKV_DTYPE_BF16 && a.cache_dtype == PKV_DTYPE_FP8_E4M3)
    return launch_write<__nv_bfloat16, __nv_fp8_e4m3>(a, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_block_copy(const int64_t* pairs, int64_t num_pairs, void* kc, void* vc, int64_t num_blocks,
                              int64_t block_bytes, unsigned* status, cudaStream_t st) {
  const int64_t vecs = block_bytes / 16;
  const int64_t per_cta = 256 * 4;
  const unsigned gx = static_cast<unsigned>((vecs + per_cta - 1) / per_cta);
  const unsigned gy = static_cast<unsigned>(num_pairs < 65535 ? num_pairs : 65535);
  return launch_pdl(kv_block_copy_kernel, dim3(gx, gy), dim3(256), 0, st, pairs, num_pairs, static_cast<uint8_t*>(kc),
                    static_cast<uint8_t*>(vc), num_blocks, block_bytes, status);
}

}  // namespace pkv

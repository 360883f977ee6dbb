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
// Copies block src of the source pool onto block dst of the destination pool
// in both caches.  The copy-on-write copy uses one pool for both; the swap
// between the device pool and a pinned host pool passes host pointers on one
// side (unified addressing: the kernel reads or writes host memory directly,
// so any number of blocks moves in one launch).
__global__ void __launch_bounds__(256)
    kv_block_copy_kernel(const int64_t* __restrict__ pairs, int64_t num_pairs, const uint8_t* src_k,
                         const uint8_t* src_v, int64_t src_blocks, uint8_t* dst_k, uint8_t* dst_v, int64_t dst_blocks,
                         int64_t block_bytes, unsigned* status) {
  constexpr int kIlp = 4;
  pdl_wait_and_release();
  const int64_t vecs = block_bytes / 16;
  for (int64_t pi = blockIdx.y; pi < num_pairs; pi += gridDim.y) {
    const int64_t src = pairs[2 * pi], dst = pairs[2 * pi + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
      if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, PKV_STATUS_BAD_COPY_PAIR);
      continue;
    }
    const uint4* ks = reinterpret_cast<const uint4*>(src_k + src * block_bytes);
    const uint4* vs = reinterpret_cast<const uint4*>(src_v + src * block_bytes);
    uint4* kd = reinterpret_cast<uint4*>(dst_k + dst * block_bytes);
    uint4* vd = reinterpret_cast<uint4*>(dst_v + dst * block_bytes);
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

// amax(|x|) of n elements into *amax_bits (the float's bits: for non-negative
// floats the unsigned order is the float order, so atomicMax works; the word
// must be zero first).  Grid-stride, 8 elements per thread per step.
template <typename T>
__global__ void __launch_bounds__(256) amax_kernel(const T* __restrict__ x, int64_t n, unsigned* amax_bits) {
  pdl_wait_and_release();
  float m = 0.f;
  const int64_t n8 = n / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    if constexpr (sizeof(T) == 2) {
      const uint4 w = reinterpret_cast<const uint4*>(x)[i];
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = fmaxf(m, fabsf(__uint_as_float(ws[k] << 16)));
        m = fmaxf(m, fabsf(__uint_as_float(ws[k] & 0xffff0000u)));
      }
    } else {
      const float4 a = reinterpret_cast<const float4*>(x)[2 * i], b = reinterpret_cast<const float4*>(x)[2 * i + 1];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
      m = fmaxf(m, fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
    }
  }
  if (blockIdx.x == 0 && threadIdx.x < n - 8 * n8) m = fmaxf(m, fabsf(Elem<T>::to_float(x[8 * n8 + threadIdx.x])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

// scale = amax / 448 (one fp32 division), or 1 when amax is 0.
__global__ void fp8_scale_finish_kernel(unsigned* word) {
  pdl_wait_and_release();
  const float amax = __uint_as_float(*word);
  *reinterpret_cast<float*>(word) = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
}

cudaError_t launch_fp8_scale(const void* x, int64_t n, int dtype, float* scale, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(scale, 0, sizeof(float), st);
  if (e != cudaSuccess) return e;
  unsigned* word = reinterpret_cast<unsigned*>(scale);
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t n8 = n / 8;
  int64_t grid = (n8 + 255) / 256;
  if (grid > 8LL * sms) grid = 8LL * sms;
  if (grid < 1) grid = 1;
  if (dtype == PKV_DTYPE_BF16)
    e = launch_pdl(amax_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st,
                   static_cast<const __nv_bfloat16*>(x), n, word);
  else
    e = launch_pdl(amax_kernel<float>, dim3(static_cast<unsigned>(grid)), dim3(256), 0, st,
                   static_cast<const float*>(x), n, word);
  if (e != cudaSuccess) return e;
  return launch_pdl(fp8_scale_finish_kernel, dim3(1), dim3(1), 0, st, word);
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

cudaError_t launch_block_copy(const int64_t* pairs, int64_t num_pairs, const void* src_k, const void* src_v,
                              int64_t src_blocks, void* dst_k, void* dst_v, int64_t dst_blocks, int64_t block_bytes,
                              unsigned* status, cudaStream_t st) {
  const int64_t vecs = block_bytes / 16;
  const int64_t per_cta = 256 * 4;
  const unsigned gx = static_cast<unsigned>((vecs + per_cta - 1) / per_cta);
  const unsigned gy = static_cast<unsigned>(num_pairs < 65535 ? num_pairs : 65535);
  return launch_pdl(kv_block_copy_kernel, dim3(gx, gy), dim3(256), 0, st, pairs, num_pairs,
                    static_cast<const uint8_t*>(src_k), static_cast<const uint8_t*>(src_v), src_blocks,
                    static_cast<uint8_t*>(dst_k), static_cast<uint8_t*>(dst_v), dst_blocks, block_bytes, status);
}

}  // namespace pkv

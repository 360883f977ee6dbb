// decode_launch.cuh -- host-side dispatch of the decode kernels for one
// (q dtype, cache dtype) pair.  Included by one .cu per pair so the template
// instances compile in parallel.
#pragma once

#include <type_traits>

#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_mma_bf16.cuh"
#include "launch.h"

namespace pkv {

template <typename TQ, typename TC, int D, int BS, int G>
static cudaError_t launch_partition(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                   int num_kv_heads, cudaStream_t st) {
  using T = DecodeTraits<TQ, TC, D, BS, G>;
  auto kern = paged_decode_partition_kernel<TQ, TC, D, BS, G>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(num_kv_heads, p.max_partitions, p.num_seqs);
  return launch_pdl(kern, grid, dim3(T::NW * 32), smem, st, kmap, vmap, p);
}

template <typename TQ, int BS>
static cudaError_t launch_mma(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p, int num_kv_heads,
                              cudaStream_t st) {
  using T = MmaTraits<BS>;
  auto kern = paged_decode_gqa8_fp8_mma_kernel<TQ, BS>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(num_kv_heads, p.max_partitions, p.num_seqs);
  return launch_pdl(kern, grid, dim3(32), smem, st, kmap, vmap, p);
}

template <int BS, int G>
static cudaError_t launch_mma_bf16(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                   int num_kv_heads, cudaStream_t st) {
  using T = MmaBf16Traits<BS>;
  auto kern = paged_decode_mma_bf16_kernel<BS, G>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(num_kv_heads, p.max_partitions, p.num_seqs);
  return launch_pdl(kern, grid, dim3(32), smem, st, kmap, vmap, p);
}

// Shared-prefix decode: grid z = the groups' shared units, then one unit per
// sequence for its own blocks; the merge always runs.
template <int BS, int G>
static cudaError_t launch_mma_bf16_grouped(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                           int num_kv_heads, int grid_partitions, cudaStream_t st) {
  using T = MmaBf16Traits<BS>;
  auto kern = paged_decode_mma_bf16_kernel<BS, G, true>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(num_kv_heads, grid_partitions, p.num_groups + p.num_seqs);
  return launch_pdl(kern, grid, dim3(32), smem, st, kmap, vmap, p);
}

template <typename TQ, int D>
static cudaError_t launch_reduce(const DecodeParams& p, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.num_seqs) * p.num_q_heads;
  if (p.max_partitions <= 8)
    return launch_pdl(paged_decode_reduce_kernel<TQ, D, 8>, dim3(static_cast<unsigned>((rows + 3) / 4)), dim3(128), 0,
                      st, p);
  return launch_pdl(paged_decode_reduce_kernel<TQ, D>, dim3(static_cast<unsigned>((rows + 3) / 4)), dim3(128), 0, st,
                    p);
}

template <typename TQ, typename TC, int D, int BS>
static cudaError_t dispatch_group(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p, int group,
                                  int num_kv_heads, cudaStream_t st) {
  if constexpr (std::is_same_v<TC, __nv_fp8_e4m3> && D == 128 && (BS == 16 || BS == 32)) {
    if (group == 8) return launch_mma<TQ, BS>(kmap, vmap, p, num_kv_heads, st);
  }
  if constexpr (std::is_same_v<TC, __nv_bfloat16> && std::is_same_v<TQ, __nv_bfloat16> && D == 128 &&
                (BS == 16 || BS == 32)) {
    switch (group) {
      case 1: break;  // MHA: CUDA-core kernel below
      case 2: return launch_mma_bf16<BS, 2>(kmap, vmap, p, num_kv_heads, st);
      case 4: return launch_mma_bf16<BS, 4>(kmap, vmap, p, num_kv_heads, st);
      case 8: return launch_mma_bf16<BS, 8>(kmap, vmap, p, num_kv_heads, st);
      default: return cudaErrorInvalidValue;
    }
  }
  // (decode_uses_mma() in launch.h makes the same choice for the tensor maps.)
  switch (group) {
    case 1: return launch_partition<TQ, TC, D, BS, 1>(kmap, vmap, p, num_kv_heads, st);
    case 2: return launch_partition<TQ, TC, D, BS, 2>(kmap, vmap, p, num_kv_heads, st);
    case 4: return launch_partition<TQ, TC, D, BS, 4>(kmap, vmap, p, num_kv_heads, st);
    case 8: return launch_partition<TQ, TC, D, BS, 8>(kmap, vmap, p, num_kv_heads, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ, typename TC, int D>
static cudaError_t dispatch_block(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p, int group,
                                  int num_kv_heads, cudaStream_t st) {
  switch (p.block_size) {
    case 8: return dispatch_group<TQ, TC, D, 8>(kmap, vmap, p, group, num_kv_heads, st);
    case 16: return dispatch_group<TQ, TC, D, 16>(kmap, vmap, p, group, num_kv_heads, st);
    case 32: return dispatch_group<TQ, TC, D, 32>(kmap, vmap, p, group, num_kv_heads, st);
    default: return cudaErrorInvalidValue;
  }
}

template <typename TQ, typename TC>
static cudaError_t dispatch_decode(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                   int head_dim, int group, int num_kv_heads, bool reduce, cudaStream_t st) {
  cudaError_t e;
  switch (head_dim) {
    case 64: e = dispatch_block<TQ, TC, 64>(kmap, vmap, p, group, num_kv_heads, st); break;
    case 128: e = dispatch_block<TQ, TC, 128>(kmap, vmap, p, group, num_kv_heads, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || !reduce) return e;
  return head_dim == 64 ? launch_reduce<TQ, 64>(p, st) : launch_reduce<TQ, 128>(p, st);
}

template <int BS>
static cudaError_t dispatch_grouped_group(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                          int group, int num_kv_heads, int grid_partitions, cudaStream_t st) {
  switch (group) {
    case 1: return launch_mma_bf16_grouped<BS, 1>(kmap, vmap, p, num_kv_heads, grid_partitions, st);
    case 2: return launch_mma_bf16_grouped<BS, 2>(kmap, vmap, p, num_kv_heads, grid_partitions, st);
    case 4: return launch_mma_bf16_grouped<BS, 4>(kmap, vmap, p, num_kv_heads, grid_partitions, st);
    case 8: return launch_mma_bf16_grouped<BS, 8>(kmap, vmap, p, num_kv_heads, grid_partitions, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pkv

#define PKV_DEFINE_DECODE(NAME, TQ, TC)                                                                       \
  namespace pkv {                                                                                             \
  cudaError_t NAME(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p, int head_dim,     \
                   int group, int num_kv_heads, bool reduce, cudaStream_t st) {                               \
    return dispatch_decode<TQ, TC>(kmap, vmap, p, head_dim, group, num_kv_heads, reduce, st);                \
  }                                                                                                           \
  }

// multiquery_launch.cuh -- launch of the mma.sync multi-query kernel, shared by
// its bf16-cache (multiquery_bf16.cu) and fp8-cache (multiquery_fp8.cu)
// instantiation units.
#pragma once

#include "launch.h"
#include "multiquery.cuh"

namespace pkv {

template <int BS, int G, int NWC, bool F8>
static cudaError_t launch_mq(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                             int n_qtiles, bool reduce, cudaStream_t st) {
  using T = MqTraits<BS, NWC, 0, F8>;
  auto kern = paged_multiquery_mma_kernel<BS, G, NWC, F8>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.num_kv_heads) * n_qtiles, p.max_partitions, p.num_seqs);
  e = launch_pdl(kern, grid, dim3(T::THREADS), smem, st, kmap, vmap, p);
  if (e != cudaSuccess || !reduce) return e;
  return launch_multiquery_reduce(p, st);
}

template <int BS, int NWC, bool F8>
static cudaError_t dispatch_mq_group(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                                     int group, int n_qtiles, bool reduce, cudaStream_t st) {
  switch (group) {
    case 1: return launch_mq<BS, 1, NWC, F8>(kmap, vmap, p, n_qtiles, reduce, st);
    case 2: return launch_mq<BS, 2, NWC, F8>(kmap, vmap, p, n_qtiles, reduce, st);
    case 4: return launch_mq<BS, 4, NWC, F8>(kmap, vmap, p, n_qtiles, reduce, st);
    case 8: return launch_mq<BS, 8, NWC, F8>(kmap, vmap, p, n_qtiles, reduce, st);
    default: return cudaErrorInvalidValue;
  }
}

// One compute warp per 16 rows of a (sequence, KV head), at most four; more
// rows are split over query-row tiles (grid x = KV heads x tiles).
template <bool F8>
static cudaError_t launch_multiquery_mma_t(const CUtensorMap& kmap, const CUtensorMap& vmap,
                                           const MultiQueryParams& p, int group, int rows_per_seq, bool reduce,
                                           cudaStream_t st) {
  const int nwc = multiquery_compute_warps(rows_per_seq);
  const int n_qtiles = (rows_per_seq + 16 * nwc - 1) / (16 * nwc);
  if (p.block_size != 16 && p.block_size != 32) return cudaErrorInvalidValue;
  const bool b16 = p.block_size == 16;
  switch (nwc) {
    case 1: return b16 ? dispatch_mq_group<16, 1, F8>(kmap, vmap, p, group, n_qtiles, reduce, st)
                       : dispatch_mq_group<32, 1, F8>(kmap, vmap, p, group, n_qtiles, reduce, st);
    case 2: return b16 ? dispatch_mq_group<16, 2, F8>(kmap, vmap, p, group, n_qtiles, reduce, st)
                       : dispatch_mq_group<32, 2, F8>(kmap, vmap, p, group, n_qtiles, reduce, st);
    case 3: return b16 ? dispatch_mq_group<16, 3, F8>(kmap, vmap, p, group, n_qtiles, reduce, st)
                       : dispatch_mq_group<32, 3, F8>(kmap, vmap, p, group, n_qtiles, reduce, st);
    default: return b16 ? dispatch_mq_group<16, 4, F8>(kmap, vmap, p, group, n_qtiles, reduce, st)
                        : dispatch_mq_group<32, 4, F8>(kmap, vmap, p, group, n_qtiles, reduce, st);
  }
}

}  // namespace pkv

// multiquery_tc.cu -- launcher of the tcgen05 multi-query attention kernel
// (bf16 and fp8 caches).
#include "launch.h"
#include "multiquery_tc.cuh"

namespace pkv {

// Persistent launch: one CTA per SM (fewer when there are fewer work units);
// each CTA takes units c, c + CTAs, ... of the longest-first unit list.
static int sm_count_of_device() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  return n;
}

template <int BS, int G, bool F8, bool STACK>
static cudaError_t launch_mq_tc_kind(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                     const MultiQueryParams& p, int n_qtiles, bool reduce, cudaStream_t st) {
  using T = MqTcTraits<BS, F8, STACK>;
  auto kern = paged_multiquery_tc_kernel<BS, G, F8, STACK>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(p.num_kv_heads) * n_qtiles * p.max_partitions * p.num_seqs;
  const int64_t ctas = units < sm_count_of_device() ? units : sm_count_of_device();
  if (ctas <= 0) return cudaSuccess;
  e = launch_pdl(kern, dim3(static_cast<unsigned>(ctas)), dim3(T::THREADS), smem, st, qmap, kmap, vmap, p);
  if (e != cudaSuccess || !reduce) return e;
  return launch_multiquery_reduce(p, st);
}

// bf16 caches with at most 64 query rows per (sequence, KV head): the stacked tile
template <int BS, int G, bool F8>
static cudaError_t launch_mq_tc(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                const MultiQueryParams& p, int n_qtiles, bool reduce, cudaStream_t st) {
  if constexpr (!F8) {
    if (p.max_q_len * G <= 64) return launch_mq_tc_kind<BS, G, F8, true>(qmap, kmap, vmap, p, 1, reduce, st);
  }
  return launch_mq_tc_kind<BS, G, F8, false>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
}

template <int BS, bool F8>
static cudaError_t dispatch_mq_tc_group(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                        const MultiQueryParams& p, int group, int n_qtiles, bool reduce,
                                        cudaStream_t st) {
  switch (group) {
    case 1: return launch_mq_tc<BS, 1, F8>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
    case 2: return launch_mq_tc<BS, 2, F8>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
    case 4: return launch_mq_tc<BS, 4, F8>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
    case 8: return launch_mq_tc<BS, 8, F8>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_multiquery_tc(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                 const MultiQueryParams& p, int group, int rows_per_seq, bool fp8, bool reduce,
                                 cudaStream_t st) {
  const int n_qtiles = (rows_per_seq + 127) / 128;
  switch (p.block_size) {
    case 16: return fp8 ? dispatch_mq_tc_group<16, true>(qmap, kmap, vmap, p, group, n_qtiles, reduce, st)
                        : dispatch_mq_tc_group<16, false>(qmap, kmap, vmap, p, group, n_qtiles, reduce, st);
    case 32: return fp8 ? dispatch_mq_tc_group<32, true>(qmap, kmap, vmap, p, group, n_qtiles, reduce, st)
                        : dispatch_mq_tc_group<32, false>(qmap, kmap, vmap, p, group, n_qtiles, reduce, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace pkv

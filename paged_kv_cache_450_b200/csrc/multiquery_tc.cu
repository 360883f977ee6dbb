// multiquery_tc.cu -- launcher of the tcgen05 multi-query attention kernel
// (bf16 and fp8 caches).
#include "launch.h"
#include "multiquery_tc.cuh"

namespace pkv {

template <int BS, int G, bool F8, int ROWS>
static cudaError_t launch_mq_tc_rows(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                     const MultiQueryParams& p, int n_qtiles, bool reduce, cudaStream_t st) {
  using T = MqTcTraits<BS, F8, ROWS>;
  auto kern = paged_multiquery_tc_kernel<BS, G, F8, ROWS>;
  const size_t smem = T::smem_bytes(p.partition_blocks);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(p.num_kv_heads) * n_qtiles, p.max_partitions, p.num_seqs);
  e = launch_pdl(kern, grid, dim3(T::THREADS), smem, st, qmap, kmap, vmap, p);
  if (e != cudaSuccess || !reduce) return e;
  return launch_multiquery_reduce(p, st);
}

// n_qtiles counts 128-row tiles.  bf16 caches with at most 64 rows per (sequence, KV head) run the
// stacked 64-row tile (one MMA per P . V k-step instead of two).
template <int BS, int G, bool F8>
static cudaError_t launch_mq_tc(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                const MultiQueryParams& p, int n_qtiles, bool reduce, cudaStream_t st) {
  if constexpr (!F8) {
    if (p.max_q_len * G <= 64) return launch_mq_tc_rows<BS, G, F8, 64>(qmap, kmap, vmap, p, 1, reduce, st);
  }
  return launch_mq_tc_rows<BS, G, F8, 128>(qmap, kmap, vmap, p, n_qtiles, reduce, st);
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

// launch.h -- internal interface between the C ABI (abi.cu) and the kernel
// translation units.  Host code only; no CUDA kernels are declared here.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace pkv {

struct DecodeParams;
struct MultiQueryParams;

// Counts one kernel launch (pkv_launch_count()).
void count_launch();

// Launches `kern` on `st` with programmatic stream serialisation (the kernel
// starts with griddepcontrol.wait, see common.cuh) and counts the launch.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

struct KvWriteArgs {
  const void* k;
  const void* v;
  const int64_t* slot_mapping;
  int64_t num_tokens;
  void* key_cache;
  void* value_cache;
  int64_t num_blocks;
  int block_size;
  int num_kv_heads;
  int head_dim;
  int in_dtype;
  int cache_dtype;
  float k_inv;  // 1/k_scale rounded to fp32 (fp8 caches)
  float v_inv;
  unsigned* status;
};

cudaError_t launch_kv_write(const KvWriteArgs& a, cudaStream_t st);
cudaError_t launch_fp8_scale(const void* x, int64_t n, int dtype, float* scale, cudaStream_t st);
cudaError_t launch_block_copy(const int64_t* pairs, int64_t num_pairs, const void* src_k, const void* src_v,
                              int64_t src_blocks, void* dst_k, void* dst_v, int64_t dst_blocks, int64_t block_bytes,
                              unsigned* status, cudaStream_t st);

// The decode grid's block-table reads alone (a measurement aid, table_scan.cu).
cudaError_t launch_table_scan(const int32_t* tables, const int32_t* lens, int num_seqs, int num_kv_heads,
                              int max_blocks_per_seq, int num_blocks, int block_size, int partition_blocks,
                              int num_partitions, unsigned* sink, unsigned* status, cudaStream_t st);

// A warp waits on an mbarrier nothing completes, with a short limit (selftest.cu).
cudaError_t launch_wait_timeout_selftest(unsigned* status, uint64_t limit_ns, unsigned* gave_up, cudaStream_t st);

// The tensor-core decode kernels serve head_dim 128 with 16- or 32-token
// blocks: fp8 caches with 8 query heads per KV head, and bf16 caches with 2,
// 4 or 8 (grouped-query attention, where CUDA-core work grows with the
// group).  Their cache tensor maps use the 128-byte swizzle (boxes of one
// 128-byte row segment).  Everything else -- MHA included, which is at the
// memory limit on CUDA cores and measured slightly faster there (more warps
// per SM keep more loads in flight) -- runs on the CUDA-core kernel.
inline bool decode_uses_mma(int cache_dtype, int head_dim, int group, int block_size) {
  if (head_dim != 128 || (block_size != 16 && block_size != 32)) return false;
  if (cache_dtype == 2 /* PKV_DTYPE_FP8_E4M3 */) return group == 8;
  if (cache_dtype == 1 /* PKV_DTYPE_BF16 */) return group == 2 || group == 4 || group == 8;
  return false;
}

// Multi-query (prefill / verification) attention: bf16 q, bf16 or fp8 caches,
// head_dim 128, bs 16/32.  Up to 16 rows per (sequence, KV head)
// -- rows = queries x query heads of the group -- run on the mma.sync kernel
// (one 16-row warp per CTA); more rows on the tcgen05 kernel with 128-row
// tiles, whose time per KV tile does not depend on how many of the rows are
// used (measured: 40 rows, 70B-GQA verification, 2.70 TB/s on mma.sync with
// three 16-row warps, 3.56 TB/s on tcgen05).  The same split for fp8 caches.
#ifndef PKV_MQ_TC_MIN_ROWS
#define PKV_MQ_TC_MIN_ROWS 16
#endif
inline bool multiquery_uses_tc(int rows_per_seq) { return rows_per_seq > PKV_MQ_TC_MIN_ROWS; }
// Compute warps (16 rows each) per CTA of the mma.sync kernel, and its
// resident CTAs per SM.
inline int multiquery_compute_warps(int rows_per_seq) {
  const int w = (rows_per_seq + 15) / 16;
  return w < 1 ? 1 : (w > 4 ? 4 : w);
}
inline int multiquery_ctas_per_sm(int compute_warps) {
  return compute_warps == 1 ? 6 : (compute_warps == 2 ? 4 : (compute_warps == 3 ? 3 : 2));
}
// The mma.sync kernel over bf16 caches and over fp8 (E4M3) caches.
cudaError_t launch_multiquery_mma_bf16(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                                       int group, int rows_per_seq, bool reduce, cudaStream_t st);
cudaError_t launch_multiquery_mma_fp8(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                                      int group, int rows_per_seq, bool reduce, cudaStream_t st);
cudaError_t launch_multiquery_tc(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vmap,
                                 const MultiQueryParams& p, int group, int rows_per_seq, bool fp8, bool reduce,
                                 cudaStream_t st);
// The split-context merge of either multi-query kernel.
cudaError_t launch_multiquery_reduce(const MultiQueryParams& p, cudaStream_t st);

// Decode launchers, one per (q dtype, cache dtype); each dispatches on
// head_dim, block_size and the query-head group.  `reduce` adds the merge
// kernel (sequences with more than one partition).
#define PKV_DECLARE_DECODE(NAME)                                                                            \
  cudaError_t NAME(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p, int head_dim, \
                   int group, int num_kv_heads, bool reduce, cudaStream_t st);
PKV_DECLARE_DECODE(launch_decode_f32_f32)
PKV_DECLARE_DECODE(launch_decode_bf16_bf16)
PKV_DECLARE_DECODE(launch_decode_f32_fp8)
PKV_DECLARE_DECODE(launch_decode_bf16_fp8)
#undef PKV_DECLARE_DECODE
// Shared-prefix decode, bf16 q and cache, head_dim 128, bs 16/32 (the merge included).
cudaError_t launch_decode_shared_prefix_bf16(const CUtensorMap& kmap, const CUtensorMap& vmap, const DecodeParams& p,
                                             int group, int num_kv_heads, int grid_partitions, cudaStream_t st);

}  // namespace pkv

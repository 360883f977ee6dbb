// multiquery_bf16.cu -- the mma.sync multi-query kernel over bf16 caches, and
// the split-context merge shared by every multi-query kernel.
#include "multiquery_launch.cuh"

namespace pkv {

// Merge of split-context partials, one warp per (query token, query head).
__global__ void __launch_bounds__(128) paged_multiquery_reduce_kernel(const MultiQueryParams p) {
  constexpr int D = 128, PVV = D / 32;
  pdl_wait_and_release();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  if (row >= static_cast<int64_t>(p.total_q) * p.num_q_heads) return;
  const int tok = static_cast<int>(row / p.num_q_heads);
  int lo = 0, hi = p.num_seqs - 1;  // the sequence owning query token tok
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (p.query_start_loc[mid] <= tok) lo = mid; else hi = mid - 1;
  }
  int q0, q_len;  // a row of no sequence, or of one the partition pass skipped, is not written
  if (!query_rows_ok(p, lo, q0, q_len) || tok < q0 || tok >= q0 + q_len) return;
  const int BS = p.block_size;
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = p.context_lens[lo];
  ctx = ctx < 0 ? 0 : (ctx > max_ctx ? max_ctx : ctx);
  const int pos = ctx - q_len + (tok - q0);
  const int nparts = ((ctx + BS - 1) / BS + p.partition_blocks - 1) / p.partition_blocks;
  if (nparts <= 1) return;  // written directly by the partition pass
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * D + lane * PVV;
  if (pos < 0) {  // a query before the context: attends nothing
#pragma unroll
    for (int e = 0; e < PVV; ++e) out[e] = __float2bfloat16_rn(0.f);
    return;
  }
  const int nvis = min(nparts, pos / (p.partition_blocks * BS) + 1);  // partitions the query can see
  const float* ml = p.ws_ml + row * p.max_partitions * 2;
  const float* o = p.ws_o + row * p.max_partitions * D;
  float M = -INFINITY;
  for (int i = lane; i < nvis; i += 32)
    if (ml[2 * i + 1] > 0.f) M = fmaxf(M, ml[2 * i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
  float acc[PVV];
#pragma unroll
  for (int e = 0; e < PVV; ++e) acc[e] = 0.f;
  float W = 0.f;
  for (int i = 0; i < nvis; ++i) {
    const float li = ml[2 * i + 1];
    const float w = li > 0.f ? li * fast_exp2((ml[2 * i] - M) * kLog2e) : 0.f;
    W += w;
    const float* oi = o + static_cast<int64_t>(i) * D + lane * PVV;
#pragma unroll
    for (int e = 0; e < PVV; ++e) acc[e] = fmaf(w, oi[e], acc[e]);
  }
#pragma unroll
  for (int e = 0; e < PVV; ++e) out[e] = __float2bfloat16_rn(W > 0.f ? acc[e] / W : 0.f);
}

cudaError_t launch_multiquery_reduce(const MultiQueryParams& p, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.total_q) * p.num_q_heads;
  return launch_pdl(paged_multiquery_reduce_kernel, dim3(static_cast<unsigned>((rows + 3) / 4)), dim3(128), 0, st, p);
}

cudaError_t launch_multiquery_mma_bf16(const CUtensorMap& kmap, const CUtensorMap& vmap, const MultiQueryParams& p,
                                       int group, int rows_per_seq, bool reduce, cudaStream_t st) {
  return launch_multiquery_mma_t<false>(kmap, vmap, p, group, rows_per_seq, reduce, st);
}

}  // namespace pkv

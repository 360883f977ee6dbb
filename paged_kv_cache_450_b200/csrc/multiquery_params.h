// multiquery_params.h -- arguments of the multi-query attention kernels
// (shared by the launcher and the C ABI).
#pragma once

#include <stdint.h>

namespace pkv {

struct MultiQueryParams {
  void* out;                       // [total_q][Hq][D] bf16
  const void* q;                   // [total_q][Hq][D] bf16
  const int32_t* block_tables;     // [B][max_blocks_per_seq]
  const int32_t* context_lens;     // [B]
  const int32_t* query_start_loc;  // [B + 1]
  float* ws_ml;                    // [total_q * Hq][P][2]
  float* ws_o;                     // [total_q * Hq][P][D]
  unsigned* status;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int max_blocks_per_seq;
  int num_blocks;
  int block_size;
  int partition_blocks;
  int max_partitions;
  int total_q;
  int max_q_len;  // q_len of any sequence must not exceed it (the grid covers that many rows)
  float q_scale;    // scale * log2(e) (* k_scale for fp8 caches)
  float out_scale;  // v_scale for fp8 caches, else 1
};

#ifdef __CUDACC__
// The query rows of sequence b, [q0, q0 + q_len).  False (nothing of the
// sequence may be touched) when they leave [0, total_q) or q_len exceeds
// max_q_len, the most rows the launch grid covers per sequence.
__device__ __forceinline__ bool query_rows_ok(const MultiQueryParams& p, int b, int& q0, int& q_len) {
  const int64_t a = p.query_start_loc[b], e = p.query_start_loc[b + 1];
  q0 = static_cast<int>(a);
  q_len = static_cast<int>(e - a);
  return a >= 0 && e >= a && e <= p.total_q && e - a <= p.max_q_len;
}
#endif

}  // namespace pkv

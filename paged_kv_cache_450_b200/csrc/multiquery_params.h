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
  float q_scale;  // scale * log2(e)
};

}  // namespace pkv

// table_scan.cu -- the block-table reads of a decode launch, alone.
//
// A measurement aid.  The decode partition pass (decode.cuh) starts every
// (kv head, partition, sequence) CTA by reading the partition's physical
// block ids from the sequence's block table -- the "one more int load" of
// "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 -- with the pool-range
// guard, and then streams the blocks.  This kernel runs the same grid and the
// same coalesced, guarded id reads and nothing else, so that its time and its
// L2 hit rate isolate what the indirection costs.  Each CTA folds its ids into
// one word written to `sink` (so the reads cannot be dropped).
#include "common.cuh"
#include "launch.h"

namespace pkv {

__global__ void __launch_bounds__(32)
    decode_table_scan_kernel(const int32_t* __restrict__ tables, const int32_t* __restrict__ lens,
                             int max_blocks_per_seq, int num_blocks, int block_size, int partition_blocks,
                             unsigned* __restrict__ sink, unsigned* status) {
  pdl_wait_and_release();
  const int hk = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int max_ctx = max_blocks_per_seq * block_size;
  int ctx = lens[b];
  if (ctx < 0 || ctx > max_ctx) {
    if (threadIdx.x == 0 && hk == 0 && part == 0) set_status(status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + block_size - 1) / block_size;
  const int nparts = (nblk + partition_blocks - 1) / partition_blocks;
  unsigned acc = 0;
  if (part < nparts) {
    const int blk0 = part * partition_blocks;
    const int nb = min(partition_blocks, nblk - blk0);
    const int32_t* row = tables + static_cast<int64_t>(b) * max_blocks_per_seq + blk0;
    for (int i = threadIdx.x; i < nb; i += 32) {
      int id = row[i];
      if (id < 0 || id >= num_blocks) {
        set_status(status, PKV_STATUS_BAD_BLOCK_ID);
        id = -1;
      }
      acc ^= static_cast<unsigned>(id) * 2654435761u + static_cast<unsigned>(i);
    }
  }
  acc = __reduce_xor_sync(kFullMask, acc);
  if (threadIdx.x == 0) sink[(static_cast<int64_t>(b) * gridDim.y + part) * gridDim.x + hk] = acc;
}

cudaError_t launch_table_scan(const int32_t* tables, const int32_t* lens, int num_seqs, int num_kv_heads,
                              int max_blocks_per_seq, int num_blocks, int block_size, int partition_blocks,
                              int num_partitions, unsigned* sink, unsigned* status, cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(num_kv_heads), static_cast<unsigned>(num_partitions),
            static_cast<unsigned>(num_seqs));
  return launch_pdl(decode_table_scan_kernel, grid, dim3(32), 0, st, tables, lens, max_blocks_per_seq, num_blocks,
                    block_size, partition_blocks, sink, status);
}

}  // namespace pkv

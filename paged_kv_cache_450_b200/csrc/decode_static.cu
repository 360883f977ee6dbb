// decode_static.cu -- paged decode attention for callers that cannot hand the
// library a scratch buffer.
//
// pkv_paged_attention_decode needs device scratch for the split-context
// partials and takes it from the caller.  Some callers have none to give:
// an engine that reserved nearly all of HBM for its KV block pool up front
// and keeps no allocator for temporaries, code that must not call cudaMalloc
// in the middle of a decode step because cudaMalloc can synchronise the whole
// device, or a binding from an environment without any device allocator.
// This entry point serves them from a fixed array compiled into the library
// and allocates nothing itself.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pagedkv.h"

namespace {

constexpr size_t kScratchBytes = PKV_DECODE_STATIC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Split-context scratch shared by every call on a device.  It lives as long
// as the library's code is loaded on that device (until the process exits).
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device.  In host code the
// symbol name is only a host-side handle, never a device pointer, so the
// address is looked up once per device (with that device current) and cached.
void* scratch_address(int* status) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = PKV_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
      *status = PKV_ERR_CUDA;
      return nullptr;
    }
    g_scratch_addr[dev] = p;
  }
  *status = PKV_OK;
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int pkv_paged_attention_decode_static(void* out, const void* q, const void* key_cache,
                                                 const void* value_cache, const int32_t* block_tables,
                                                 const int32_t* context_lens, int num_seqs, int num_q_heads,
                                                 int num_kv_heads, int head_dim, int block_size,
                                                 int max_blocks_per_seq, int64_t num_blocks, float scale,
                                                 float k_scale, float v_scale, int q_dtype, int cache_dtype,
                                                 int partition_tokens, void* stream) {
  const size_t need = pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                 max_blocks_per_seq, cache_dtype, partition_tokens);
  if (need == 0 || need > kScratchBytes) {
    // No partials (one partition per sequence, an empty batch or arguments the
    // decode rejects), or more than the array holds: the workspace entry point
    // without a workspace gives the same answer -- its argument errors first,
    // PKV_OK for an empty batch, PKV_ERR_WORKSPACE (nothing launched) when
    // partials are needed -- and the array's address is not looked up.
    return pkv_paged_attention_decode(out, q, key_cache, value_cache, block_tables, context_lens, num_seqs,
                                      num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                                      num_blocks, scale, k_scale, v_scale, q_dtype, cache_dtype, partition_tokens,
                                      nullptr, 0, /*validate=*/0, stream);
  }
  int status = PKV_OK;
  void* scratch = scratch_address(&status);
  if (!scratch) return status;
  // The partials are written before they are read, so nothing is cleared.
  return pkv_paged_attention_decode(out, q, key_cache, value_cache, block_tables, context_lens, num_seqs,
                                    num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
                                    scale, k_scale, v_scale, q_dtype, cache_dtype, partition_tokens, scratch,
                                    kScratchBytes, /*validate=*/0, stream);
}

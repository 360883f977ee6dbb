// step_host.cu -- one decode step whose per-step inputs and output live in
// host memory: the copies in, the three operations and the copy out, all
// enqueued on the caller's stream by one call (for serving loops that keep
// the KV cache on the device and everything else on the host).
#include <cuda_runtime.h>

#include "../../include/pagedkv.h"

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t dtype_bytes(int dtype) {
  switch (dtype) {
    case PKV_DTYPE_F32: return 4;
    case PKV_DTYPE_BF16: return 2;
    case PKV_DTYPE_FP8_E4M3: return 1;
    default: return 0;
  }
}

// Offsets of the staged pieces inside the staging buffer.
struct StagingLayout {
  size_t q, out, k, v, slots, tables, lens, pairs, workspace, workspace_bytes, total;
};

bool layout(StagingLayout* L, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
            int max_blocks_per_seq, int q_dtype, int cache_dtype, int partition_tokens, int64_t num_tokens,
            int64_t num_pairs) {
  const size_t es = dtype_bytes(q_dtype);
  if (!es || num_seqs < 0 || num_tokens < 0 || num_pairs < 0 || max_blocks_per_seq <= 0) return false;
  const size_t qb = static_cast<size_t>(num_seqs) * num_q_heads * head_dim * es;
  const size_t kb = static_cast<size_t>(num_tokens) * num_kv_heads * head_dim * es;
  size_t off = 0;
  L->q = off;
  off = align256(off + qb);
  L->out = off;
  off = align256(off + qb);
  L->k = off;
  off = align256(off + kb);
  L->v = off;
  off = align256(off + kb);
  L->slots = off;
  off = align256(off + static_cast<size_t>(num_tokens) * sizeof(int64_t));
  L->tables = off;
  off = align256(off + static_cast<size_t>(num_seqs) * max_blocks_per_seq * sizeof(int32_t));
  L->lens = off;
  off = align256(off + static_cast<size_t>(num_seqs) * sizeof(int32_t));
  L->pairs = off;
  off = align256(off + static_cast<size_t>(num_pairs) * 2 * sizeof(int64_t));
  L->workspace = off;
  L->workspace_bytes = num_seqs > 0 ? pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                                                 block_size, max_blocks_per_seq, cache_dtype,
                                                                 partition_tokens)
                                    : 0;
  L->total = align256(off + L->workspace_bytes);
  return true;
}

bool h2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return true;
  return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st) == cudaSuccess;
}

}  // namespace

extern "C" size_t pkv_decode_step_staging_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                                int block_size, int max_blocks_per_seq, int q_dtype, int cache_dtype,
                                                int partition_tokens, int64_t num_tokens, int64_t num_pairs) {
  StagingLayout L;
  if (!layout(&L, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, q_dtype,
              cache_dtype, partition_tokens, num_tokens, num_pairs))
    return 0;
  return L.total;
}

namespace {

// Records an event on `from` and makes `to` wait for it (nothing when the
// streams are the same).  The event is released at once; CUDA keeps it alive
// until the wait has been satisfied.
bool order(cudaStream_t from, cudaStream_t to) {
  if (from == to) return true;
  cudaEvent_t ev;
  if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return false;
  const bool ok = cudaEventRecord(ev, from) == cudaSuccess && cudaStreamWaitEvent(to, ev, 0) == cudaSuccess;
  cudaEventDestroy(ev);
  return ok;
}

// The step with its copies in on `in`, kernels on `comp`, copy out on `out`;
// `wait_ev` (optional) gates the copies in, `done_ev` (optional) is recorded
// after the copy out.
int step_host(void* out_host, const void* q_host, const void* k_host, const void* v_host,
              const int64_t* slot_mapping_host, int64_t num_tokens, const int32_t* block_tables_host,
              const int32_t* context_lens_host, const int64_t* copy_pairs_host, int64_t num_pairs, void* key_cache,
              void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
              int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale, float v_scale, int q_dtype,
              int cache_dtype, int partition_tokens, void* staging, size_t staging_bytes, cudaStream_t in,
              cudaStream_t comp, cudaStream_t outs, cudaEvent_t wait_ev, cudaEvent_t done_ev) {
  if (num_seqs < 0 || num_tokens < 0 || num_pairs < 0) return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0 && num_tokens == 0 && num_pairs == 0) return PKV_OK;
  if (!staging || !key_cache || !value_cache) return PKV_ERR_NULL_POINTER;
  if (num_seqs > 0 && (!out_host || !q_host || !block_tables_host || !context_lens_host)) return PKV_ERR_NULL_POINTER;
  if (num_tokens > 0 && (!k_host || !v_host || !slot_mapping_host)) return PKV_ERR_NULL_POINTER;
  if (num_pairs > 0 && !copy_pairs_host) return PKV_ERR_NULL_POINTER;
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return PKV_ERR_MISALIGNED;
  const int pt = num_seqs > 0 ? pkv_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                            max_blocks_per_seq, cache_dtype, partition_tokens)
                              : 0;
  if (pt < 0) return pt;
  StagingLayout L;
  if (!layout(&L, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, q_dtype, cache_dtype,
              partition_tokens, num_tokens, num_pairs))
    return PKV_ERR_BAD_DTYPE;
  if (staging_bytes < L.total) return PKV_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(staging);
  cudaStream_t st = in;
  void* stream = static_cast<void*>(comp);  // the kernels' stream
  const size_t es = dtype_bytes(q_dtype);
  const size_t qb = static_cast<size_t>(num_seqs) * num_q_heads * head_dim * es;
  const size_t kb = static_cast<size_t>(num_tokens) * num_kv_heads * head_dim * es;
  // Copies in (after the caller's event: the previous user of this staging buffer is done).
  if (wait_ev && cudaStreamWaitEvent(in, wait_ev, 0) != cudaSuccess) return PKV_ERR_CUDA;
  if (!h2d(base + L.q, q_host, qb, st) || !h2d(base + L.k, k_host, kb, st) || !h2d(base + L.v, v_host, kb, st) ||
      !h2d(base + L.slots, slot_mapping_host, static_cast<size_t>(num_tokens) * sizeof(int64_t), st) ||
      !h2d(base + L.tables, block_tables_host,
           static_cast<size_t>(num_seqs) * max_blocks_per_seq * sizeof(int32_t), st) ||
      !h2d(base + L.lens, context_lens_host, static_cast<size_t>(num_seqs) * sizeof(int32_t), st) ||
      !h2d(base + L.pairs, copy_pairs_host, static_cast<size_t>(num_pairs) * 2 * sizeof(int64_t), st))
    return PKV_ERR_CUDA;
  if (!order(in, comp)) return PKV_ERR_CUDA;
  int rc;
  if (num_pairs > 0) {
    const int64_t block_bytes =
        static_cast<int64_t>(block_size) * num_kv_heads * head_dim * static_cast<int64_t>(dtype_bytes(cache_dtype));
    rc = pkv_kv_block_copy(reinterpret_cast<const int64_t*>(base + L.pairs), num_pairs, key_cache, value_cache,
                           num_blocks, block_bytes, 0, stream);
    if (rc) return rc;
  }
  if (num_tokens > 0) {
    rc = pkv_paged_kv_write(base + L.k, base + L.v, reinterpret_cast<const int64_t*>(base + L.slots), num_tokens,
                            key_cache, value_cache, num_blocks, block_size, num_kv_heads, head_dim, q_dtype,
                            cache_dtype, k_scale, v_scale, 0, stream);
    if (rc) return rc;
  }
  if (num_seqs > 0) {
    rc = pkv_paged_attention_decode(base + L.out, base + L.q, key_cache, value_cache,
                                    reinterpret_cast<const int32_t*>(base + L.tables),
                                    reinterpret_cast<const int32_t*>(base + L.lens), num_seqs, num_q_heads,
                                    num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale,
                                    v_scale, q_dtype, cache_dtype, pt, base + L.workspace, L.workspace_bytes, 0,
                                    stream);
    if (rc) return rc;
    // Copy out.
    if (!order(comp, outs)) return PKV_ERR_CUDA;
    if (cudaMemcpyAsync(out_host, base + L.out, qb, cudaMemcpyDeviceToHost, outs) != cudaSuccess) return PKV_ERR_CUDA;
  } else if (!order(comp, outs)) {
    return PKV_ERR_CUDA;
  }
  if (done_ev && cudaEventRecord(done_ev, outs) != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

}  // namespace

extern "C" int pkv_decode_step_host(void* out_host, const void* q_host, const void* k_host, const void* v_host,
                                    const int64_t* slot_mapping_host, int64_t num_tokens,
                                    const int32_t* block_tables_host, const int32_t* context_lens_host,
                                    const int64_t* copy_pairs_host, int64_t num_pairs, void* key_cache,
                                    void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                                    int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale,
                                    float k_scale, float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                                    void* staging, size_t staging_bytes, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return step_host(out_host, q_host, k_host, v_host, slot_mapping_host, num_tokens, block_tables_host,
                   context_lens_host, copy_pairs_host, num_pairs, key_cache, value_cache, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale, v_scale,
                   q_dtype, cache_dtype, partition_tokens, staging, staging_bytes, st, st, st, nullptr, nullptr);
}

extern "C" int pkv_decode_step_host_async(void* out_host, const void* q_host, const void* k_host,
                                          const void* v_host, const int64_t* slot_mapping_host, int64_t num_tokens,
                                          const int32_t* block_tables_host, const int32_t* context_lens_host,
                                          const int64_t* copy_pairs_host, int64_t num_pairs, void* key_cache,
                                          void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads,
                                          int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks,
                                          float scale, float k_scale, float v_scale, int q_dtype, int cache_dtype,
                                          int partition_tokens, void* staging, size_t staging_bytes,
                                          void* copy_in_stream, void* compute_stream, void* copy_out_stream,
                                          void* staging_free_event, void* done_event) {
  return step_host(out_host, q_host, k_host, v_host, slot_mapping_host, num_tokens, block_tables_host,
                   context_lens_host, copy_pairs_host, num_pairs, key_cache, value_cache, num_seqs, num_q_heads,
                   num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale, v_scale,
                   q_dtype, cache_dtype, partition_tokens, staging, staging_bytes,
                   static_cast<cudaStream_t>(copy_in_stream), static_cast<cudaStream_t>(compute_stream),
                   static_cast<cudaStream_t>(copy_out_stream), static_cast<cudaEvent_t>(staging_free_event),
                   static_cast<cudaEvent_t>(done_event));
}

// ---- the same step over groups that share their prompt's blocks (parallel sampling) --------------

namespace {

// Staging of the shared-prefix step: q, out, the sequences' new tokens (one per sequence), tables,
// lens, group starts, shared-block counts, copy pairs, then the shared-prefix decode's workspace.
struct SpLayout {
  size_t q, out, k, v, tables, lens, gstart, shared, pairs, workspace, workspace_bytes, total;
};

bool layout_sp(SpLayout* L, int num_seqs, int num_groups, int num_q_heads, int num_kv_heads, int head_dim,
               int block_size, int max_blocks_per_seq, int q_dtype, int partition_tokens, int64_t num_pairs) {
  const size_t es = dtype_bytes(q_dtype);
  if (!es || num_seqs < 0 || num_groups < 0 || num_pairs < 0 || max_blocks_per_seq <= 0) return false;
  const size_t qb = static_cast<size_t>(num_seqs) * num_q_heads * head_dim * es;
  const size_t kb = static_cast<size_t>(num_seqs) * num_kv_heads * head_dim * es;
  size_t off = 0;
  L->q = off;
  off = align256(off + qb);
  L->out = off;
  off = align256(off + qb);
  L->k = off;
  off = align256(off + kb);
  L->v = off;
  off = align256(off + kb);
  L->tables = off;
  off = align256(off + static_cast<size_t>(num_seqs) * max_blocks_per_seq * sizeof(int32_t));
  L->lens = off;
  off = align256(off + static_cast<size_t>(num_seqs) * sizeof(int32_t));
  L->gstart = off;
  off = align256(off + static_cast<size_t>(num_groups + 1) * sizeof(int32_t));
  L->shared = off;
  off = align256(off + static_cast<size_t>(num_groups) * sizeof(int32_t));
  L->pairs = off;
  off = align256(off + static_cast<size_t>(num_pairs) * 2 * sizeof(int64_t));
  L->workspace = off;
  L->workspace_bytes = num_seqs > 0 ? pkv_decode_shared_prefix_workspace_bytes(num_seqs, num_groups, num_q_heads,
                                                                                num_kv_heads, head_dim, block_size,
                                                                                max_blocks_per_seq, partition_tokens)
                                    : 0;
  L->total = align256(off + L->workspace_bytes);
  return true;
}

int step_host_shared_prefix(void* out_host, const void* q_host, const void* k_host, const void* v_host,
                            const int32_t* block_tables_host, const int32_t* context_lens_host,
                            const int32_t* group_start_host, const int32_t* shared_blocks_host, int num_groups,
                            int max_group_size, const int64_t* copy_pairs_host, int64_t num_pairs, void* key_cache,
                            void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                            int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale, int q_dtype,
                            int cache_dtype, int partition_tokens, void* staging, size_t staging_bytes,
                            cudaStream_t in, cudaStream_t comp, cudaStream_t outs, cudaEvent_t wait_ev,
                            cudaEvent_t done_ev) {
  if (num_seqs < 0 || num_groups < 0 || num_pairs < 0) return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0 && num_pairs == 0) return PKV_OK;
  if (!staging || !key_cache || !value_cache) return PKV_ERR_NULL_POINTER;
  if (num_seqs > 0 && (!out_host || !q_host || !block_tables_host || !context_lens_host || !group_start_host ||
                       (num_groups > 0 && !shared_blocks_host)))
    return PKV_ERR_NULL_POINTER;
  if ((k_host == nullptr) != (v_host == nullptr)) return PKV_ERR_NULL_POINTER;
  if (num_pairs > 0 && !copy_pairs_host) return PKV_ERR_NULL_POINTER;
  if ((reinterpret_cast<uintptr_t>(staging) & 255u) != 0) return PKV_ERR_MISALIGNED;
  const int pt = num_seqs > 0 ? pkv_decode_shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size,
                                                                          max_blocks_per_seq, partition_tokens)
                              : 0;
  if (pt < 0) return pt;
  SpLayout L;
  if (!layout_sp(&L, num_seqs, num_groups, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                 q_dtype, pt, num_pairs))
    return PKV_ERR_BAD_DTYPE;
  if (staging_bytes < L.total) return PKV_ERR_WORKSPACE;
  uint8_t* base = static_cast<uint8_t*>(staging);
  void* stream = static_cast<void*>(comp);  // the kernels' stream
  const size_t es = dtype_bytes(q_dtype);
  const size_t qb = static_cast<size_t>(num_seqs) * num_q_heads * head_dim * es;
  const size_t kb = k_host ? static_cast<size_t>(num_seqs) * num_kv_heads * head_dim * es : 0;
  if (wait_ev && cudaStreamWaitEvent(in, wait_ev, 0) != cudaSuccess) return PKV_ERR_CUDA;
  if (!h2d(base + L.q, q_host, qb, in) || !h2d(base + L.k, k_host, kb, in) || !h2d(base + L.v, v_host, kb, in) ||
      !h2d(base + L.tables, block_tables_host,
           static_cast<size_t>(num_seqs) * max_blocks_per_seq * sizeof(int32_t), in) ||
      !h2d(base + L.lens, context_lens_host, static_cast<size_t>(num_seqs) * sizeof(int32_t), in) ||
      !h2d(base + L.gstart, group_start_host, num_seqs > 0 ? static_cast<size_t>(num_groups + 1) * sizeof(int32_t) : 0,
           in) ||
      !h2d(base + L.shared, shared_blocks_host, num_seqs > 0 ? static_cast<size_t>(num_groups) * sizeof(int32_t) : 0,
           in) ||
      !h2d(base + L.pairs, copy_pairs_host, static_cast<size_t>(num_pairs) * 2 * sizeof(int64_t), in))
    return PKV_ERR_CUDA;
  if (!order(in, comp)) return PKV_ERR_CUDA;
  int rc;
  if (num_pairs > 0) {  // copy first, then write: the new tokens may land in the copied blocks
    const int64_t block_bytes =
        static_cast<int64_t>(block_size) * num_kv_heads * head_dim * static_cast<int64_t>(dtype_bytes(cache_dtype));
    rc = pkv_kv_block_copy(reinterpret_cast<const int64_t*>(base + L.pairs), num_pairs, key_cache, value_cache,
                           num_blocks, block_bytes, 0, stream);
    if (rc) return rc;
  }
  if (num_seqs > 0) {
    rc = pkv_paged_attention_decode_shared_prefix(
        base + L.out, base + L.q, k_host ? base + L.k : nullptr, v_host ? base + L.v : nullptr, key_cache,
        value_cache, reinterpret_cast<const int32_t*>(base + L.tables), reinterpret_cast<const int32_t*>(base + L.lens),
        reinterpret_cast<const int32_t*>(base + L.gstart), reinterpret_cast<const int32_t*>(base + L.shared), num_seqs,
        num_groups, max_group_size, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks,
        scale, q_dtype, cache_dtype, pt, base + L.workspace, L.workspace_bytes, 0, stream);
    if (rc) return rc;
    if (!order(comp, outs)) return PKV_ERR_CUDA;
    if (cudaMemcpyAsync(out_host, base + L.out, qb, cudaMemcpyDeviceToHost, outs) != cudaSuccess) return PKV_ERR_CUDA;
  } else if (!order(comp, outs)) {
    return PKV_ERR_CUDA;
  }
  if (done_ev && cudaEventRecord(done_ev, outs) != cudaSuccess) return PKV_ERR_CUDA;
  return PKV_OK;
}

}  // namespace

extern "C" size_t pkv_decode_step_shared_prefix_staging_bytes(int num_seqs, int num_groups, int num_q_heads,
                                                              int num_kv_heads, int head_dim, int block_size,
                                                              int max_blocks_per_seq, int q_dtype,
                                                              int partition_tokens, int64_t num_pairs) {
  const int pt = num_seqs > 0 ? pkv_decode_shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size,
                                                                          max_blocks_per_seq, partition_tokens)
                              : 0;
  if (pt < 0) return 0;
  SpLayout L;
  if (!layout_sp(&L, num_seqs, num_groups, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                 q_dtype, pt, num_pairs))
    return 0;
  return L.total;
}

extern "C" int pkv_decode_step_host_shared_prefix_async(
    void* out_host, const void* q_host, const void* k_new_host, const void* v_new_host,
    const int32_t* block_tables_host, const int32_t* context_lens_host, const int32_t* group_start_host,
    const int32_t* shared_blocks_host, int num_groups, int max_group_size, const int64_t* copy_pairs_host,
    int64_t num_pairs, void* key_cache, void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads,
    int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale, int q_dtype,
    int cache_dtype, int partition_tokens, void* staging, size_t staging_bytes, void* copy_in_stream,
    void* compute_stream, void* copy_out_stream, void* staging_free_event, void* done_event) {
  return step_host_shared_prefix(
      out_host, q_host, k_new_host, v_new_host, block_tables_host, context_lens_host, group_start_host,
      shared_blocks_host, num_groups, max_group_size, copy_pairs_host, num_pairs, key_cache, value_cache, num_seqs,
      num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, q_dtype, cache_dtype,
      partition_tokens, staging, staging_bytes, static_cast<cudaStream_t>(copy_in_stream),
      static_cast<cudaStream_t>(compute_stream), static_cast<cudaStream_t>(copy_out_stream),
      static_cast<cudaEvent_t>(staging_free_event), static_cast<cudaEvent_t>(done_event));
}

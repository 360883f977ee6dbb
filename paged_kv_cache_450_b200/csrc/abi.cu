// abi.cu -- the C ABI of libpagedkv (declared in include/pagedkv.h):
// argument checks, optional host-side validation of index arrays, TMA
// descriptor encoding for the caches, the split-context partition choice and
// the kernel dispatch.
#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "launch.h"
#include "multiquery_params.h"

namespace pkv {

// The device status word (PKV_STATUS_* bits), one per device that loads the module.
__device__ unsigned g_status_word;

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

constexpr int kMaxDevices = 64;
static std::mutex g_mu;

static unsigned* status_word() {
  static unsigned* ptr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptr[dev] = static_cast<unsigned*>(p);
  }
  return ptr[dev];
}

static int sm_count() {
  static int cached[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map of one cache [NB][BS][Hkv][D] seen as a 4-D tensor
// (D, Hkv, BS, NB) innermost first; the box is one (block, kv head) tile.
// With `swizzle128` the tile lands in shared memory with the 128-byte swizzle
// (16-byte chunk q of row t at chunk q ^ (t % 8)); rows must be a multiple of 128 bytes.
static bool encode_cache_map(CUtensorMap* map, const void* base, int64_t num_blocks, int block_size, int num_kv_heads,
                             int head_dim, int dtype, bool swizzle128) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  CUtensorMapDataType dt;
  int es;
  switch (dtype) {
    case PKV_DTYPE_F32: dt = CU_TENSOR_MAP_DATA_TYPE_FLOAT32; es = 4; break;
    case PKV_DTYPE_BF16: dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; es = 2; break;
    case PKV_DTYPE_FP8_E4M3: dt = CU_TENSOR_MAP_DATA_TYPE_UINT8; es = 1; break;
    default: return false;
  }
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(head_dim), static_cast<cuuint64_t>(num_kv_heads),
                              static_cast<cuuint64_t>(block_size), static_cast<cuuint64_t>(num_blocks)};
  const cuuint64_t row = static_cast<cuuint64_t>(head_dim) * es;
  const cuuint64_t strides[3] = {row, row * num_kv_heads, row * num_kv_heads * block_size};
  // Swizzled maps move one 128-byte segment of a row per box (a whole fp8
  // row, half a bf16 row); the kernels issue one box per segment.
  const cuuint32_t box0 = swizzle128 ? static_cast<cuuint32_t>(128 / es) : static_cast<cuuint32_t>(head_dim);
  const cuuint32_t box[4] = {box0, 1, static_cast<cuuint32_t>(block_size), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  if (swizzle128 && (row % 128) != 0) return false;
  return fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over the bf16 queries [total_q][num_q_heads][128] of the tcgen05
// multi-query kernel: one box = 128 / group queries x the group's query heads
// x one 64-dim half (128 bytes, 128-byte swizzle), i.e. 128 MMA rows ordered
// (query, head) with the head fastest.  Rows past total_q read as zeros.
static bool encode_query_map(CUtensorMap* map, const void* q, int total_q, int num_q_heads, int group) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(num_q_heads), static_cast<cuuint64_t>(total_q)};
  const cuuint64_t strides[2] = {128 * 2, static_cast<cuuint64_t>(num_q_heads) * 128 * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(group), static_cast<cuuint32_t>(128 / group)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <typename T>
static bool copy_to_host(std::vector<T>& dst, const T* src, size_t n, cudaStream_t st) {
  dst.resize(n);
  if (n == 0) return true;
  if (cudaMemcpyAsync(dst.data(), src, n * sizeof(T), cudaMemcpyDeviceToHost, st) != cudaSuccess) return false;
  return cudaStreamSynchronize(st) == cudaSuccess;
}

constexpr int kMaxPartitionTokens = 16384;

// Resident CTAs per SM of the decode kernel that serves these arguments
// (from the kernels' shared-memory and register budgets on B200).
static int decode_ctas_per_sm(int cache_dtype, int head_dim, int group, int block_size) {
  if (decode_uses_mma(cache_dtype, head_dim, group, block_size))
    return cache_dtype == PKV_DTYPE_FP8_E4M3 ? 16 : 8;  // one warp, 13 KB / 25 KB of stages
  return 6;                                            // four warps, ~34 KB
}

// Automatic split-context partition length (see pkv_decode_partition_tokens).
// Longer partitions cost less per token (one CTA set-up and one partial per
// partition, and no merge pass at all for a single one).  With fewer
// (sequence, KV head) pairs than four waves of resident CTAs, at least 4
// partitions per long context keep mixed lengths balanced and at least three
// quarters of a wave of CTAs keeps the SMs busy (a full single wave measured
// faster than 1.7 waves of half-length CTAs).  With more pairs than that, the
// pairs alone balance the load: partitions of up to 2048 tokens, a single one
// for shorter contexts (measured 22% faster than four on the 128-sequence
// parallel-sampling batch).
static int auto_partition_tokens(int num_seqs, int num_kv_heads, int block_size, int max_blocks_per_seq,
                                 int ctas_per_sm, int64_t few_pairs_min_parts = 4) {
  const int64_t max_ctx = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  const int64_t pairs = static_cast<int64_t>(num_seqs) * num_kv_heads;
  if (max_ctx <= 512) return static_cast<int>(cdiv64(max_ctx, block_size) * block_size);
  const int64_t slots = static_cast<int64_t>(ctas_per_sm) * sm_count();
  const bool many = pairs >= 4 * slots;
  const int64_t min_parts = many ? 1 : few_pairs_min_parts;
  int pt = many ? 2048 : 4096;
  while (pt > 128 && (cdiv64(max_ctx, pt) < min_parts || 4 * pairs * cdiv64(max_ctx, pt) < 3 * slots)) pt /= 2;
  return pt < block_size ? block_size : pt;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_NULL_POINTER: return "a required pointer is NULL";
    case PKV_ERR_BAD_DTYPE: return "unsupported dtype or dtype combination";
    case PKV_ERR_HEAD_DIM: return "head_dim must be 64 or 128";
    case PKV_ERR_BLOCK_SIZE: return "block_size must be 8, 16 or 32";
    case PKV_ERR_HEAD_GROUPING: return "num_q_heads / num_kv_heads must be 1, 2, 4 or 8";
    case PKV_ERR_WORKSPACE: return "workspace missing or too small";
    case PKV_ERR_BAD_SHAPE: return "bad size argument";
    case PKV_ERR_OUT_OF_RANGE: return "an index (block id, slot, context length) is outside the pool";
    case PKV_ERR_BAD_COPY_PAIRS: return "copy pairs repeat a destination or use a destination as a source";
    case PKV_ERR_MISALIGNED: return "a data pointer is not 16-byte aligned";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_TENSOR_MAP: return "TMA descriptor encoding failed";
    case PKV_ERR_PARTITION: return "partition_tokens must be a positive multiple of block_size (at most 16384)";
    default: return "unknown status";
  }
}

uint64_t pkv_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int pkv_device_status(unsigned* status, int clear, void* stream) {
  if (!status) return PKV_ERR_NULL_POINTER;
  unsigned* w = status_word();
  if (!w) return PKV_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status, w, sizeof(unsigned), cudaMemcpyDeviceToHost, st) != cudaSuccess) return PKV_ERR_CUDA;
  if (clear && cudaMemsetAsync(w, 0, sizeof(unsigned), st) != cudaSuccess) return PKV_ERR_CUDA;
  return cudaStreamSynchronize(st) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_paged_kv_write(const void* k, const void* v, const int64_t* slot_mapping, int64_t num_tokens,
                       void* key_cache, void* value_cache, int64_t num_blocks, int block_size, int num_kv_heads,
                       int head_dim, int in_dtype, int cache_dtype, float k_scale, float v_scale, int validate,
                       void* stream) {
  if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return PKV_ERR_BAD_SHAPE;
  if (num_tokens == 0) return PKV_OK;
  if (!k || !v || !slot_mapping || !key_cache || !value_cache) return PKV_ERR_NULL_POINTER;
  if (in_dtype != PKV_DTYPE_F32 && in_dtype != PKV_DTYPE_BF16) return PKV_ERR_BAD_DTYPE;
  if (cache_dtype != in_dtype && cache_dtype != PKV_DTYPE_FP8_E4M3) return PKV_ERR_BAD_DTYPE;
  if (head_dim % 16 != 0) return PKV_ERR_HEAD_DIM;
  if (num_tokens > 0x7fffffffLL) return PKV_ERR_BAD_SHAPE;
  if (!aligned16(k) || !aligned16(v) || !aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_MISALIGNED;
  if (cache_dtype == PKV_DTYPE_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_ERR_BAD_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    std::vector<int64_t> h;
    if (!copy_to_host(h, slot_mapping, static_cast<size_t>(num_tokens), st)) return PKV_ERR_CUDA;
    const int64_t slots = num_blocks * block_size;
    std::vector<int64_t> seen;
    for (int64_t s : h) {
      if (s >= slots) return PKV_ERR_OUT_OF_RANGE;
      if (s >= 0) seen.push_back(s);
    }
    std::sort(seen.begin(), seen.end());
    for (size_t i = 1; i < seen.size(); ++i)
      if (seen[i] == seen[i - 1]) return PKV_ERR_OUT_OF_RANGE;
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  KvWriteArgs a;
  a.k = k;
  a.v = v;
  a.slot_mapping = slot_mapping;
  a.num_tokens = num_tokens;
  a.key_cache = key_cache;
  a.value_cache = value_cache;
  a.num_blocks = num_blocks;
  a.block_size = block_size;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.in_dtype = in_dtype;
  a.cache_dtype = cache_dtype;
  a.k_inv = 1.0f / k_scale;  // rounded once to fp32 on the host
  a.v_inv = 1.0f / v_scale;
  a.status = status;
  return launch_kv_write(a, st) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_decode_partition_tokens(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_blocks_per_seq, int cache_dtype, int partition_tokens) {
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0) return PKV_ERR_BAD_SHAPE;
  if (partition_tokens != 0) {
    if (partition_tokens < 0 || partition_tokens % block_size != 0 || partition_tokens > kMaxPartitionTokens)
      return PKV_ERR_PARTITION;
    return partition_tokens;
  }
  const int group = num_q_heads % num_kv_heads == 0 ? num_q_heads / num_kv_heads : 0;
  return auto_partition_tokens(num_seqs, num_kv_heads, block_size, max_blocks_per_seq,
                               decode_ctas_per_sm(cache_dtype, head_dim, group, block_size));
}

int pkv_decode_max_partitions(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int cache_dtype, int partition_tokens) {
  const int pt = pkv_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                             max_blocks_per_seq, cache_dtype, partition_tokens);
  if (pt < 0) return pt;
  return static_cast<int>(cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt));
}

size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int cache_dtype, int partition_tokens) {
  const int P = pkv_decode_max_partitions(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                          max_blocks_per_seq, cache_dtype, partition_tokens);
  if (P <= 1 || head_dim <= 0) return 0;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * P;
  return align256(rows * 2 * sizeof(float)) + rows * head_dim * sizeof(float);
}

}  // extern "C"

// Decode, optionally with the fused append of one new token per sequence
// (k_new / v_new non-NULL).
static int decode_impl(void* out, const void* q, const void* k_new, const void* v_new, const void* key_cache,
                       const void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                       int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale, float v_scale,
                       int q_dtype, int cache_dtype, int partition_tokens, void* workspace, size_t workspace_bytes,
                       int validate, void* stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0)
    return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0) return PKV_OK;
  if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens) return PKV_ERR_NULL_POINTER;
  if ((k_new == nullptr) != (v_new == nullptr)) return PKV_ERR_NULL_POINTER;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PKV_ERR_MISALIGNED;
  if (q_dtype != PKV_DTYPE_F32 && q_dtype != PKV_DTYPE_BF16) return PKV_ERR_BAD_DTYPE;
  if (cache_dtype != q_dtype && cache_dtype != PKV_DTYPE_FP8_E4M3) return PKV_ERR_BAD_DTYPE;
  if (head_dim != 64 && head_dim != 128) return PKV_ERR_HEAD_DIM;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_HEAD_GROUPING;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_HEAD_GROUPING;
  if (num_blocks > 0x7fffffffLL || num_seqs > 65535) return PKV_ERR_BAD_SHAPE;
  if (static_cast<int64_t>(max_blocks_per_seq) * block_size > 0x7fffffffLL) return PKV_ERR_BAD_SHAPE;
  if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_MISALIGNED;
  if (cache_dtype == PKV_DTYPE_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_ERR_BAD_SHAPE;
  const int pt = pkv_decode_partition_tokens(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                             max_blocks_per_seq, cache_dtype, partition_tokens);
  if (pt < 0) return pt;
  const int P = static_cast<int>(cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt));
  if (P > 65535) return PKV_ERR_PARTITION;
  const size_t need = pkv_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                                                 max_blocks_per_seq, cache_dtype, partition_tokens);
  if (need > 0 && (!workspace || workspace_bytes < need)) return PKV_ERR_WORKSPACE;
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    std::vector<int32_t> lens, tables;
    if (!copy_to_host(lens, context_lens, static_cast<size_t>(num_seqs), st)) return PKV_ERR_CUDA;
    if (!copy_to_host(tables, block_tables, static_cast<size_t>(num_seqs) * max_blocks_per_seq, st))
      return PKV_ERR_CUDA;
    for (int b = 0; b < num_seqs; ++b) {
      const int64_t ctx = lens[b];
      if (ctx < 0 || ctx > static_cast<int64_t>(max_blocks_per_seq) * block_size) return PKV_ERR_OUT_OF_RANGE;
      for (int64_t j = 0; j < cdiv64(ctx, block_size); ++j) {
        const int64_t id = tables[static_cast<size_t>(b) * max_blocks_per_seq + j];
        if (id < 0 || id >= num_blocks) return PKV_ERR_OUT_OF_RANGE;
      }
    }
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  CUtensorMap kmap, vmap;
  const bool mma = decode_uses_mma(cache_dtype, head_dim, group, block_size);
  if (!encode_cache_map(&kmap, key_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, mma) ||
      !encode_cache_map(&vmap, value_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, mma))
    return PKV_ERR_TENSOR_MAP;

  DecodeParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.ws_ml = nullptr;
  p.ws_o = nullptr;
  if (need > 0) {
    const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * P;
    p.ws_ml = static_cast<float*>(workspace);
    p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * 2 * sizeof(float)));
  }
  p.status = status;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = static_cast<int>(num_blocks);
  p.block_size = block_size;
  p.partition_blocks = pt / block_size;
  p.max_partitions = P;
  const bool fp8 = cache_dtype == PKV_DTYPE_FP8_E4M3;
  p.q_scale = scale * kLog2e * (fp8 ? k_scale : 1.0f);
  p.out_scale = fp8 ? v_scale : 1.0f;
  p.new_k = k_new;
  p.new_v = v_new;
  p.key_cache = const_cast<void*>(key_cache);
  p.value_cache = const_cast<void*>(value_cache);
  p.k_inv = fp8 ? 1.0f / k_scale : 1.0f;  // rounded once to fp32 on the host, as for pkv_paged_kv_write
  p.v_inv = fp8 ? 1.0f / v_scale : 1.0f;
  const bool reduce = P > 1;

  cudaError_t e;
  if (q_dtype == PKV_DTYPE_F32 && cache_dtype == PKV_DTYPE_F32)
    e = launch_decode_f32_f32(kmap, vmap, p, head_dim, group, num_kv_heads, reduce, st);
  else if (q_dtype == PKV_DTYPE_BF16 && cache_dtype == PKV_DTYPE_BF16)
    e = launch_decode_bf16_bf16(kmap, vmap, p, head_dim, group, num_kv_heads, reduce, st);
  else if (q_dtype == PKV_DTYPE_F32)
    e = launch_decode_f32_fp8(kmap, vmap, p, head_dim, group, num_kv_heads, reduce, st);
  else
    e = launch_decode_bf16_fp8(kmap, vmap, p, head_dim, group, num_kv_heads, reduce, st);
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

extern "C" {

int pkv_paged_attention_decode(void* out, const void* q, const void* key_cache, const void* value_cache,
                               const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                               float v_scale, int q_dtype, int cache_dtype, int partition_tokens, void* workspace,
                               size_t workspace_bytes, int validate, void* stream) {
  return decode_impl(out, q, nullptr, nullptr, key_cache, value_cache, block_tables, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale,
                     v_scale, q_dtype, cache_dtype, partition_tokens, workspace, workspace_bytes, validate, stream);
}

int pkv_paged_decode_append(void* out, const void* q, const void* k_new, const void* v_new, void* key_cache,
                            void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale, float v_scale,
                            int q_dtype, int cache_dtype, int partition_tokens, void* workspace,
                            size_t workspace_bytes, int validate, void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return PKV_ERR_NULL_POINTER;
  if (cache_dtype == PKV_DTYPE_FP8_E4M3 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_ERR_BAD_SHAPE;
  return decode_impl(out, q, k_new, v_new, key_cache, value_cache, block_tables, context_lens, num_seqs,
                     num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, scale, k_scale,
                     v_scale, q_dtype, cache_dtype, partition_tokens, workspace, workspace_bytes, validate, stream);
}

// Host-side check of copy pairs (validate): ids in range; destinations distinct
// and, when both sides are one pool, never also a source.
static int check_pairs(const int64_t* pairs, int64_t num_pairs, int64_t src_blocks, int64_t dst_blocks, bool same_pool,
                       cudaStream_t st) {
  std::vector<int64_t> h;
  if (!copy_to_host(h, pairs, static_cast<size_t>(num_pairs) * 2, st)) return PKV_ERR_CUDA;
  std::vector<int64_t> dsts, srcs;
  for (int64_t i = 0; i < num_pairs; ++i) {
    const int64_t s = h[2 * i], d = h[2 * i + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) return PKV_ERR_OUT_OF_RANGE;
    srcs.push_back(s);
    dsts.push_back(d);
  }
  std::sort(dsts.begin(), dsts.end());
  std::sort(srcs.begin(), srcs.end());
  for (size_t i = 1; i < dsts.size(); ++i)
    if (dsts[i] == dsts[i - 1]) return PKV_ERR_BAD_COPY_PAIRS;
  if (same_pool)
    for (int64_t d : dsts)
      if (std::binary_search(srcs.begin(), srcs.end(), d)) return PKV_ERR_BAD_COPY_PAIRS;
  return PKV_OK;
}

int pkv_kv_block_copy(const int64_t* src_dst_pairs, int64_t num_pairs, void* key_cache, void* value_cache,
                      int64_t num_blocks, int64_t block_bytes, int validate, void* stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_bytes <= 0 || block_bytes % 16 != 0) return PKV_ERR_BAD_SHAPE;
  if (num_pairs == 0) return PKV_OK;
  if (!src_dst_pairs || !key_cache || !value_cache) return PKV_ERR_NULL_POINTER;
  if (!aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    const int rc = check_pairs(src_dst_pairs, num_pairs, num_blocks, num_blocks, true, st);
    if (rc) return rc;
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  return launch_block_copy(src_dst_pairs, num_pairs, key_cache, value_cache, num_blocks, key_cache, value_cache,
                           num_blocks, block_bytes, status, st) == cudaSuccess
             ? PKV_OK
             : PKV_ERR_CUDA;
}

// Split-context partition length of the multi-query kernel: one partition
// when (sequences x KV heads x query-row tiles) already gives about two waves
// of the kernel's resident CTAs, else the context split so that it does
// (multiples of 256 tokens).
static int mq_partition_tokens(int num_seqs, int num_kv_heads, int group, int max_q_len, int block_size,
                               int max_blocks_per_seq, bool fp8, int partition_tokens) {
  if (partition_tokens != 0) {
    if (partition_tokens < 0 || partition_tokens % block_size != 0 || partition_tokens > kMaxPartitionTokens)
      return PKV_ERR_PARTITION;
    return partition_tokens;
  }
  const int64_t max_ctx = static_cast<int64_t>(max_blocks_per_seq) * block_size;
  const int64_t rows = static_cast<int64_t>(max_q_len) * group;
  // CTAs per (sequence, KV head) and resident CTAs per SM of the kernel that
  // serves these rows: 16- to 64-row mma.sync CTAs (6 to 2 per SM), or 128-row
  // tcgen05 CTAs (1 per SM)
  (void)fp8;  // the same kernel split for both cache types
  const bool tc = multiquery_uses_tc(static_cast<int>(rows > 0x7fffffff ? 0x7fffffff : rows));
  const int nwc = multiquery_compute_warps(static_cast<int>(rows > 64 ? 64 : rows));
  const int tile = tc ? 128 : 16 * nwc;
  const int per_sm = tc ? 1 : multiquery_ctas_per_sm(nwc);
  const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads * cdiv64(rows, tile);
  const int64_t want = 2LL * per_sm * sm_count();
  int64_t P = units >= want ? 1 : cdiv64(want, units > 0 ? units : 1);
  int64_t pt = cdiv64(max_ctx, P);
  pt = cdiv64(pt, 256) * 256;
  if (pt < 256) pt = 256;
  if (pt >= max_ctx) pt = cdiv64(max_ctx, block_size) * block_size;
  if (pt > kMaxPartitionTokens) pt = kMaxPartitionTokens;
  return static_cast<int>(pt);
}

int pkv_multiquery_partition_tokens(int num_seqs, int max_q_len, int num_q_heads, int num_kv_heads, int block_size,
                                    int max_blocks_per_seq, int cache_dtype, int partition_tokens) {
  if (block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (num_seqs < 0 || max_q_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0)
    return PKV_ERR_BAD_SHAPE;
  if (cache_dtype != PKV_DTYPE_BF16 && cache_dtype != PKV_DTYPE_FP8_E4M3) return PKV_ERR_BAD_DTYPE;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_HEAD_GROUPING;
  return mq_partition_tokens(num_seqs, num_kv_heads, num_q_heads / num_kv_heads, max_q_len, block_size,
                             max_blocks_per_seq, cache_dtype == PKV_DTYPE_FP8_E4M3, partition_tokens);
}

size_t pkv_multiquery_workspace_bytes(int num_seqs, int total_q, int max_q_len, int num_q_heads, int num_kv_heads,
                                      int head_dim, int block_size, int max_blocks_per_seq, int cache_dtype,
                                      int partition_tokens) {
  const int pt = pkv_multiquery_partition_tokens(num_seqs, max_q_len, num_q_heads, num_kv_heads, block_size,
                                                 max_blocks_per_seq, cache_dtype, partition_tokens);
  if (pt < 0 || total_q <= 0 || head_dim <= 0) return 0;
  const int64_t P = cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt);
  if (P <= 1) return 0;
  const size_t rows = static_cast<size_t>(total_q) * num_q_heads * P;
  return align256(rows * 2 * sizeof(float)) + rows * head_dim * sizeof(float);
}

int pkv_paged_attention_multiquery(void* out, const void* q, const void* key_cache, const void* value_cache,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   const int32_t* query_start_loc, int num_seqs, int total_q, int max_q_len,
                                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                                   float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                                   void* workspace, size_t workspace_bytes, int validate, void* stream) {
  if (num_seqs < 0 || total_q < 0 || max_q_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      max_blocks_per_seq <= 0 || num_blocks <= 0)
    return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0 || total_q == 0) return PKV_OK;
  if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens || !query_start_loc)
    return PKV_ERR_NULL_POINTER;
  if (q_dtype != PKV_DTYPE_BF16 || (cache_dtype != PKV_DTYPE_BF16 && cache_dtype != PKV_DTYPE_FP8_E4M3))
    return PKV_ERR_BAD_DTYPE;
  const bool fp8 = cache_dtype == PKV_DTYPE_FP8_E4M3;
  if (fp8 && !(k_scale > 0.f && v_scale > 0.f)) return PKV_ERR_BAD_SHAPE;
  if (head_dim != 128) return PKV_ERR_HEAD_DIM;
  if (block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_HEAD_GROUPING;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_HEAD_GROUPING;
  if (num_blocks > 0x7fffffffLL || num_seqs > 65535) return PKV_ERR_BAD_SHAPE;
  if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_MISALIGNED;
  const int pt = mq_partition_tokens(num_seqs, num_kv_heads, group, max_q_len, block_size, max_blocks_per_seq, fp8,
                                     partition_tokens);
  if (pt < 0) return pt;
  const int P = static_cast<int>(cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt));
  if (P > 65535) return PKV_ERR_PARTITION;
  const size_t need = pkv_multiquery_workspace_bytes(num_seqs, total_q, max_q_len, num_q_heads, num_kv_heads,
                                                     head_dim, block_size, max_blocks_per_seq, cache_dtype,
                                                     partition_tokens);
  if (need > 0 && (!workspace || workspace_bytes < need)) return PKV_ERR_WORKSPACE;
  if (need > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    std::vector<int32_t> lens, tables, qsl;
    if (!copy_to_host(lens, context_lens, static_cast<size_t>(num_seqs), st) ||
        !copy_to_host(qsl, query_start_loc, static_cast<size_t>(num_seqs) + 1, st) ||
        !copy_to_host(tables, block_tables, static_cast<size_t>(num_seqs) * max_blocks_per_seq, st))
      return PKV_ERR_CUDA;
    if (qsl[0] != 0 || qsl[num_seqs] != total_q) return PKV_ERR_OUT_OF_RANGE;
    for (int b = 0; b < num_seqs; ++b) {
      const int64_t ctx = lens[b], ql = static_cast<int64_t>(qsl[b + 1]) - qsl[b];
      if (ql < 0 || ql > max_q_len || ctx < ql || ctx > static_cast<int64_t>(max_blocks_per_seq) * block_size)
        return PKV_ERR_OUT_OF_RANGE;
      for (int64_t j = 0; j < cdiv64(ctx, block_size); ++j) {
        const int64_t id = tables[static_cast<size_t>(b) * max_blocks_per_seq + j];
        if (id < 0 || id >= num_blocks) return PKV_ERR_OUT_OF_RANGE;
      }
    }
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  CUtensorMap kmap, vmap;
  if (!encode_cache_map(&kmap, key_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, true) ||
      !encode_cache_map(&vmap, value_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, true))
    return PKV_ERR_TENSOR_MAP;
  MultiQueryParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  p.query_start_loc = query_start_loc;
  p.ws_ml = nullptr;
  p.ws_o = nullptr;
  if (need > 0) {
    const size_t rows = static_cast<size_t>(total_q) * num_q_heads * P;
    p.ws_ml = static_cast<float*>(workspace);
    p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * 2 * sizeof(float)));
  }
  p.status = status;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = static_cast<int>(num_blocks);
  p.block_size = block_size;
  p.partition_blocks = pt / block_size;
  p.max_partitions = P;
  p.total_q = total_q;
  p.max_q_len = max_q_len;
  p.q_scale = scale * kLog2e * (fp8 ? k_scale : 1.f);
  p.out_scale = fp8 ? v_scale : 1.f;
  const int rows_per_seq = max_q_len * group;
  if (rows_per_seq <= 0) return PKV_OK;
  if (multiquery_uses_tc(rows_per_seq)) {
    CUtensorMap qmap;
    if (!encode_query_map(&qmap, q, total_q, num_q_heads, group)) return PKV_ERR_TENSOR_MAP;
    return launch_multiquery_tc(qmap, kmap, vmap, p, group, rows_per_seq, fp8, P > 1, st) == cudaSuccess
               ? PKV_OK
               : PKV_ERR_CUDA;
  }
  const cudaError_t e = fp8 ? launch_multiquery_mma_fp8(kmap, vmap, p, group, rows_per_seq, P > 1, st)
                            : launch_multiquery_mma_bf16(kmap, vmap, p, group, rows_per_seq, P > 1, st);
  return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

// Partition length and slot counts of the shared-prefix decode: the automatic
// choice is made for the groups' shared units (one per group and KV head, the
// bulk of the bytes) on the bf16 tensor-core kernel.
static int shared_prefix_partition_tokens(int num_groups, int num_kv_heads, int block_size, int max_blocks_per_seq,
                                          int partition_tokens) {
  if (partition_tokens != 0) {
    if (partition_tokens < 0 || partition_tokens % block_size != 0 || partition_tokens > kMaxPartitionTokens)
      return PKV_ERR_PARTITION;
    return partition_tokens;
  }
  // The members' own units (one per sequence and KV head) run beside the shared ones and fill
  // the gaps of the last wave, so the shared part takes three splits at least rather than four
  // (measured on 32 prompts of 1024 tokens x 4 candidates x 40 heads: 512-token partitions
  // 2.4% faster than 256, 128 19% slower).
  return auto_partition_tokens(num_groups, num_kv_heads, block_size, max_blocks_per_seq,
                               decode_ctas_per_sm(PKV_DTYPE_BF16, 128, 2, block_size), 3);
}

int pkv_decode_shared_prefix_partition_tokens(int num_groups, int num_kv_heads, int block_size,
                                              int max_blocks_per_seq, int partition_tokens) {
  if (num_groups <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0) return PKV_ERR_BAD_SHAPE;
  if (block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  return shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size, max_blocks_per_seq, partition_tokens);
}

size_t pkv_decode_shared_prefix_workspace_bytes(int num_seqs, int num_groups, int num_q_heads, int num_kv_heads,
                                                int head_dim, int block_size, int max_blocks_per_seq,
                                                int partition_tokens) {
  if (num_seqs <= 0 || num_groups <= 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq <= 0 || (block_size != 16 && block_size != 32))
    return 0;
  const int pt = shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size, max_blocks_per_seq,
                                                partition_tokens);
  if (pt < 0) return 0;
  const int64_t P = 2 * cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt);
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * P;
  return align256(rows * 2 * sizeof(float)) + rows * head_dim * sizeof(float);
}

int pkv_paged_attention_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                                             void* key_cache, void* value_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, const int32_t* group_start,
                                             const int32_t* shared_blocks, int num_seqs, int num_groups,
                                             int max_group_size, int num_q_heads, int num_kv_heads, int head_dim,
                                             int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale,
                                             int q_dtype, int cache_dtype, int partition_tokens, void* workspace,
                                             size_t workspace_bytes, int validate, void* stream) {
  if (num_seqs < 0 || num_groups < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 ||
      num_blocks <= 0)
    return PKV_ERR_BAD_SHAPE;
  if (num_seqs == 0) return PKV_OK;
  if (num_groups < 1 || num_groups > num_seqs || max_group_size < 1) return PKV_ERR_BAD_SHAPE;
  if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens || !group_start || !shared_blocks)
    return PKV_ERR_NULL_POINTER;
  if ((k_new == nullptr) != (v_new == nullptr)) return PKV_ERR_NULL_POINTER;
  if (q_dtype != PKV_DTYPE_BF16 || cache_dtype != PKV_DTYPE_BF16) return PKV_ERR_BAD_DTYPE;
  if (head_dim != 128) return PKV_ERR_HEAD_DIM;
  if (block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (num_q_heads % num_kv_heads != 0) return PKV_ERR_HEAD_GROUPING;
  const int group = num_q_heads / num_kv_heads;
  if (group != 1 && group != 2 && group != 4 && group != 8) return PKV_ERR_HEAD_GROUPING;
  if (static_cast<int64_t>(max_group_size) * group > 8) return PKV_ERR_BAD_SHAPE;  // members x heads: 8 columns
  if (num_blocks > 0x7fffffffLL || num_seqs + num_groups > 65535) return PKV_ERR_BAD_SHAPE;
  if (static_cast<int64_t>(max_blocks_per_seq) * block_size > 0x7fffffffLL) return PKV_ERR_BAD_SHAPE;
  if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache)) return PKV_ERR_MISALIGNED;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return PKV_ERR_MISALIGNED;
  const int pt = shared_prefix_partition_tokens(num_groups, num_kv_heads, block_size, max_blocks_per_seq,
                                                partition_tokens);
  if (pt < 0) return pt;
  const int Ph = static_cast<int>(cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, pt));
  if (Ph > 32767) return PKV_ERR_PARTITION;
  const size_t need = pkv_decode_shared_prefix_workspace_bytes(num_seqs, num_groups, num_q_heads, num_kv_heads,
                                                               head_dim, block_size, max_blocks_per_seq,
                                                               partition_tokens);
  if (!workspace || workspace_bytes < need) return PKV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return PKV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    std::vector<int32_t> lens, tables, gs, sh;
    if (!copy_to_host(lens, context_lens, static_cast<size_t>(num_seqs), st) ||
        !copy_to_host(tables, block_tables, static_cast<size_t>(num_seqs) * max_blocks_per_seq, st) ||
        !copy_to_host(gs, group_start, static_cast<size_t>(num_groups) + 1, st) ||
        !copy_to_host(sh, shared_blocks, static_cast<size_t>(num_groups), st))
      return PKV_ERR_CUDA;
    if (gs[0] != 0 || gs[num_groups] != num_seqs) return PKV_ERR_OUT_OF_RANGE;
    for (int g = 0; g < num_groups; ++g) {
      const int n = gs[g + 1] - gs[g];
      if (n < 1 || n > max_group_size || sh[g] < 0) return PKV_ERR_OUT_OF_RANGE;
      for (int b = gs[g]; b < gs[g + 1]; ++b) {
        // the shared blocks are whole blocks of every member's context (and the appended token is its own)
        if (static_cast<int64_t>(sh[g]) * block_size > static_cast<int64_t>(lens[b]) - (k_new ? 1 : 0))
          return PKV_ERR_OUT_OF_RANGE;
        for (int j = 0; j < sh[g]; ++j)
          if (tables[static_cast<size_t>(b) * max_blocks_per_seq + j] !=
              tables[static_cast<size_t>(gs[g]) * max_blocks_per_seq + j])
            return PKV_ERR_OUT_OF_RANGE;
      }
    }
    for (int b = 0; b < num_seqs; ++b) {
      const int64_t ctx = lens[b];
      if (ctx < 0 || ctx > static_cast<int64_t>(max_blocks_per_seq) * block_size) return PKV_ERR_OUT_OF_RANGE;
      for (int64_t j = 0; j < cdiv64(ctx, block_size); ++j) {
        const int64_t id = tables[static_cast<size_t>(b) * max_blocks_per_seq + j];
        if (id < 0 || id >= num_blocks) return PKV_ERR_OUT_OF_RANGE;
      }
    }
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  CUtensorMap kmap, vmap;
  if (!encode_cache_map(&kmap, key_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, true) ||
      !encode_cache_map(&vmap, value_cache, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype, true))
    return PKV_ERR_TENSOR_MAP;
  DecodeParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.context_lens = context_lens;
  const size_t rows = static_cast<size_t>(num_seqs) * num_q_heads * (2 * Ph);
  p.ws_ml = static_cast<float*>(workspace);
  p.ws_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align256(rows * 2 * sizeof(float)));
  p.status = status;
  p.num_seqs = num_seqs;
  p.num_q_heads = num_q_heads;
  p.num_kv_heads = num_kv_heads;
  p.max_blocks_per_seq = max_blocks_per_seq;
  p.num_blocks = static_cast<int>(num_blocks);
  p.block_size = block_size;
  p.partition_blocks = pt / block_size;
  p.max_partitions = 2 * Ph;
  p.q_scale = scale * kLog2e;
  p.out_scale = 1.f;
  p.new_k = k_new;
  p.new_v = v_new;
  p.key_cache = key_cache;
  p.value_cache = value_cache;
  p.k_inv = 1.f;
  p.v_inv = 1.f;
  p.group_start = group_start;
  p.shared_blocks = shared_blocks;
  p.num_groups = num_groups;
  p.shared_partitions = Ph;
  return launch_decode_shared_prefix_bf16(kmap, vmap, p, group, num_kv_heads, Ph, st) == cudaSuccess ? PKV_OK
                                                                                                     : PKV_ERR_CUDA;
}

int pkv_selftest_wait_timeout(int64_t limit_ns, unsigned* gave_up, void* stream) {
  if (limit_ns <= 0 || limit_ns > 100000000LL) return PKV_ERR_BAD_SHAPE;
  if (!gave_up) return PKV_ERR_NULL_POINTER;
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  return launch_wait_timeout_selftest(status, static_cast<uint64_t>(limit_ns), gave_up,
                                      static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PKV_OK
             : PKV_ERR_CUDA;
}

int pkv_decode_table_scan(const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_kv_heads,
                          int block_size, int max_blocks_per_seq, int64_t num_blocks, int partition_tokens,
                          unsigned* sink, size_t sink_words, void* stream) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0) return PKV_ERR_BAD_SHAPE;
  if (block_size != 8 && block_size != 16 && block_size != 32) return PKV_ERR_BLOCK_SIZE;
  if (partition_tokens <= 0 || partition_tokens % block_size != 0 || partition_tokens > kMaxPartitionTokens)
    return PKV_ERR_PARTITION;
  if (num_seqs == 0) return PKV_OK;
  if (!block_tables || !context_lens || !sink) return PKV_ERR_NULL_POINTER;
  if (num_blocks > 0x7fffffffLL || num_seqs > 65535 || num_kv_heads > 65535) return PKV_ERR_BAD_SHAPE;
  if (static_cast<int64_t>(max_blocks_per_seq) * block_size > 0x7fffffffLL) return PKV_ERR_BAD_SHAPE;
  const int64_t P = cdiv64(static_cast<int64_t>(max_blocks_per_seq) * block_size, partition_tokens);
  if (P > 65535) return PKV_ERR_PARTITION;
  if (sink_words < static_cast<size_t>(num_seqs) * num_kv_heads * P) return PKV_ERR_WORKSPACE;
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  return launch_table_scan(block_tables, context_lens, num_seqs, num_kv_heads, max_blocks_per_seq,
                           static_cast<int>(num_blocks), block_size, partition_tokens / block_size,
                           static_cast<int>(P), sink, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PKV_OK
             : PKV_ERR_CUDA;
}

int pkv_fp8_scale_from_amax(const void* x, int64_t n, int dtype, float* scale, void* stream) {
  if (n < 0) return PKV_ERR_BAD_SHAPE;
  if (!x || !scale) return PKV_ERR_NULL_POINTER;
  if (dtype != PKV_DTYPE_F32 && dtype != PKV_DTYPE_BF16) return PKV_ERR_BAD_DTYPE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0) return PKV_ERR_MISALIGNED;
  return launch_fp8_scale(x, n, dtype, scale, static_cast<cudaStream_t>(stream)) == cudaSuccess ? PKV_OK
                                                                                                  : PKV_ERR_CUDA;
}

int pkv_swap_blocks(const int64_t* src_dst_pairs, int64_t num_pairs, const void* src_key, const void* src_value,
                    int64_t src_num_blocks, void* dst_key, void* dst_value, int64_t dst_num_blocks,
                    int64_t block_bytes, int validate, void* stream) {
  if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || block_bytes <= 0 || block_bytes % 16 != 0)
    return PKV_ERR_BAD_SHAPE;
  if (num_pairs == 0) return PKV_OK;
  if (!src_dst_pairs || !src_key || !src_value || !dst_key || !dst_value) return PKV_ERR_NULL_POINTER;
  if (!aligned16(src_key) || !aligned16(src_value) || !aligned16(dst_key) || !aligned16(dst_value))
    return PKV_ERR_MISALIGNED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (validate) {
    const bool same = src_key == dst_key || src_value == dst_value;
    const int rc = check_pairs(src_dst_pairs, num_pairs, src_num_blocks, dst_num_blocks, same, st);
    if (rc) return rc;
  }
  unsigned* status = status_word();
  if (!status) return PKV_ERR_CUDA;
  return launch_block_copy(src_dst_pairs, num_pairs, src_key, src_value, src_num_blocks, dst_key, dst_value,
                           dst_num_blocks, block_bytes, status, st) == cudaSuccess
             ? PKV_OK
             : PKV_ERR_CUDA;
}

}  // extern "C"

/*
 * pagedkv.h -- C ABI of libpagedkv, the B200 (sm_100a) paged KV-cache decode path.
 *
 * Three operations, as the PagedAttention pages state the problem:
 *
 *   pkv_paged_kv_write          write each new token's K/V into its cache slot
 *   pkv_paged_attention_decode  single-query attention over a block-paged cache
 *   pkv_kv_block_copy           copy-on-write copies of shared blocks
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers marked "device" are CUDA device memory owned by the caller.  The
 *   library allocates no device memory; the caller passes the decode
 *   workspace.  Pointers must be 16-byte aligned (cache and q/k/v bases);
 *   integer arrays need natural alignment.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and return PKV_OK or a negative PKV_ERR_* code.  A negative code
 *   means nothing was launched.
 * - `validate` != 0 copies the index arrays (block tables, context lengths,
 *   slots, copy pairs) to the host, checks every id against the pool and
 *   returns PKV_ERR_OUT_OF_RANGE / PKV_ERR_BAD_COPY_PAIRS before launching.
 *   This synchronises the stream; it is meant for tests and debugging.
 * - Independently of `validate`, the kernels check every index they
 *   dereference.  An id outside the pool is never read or written: the access
 *   is skipped (reads yield zeros) and a bit is set in the library's device
 *   status word, read back with pkv_device_status().
 * - Cache layout (both caches, every dtype):
 *       [num_blocks][block_size][num_kv_heads][head_dim], contiguous.
 *   The pages give only the block's byte count (block_size x num_kv_heads x
 *   head_dim x dtype bytes, "vLLM — 把操作系统的分页搬进 GPU KV cache",
 *   实践案例 1); the dimension order is this library's choice.  A physical
 *   block is one contiguous span of block_size * num_kv_heads * head_dim
 *   elements.
 * - Element types: PKV_DTYPE_F32, PKV_DTYPE_BF16, PKV_DTYPE_FP8_E4M3 (OCP E4M3,
 *   per-tensor scale: a stored code c reads back as value(c) * scale).
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element types */
#define PKV_DTYPE_F32 0
#define PKV_DTYPE_BF16 1
#define PKV_DTYPE_FP8_E4M3 2

/* status codes */
#define PKV_OK 0
#define PKV_ERR_NULL_POINTER (-1)       /* a required pointer is NULL */
#define PKV_ERR_BAD_DTYPE (-2)          /* dtype code or dtype combination not supported */
#define PKV_ERR_HEAD_DIM (-3)           /* head_dim not in {64, 128} */
#define PKV_ERR_BLOCK_SIZE (-4)         /* block_size not in {8, 16, 32} */
#define PKV_ERR_HEAD_GROUPING (-5)      /* num_q_heads % num_kv_heads != 0, or group not in {1,2,4,8} */
#define PKV_ERR_WORKSPACE (-6)          /* workspace NULL or smaller than pkv_decode_workspace_bytes() */
#define PKV_ERR_BAD_SHAPE (-7)          /* a negative or zero size where a positive one is needed */
#define PKV_ERR_OUT_OF_RANGE (-8)       /* validate: a block id, slot or context length outside the pool */
#define PKV_ERR_BAD_COPY_PAIRS (-9)     /* validate: copy pairs whose result would depend on their order */
#define PKV_ERR_MISALIGNED (-10)        /* a data pointer is not 16-byte aligned */
#define PKV_ERR_CUDA (-11)              /* a CUDA runtime call or kernel launch failed */
#define PKV_ERR_TENSOR_MAP (-12)        /* the TMA descriptor for a cache could not be encoded */
#define PKV_ERR_PARTITION (-13)         /* partition_tokens not a positive multiple of block_size */

/* bits of the device status word (pkv_device_status) */
#define PKV_STATUS_BAD_BLOCK_ID 0x1u    /* decode met a block id outside [0, num_blocks) */
#define PKV_STATUS_BAD_CONTEXT 0x2u     /* decode met context_len < 0 or > max_blocks_per_seq * block_size */
#define PKV_STATUS_BAD_SLOT 0x4u        /* write met a slot >= num_blocks * block_size */
#define PKV_STATUS_BAD_COPY_PAIR 0x8u   /* block copy met an id outside [0, num_blocks) */
#define PKV_STATUS_WAIT_TIMEOUT 0x10u   /* a bounded wait inside a kernel gave up */
#define PKV_STATUS_BAD_QUERY_LOC 0x20u  /* multi-query met query_start_loc entries outside [0, total_q] or a
                                           q_len above max_q_len: that sequence's rows are left unwritten */
#define PKV_STATUS_BAD_GROUP 0x40u      /* shared-prefix decode met a group outside [0, num_seqs), empty, or
                                           wider than 8 columns: its shared unit was skipped */

/*
 * Human-readable name of a PKV_* status code (static storage).
 */
const char* pkv_status_string(int status);

/*
 * New-token KV write ("reshape_and_cache").
 *
 * Source: "vLLM 与 KV Cache", KV Cache：为什么需要缓存 -- each decode step
 * computes K and V of the new token only and appends them to the cache;
 * "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 -- the cache is a pool
 * of fixed-size blocks addressed through the sequence's block table.
 *
 * k, v            device, [num_tokens][num_kv_heads][head_dim] of in_dtype
 *                 (F32 or BF16), contiguous.
 * slot_mapping    device int64 [num_tokens]: the flat slot of each token,
 *                 block = slot / block_size, row = slot % block_size.  A
 *                 negative slot is a padding token and is skipped.  Slots
 *                 must be distinct (two tokens on one slot race); validate
 *                 rejects a repeated slot with PKV_ERR_OUT_OF_RANGE.
 * key_cache,      device, [num_blocks][block_size][num_kv_heads][head_dim] of
 * value_cache     cache_dtype; written in place.
 * cache_dtype     == in_dtype (the bytes are copied), or FP8_E4M3: the stored
 *                 code is E4M3(x * r) with r = 1/k_scale (1/v_scale for V)
 *                 rounded once to fp32 on the host, one fp32 multiply, round
 *                 to nearest even, saturating to +-448.
 * k_scale,        fp8 dequantisation scales (ignored for other cache types).
 * v_scale
 * Errors: PKV_ERR_NULL_POINTER, _BAD_DTYPE, _BAD_SHAPE, _MISALIGNED,
 * _OUT_OF_RANGE (validate), _CUDA.  num_tokens == 0 launches nothing.
 */
int pkv_paged_kv_write(const void* k, const void* v, const int64_t* slot_mapping, int64_t num_tokens,
                       void* key_cache, void* value_cache, int64_t num_blocks, int block_size,
                       int num_kv_heads, int head_dim, int in_dtype, int cache_dtype, float k_scale,
                       float v_scale, int validate, void* stream);

/*
 * Paged single-query decode attention.
 *
 * Source: "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 -- the kernel
 * reads the physical block id from the sequence's block_table, computes the
 * offset ("one more int load and one multiply"), then computes attention as
 * before; "vLLM KV Cache 实现机制", 1.2 -- logically contiguous, physically
 * scattered.  For every sequence b and query head hq:
 *     s_t = scale * <q[b,hq], K_t>  (t < context_lens[b]),
 *     out[b,hq] = sum_t softmax(s)_t V_t,
 * K_t / V_t being row t % block_size of physical block
 * block_tables[b][t / block_size], KV head hq / (num_q_heads / num_kv_heads).
 *
 * out             device, [num_seqs][num_q_heads][head_dim] of q_dtype.
 * q               device, [num_seqs][num_q_heads][head_dim] of q_dtype (F32 or BF16).
 * key_cache,      device, cache layout above, cache_dtype == q_dtype or FP8_E4M3.
 * value_cache
 * block_tables    device int32 [num_seqs][max_blocks_per_seq].
 * context_lens    device int32 [num_seqs]: tokens to attend, including the
 *                 one written by this step's pkv_paged_kv_write.  0 gives a
 *                 zero output row.
 * scale           softmax scale (usually 1/sqrt(head_dim)).
 * k_scale,        fp8 dequantisation scales (ignored for other cache types).
 * v_scale
 * partition_tokens  0 = automatic; otherwise the split-context partition
 *                 length in tokens (a positive multiple of block_size).  Each
 *                 (sequence, kv head, partition) is one CTA; sequences with
 *                 more than one partition are merged by a second kernel.
 * workspace       device scratch of at least pkv_decode_workspace_bytes(...)
 *                 bytes (same arguments); not read before it is written.
 *                 Layout, with P = pkv_decode_max_partitions(...):
 *                 float ml[num_seqs][num_q_heads][P][2] = (m, l): a reference
 *                 logit m (natural units, at most the partition's max) and
 *                 l = sum e^{s - m}, so m + ln l is the partition's log-sum-exp;
 *                 then float o[num_seqs][num_q_heads][P][head_dim] (normalised
 *                 partial outputs), starting at a 256-byte aligned offset.
 * Supported: head_dim in {64, 128}, block_size in {8, 16, 32}, query heads
 * per KV head in {1, 2, 4, 8}.
 * Errors: PKV_ERR_NULL_POINTER, _BAD_DTYPE, _HEAD_DIM, _BLOCK_SIZE,
 * _HEAD_GROUPING, _WORKSPACE, _BAD_SHAPE, _MISALIGNED, _PARTITION,
 * _OUT_OF_RANGE (validate), _TENSOR_MAP, _CUDA.  num_seqs == 0 launches nothing.
 */
int pkv_paged_attention_decode(void* out, const void* q, const void* key_cache, const void* value_cache,
                               const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                               float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                               void* workspace, size_t workspace_bytes, int validate, void* stream);

/*
 * Decode step with the new-token write fused in: append, then attend.
 *
 * Source: "vLLM 与 KV Cache", KV Cache：为什么需要缓存 -- each decode step
 * computes the new token's K,V, appends them to the cache and attends over
 * all cached tokens.  For every sequence b with context_lens[b] >= 1, the
 * new token k_new[b] / v_new[b] is written to logical position
 * context_lens[b] - 1, i.e. row (ctx-1) % block_size of physical block
 * block_tables[b][(ctx-1) / block_size] (that block must be allocated), with
 * the same bytes pkv_paged_kv_write would store for that slot; then the
 * result equals pkv_paged_attention_decode's.  One kernel launch (plus the
 * split-context merge) instead of two: the CTA that reads the sequence's last
 * block writes its KV head's slice of the new token first.
 *
 * k_new, v_new   device [num_seqs][num_kv_heads][head_dim] of q_dtype, 16-byte aligned.
 * Other arguments and errors: as pkv_paged_attention_decode (key_cache and
 * value_cache are written).
 */
int pkv_paged_decode_append(void* out, const void* q, const void* k_new, const void* v_new, void* key_cache,
                            void* value_cache, const int32_t* block_tables, const int32_t* context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale, float v_scale,
                            int q_dtype, int cache_dtype, int partition_tokens, void* workspace,
                            size_t workspace_bytes, int validate, void* stream);

/*
 * Paged decode attention with shared prefixes read once.
 *
 * Source: "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 and 实践案例 2 --
 * the n candidates of parallel sampling share their prompt's physical blocks
 * (ref_count n), one copy of the prompt's KV for all of them; the attention is
 * pkv_paged_attention_decode's.  This call computes exactly that attention
 * (every output row equals pkv_paged_attention_decode's for the same
 * arguments, up to rounding order), but reads each shared block once for all
 * the sequences that share it: the queries of a group's members are the
 * columns of one tensor-core tile over the group's shared blocks, each member
 * then attends its own blocks, and the two partial softmaxes are merged by the
 * softmax identity.  With k_new / v_new (both or neither) each sequence's new
 * token is written first, as by pkv_paged_decode_append.
 *
 * group_start     device int32 [num_groups + 1]: the sequences of group g are
 *                 group_start[g] .. group_start[g+1] - 1 (consecutive; every
 *                 sequence in exactly one group; a group of one is allowed).
 * shared_blocks   device int32 [num_groups]: the first shared_blocks[g] logical
 *                 blocks of every member of group g are the same physical
 *                 blocks (the group's first member's table is read for them),
 *                 and lie within every member's context -- before its new
 *                 token when k_new is given.  validate checks all of this; a
 *                 wrong grouping without validate gives wrong results.
 * max_group_size  the largest group; max_group_size x (num_q_heads /
 *                 num_kv_heads) <= 8 (the tile's columns), else PKV_ERR_BAD_SHAPE.
 * workspace       device scratch of pkv_decode_shared_prefix_workspace_bytes()
 *                 bytes, 256-byte aligned (the shared and own partials of every
 *                 (sequence, head)).
 * Supported: bf16 q and caches, head_dim 128, block_size 16 or 32, 1/2/4/8
 * query heads per KV head.  Other arguments and errors: as
 * pkv_paged_decode_append.  num_seqs == 0 launches nothing.
 */
int pkv_paged_attention_decode_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                                             void* key_cache, void* value_cache, const int32_t* block_tables,
                                             const int32_t* context_lens, const int32_t* group_start,
                                             const int32_t* shared_blocks, int num_seqs, int num_groups,
                                             int max_group_size, int num_q_heads, int num_kv_heads, int head_dim,
                                             int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale,
                                             int q_dtype, int cache_dtype, int partition_tokens, void* workspace,
                                             size_t workspace_bytes, int validate, void* stream);

/* Partition length pkv_paged_attention_decode_shared_prefix uses: partition_tokens
 * when non-zero (a positive multiple of block_size, at most 16384, else
 * PKV_ERR_PARTITION), otherwise the automatic choice of pkv_decode_partition_tokens
 * made for the groups' shared units (num_groups x num_kv_heads) on the bf16
 * tensor-core kernel, with at least three partitions per long context instead of
 * four (the members' own units fill the last wave).  Negative PKV_ERR_* on bad
 * arguments.  A sizing helper of this library. */
int pkv_decode_shared_prefix_partition_tokens(int num_groups, int num_kv_heads, int block_size,
                                              int max_blocks_per_seq, int partition_tokens);

/* Workspace bytes of pkv_paged_attention_decode_shared_prefix (0 for
 * unsupported arguments): 2 x ceil(max_blocks_per_seq x block_size / P)
 * partial slots per (sequence, query head), P the partition length above. */
size_t pkv_decode_shared_prefix_workspace_bytes(int num_seqs, int num_groups, int num_q_heads, int num_kv_heads,
                                                int head_dim, int block_size, int max_blocks_per_seq,
                                                int partition_tokens);

/*
 * Paged decode attention that allocates nothing and takes no workspace.
 *
 * The PagedAttention pages have no counterpart of this call; it is a
 * convenience of this library.  pkv_paged_attention_decode needs device
 * scratch for its split-context partials and takes it from the caller.
 * Some callers have none to give at that point: an engine that reserved
 * nearly all device memory for its KV block pool up front and keeps no
 * allocator for temporaries, code that must not call cudaMalloc inside a
 * decode step (cudaMalloc can synchronise the whole device), or a binding
 * from an environment without a device allocator.  This call computes
 * exactly what pkv_paged_attention_decode computes, with the same arguments
 * (minus workspace, workspace_bytes and validate) and the same kernels, but
 * keeps the partials in a fixed array of PKV_DECODE_STATIC_SCRATCH_BYTES
 * compiled into the library.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * - Every GPU on which the library's device code is loaded holds that array
 *   until the process exits.
 * - The first call on each device that needs partials looks up the array's
 *   device address (cudaGetSymbolAddress, with that device current) and
 *   caches it; make that first call before any stream capture.  Calls that
 *   need no partials (pkv_decode_workspace_bytes() == 0, e.g. num_seqs == 0
 *   or one partition per sequence) do not touch the array.
 * - All calls on a device share the array, and it keeps the partials of the
 *   last call.  Nothing in it has to start at zero.  Calls that may run at
 *   the same time on the GPU (other streams, or host threads without an
 *   order between them) race on the array and give wrong results: order
 *   them on one stream.
 * - A call whose partials need more than PKV_DECODE_STATIC_SCRATCH_BYTES
 *   (pkv_decode_workspace_bytes() for the same call) returns
 *   PKV_ERR_WORKSPACE and launches nothing; a larger partition_tokens lowers
 *   the need.  Argument errors take precedence over it, in the order
 *   pkv_paged_attention_decode checks them.
 * Other errors: as pkv_paged_attention_decode.
 */
#define PKV_DECODE_STATIC_SCRATCH_BYTES ((size_t)16 << 20)
int pkv_paged_attention_decode_static(void* out, const void* q, const void* key_cache, const void* value_cache,
                                      const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                                      int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                      int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                                      float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                                      void* stream);

/*
 * Partition length (tokens) the decode call uses for these arguments:
 * partition_tokens if it is non-zero, else the automatic choice.  The
 * automatic choice depends on the shape, on which kernel serves it
 * (cache_dtype, head_dim and the query-head group select it) and on the
 * current device's SM count.  A single partition when the longest possible
 * context (max_blocks_per_seq * block_size) is 512 tokens or less.  With
 * fewer (sequence, KV head) pairs than four waves of the kernel's resident
 * CTAs: the largest power of two <= 4096 that splits that context into at
 * least 4 partitions and gives at least three quarters of a wave of CTAs.
 * With more pairs: the largest power of two <= 2048 that gives three quarters
 * of a wave (so one partition for contexts up to 2048 tokens).
 * Returns a negative PKV_ERR_* code for unsupported arguments.  (This and the
 * other sizing helpers below are this library's; the pages have no
 * counterpart: the split-context partition is its design for long contexts.)
 */
int pkv_decode_partition_tokens(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_blocks_per_seq, int cache_dtype, int partition_tokens);

/* Partitions per sequence the workspace must hold (max over sequences); same arguments. */
int pkv_decode_max_partitions(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int max_blocks_per_seq, int cache_dtype, int partition_tokens);

/* Workspace bytes pkv_paged_attention_decode needs for these arguments
 * (0 when no sequence can need more than one partition). */
size_t pkv_decode_workspace_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int cache_dtype, int partition_tokens);

/*
 * Copy-on-write block copy.
 *
 * Source: "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 (引用计数 +
 * copy-on-write), 实践案例 2 and 踩过的坑 -- blocks shared by n sequences
 * carry ref_count n; a sequence about to write into a shared block first
 * gets a private copy (n-1 copies on the first parallel-sampling step).
 *
 * src_dst_pairs   device int64 [num_pairs][2] of (src, dst) physical block ids.
 *                 Every pair copies block src onto block dst in BOTH caches,
 *                 byte for byte.  The destinations must be distinct and no
 *                 destination may also be a source (so the result does not
 *                 depend on order); validate checks this.
 * key_cache,      device pools of num_blocks blocks of block_bytes bytes each.
 * value_cache
 * block_bytes     bytes of one block of one cache: block_size * num_kv_heads
 *                 * head_dim * dtype size; a multiple of 16.
 * Errors: PKV_ERR_NULL_POINTER, _BAD_SHAPE, _MISALIGNED, _OUT_OF_RANGE /
 * _BAD_COPY_PAIRS (validate), _CUDA.  num_pairs == 0 launches nothing.
 */
int pkv_kv_block_copy(const int64_t* src_dst_pairs, int64_t num_pairs, void* key_cache, void* value_cache,
                      int64_t num_blocks, int64_t block_bytes, int validate, void* stream);

/*
 * Multi-query paged attention: several new query tokens per sequence
 * (chunked prefill, speculative-decoding verification), causal over the
 * paged cache.
 *
 * Source: the decode step's attention ("vLLM — 把操作系统的分页搬进 GPU KV
 * cache", 核心要点; "vLLM 与 KV Cache", KV Cache：为什么需要缓存) with several
 * new tokens per step -- an extension of this library; the pages describe one
 * new token per step.  The q_len_b = query_start_loc[b+1] - query_start_loc[b]
 * queries of sequence b are its LAST q_len_b positions (their K/V already in
 * the cache, written with pkv_paged_kv_write): query i sits at position
 * p = context_lens[b] - q_len_b + i and attends the logical tokens 0..p.
 *
 * out, q            device [total_q][num_q_heads][head_dim] bf16; rows of
 *                   sequence b are query_start_loc[b] .. query_start_loc[b+1]-1.
 * key_cache,        device, cache layout above: BF16, or FP8_E4M3 with the
 * value_cache       dequantisation scales k_scale, v_scale (both > 0; ignored
 *                   for BF16).
 * query_start_loc   device int32 [num_seqs + 1], non-decreasing, starting at 0,
 *                   ending at total_q; every q_len_b <= max_q_len and
 *                   <= context_lens[b] (validate checks all of this; without
 *                   validate, the first q_len_b - context_lens[b] queries of a
 *                   sequence with more queries than context tokens sit at
 *                   negative positions and get zero rows).  Independently of
 *                   validate, the kernels skip a sequence whose rows would fall
 *                   outside [0, total_q) or whose q_len_b exceeds max_q_len:
 *                   nothing of it is read or written (its rows of out keep their
 *                   previous bytes) and PKV_STATUS_BAD_QUERY_LOC is set.
 * workspace         device scratch of pkv_multiquery_workspace_bytes(...) bytes
 *                   (same arguments; 0 when no split is needed), 256-byte aligned.
 * Supported: bf16 q, bf16 or fp8 E4M3 caches, head_dim 128, block_size 16 or
 * 32, 1/2/4/8 query heads per KV head.  Runs on the tensor cores: up to 16
 * rows per (sequence, KV head) -- rows = max_q_len x query heads per KV head
 * -- on mma.sync m16n8k16; more rows (prefill, grouped verification) on
 * tcgen05 with 128-row tiles and 128-token KV tiles.  bf16 caches: bf16
 * operands, P as a bf16 high part and residual (~16 significant bits).  fp8
 * caches: the codes widened exactly to fp16 in shared memory, q rounded once
 * to fp16 (exact for |q| in [2^-14, 65504]), fp16 operands and one fp16 P, in
 * both kernels.  Other arguments and errors: as pkv_paged_attention_decode.
 */
int pkv_paged_attention_multiquery(void* out, const void* q, const void* key_cache, const void* value_cache,
                                   const int32_t* block_tables, const int32_t* context_lens,
                                   const int32_t* query_start_loc, int num_seqs, int total_q, int max_q_len,
                                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                   int max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                                   float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                                   void* workspace, size_t workspace_bytes, int validate, void* stream);

/* Split-context partition length pkv_paged_attention_multiquery uses:
 * partition_tokens if non-zero (a multiple of block_size, at most 16384), else
 * automatic -- one partition when (sequences x KV heads x query-row tiles of
 * the kernel that serves these rows and cache_dtype) already gives two waves
 * of its resident CTAs, else the longest context split so that it does, in
 * multiples of 256 tokens.  Negative PKV_ERR_* for unsupported arguments.  A
 * sizing helper of this library (no counterpart on the pages). */
int pkv_multiquery_partition_tokens(int num_seqs, int max_q_len, int num_q_heads, int num_kv_heads, int block_size,
                                    int max_blocks_per_seq, int cache_dtype, int partition_tokens);

/* Workspace bytes pkv_paged_attention_multiquery needs (0 when no context is
 * split): float (m, l) then, at a 256-byte boundary, float o[d] per (query
 * token, query head, partition).  A sizing helper of this library. */
size_t pkv_multiquery_workspace_bytes(int num_seqs, int total_q, int max_q_len, int num_q_heads, int num_kv_heads,
                                      int head_dim, int block_size, int max_blocks_per_seq, int cache_dtype,
                                      int partition_tokens);

/*
 * Per-tensor fp8 scale on the device: *scale = amax(|x|) / 448 (one fp32
 * division; 1.0 when x is all zeros), the scale that maps the largest
 * magnitude onto the largest finite E4M3 value.
 *
 * Source: the "--kv-cache-dtype fp8" option of "vLLM KV Cache 实现机制", 2.3;
 * the pages give no calibration rule -- amax / 448 per tensor is this
 * library's reading.  Pass the value as k_scale / v_scale of the other calls
 * (copy it to the host first).
 *
 * x       device, n elements of dtype (F32 or BF16), 16-byte aligned.
 * scale   device float, written on `stream` (its previous content is ignored).
 * NaN elements are ignored (fmax semantics).  Errors: PKV_ERR_NULL_POINTER, _BAD_DTYPE,
 * _BAD_SHAPE, _MISALIGNED, _CUDA.
 */
int pkv_fp8_scale_from_amax(const void* x, int64_t n, int dtype, float* scale, void* stream);

/*
 * Block swap between two pools (device <-> pinned host, or any two pools).
 *
 * Source: "vLLM KV Cache 实现机制", 1.2 (blocks migrate between GPU memory and
 * CPU RAM block by block when GPU memory runs short) and 2.1 (CPU offloading
 * tier); "vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 3 (SWAP: copy the
 * blocks to CPU memory and back when needed).
 * Each (src, dst) pair of src_dst_pairs copies block src of the source pool
 * (src_key / src_value) onto block dst of the destination pool (dst_key /
 * dst_value), byte for byte, in ONE kernel launch for all pairs.  Either pool
 * may live in page-locked host memory allocated with cudaHostAlloc /
 * cudaMallocHost (or registered with cudaHostRegister): the kernel reads or
 * writes it directly through unified addressing.  Pageable host memory is not
 * supported.  Both pools use the cache layout above with the same block_bytes.
 *
 * src_dst_pairs   device int64 [num_pairs][2] (src block id, dst block id).
 *                 Destinations must be distinct (and, within one pool, never a
 *                 source); validate checks this.
 * Errors: PKV_ERR_NULL_POINTER, _BAD_SHAPE, _MISALIGNED, _OUT_OF_RANGE /
 * _BAD_COPY_PAIRS (validate), _CUDA.  num_pairs == 0 launches nothing.
 */
int pkv_swap_blocks(const int64_t* src_dst_pairs, int64_t num_pairs, const void* src_key, const void* src_value,
                    int64_t src_num_blocks, void* dst_key, void* dst_value, int64_t dst_num_blocks,
                    int64_t block_bytes, int validate, void* stream);

/*
 * One whole decode step with the per-step inputs and the output in HOST memory.
 *
 * Source: the decode step of "vLLM 与 KV Cache", KV Cache：为什么需要缓存 (append
 * the new token's K,V, then attend over the cache) with the copy-on-write of
 * "vLLM — 把操作系统的分页搬进 GPU KV cache", 核心要点 (copy first, then write).
 * Enqueued on `stream`, in order: host -> device copies of every per-step
 * input into `staging`; pkv_kv_block_copy (if num_pairs > 0);
 * pkv_paged_kv_write (if num_tokens > 0); pkv_paged_attention_decode; the
 * device -> host copy of the output.  Synchronise `stream` before reading
 * out_host or reusing the input buffers.  The host buffers should be pinned
 * (page-locked): pageable buffers make the copies synchronous.
 *
 * out_host, q_host      host [num_seqs][num_q_heads][head_dim] of q_dtype.
 * k_host, v_host,       host [num_tokens][num_kv_heads][head_dim] of q_dtype and
 * slot_mapping_host     host int64 [num_tokens] (see pkv_paged_kv_write).
 * block_tables_host,    host int32 [num_seqs][max_blocks_per_seq], [num_seqs].
 * context_lens_host
 * copy_pairs_host       host int64 [num_pairs][2] (may be NULL when num_pairs == 0).
 * key_cache, value_cache  device caches (layout above).
 * staging               device scratch of at least pkv_decode_step_staging_bytes(...)
 *                       bytes, 256-byte aligned, caller-owned; holds the copied
 *                       inputs, the output and the decode workspace.
 * Other arguments and errors: as pkv_paged_attention_decode / pkv_paged_kv_write /
 * pkv_kv_block_copy (without validation).  Argument errors are returned before
 * anything is enqueued.
 */
int pkv_decode_step_host(void* out_host, const void* q_host, const void* k_host, const void* v_host,
                         const int64_t* slot_mapping_host, int64_t num_tokens, const int32_t* block_tables_host,
                         const int32_t* context_lens_host, const int64_t* copy_pairs_host, int64_t num_pairs,
                         void* key_cache, void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale,
                         float k_scale, float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                         void* staging, size_t staging_bytes, void* stream);

/* Staging bytes pkv_decode_step_host / _async need for these arguments (a
 * sizing helper of this library). */
size_t pkv_decode_step_staging_bytes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                     int max_blocks_per_seq, int q_dtype, int cache_dtype, int partition_tokens,
                                     int64_t num_tokens, int64_t num_pairs);

/*
 * pkv_decode_step_host with its three parts on three streams, so that a caller
 * can keep several steps in flight: the host -> device copies on
 * copy_in_stream, the kernels on compute_stream (after those copies), the
 * device -> host copy of the output on copy_out_stream (after the kernels).
 * The library orders the parts of one step with events of its own; the order
 * BETWEEN steps is the caller's: the kernels of consecutive steps follow each
 * other on compute_stream, and a staging buffer (and its host output) may be
 * reused only after the step that last used it has copied its output out.
 *
 * Source: as pkv_decode_step_host (the pages' decode step); the overlap of the
 * next step's input copies with this step's kernels is this library's.
 *
 * staging_free_event  cudaEvent_t or NULL: copy_in_stream waits for it before
 *                     the copies in (pass the done_event of the step that last
 *                     used this staging buffer).
 * done_event          cudaEvent_t or NULL: recorded on copy_out_stream after
 *                     the copy out; out_host is valid once it has completed.
 * All other arguments, the order of operations inside the step and the errors:
 * as pkv_decode_step_host.  The three streams may be the same stream.
 */
int pkv_decode_step_host_async(void* out_host, const void* q_host, const void* k_host, const void* v_host,
                               const int64_t* slot_mapping_host, int64_t num_tokens, const int32_t* block_tables_host,
                               const int32_t* context_lens_host, const int64_t* copy_pairs_host, int64_t num_pairs,
                               void* key_cache, void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads,
                               int head_dim, int block_size, int max_blocks_per_seq, int64_t num_blocks, float scale,
                               float k_scale, float v_scale, int q_dtype, int cache_dtype, int partition_tokens,
                               void* staging, size_t staging_bytes, void* copy_in_stream, void* compute_stream,
                               void* copy_out_stream, void* staging_free_event, void* done_event);

/*
 * pkv_decode_step_host_async for groups of sequences that share their
 * prompt's blocks: the decode is pkv_paged_attention_decode_shared_prefix
 * (each shared block read once for the whole group), with each sequence's new
 * token written first inside it.
 *
 * Source: "vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 2 (n candidates
 * share the prompt's blocks) and 核心要点 (copy-on-write before the write);
 * the step with host buffers is this library's.
 * Enqueued in order: the host -> device copies (on copy_in_stream, after
 * staging_free_event); pkv_kv_block_copy of copy_pairs (if num_pairs > 0);
 * the shared-prefix decode with the new tokens fused in (on compute_stream);
 * the device -> host copy of the output (on copy_out_stream), then done_event.
 *
 * k_new_host,          host [num_seqs][num_kv_heads][head_dim] of q_dtype: the
 * v_new_host           token each sequence appends at position
 *                      context_lens[b] - 1 (both, or both NULL for none).
 * group_start_host,    host int32 [num_groups + 1] and [num_groups]: the groups
 * shared_blocks_host   (see pkv_paged_attention_decode_shared_prefix).
 * max_group_size       the largest group.
 * staging              device scratch of at least
 *                      pkv_decode_step_shared_prefix_staging_bytes(...) bytes,
 *                      256-byte aligned, caller-owned.
 * Other arguments, errors and the stream / event contract: as
 * pkv_decode_step_host_async and pkv_paged_attention_decode_shared_prefix
 * (bf16 only; no validation).  Argument errors are returned before anything
 * is enqueued.
 */
int pkv_decode_step_host_shared_prefix_async(void* out_host, const void* q_host, const void* k_new_host,
                                             const void* v_new_host, const int32_t* block_tables_host,
                                             const int32_t* context_lens_host, const int32_t* group_start_host,
                                             const int32_t* shared_blocks_host, int num_groups, int max_group_size,
                                             const int64_t* copy_pairs_host, int64_t num_pairs, void* key_cache,
                                             void* value_cache, int num_seqs, int num_q_heads, int num_kv_heads,
                                             int head_dim, int block_size, int max_blocks_per_seq,
                                             int64_t num_blocks, float scale, int q_dtype, int cache_dtype,
                                             int partition_tokens, void* staging, size_t staging_bytes,
                                             void* copy_in_stream, void* compute_stream, void* copy_out_stream,
                                             void* staging_free_event, void* done_event);

/* Staging bytes pkv_decode_step_host_shared_prefix_async needs for these
 * arguments (0 for unsupported ones; a sizing helper of this library). */
size_t pkv_decode_step_shared_prefix_staging_bytes(int num_seqs, int num_groups, int num_q_heads, int num_kv_heads,
                                                   int head_dim, int block_size, int max_blocks_per_seq,
                                                   int q_dtype, int partition_tokens, int64_t num_pairs);

/*
 * Prefix caching by hash chain (host side; no device work).
 *
 * Source: "vLLM KV Cache 实现机制", 4.2 -- a full block is identified by a hash
 * of (the parent block's hash, the exact tokens in the block, an extra hash
 * for multimodal inputs), and requests whose prompts share a prefix reuse the
 * cached blocks; 3.2 -- reference counts keep shared blocks from eviction,
 * which is least-recently-used.  The hash is FNV-1a 64 over the little-endian
 * bytes of (parent hash, the block's int32 tokens, extra_hash); the first
 * block's parent hash is 0.  Only full blocks are hashed or cached.  Every
 * cache hit also compares the stored tokens, parent and extra hash, so two
 * blocks with colliding hashes are never shared.  The cache maps blocks to the
 * caller's physical block ids; it never allocates or frees device blocks.
 * The functions of one cache are thread-safe.
 *
 * pkv_prefix_block_hashes: hashes of the num_tokens / block_size full blocks
 *   (chained from parent_hash) into hashes_out; returns that count.
 * pkv_prefix_cache_create / _destroy: a cache of at most capacity_blocks
 *   entries for blocks of block_size tokens (NULL on bad arguments).
 * pkv_prefix_cache_match: the longest cached prefix of `tokens` (at most
 *   max_blocks blocks): writes its physical block ids, takes one reference
 *   on each and marks them recently used; returns the number of blocks.
 * pkv_prefix_cache_insert: registers the first num_blocks full blocks of
 *   `tokens` with physical ids block_ids (one reference each, held by the
 *   caller); blocks already cached get one more reference instead.  Returns
 *   the number of new entries, or PKV_ERR_OUT_OF_RANGE (inserting nothing)
 *   when they would exceed the capacity -- evict first.
 * pkv_prefix_cache_release: drops one reference from each of the first
 *   num_blocks cached blocks of `tokens`; returns how many were released.
 * pkv_prefix_cache_evict: removes up to max_evict unreferenced entries, least
 *   recently used first, writing their physical ids (now free for the
 *   caller's pool); returns the count.
 * pkv_prefix_cache_size: number of entries.
 * Errors: PKV_ERR_NULL_POINTER, PKV_ERR_BAD_SHAPE, PKV_ERR_OUT_OF_RANGE.
 */
int64_t pkv_prefix_block_hashes(const int32_t* tokens, int64_t num_tokens, int block_size, uint64_t parent_hash,
                                uint64_t extra_hash, uint64_t* hashes_out);
void* pkv_prefix_cache_create(int block_size, int64_t capacity_blocks);
void pkv_prefix_cache_destroy(void* cache);
int64_t pkv_prefix_cache_size(void* cache);
int64_t pkv_prefix_cache_match(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                               int32_t* block_ids_out, int64_t max_blocks);
int64_t pkv_prefix_cache_insert(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                                const int32_t* block_ids, int64_t num_blocks);
int64_t pkv_prefix_cache_release(void* cache, const int32_t* tokens, int64_t num_tokens, uint64_t extra_hash,
                                 int64_t num_blocks);
int64_t pkv_prefix_cache_evict(void* cache, int64_t max_evict, int32_t* evicted_ids_out);

/*
 * The block-table reads of a decode launch, alone (a measurement aid; the
 * pages have no counterpart).  Runs the decode grid -- one CTA per (kv head,
 * partition of partition_tokens tokens, sequence) -- and in each CTA only the
 * coalesced, range-checked reads of that partition's physical block ids from
 * block_tables, the "one more int load" of "vLLM — 把操作系统的分页搬进 GPU KV
 * cache", 核心要点.  No KV byte is read.  Its time and L2 hit rate, next to the
 * decode's, show what the indirection costs.
 *
 * block_tables,   device, as pkv_paged_attention_decode.
 * context_lens
 * partition_tokens  the decode's partition length (pkv_decode_partition_tokens),
 *                 a positive multiple of block_size; there is no automatic choice.
 * sink            device unsigned [num_seqs][P][num_kv_heads], P = ceil(max_blocks_per_seq
 *                 * block_size / partition_tokens): one word per CTA (a hash of its ids).
 * Out-of-pool ids and context lengths set the status bits the decode sets.
 * Errors: PKV_ERR_BAD_SHAPE, _BLOCK_SIZE, _PARTITION, _NULL_POINTER,
 * _WORKSPACE (sink_words too small), _CUDA.  num_seqs == 0 launches nothing.
 */
int pkv_decode_table_scan(const int32_t* block_tables, const int32_t* context_lens, int num_seqs, int num_kv_heads,
                          int block_size, int max_blocks_per_seq, int64_t num_blocks, int partition_tokens,
                          unsigned* sink, size_t sink_words, void* stream);

/*
 * Self-test of the failure reporting (the pages have no counterpart).  Every
 * wait inside the library's kernels gives up after a time limit, sets
 * PKV_STATUS_WAIT_TIMEOUT in the device status word and lets the kernel
 * return.  This call runs that path on purpose: one warp waits, through the
 * same bounded-wait helper, on an mbarrier that nothing completes, for
 * limit_ns nanoseconds (at most 0.1 s); no copy or MMA is started, so nothing
 * is in flight when it gives up.  Afterwards PKV_STATUS_WAIT_TIMEOUT is set
 * and *gave_up (device unsigned) is 1; the context stays usable.
 * Errors: PKV_ERR_BAD_SHAPE (limit outside (0, 1e8]), _NULL_POINTER, _CUDA.
 */
int pkv_selftest_wait_timeout(int64_t limit_ns, unsigned* gave_up, void* stream);

/*
 * Reads the current device's status word (PKV_STATUS_* bits) into *status,
 * after synchronising `stream`; clears it if `clear` != 0.  The library's
 * failure reporting (in-kernel guards and bounded waits set the bits); the
 * pages have no counterpart.
 */
int pkv_device_status(unsigned* status, int clear, void* stream);

/* Number of kernel launches this library issued on this process (all devices):
 * the library's own accounting, no counterpart on the pages. */
uint64_t pkv_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */

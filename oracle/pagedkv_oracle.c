/*
 * pagedkv_oracle.c -- plain, slow CPU oracle for the paged KV-cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The
 * product (paged_kv_cache_450_b200 and its CUDA library) never imports,
 * links or calls it, and it shares no code, header, table or constant with
 * the product.
 *
 * What it computes, and where the pages say so:
 *
 *  - Paged decode attention.  "vLLM — 把操作系统的分页搬进 GPU KV cache",
 *    section 核心要点 (间接寻址): every sequence owns a block_table that maps
 *    its logical block N to a physical block M anywhere in the pool; the
 *    attention kernel first looks up the physical block id, then computes
 *    the offset, and otherwise computes attention unchanged.  "vLLM KV Cache
 *    实现机制", section 1.2: the logical view is contiguous while the
 *    physical blocks are scattered.  The result is therefore exactly dense
 *    single-query attention over the logically gathered K/V:
 *        s_t = scale * <q, K_t>,  out = sum_t e^{s_t - m} V_t / sum_t e^{s_t - m},
 *    m = max_t s_t (max subtraction does not change the value).  Everything
 *    here is fp64 with libm exp.
 *
 *  - New-token KV write.  "vLLM 与 KV Cache", section "KV Cache：为什么需要
 *    缓存": each step computes K,V of the new token only and appends them to
 *    the cache.  A token with slot s lands in physical block s / block_size,
 *    row s % block_size (the slot is the caller's flat index into the pool);
 *    a negative slot marks a padding token that is skipped.
 *
 *  - Copy-on-write block copy.  "vLLM — 把操作系统的分页搬进 GPU KV cache",
 *    section 核心要点 (引用计数 + copy-on-write) and 实践案例 2: before a
 *    sequence writes into a block shared with others it gets a private copy.
 *    The copy is byte-for-byte.
 *
 *  - Split-context partials and their merge: the partition pass computes,
 *    over a token range, (m_p, l_p = sum e^{s-m_p}, o_p = sum e^{s-m_p} V / l_p);
 *    the merge rescales to the global max M:
 *        out = sum_p l_p e^{m_p-M} o_p / sum_p l_p e^{m_p-M}.
 *    This is the softmax identity, written out; the pages do not describe a
 *    split (it is part of the decode step as specified for this library).
 *
 *  - FP8 E4M3 (the "--kv-cache-dtype fp8" option of "vLLM KV Cache 实现机制",
 *    section 2.3).  The pages give no format details; the encoding used is the
 *    OCP 8-bit floating point E4M3 definition: 1 sign bit, 4 exponent bits
 *    with bias 7, 3 mantissa bits, subnormals at exponent field 0, no
 *    infinities, NaN only at S.1111.111, largest finite value 448.  Values are
 *    stored as E4M3(x * (1/scale)) with round-to-nearest-even and saturation
 *    to +-448; they read back as code_value * scale.  The reciprocal 1/scale
 *    is rounded to fp32 once, and the product x * (1/scale) is one fp32
 *    multiply (both are reading choices of this library, applied identically
 *    on both sides).
 *
 * Cache layout (the pages give only the byte count block_size x num_kv_heads
 * x head_dim x 2 in "vLLM — 把操作系统的分页搬进 GPU KV cache", 实践案例 1; the
 * order of the dimensions is this library's reading): key_cache and
 * value_cache are [num_blocks][block_size][num_kv_heads][head_dim].
 *
 * Grouped-query attention: query head hq reads KV head hq / (Hq / Hkv).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

#define ORC_OK 0
#define ORC_EINVAL (-1)
#define ORC_ERANGE (-2)

/* ---------- element formats ---------------------------------------------- */

static int elem_size(int dtype) {
  switch (dtype) {
    case ORC_F32: return 4;
    case ORC_BF16: return 2;
    case ORC_E4M3: return 1;
    default: return 0;
  }
}

/* bf16 is the top half of an IEEE binary32; the value is exact in double. */
static double bf16_bits_to_double(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* OCP E4M3: value of one code, from the format definition. */
double orc_e4m3_to_double(uint8_t c) {
  int sign = (c >> 7) & 1;
  int e = (c >> 3) & 0xF;
  int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = ldexp((double)m / 8.0, -6); /* subnormal: 0.mmm x 2^(1-7) */
  else
    v = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -v : v;
}

/* OCP E4M3 encoding of a binary32 value: round to nearest, ties to the even
 * code (even mantissa), saturate finite overflow and infinities to +-448,
 * NaN to the NaN code.  Written from the definition: find the spacing of
 * representable values at |x|, round |x| to a multiple of it, then split the
 * rounded value into exponent and mantissa fields. */
uint8_t orc_e4m3_from_float(float xf) {
  double x = (double)xf;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (isnan(x)) return (uint8_t)(sign | 0x7F);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E); /* satfinite: +-448 */
  if (a == 0.0) return sign;
  int e2; /* a = f * 2^e2 with f in [0.5, 1) -> unbiased exponent e2 - 1 */
  frexp(a, &e2);
  int ue = e2 - 1;
  if (ue < -6) ue = -6;                 /* subnormal range shares 2^-6's spacing */
  double quantum = ldexp(1.0, ue - 3);  /* 3 mantissa bits */
  double r = nearbyint(a / quantum);    /* a / quantum is exact; default mode = nearest-even */
  double v = r * quantum;
  if (v >= 448.0) return (uint8_t)(sign | 0x7E);
  if (v == 0.0) return sign;
  if (v < ldexp(1.0, -6)) { /* subnormal: v = m * 2^-9 */
    int m = (int)(v / ldexp(1.0, -9));
    return (uint8_t)(sign | m);
  }
  frexp(v, &e2);
  int be = (e2 - 1) + 7;
  double frac = v / ldexp(1.0, e2 - 1) - 1.0; /* in [0, 1) in steps of 1/8 */
  int m = (int)(frac * 8.0);
  return (uint8_t)(sign | (be << 3) | m);
}

static double load_elem(const void* base, int64_t idx, int dtype, double fp8_scale) {
  switch (dtype) {
    case ORC_F32: {
      float f;
      memcpy(&f, (const char*)base + idx * 4, 4);
      return (double)f;
    }
    case ORC_BF16: {
      uint16_t h;
      memcpy(&h, (const char*)base + idx * 2, 2);
      return bf16_bits_to_double(h);
    }
    case ORC_E4M3:
      return orc_e4m3_to_double(((const uint8_t*)base)[idx]) * fp8_scale;
    default:
      return NAN;
  }
}

/* ---------- shape checks ---------------------------------------------------- */

static int check_decode_shapes(int64_t num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                               int block_size, int64_t max_blocks_per_seq, int64_t num_blocks,
                               const int32_t* block_tables, const int32_t* context_lens) {
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
      max_blocks_per_seq < 0 || num_blocks < 0)
    return ORC_EINVAL;
  if (num_q_heads % num_kv_heads != 0) return ORC_EINVAL;
  for (int64_t b = 0; b < num_seqs; ++b) {
    int64_t ctx = context_lens[b];
    if (ctx < 0 || ctx > max_blocks_per_seq * (int64_t)block_size) return ORC_ERANGE;
    int64_t nblk = (ctx + block_size - 1) / block_size;
    for (int64_t j = 0; j < nblk; ++j) {
      int64_t phys = block_tables[b * max_blocks_per_seq + j];
      if (phys < 0 || phys >= num_blocks) return ORC_ERANGE;
    }
  }
  return ORC_OK;
}

/* Physical element index of logical token t, kv head h, dim i of sequence b:
 * the block-table lookup plus the offset ("one extra int load and one
 * multiply" of the page's 核心要点). */
static int64_t cache_index(const int32_t* block_tables, int64_t max_blocks_per_seq, int64_t b,
                           int64_t t, int block_size, int num_kv_heads, int head_dim, int h, int i) {
  int64_t phys = block_tables[b * max_blocks_per_seq + t / block_size];
  int64_t row = t % block_size;
  return ((phys * block_size + row) * num_kv_heads + h) * (int64_t)head_dim + i;
}

/* Gather the logical K (or V) of one (sequence, kv head) into dst[ctx][head_dim]. */
static void gather_logical(double* dst, const void* cache, int cache_dtype, double fp8_scale,
                           const int32_t* block_tables, int64_t max_blocks_per_seq, int64_t b,
                           int64_t ctx, int block_size, int num_kv_heads, int head_dim, int h) {
  for (int64_t t = 0; t < ctx; ++t)
    for (int i = 0; i < head_dim; ++i)
      dst[t * head_dim + i] = load_elem(
          cache, cache_index(block_tables, max_blocks_per_seq, b, t, block_size, num_kv_heads, head_dim, h, i),
          cache_dtype, fp8_scale);
}

/* ---------- paged decode attention ----------------------------------------- */

/* One (sequence b, query head hq): dense softmax attention over the logical
 * K/V of tokens [t0, t1).  Writes o[head_dim] = sum e^{s-m} V / l and returns
 * m and l through the pointers.  An empty range gives m = -inf, l = 0, o = 0. */
static void attend_range(double* o, double* m_out, double* l_out, const double* qv, const double* K,
                         const double* V, int64_t t0, int64_t t1, int head_dim, double scale) {
  double m = -INFINITY, l = 0.0;
  for (int i = 0; i < head_dim; ++i) o[i] = 0.0;
  if (t1 <= t0) {
    *m_out = m;
    *l_out = l;
    return;
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)(t1 - t0));
  for (int64_t t = t0; t < t1; ++t) {
    double dot = 0.0;
    for (int i = 0; i < head_dim; ++i) dot += qv[i] * K[t * head_dim + i];
    s[t - t0] = scale * dot;
    if (s[t - t0] > m) m = s[t - t0];
  }
  for (int64_t t = t0; t < t1; ++t) {
    double w = exp(s[t - t0] - m);
    l += w;
    for (int i = 0; i < head_dim; ++i) o[i] += w * V[t * head_dim + i];
  }
  for (int i = 0; i < head_dim; ++i) o[i] /= l;
  free(s);
  *m_out = m;
  *l_out = l;
}

/*
 * out[n][head_dim] for the selected rows (row = b * num_q_heads + hq), or for
 * every row when sel == NULL (n = num_seqs * num_q_heads).
 * q: [num_seqs][num_q_heads][head_dim] of q_dtype (f32 or bf16).
 * key_cache/value_cache: [num_blocks][block_size][num_kv_heads][head_dim] of
 * cache_dtype; k_scale/v_scale multiply fp8 codes and are ignored otherwise.
 * context_len 0 gives a zero row.  Returns ORC_OK or a negative code (bad
 * shapes, block id or context length out of range) without reading out of
 * bounds.
 */
int orc_paged_attention_decode(double* out, const void* q, int q_dtype, const void* key_cache,
                               const void* value_cache, int cache_dtype, const int32_t* block_tables,
                               const int32_t* context_lens, int64_t num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, int block_size, int64_t max_blocks_per_seq,
                               int64_t num_blocks, float scale, float k_scale, float v_scale,
                               const int64_t* sel, int64_t n_sel, int num_threads) {
  if (q_dtype != ORC_F32 && q_dtype != ORC_BF16) return ORC_EINVAL;
  if (!elem_size(cache_dtype)) return ORC_EINVAL;
  int rc = check_decode_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                               max_blocks_per_seq, num_blocks, block_tables, context_lens);
  if (rc) return rc;
  int64_t n = sel ? n_sel : num_seqs * num_q_heads;
  for (int64_t r = 0; r < n; ++r) {
    int64_t row = sel ? sel[r] : r;
    if (row < 0 || row >= num_seqs * num_q_heads) return ORC_ERANGE;
  }
  const int group = num_q_heads / num_kv_heads;
  const double ks = (double)k_scale, vs = (double)v_scale, sc = (double)scale;
  if (num_threads < 1) num_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
  for (int64_t r = 0; r < n; ++r) {
    int64_t row = sel ? sel[r] : r;
    int64_t b = row / num_q_heads;
    int hq = (int)(row % num_q_heads);
    int hk = hq / group;
    int64_t ctx = context_lens[b];
    double* o = out + r * head_dim;
    double* qv = (double*)malloc(sizeof(double) * head_dim);
    double* K = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * head_dim);
    for (int i = 0; i < head_dim; ++i) qv[i] = load_elem(q, row * head_dim + i, q_dtype, 1.0);
    gather_logical(K, key_cache, cache_dtype, ks, block_tables, max_blocks_per_seq, b, ctx, block_size,
                   num_kv_heads, head_dim, hk);
    gather_logical(V, value_cache, cache_dtype, vs, block_tables, max_blocks_per_seq, b, ctx, block_size,
                   num_kv_heads, head_dim, hk);
    double m, l;
    attend_range(o, &m, &l, qv, K, V, 0, ctx, head_dim, sc);
    free(qv);
    free(K);
    free(V);
  }
  return ORC_OK;
}

/*
 * Split-context partials: for every row (b, hq) and partition p in
 * [0, max_partitions), the token range [p*P, min((p+1)*P, ctx)) with
 * P = partition_tokens gives m[row][p], l[row][p], o[row][p][head_dim]
 * (see attend_range).  Partitions past the context get m = -inf, l = 0, o = 0.
 */
int orc_decode_partials(double* m_out, double* l_out, double* o_out, const void* q, int q_dtype,
                        const void* key_cache, const void* value_cache, int cache_dtype,
                        const int32_t* block_tables, const int32_t* context_lens, int64_t num_seqs,
                        int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                        int64_t max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                        float v_scale, int64_t partition_tokens, int64_t max_partitions, int num_threads) {
  if (q_dtype != ORC_F32 && q_dtype != ORC_BF16) return ORC_EINVAL;
  if (!elem_size(cache_dtype) || partition_tokens <= 0 || max_partitions <= 0) return ORC_EINVAL;
  int rc = check_decode_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                               max_blocks_per_seq, num_blocks, block_tables, context_lens);
  if (rc) return rc;
  for (int64_t b = 0; b < num_seqs; ++b)
    if ((context_lens[b] + partition_tokens - 1) / partition_tokens > max_partitions) return ORC_ERANGE;
  const int group = num_q_heads / num_kv_heads;
  const int64_t rows = num_seqs * num_q_heads;
  if (num_threads < 1) num_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
  for (int64_t row = 0; row < rows; ++row) {
    int64_t b = row / num_q_heads;
    int hq = (int)(row % num_q_heads);
    int hk = hq / group;
    int64_t ctx = context_lens[b];
    double* qv = (double*)malloc(sizeof(double) * head_dim);
    double* K = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)(ctx > 0 ? ctx : 1) * head_dim);
    for (int i = 0; i < head_dim; ++i) qv[i] = load_elem(q, row * head_dim + i, q_dtype, 1.0);
    gather_logical(K, key_cache, cache_dtype, (double)k_scale, block_tables, max_blocks_per_seq, b, ctx,
                   block_size, num_kv_heads, head_dim, hk);
    gather_logical(V, value_cache, cache_dtype, (double)v_scale, block_tables, max_blocks_per_seq, b, ctx,
                   block_size, num_kv_heads, head_dim, hk);
    for (int64_t p = 0; p < max_partitions; ++p) {
      int64_t t0 = p * partition_tokens;
      int64_t t1 = t0 + partition_tokens < ctx ? t0 + partition_tokens : ctx;
      int64_t k = row * max_partitions + p;
      attend_range(o_out + k * head_dim, &m_out[k], &l_out[k], qv, K, V, t0, t1, head_dim, (double)scale);
    }
    free(qv);
    free(K);
    free(V);
  }
  return ORC_OK;
}

/* Merge of split-context partials (softmax identity): per row,
 * M = max_p m_p over partitions with l_p > 0, w_p = l_p e^{m_p - M},
 * out = sum_p w_p o_p / sum_p w_p.  A row with no partition gives zeros. */
void orc_merge_partials(double* out, const double* m, const double* l, const double* o, int64_t rows,
                        int64_t num_parts, int head_dim) {
  for (int64_t r = 0; r < rows; ++r) {
    double M = -INFINITY;
    for (int64_t p = 0; p < num_parts; ++p)
      if (l[r * num_parts + p] > 0.0 && m[r * num_parts + p] > M) M = m[r * num_parts + p];
    double W = 0.0;
    for (int i = 0; i < head_dim; ++i) out[r * head_dim + i] = 0.0;
    for (int64_t p = 0; p < num_parts; ++p) {
      int64_t k = r * num_parts + p;
      if (!(l[k] > 0.0)) continue;
      double w = l[k] * exp(m[k] - M);
      W += w;
      for (int i = 0; i < head_dim; ++i) out[r * head_dim + i] += w * o[k * head_dim + i];
    }
    if (W > 0.0)
      for (int i = 0; i < head_dim; ++i) out[r * head_dim + i] /= W;
  }
}

/* ---------- new-token KV write ---------------------------------------------- */

/*
 * k, v: [num_tokens][num_kv_heads][head_dim] of in_dtype (f32 or bf16).
 * Token t with slot s = slot_mapping[t] >= 0 goes to block s / block_size,
 * row s % block_size of both caches; s < 0 is skipped.  With cache_dtype ==
 * in_dtype the bytes are copied; with an E4M3 cache the stored code is
 * E4M3(x * (1/k_scale)) (V likewise with v_scale).  Returns ORC_ERANGE,
 * writing nothing, if any slot is past the pool.
 */
int orc_paged_kv_write(const void* k, const void* v, int in_dtype, const int64_t* slot_mapping,
                       int64_t num_tokens, void* key_cache, void* value_cache, int cache_dtype,
                       int64_t num_blocks, int block_size, int num_kv_heads, int head_dim, float k_scale,
                       float v_scale) {
  if (in_dtype != ORC_F32 && in_dtype != ORC_BF16) return ORC_EINVAL;
  if (cache_dtype != in_dtype && cache_dtype != ORC_E4M3) return ORC_EINVAL;
  if (num_tokens < 0 || num_blocks < 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
    return ORC_EINVAL;
  for (int64_t t = 0; t < num_tokens; ++t)
    if (slot_mapping[t] >= num_blocks * (int64_t)block_size) return ORC_ERANGE;
  const int es = elem_size(in_dtype);
  const int64_t row_elems = (int64_t)num_kv_heads * head_dim;
  const float k_inv = 1.0f / k_scale, v_inv = 1.0f / v_scale;
  for (int64_t t = 0; t < num_tokens; ++t) {
    int64_t s = slot_mapping[t];
    if (s < 0) continue;
    int64_t blk = s / block_size, row = s % block_size;
    int64_t dst0 = (blk * block_size + row) * row_elems; /* element index of (blk, row, 0, 0) */
    int64_t src0 = t * row_elems;
    if (cache_dtype == in_dtype) {
      memcpy((char*)key_cache + dst0 * es, (const char*)k + src0 * es, (size_t)(row_elems * es));
      memcpy((char*)value_cache + dst0 * es, (const char*)v + src0 * es, (size_t)(row_elems * es));
    } else {
      for (int64_t i = 0; i < row_elems; ++i) {
        float xk = (float)load_elem(k, src0 + i, in_dtype, 1.0);
        float xv = (float)load_elem(v, src0 + i, in_dtype, 1.0);
        volatile float pk = xk * k_inv; /* one binary32 multiply */
        volatile float pv = xv * v_inv;
        ((uint8_t*)key_cache)[dst0 + i] = orc_e4m3_from_float(pk);
        ((uint8_t*)value_cache)[dst0 + i] = orc_e4m3_from_float(pv);
      }
    }
  }
  return ORC_OK;
}

/* ---------- copy-on-write block copy ---------------------------------------- */

/*
 * pairs: [num_pairs][2] (src, dst) block ids.  Each pair copies the
 * block_bytes of block src to block dst in both caches.  The pairs must be
 * order-independent: every id in range, no dst repeated, no dst also a src;
 * otherwise ORC_ERANGE / ORC_EINVAL and nothing is written.
 */
int orc_kv_block_copy(const int64_t* pairs, int64_t num_pairs, void* key_cache, void* value_cache,
                      int64_t num_blocks, int64_t block_bytes) {
  if (num_pairs < 0 || num_blocks < 0 || block_bytes <= 0) return ORC_EINVAL;
  for (int64_t i = 0; i < num_pairs; ++i) {
    int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return ORC_ERANGE;
    for (int64_t j = 0; j < num_pairs; ++j) {
      if (j != i && pairs[2 * j + 1] == d) return ORC_EINVAL;
      if (pairs[2 * j] == d) return ORC_EINVAL;
    }
  }
  for (int64_t i = 0; i < num_pairs; ++i) {
    int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    memcpy((char*)key_cache + d * block_bytes, (const char*)key_cache + s * block_bytes, (size_t)block_bytes);
    memcpy((char*)value_cache + d * block_bytes, (const char*)value_cache + s * block_bytes,
           (size_t)block_bytes);
  }
  return ORC_OK;
}

/* Element-wise E4M3 encoding of an fp32 array (test convenience). */
void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_float(x[i]);
}

/* ---------- block swap between two pools ------------------------------------ */

/*
 * Block swap ("vLLM KV Cache 实现机制", 1.2 and 2.1; "vLLM — 把操作系统的分页搬进
 * GPU KV cache", 实践案例 3): block src of the source pool is copied onto block
 * dst of the destination pool, in both caches, byte for byte.  Destinations
 * must be distinct and in range (sources in range); otherwise nothing is
 * written and ORC_ERANGE / ORC_EINVAL is returned.
 */
int orc_swap_blocks(const int64_t* pairs, int64_t num_pairs, const void* src_k, const void* src_v,
                    int64_t src_blocks, void* dst_k, void* dst_v, int64_t dst_blocks, int64_t block_bytes) {
  if (num_pairs < 0 || src_blocks < 0 || dst_blocks < 0 || block_bytes <= 0) return ORC_EINVAL;
  for (int64_t i = 0; i < num_pairs; ++i) {
    int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) return ORC_ERANGE;
    for (int64_t j = 0; j < i; ++j)
      if (pairs[2 * j + 1] == d) return ORC_EINVAL;
  }
  for (int64_t i = 0; i < num_pairs; ++i) {
    int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
    memcpy((char*)dst_k + d * block_bytes, (const char*)src_k + s * block_bytes, (size_t)block_bytes);
    memcpy((char*)dst_v + d * block_bytes, (const char*)src_v + s * block_bytes, (size_t)block_bytes);
  }
  return ORC_OK;
}

/* ---------- per-tensor fp8 scale ---------------------------------------------- */

/* amax(|x|) over n elements (exact in fp64), then amax / 448 as one binary32
 * division (the largest finite E4M3 value is 448); 1 when amax is 0.  The
 * calibration rule is this library's reading: the pages name fp8 KV caches
 * ("vLLM KV Cache 实现机制", 2.3) without one. */
float orc_fp8_scale(const void* x, int64_t n, int dtype) {
  double amax = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double a = fabs(load_elem(x, i, dtype, 1.0));
    if (a > amax) amax = a;
  }
  if (!(amax > 0.0)) return 1.0f;
  volatile float af = (float)amax; /* exact: amax is one of the inputs */
  volatile float s = af / 448.0f;
  return s;
}

/* ---------- multi-query paged attention (chunked prefill, speculative verify) -- */

/*
 * Several new query tokens per sequence over the paged cache, each attending
 * causally: the q_len_b = query_start_loc[b+1] - query_start_loc[b] queries of
 * sequence b are the last q_len_b positions of its context, so query i sits
 * at position p = context_lens[b] - q_len_b + i and attends the logical
 * tokens 0..p ("vLLM 与 KV Cache", KV Cache：为什么需要缓存: every new token
 * attends all earlier ones; the paged addressing is the decode path's).  The
 * pages describe only one new token per step; the several-token case is this
 * library's extension (prefill chunks and draft-token verification).
 * q and out: [total_q][num_q_heads][head_dim]; rows are q-token * Hq + hq.
 * A query whose position is negative (q_len_b > context_lens[b]) attends
 * nothing and gives zeros.  Everything in fp64; sel selects flat rows (NULL: all).
 */
int orc_paged_attention_multiquery(double* out, const void* q, int q_dtype, const int32_t* query_start_loc,
                                   const void* key_cache, const void* value_cache, int cache_dtype,
                                   const int32_t* block_tables, const int32_t* context_lens, int64_t num_seqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                                   int64_t max_blocks_per_seq, int64_t num_blocks, float scale, float k_scale,
                                   float v_scale, const int64_t* sel, int64_t n_sel, int num_threads) {
  if (q_dtype != ORC_F32 && q_dtype != ORC_BF16) return ORC_EINVAL;
  if (!elem_size(cache_dtype)) return ORC_EINVAL;
  int rc = check_decode_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                               num_blocks, block_tables, context_lens);
  if (rc) return rc;
  if (query_start_loc[0] != 0) return ORC_EINVAL;
  for (int64_t b = 0; b < num_seqs; ++b)
    if (query_start_loc[b + 1] < query_start_loc[b]) return ORC_EINVAL;
  const int64_t total_q = query_start_loc[num_seqs];
  const int64_t rows = total_q * num_q_heads;
  int64_t n = sel ? n_sel : rows;
  for (int64_t r = 0; r < n; ++r) {
    int64_t row = sel ? sel[r] : r;
    if (row < 0 || row >= rows) return ORC_ERANGE;
  }
  const int group = num_q_heads / num_kv_heads;
  if (num_threads < 1) num_threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads)
  for (int64_t r = 0; r < n; ++r) {
    int64_t row = sel ? sel[r] : r;
    int64_t tok = row / num_q_heads;
    int hq = (int)(row % num_q_heads);
    int64_t b = 0;
    while (query_start_loc[b + 1] <= tok) ++b; /* the sequence owning query token tok */
    int64_t q_len = query_start_loc[b + 1] - query_start_loc[b];
    int64_t ctx = context_lens[b];
    int64_t pos = ctx - q_len + (tok - query_start_loc[b]);
    double* o = out + r * head_dim;
    double* qv = (double*)malloc(sizeof(double) * head_dim);
    int64_t nk = pos + 1 > 0 ? pos + 1 : 0;
    double* K = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * head_dim);
    double* V = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * head_dim);
    for (int i = 0; i < head_dim; ++i) qv[i] = load_elem(q, row * head_dim + i, q_dtype, 1.0);
    gather_logical(K, key_cache, cache_dtype, (double)k_scale, block_tables, max_blocks_per_seq, b, nk, block_size,
                   num_kv_heads, head_dim, hq / group);
    gather_logical(V, value_cache, cache_dtype, (double)v_scale, block_tables, max_blocks_per_seq, b, nk, block_size,
                   num_kv_heads, head_dim, hq / group);
    double m, l;
    attend_range(o, &m, &l, qv, K, V, 0, nk, head_dim, (double)scale);
    free(qv);
    free(K);
    free(V);
  }
  return ORC_OK;
}

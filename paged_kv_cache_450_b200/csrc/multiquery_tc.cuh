// multiquery_tc.cuh -- multi-query paged attention on the tcgen05 tensor cores
// for more than 16 rows (queries x query heads of a group) per sequence and
// KV head: chunked prefill, grouped-query draft verification.
//
// Same operation as multiquery.cuh (causal over the paged cache, queries are
// the sequence's last q_len positions), written for the Blackwell MMA:
//
//   a work unit = 128 query rows (query i, head g; g fastest) x one KV head x
//   one split-context partition; KV tiles of 128 tokens (8 blocks of 16 or 4
//   of 32) from the partition's start (a partition that is not a multiple of
//   128 tokens ends in a partial tile, masked like the context end).
//   S = Q . K^T      M = 128 rows, N = 128 tokens, K = 128 dims -> TMEM columns [0, 128)
//   O_h += P_h . V_h M = 128 rows, N = 128 dims,   K = 64 tokens (half h of the tile)
//                    -> TMEM columns [128, 256) (h = 0) and [256, 384) (h = 1)
// (Every MMA is as wide as the operands allow: the single issuing thread pays
// ~64 cycles per instruction whatever M and N -- an N = 128 MMA executes in
// ~81 -- and ~50-100 per barrier wait, fence or commit, so it waits on as few
// barriers per tile as the data flow allows.)
//
// Persistent CTAs: one CTA per SM (the launch has min(units, SMs) CTAs) takes
// one unit of every round of CTAs-many units of the unit list, which is ordered
// by KV tiles, most first: unit c of even rounds, unit CTAs - 1 - c of odd
// rounds (a CTA that got one of the longest units of a round gets one of the
// shortest of the next).  Barrier
// phases and ring stages run on per-CTA counters across units, so the next
// unit's Q and first K / V tiles load while the current unit finishes, and the
// TMEM allocation, the barrier set-up and the CTA launch are paid once per SM
// instead of once per unit (measured ~8 us per unit: a third of a prefill
// unit of 8-9 tiles).
//
// Q, K and V sit in shared memory in the 128-byte-swizzled layout (two
// 64-element halves of every 256-byte row) as TMA delivers them; Q and K are
// K-major operands, V (stored token-major, dims contiguous) is the N-major B
// operand of P . V, so no transpose is ever made.  P never touches shared
// memory: it is the TMEM A operand of P . V (columns [384, 512)).  With bf16
// caches it is split into a bf16 high part and a bf16 residual -- two MMAs per
// k-step -- so each probability keeps ~16 significant bits (a bf16 P alone
// costs up to ~3e-3 absolute on short contexts), packed with integer byte
// permutes.  (One fp16 P over V converted to fp16 in shared memory halves the
// P . V MMAs but measured 1.7x slower: the conversions compete with the
// exponentials.)  Thirteen warps (warp w runs on sub-partition w % 4):
//   warps 0-7  softmax: warp w serves the rows in TMEM lanes 32 (w & 3) .. +31
//              (the lanes its sub-partition may touch) and half h = w >> 2 of
//              every KV tile's tokens.  The two halves are independent online
//              softmaxes -- each with its own running max, row sum and
//              accumulator O_h -- so the two warps of a sub-partition wait for
//              each other only through the tile's P barrier, and their
//              special-function (exp) and integer / FMA (P packing) phases
//              interleave; they are merged
//              once per unit, in the epilogue (the (m, l) exchange goes through
//              TMEM columns of P, free by then).  Per tile a thread reads its 64
//              scores from TMEM, applies the causal / context mask, keeps a
//              reference max (O_h is rescaled only when a score passes it by
//              more than 2^8), and writes its 64 probabilities into P_h.
//   warp 8     TMA producer of Q and the K tiles (a ring of 2-3 stages; one 4-D box
//              per block and 64-dim half); owns the TMEM allocation.
//   warp 10    TMA producer of the V tiles (a ring of 3-4 stages; warp 12 with
//              fp8 caches).
//   warp 11    MMA issuer: one thread issues S_j as soon as the softmax has
//              taken S_{j-1} into registers; completion is signalled through
//              tcgen05.commit on mbarriers.
//   warp 9     bf16 caches: the P_j . V_j issuer (its own waits and commits, so
//              the two issuing threads' barrier work overlaps the other's MMAs).
//   fp8 caches: warps 10 and 11 widen the K and V tiles (sub-partitions 2 and
//              3, idle in grouped verification, whose rows fill only lane
//              quarters 0 and 1), warp 9 issues the S MMAs, warp 13 the
//              P . V MMAs, and warp 12 produces V.
// Caches of fp8 (E4M3, F8 = true): the producer warps TMA each tile's raw codes
// (128 bytes per token row) into the upper half of the tile's own ring stage;
// warps 10 and 11 then widen them exactly to fp16 in place (one thread per token
// row reads the raw row whole, then writes its two fp16 halves; V rows that
// must not contribute are zeroed there) -- the rings have the bf16 layout and
// depths, so widening overlaps the MMAs; the softmax warps round their Q rows to
// fp16 once per unit; both MMAs run on fp16 operands, and P is one fp16 value
// (11 significant bits; columns [384, 448)).  The K scale is folded into the
// logit scale, the V scale into the output.
// Every wait is bounded (2 s); on a timeout the status bit is set, the
// producer and issuer loops stop, the softmax warps skip their remaining
// waits, in-flight work is drained with bounded waits and TMEM is freed.
#pragma once

#include "common.cuh"
#include "multiquery_params.h"
#include "tcgen05.cuh"

namespace pkv {

// STACK (bf16 caches, at most 64 query rows per (sequence, KV head), as in
// grouped verification: 5 queries x 8 heads = 40): MMA rows 64-127 repeat rows
// 0-63 (the softmax warps of TMEM lanes 64-127 copy the Q tile's first 64 rows
// below them), so S holds every score twice; the warps of lanes 0-63 write P's
// bf16 high part and those of lanes 64-127 its residual for the same rows, and
// each P . V k-step is ONE M = 128 MMA whose accumulator rows 64-127 collect the
// residual's share -- 16 MMAs per tile instead of 24 for the single issuing
// thread.  The epilogue adds the residual's share back through the Q tile, so
// the next unit's Q loads once the epilogue is done (o_free) rather than once
// the unit's S MMAs are (q_empty).
template <int BS, bool F8 = false, bool STACK_ = false>
struct MqTcTraits {
  static constexpr int D = 128;
  static constexpr bool STACK = STACK_;
  static_assert(!(STACK && F8), "stacked rows: bf16 caches");
  static constexpr int ROWS = STACK ? 64 : 128;  // query rows per unit
  static constexpr int TOK = 128;            // tokens per KV tile
  static constexpr int BPT = TOK / BS;       // blocks per KV tile
  static constexpr int HALF = 128 * 128;     // 128 rows x 128 bytes (64 bf16 / fp16)
  static constexpr int TILE = 2 * HALF;      // 32 KB: 128 rows x 128 16-bit values
  // K and V rings (fp8 caches: the raw codes land in a stage's upper half and
  // are widened to fp16 in place).  Three V stages: a V tile is issued once the
  // P . V two tiles back has read its stage, so it has about two tiles' time
  // to land.
  // (stacked rows: two K stages -- K is read by the S MMAs alone, issued as soon as it lands -- and the
  // third stage's space holds the P exchange buffers below.  Unstacked bf16: two K stages and four V
  // stages -- a V stage is freed only by the P . V a tile after the S that frees a K stage, and the
  // V tiles of the last, ragged tile of a unit held the softmax warps back.)
  static constexpr int NSK = (STACK || !F8) ? 2 : 3, NSV = (!STACK && !F8) ? 4 : 3;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + NSK * TILE;
  // stacked rows: the two warps of a row pair (TMEM lanes r and r + 64) split each tile's exponentials
  // and swap what the other stores -- 16 words per thread, two buffers by tile parity -- plus one float
  // per thread for the row-sum parts at the end of a unit
  static constexpr int XCH_OFF = V_OFF + NSV * TILE;
  static constexpr int XCH_TILE = 256 * 16 * 4;
  static constexpr int XCH_BYTES = STACK ? 2 * XCH_TILE + 256 * 4 : 0;
  // (the epilogue's residual shares, 64 rows x 128 fp32, reuse the two exchange buffers)
  static_assert(!STACK || 2 * XCH_TILE >= 64 * 128 * 4, "exchange buffers hold the residual shares");
  static constexpr int BAR_OFF = XCH_OFF + XCH_BYTES;
  // mbarriers: q_full, q_empty, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full, s_free,
  // p_full[NPB], pv_done[NPB] (both token halves of a tile; by tile parity), o_free, mma_done; fp8 caches add
  // q_ready, k_ready[NSK],
  // v_ready[NSV]
  // P buffers in TMEM: two (tile parity) when P is one 16-bit value per probability row (stacked rows,
  // fp8 caches), so the softmax writes P of tile t while P . V of tile t - 1 still reads the other; one
  // (hi and residual parts) for bf16 caches otherwise
  static constexpr int NPB = (STACK || F8) ? 2 : 1;
  static constexpr int NBAR = 2 + 2 * NSK + 2 * NSV + 8 + (F8 ? 1 + NSK + NSV : STACK ? 1 : 0);
  static constexpr int SLOT_OFF = BAR_OFF + NBAR * 8;   // TMEM base address written by tcgen05.alloc
  // the rank group of each of the CTA's first MAX_UNITS units
  static constexpr int MAX_UNITS = 64;
  static constexpr int UNIT_OFF = SLOT_OFF + 16;
  // 14 warps with fp8 caches (the two widening warps and a second issuer), 12 otherwise: each
  // sub-partition's registers hold at most three warps of the bf16 kernel's ~155 registers (four would
  // cap them at 128); the fp8 instances take ~125
  static constexpr int THREADS = F8 ? 448 : 384;
  // warp w runs on sub-partition w % 4.  fp8 caches: the two widening warps on sub-partitions 2 and 3,
  // whose softmax warps have no rows when a (sequence, KV head) has at most 64 (grouped verification),
  // the two MMA issuers (S: warp 9, P . V: warp 13) on 1 and the V producer on 0
  static constexpr int W_K = 8, W_KWIDEN = F8 ? 10 : 9, W_V = F8 ? 12 : 10, W_MMA = F8 ? 9 : 11,
                       W_VWIDEN = F8 ? 11 : 12;
  // the P . V issuer (its own waits and commits beside the S issuer's)
  static constexpr int W_PV = F8 ? 13 : 9;
  static constexpr int N_ISSUERS = 2;
  // S 128 | O_0 128 | O_1 128 | P: bf16 hi 0,1 (32 + 32) and lo 0,1 (32 + 32), or (stacked bf16, fp16)
  // buffer 0: halves 0,1 (32 + 32), buffer 1: halves 0,1 (32 + 32)
  static constexpr uint32_t TMEM_COLS = 512;
  // (block ids are read from the table as the tiles are issued: nothing depends on the partition length)
  static constexpr size_t smem_bytes(int /*partition_blocks*/) { return 1024 + UNIT_OFF + 4 * MAX_UNITS; }
  static_assert(1024 + UNIT_OFF + 4 * MAX_UNITS + 64 <= 232448, "shared memory of one CTA");
};

// 3-D tiled TMA load (coordinates innermost first; c0 is 0 or 64 elements).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// 32-byte global store of eight 32-bit words (sm_100); the address must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* ptr, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// max(a, b, c) in one instruction (sm_100).
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Waits of this kernel: the thread sleeps inside mbarrier.try_wait (the hardware
// wakes it when the phase completes, or after the hint of 20 us) instead of
// polling.  Four to five warps share each sub-partition; a warp polling a
// barrier takes issue slots from the softmax warps beside it (measured: the
// softmax warps of the MMA issuer's sub-partition ran ~1000 cycles per tile
// behind the others).  Still bounded: gives up after kWaitLimitNs in all.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20000u)
      : "memory");
  return ok != 0;
}
// Non-blocking probe of the phase (no suspend): the common case of a phase already complete costs
// least this way.
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, unsigned* status) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      set_status(status, PKV_STATUS_WAIT_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait taken by every lane of a warp; the result is the same on every
// lane (false if any lane gave up), so the warp stays converged for the
// .sync.aligned tensor-memory instructions that follow.
__device__ __forceinline__ bool warp_wait_bounded(uint32_t bar, uint32_t parity, unsigned* status) {
  return __all_sync(kFullMask, mbar_wait_sleep(bar, parity, status));
}

// One work unit: query tile qt and KV head hk of sequence b, partition part.
// Every thread of the CTA computes the same description from the same global
// data.
struct MqUnit {
  int b, hk, qt, part;
  int q0, q_len, rows_total, base_pos, row_last;
  int tok_begin, tok_end, nt, nb, nparts;
  const int32_t* table;  // the partition's block ids
  int kind;              // kRun, kSkip (nothing to do), kZero (write zero rows, then nothing), kBadQuery
};
enum { kRun = 0, kSkip = 1, kZero = 2, kBadQuery = 3 };

template <int BS, int G>
__device__ __forceinline__ MqUnit mq_unit(const MultiQueryParams& p, int b, int hk, int qt, int y) {
  MqUnit U;
  U.b = b;
  U.hk = hk;
  U.qt = qt;
  U.part = y;
  U.table = nullptr;
  U.nt = U.nb = U.nparts = 0;
  // the sequence's context length is loaded beside its query range (b < num_seqs: in bounds), so the
  // unit's description costs one memory latency, not two -- it sits between units on every warp's path
  const int ctx_loaded = p.context_lens[b];
  if (!query_rows_ok(p, b, U.q0, U.q_len)) {  // before any access through the query range
    U.kind = kBadQuery;
    return U;
  }
  U.rows_total = U.q_len * G;
  U.kind = kSkip;
  if (U.q_len <= 0 || U.qt * 128 >= U.rows_total) return U;
  const int max_ctx = p.max_blocks_per_seq * BS;
  int ctx = ctx_loaded;
  if (ctx < 0 || ctx > max_ctx) {
    if (threadIdx.x == 0 && U.hk == 0 && U.part == 0 && U.qt == 0) set_status(p.status, PKV_STATUS_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : max_ctx;
  }
  const int nblk = (ctx + BS - 1) / BS;
  const int pb = p.partition_blocks;
  const int nparts = (nblk + pb - 1) / pb;
  U.nparts = nparts;
  U.base_pos = ctx - U.q_len;
  U.row_last = min(U.rows_total, (U.qt + 1) * 128) - 1;
  const int pos_last = U.base_pos + U.row_last / G;
  if (nparts == 0 || pos_last < 0) {  // nothing to attend: zero rows (partition 0 writes them)
    if (U.part == 0) U.kind = kZero;
    return U;
  }
  if (U.part >= nparts) return U;
  U.tok_begin = U.part * pb * BS;
  // tokens this unit's rows can see in the partition: [tok_begin, tok_end)
  U.tok_end = min(min(ctx, U.tok_begin + pb * BS), pos_last + 1);
  if (U.tok_end <= U.tok_begin) return U;  // every row sits before this partition (never merged)
  U.nt = (U.tok_end - U.tok_begin + 127) / 128;
  U.nb = (U.tok_end - U.tok_begin + BS - 1) / BS;
  U.table = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq + U.part * pb;
  U.kind = kRun;
  return U;
}

// Unit k of this CTA: round k, position c or CTAs - 1 - c (see above); may be
// past the last unit (n_all) in the last round.
__device__ __forceinline__ int64_t cta_unit(int k) {
  const int64_t c = (k & 1) ? gridDim.x - 1 - blockIdx.x : blockIdx.x;
  return static_cast<int64_t>(k) * gridDim.x + c;
}

// Longest work first.  The units are ranked in groups that take the same
// time: with at most MAX_GROUPS (sequence, partition, query tile) triples, a
// group is one triple (its KV heads' units, keyed by the triple's KV tiles);
// otherwise, with at most MAX_GROUPS sequences, a group is a whole sequence
// (keyed by its context length).  Group rank r (descending key, ties by group
// index: a permutation) takes units r * per_group .. of the unit list, so the
// units that start last are the short ones.  Each thread ranks whole groups
// from the keys staged in `scratch` (shared memory no load has reached yet)
// and records the group of every unit of this CTA with that rank.
enum { kRankNone = 0, kRankSeqs = 1, kRankGroups = 2 };
constexpr int MAX_GROUPS = 1024;

template <typename Key>
__device__ __forceinline__ void rank_unit_groups(int n_groups, int per_group, int n_rounds, int* scratch,
                                                 int* unit_g, Key key) {
  for (int i = threadIdx.x; i < n_groups; i += blockDim.x) scratch[i] = key(i);
  __syncthreads();
  for (int t = threadIdx.x; t < n_groups; t += blockDim.x) {
    const int lt = scratch[t];
    int r = 0;
#pragma unroll 4
    for (int j = 0; j < n_groups; ++j) {
      const int lj = scratch[j];
      r += (lj > lt) || (lj == lt && j < t);
    }
    // this CTA's units u with u / per_group == r lie in rounds u_lo / CTAs .. (u_hi - 1) / CTAs
    const int64_t u_lo = static_cast<int64_t>(r) * per_group, u_hi = u_lo + per_group;  // [u_lo, u_hi)
    const int64_t k_hi = min(static_cast<int64_t>(n_rounds) - 1, (u_hi - 1) / gridDim.x);
    for (int64_t k = u_lo / gridDim.x; k <= k_hi; ++k) {
      const int64_t u = cta_unit(static_cast<int>(k));
      if (u >= u_lo && u < u_hi) unit_g[k] = t;
    }
  }
  fence_proxy_async_smem();  // the scratch writes before the tile loads that later land there
  __syncthreads();
}

// Widens one KV tile of raw E4M3 codes in place.  The raw codes of token row
// t (128 codes, 128 bytes) sit in the stage's upper half at line t, 16-byte
// chunk q (dims 16q .. 16q+15) at position q ^ (t & 7) (128-byte swizzle);
// the fp16 result is the operand layout -- dims 0..63 in the lower half,
// 64..127 in the upper half, line t, chunk c at position c ^ (t & 7), raw
// chunk q giving chunks 2(q % 4) and 2(q % 4) + 1 of half q / 4.  Each thread
// takes whole rows (t = lane, lane + 32, ...): it reads the raw line fully
// before it writes the same line, so no row is read after another thread
// wrote it.  Rows for which zero_row(t) holds are written as zeros.  One warp;
// each lane then orders its writes before the tensor core's (async proxy)
// reads.
template <typename ZeroRow>
__device__ __forceinline__ void widen_e4m3_tile_in_place(uint8_t* stage, int lane, ZeroRow zero_row) {
  constexpr int HALF = 128 * 128;
#pragma unroll 1
  for (int t = lane; t < 128; t += 32) {
    uint8_t* line0 = stage + t * 128;
    uint8_t* line1 = stage + HALF + t * 128;
    const int sw = t & 7;
    if (zero_row(t)) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        *reinterpret_cast<uint4*>(line0 + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(line1 + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
      }
      continue;
    }
    uint4 w[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) w[q] = *reinterpret_cast<const uint4*>(line1 + ((q ^ sw) << 4));
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      uint32_t f[8];
      e4m3x4_to_f16x2x2(w[q].x, f[0], f[1]);
      e4m3x4_to_f16x2x2(w[q].y, f[2], f[3]);
      e4m3x4_to_f16x2x2(w[q].z, f[4], f[5]);
      e4m3x4_to_f16x2x2(w[q].w, f[6], f[7]);
      uint8_t* line = q < 4 ? line0 : line1;
      const int c0 = 2 * (q & 3);
      *reinterpret_cast<uint4*>(line + ((c0 ^ sw) << 4)) = make_uint4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<uint4*>(line + (((c0 + 1) ^ sw) << 4)) = make_uint4(f[4], f[5], f[6], f[7]);
    }
  }
  fence_proxy_async_smem();
}

template <int BS, int G, bool F8, bool STACK = false>
__global__ void __launch_bounds__(MqTcTraits<BS, F8, STACK>::THREADS, 1)
    paged_multiquery_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                               const __grid_constant__ CUtensorMap vmap, const MultiQueryParams p) {
  using T = MqTcTraits<BS, F8, STACK>;
  constexpr int D = T::D;
  constexpr int QPT = T::ROWS / G;  // queries per unit
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* data = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hkv = p.num_kv_heads, Hq = p.num_q_heads;
  const int n_qt = (p.max_q_len * G + T::ROWS - 1) / T::ROWS;
  const int gx = Hkv * n_qt, gy = p.max_partitions;
  const int64_t n_all = static_cast<int64_t>(gx) * gy * p.num_seqs;
  const int n_units = static_cast<int>((n_all + gridDim.x - 1) / gridDim.x);  // rounds (the last may miss this CTA)
  // the group of each of this CTA's units (see rank_unit_groups)
  int* unit_g = reinterpret_cast<int*>(data + T::UNIT_OFF);
  const int64_t n_triples = static_cast<int64_t>(p.num_seqs) * gy * n_qt;
  const int rank_mode = n_units > T::MAX_UNITS         ? kRankNone
                        : n_triples <= MAX_GROUPS      ? kRankGroups
                        : p.num_seqs <= MAX_GROUPS     ? kRankSeqs
                                                       : kRankNone;
  int* scratch = reinterpret_cast<int*>(data + T::V_OFF);
  if (rank_mode == kRankGroups) {
    // triple g = (b * gy + y) * n_qt + (n_qt - 1 - qt), keyed by its KV tiles (0 when it has none)
    rank_unit_groups(static_cast<int>(n_triples), Hkv, n_units, scratch, unit_g, [&](int g) {
      const MqUnit U = mq_unit<BS, G>(p, g / (n_qt * gy), 0, n_qt - 1 - g % n_qt, (g / n_qt) % gy);
      return U.kind == kRun ? U.nt : 0;
    });
  } else if (rank_mode == kRankSeqs) {
    rank_unit_groups(p.num_seqs, gx * gy, n_units, scratch, unit_g, [&](int b) { return p.context_lens[b]; });
  }
  // unit k of this CTA (kind kSkip past the last unit).  In sequence order, unit u is x = u % gx (KV head
  // fastest, then the query tiles from the last: it sees the most tokens), partition (u / gx) % gy,
  // sequence u / (gx * gy).
  auto unit_at = [&](int k) {
    const int64_t u = cta_unit(k);
    if (u >= n_all) {
      MqUnit U;
      U.kind = kSkip;
      U.nt = 0;
      return U;
    }
    if (rank_mode == kRankGroups) {
      const int g = unit_g[k];
      return mq_unit<BS, G>(p, g / (n_qt * gy), static_cast<int>(u % Hkv), n_qt - 1 - g % n_qt, (g / n_qt) % gy);
    }
    const int x = static_cast<int>(u % gx), y = static_cast<int>((u / gx) % gy);
    const int b = rank_mode == kRankSeqs ? unit_g[k] : static_cast<int>(u / (static_cast<int64_t>(gx) * gy));
    return mq_unit<BS, G>(p, b, x % Hkv, n_qt - 1 - x / Hkv, y);
  };
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
  // 32-byte output stores need 32-byte aligned rows (rows are 256 bytes; the bases only promise 16)
  const bool out_v8 = (reinterpret_cast<uintptr_t>(p.out) & 31) == 0;
  const bool ws_v8 = (reinterpret_cast<uintptr_t>(p.ws_o) & 31) == 0;

  const uint32_t base = smem_u32(data);
  const uint32_t bar0 = base + T::BAR_OFF;
  const uint32_t q_full = bar0, q_empty = bar0 + 8;
  auto k_full = [&](int s) { return bar0 + 8 * (2 + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (2 + T::NSK + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (2 + 2 * T::NSK + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (2 + 2 * T::NSK + T::NSV + s); };
  constexpr int B2 = 2 + 2 * T::NSK + 2 * T::NSV;
  const uint32_t s_full = bar0 + 8 * B2, s_free = bar0 + 8 * (B2 + 1);
  // tile t: P of both token halves stored (8 softmax warps) on p_full(t & 1), phase t >> 1; both halves'
  // P . V of the tile complete on pv_done(t & 1), phase t >> 1
  auto p_full = [&](int t) { return bar0 + 8 * (B2 + 2 + (t & 1)); };
  auto pv_done = [&](int t) { return bar0 + 8 * (B2 + 4 + (t & 1)); };
  const uint32_t o_free = bar0 + 8 * (B2 + 6), mma_done = bar0 + 8 * (B2 + 7);
  // fp8 caches: Q rounded to fp16, K / V stages widened (k_full / v_full: their raw codes landed)
  constexpr int B3 = B2 + 8;
  const uint32_t q_ready = bar0 + 8 * B3;
  auto k_ready = [&](int s) { return bar0 + 8 * (B3 + 1 + s); };
  auto v_ready = [&](int s) { return bar0 + 8 * (B3 + 1 + T::NSK + s); };
  const uint64_t policy = l2_policy_evict_first();
  // physical id of block i of the unit's partition (i < nb), -1 when outside the pool
  auto block_id = [&](const MqUnit& U, int i) {
    const int id = U.table[i];
    return id < 0 || id >= p.num_blocks ? -1 : id;
  };
  // producers: lane i < BPT takes block i of tile j (-1 past the partition's blocks or outside the pool)
  auto tile_block = [&](const MqUnit& U, int j) {
    const int i = j * T::BPT + lane;
    return lane < T::BPT && i < U.nb ? block_id(U, i) : -1;
  };

  if (threadIdx.x == T::W_K * 32) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < T::NSK; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
    }
    for (int s = 0; s < T::NSV; ++s) {
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(p_full(b), 8);
      mbar_init(pv_done(b), 1);
    }
    mbar_init(o_free, 8);
    mbar_init(mma_done, T::N_ISSUERS);
    if constexpr (F8) {
      mbar_init(q_ready, 8);
      for (int s = 0; s < T::NSK; ++s) mbar_init(k_ready(s), 1);
      for (int s = 0; s < T::NSV; ++s) mbar_init(v_ready(s), 1);
    }
    if constexpr (STACK) mbar_init(q_ready, 4);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == T::W_K) {
    tmem_alloc(base + T::SLOT_OFF, T::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(data + T::SLOT_OFF);
  const uint32_t tmem_s = tmem;
  auto tmem_o = [&](int h) { return tmem + 128 + 128 * h; };
  // P of tile t, tokens 64h .. 64h+63 packed in pairs: hi / fp16
  auto tmem_p = [&](int h, int t) { return tmem + 384 + 64 * (T::NPB == 2 ? (t & 1) : 0) + 32 * h; };
  auto tmem_plo = [&](int h) { return tmem + 448 + 32 * h; };  // bf16 caches: the residual

  if (warp == T::W_K || warp == T::W_V) {  // ---------------- TMA producers of Q and K, and of V --------
    // whole warp: lane i < BPT loads block i of each tile; ring stages and phases run on the tile
    // count g across the CTA's units
    const bool is_k = warp == T::W_K;
    const int ns = is_k ? T::NSK : T::NSV;
    const CUtensorMap* map = is_k ? &kmap : &vmap;
    const uint32_t area = base + (is_k ? T::K_OFF : T::V_OFF);
    int g = 0, ku = 0;
    bool ok = true;
    for (int k = 0; ok && k < n_units; ++k) {
      const MqUnit U = unit_at(k);
      if (U.kind != kRun) continue;
      if (is_k) {  // Q of this unit once the previous unit is done with the Q tile (its S MMAs; stacked:
                   // its epilogue too)
        if (ku > 0 && !(ok = warp_wait_bounded(q_empty, (ku - 1) & 1, p.status))) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, T::TILE);
          tma_load_3d(base + T::Q_OFF, &qmap, q_full, 0, U.hk * G, U.q0 + U.qt * QPT);
          tma_load_3d(base + T::Q_OFF + T::HALF, &qmap, q_full, 64, U.hk * G, U.q0 + U.qt * QPT);
        }
        ++ku;
      }
      int id = tile_block(U, 0);  // the block ids of tile j + 1 are read while tile j is issued
      for (int j = 0; j < U.nt; ++j, ++g) {
        const int s = g % ns, use = g / ns;
        if (use > 0 && !(ok = warp_wait_bounded(is_k ? k_empty(s) : v_empty(s), (use - 1) & 1, p.status))) break;
        const unsigned vm = __ballot_sync(kFullMask, id >= 0);
        if (is_k && lane == 0 && __popc(vm) < min(T::BPT, U.nb - j * T::BPT))
          set_status(p.status, PKV_STATUS_BAD_BLOCK_ID);
        const uint32_t full = is_k ? k_full(s) : v_full(s);
        if (lane == 0) {
          const uint32_t bytes = static_cast<uint32_t>(__popc(vm)) * (F8 ? 1u : 2u) * BS * 128u;
          if (bytes) mbar_arrive_expect_tx(full, bytes); else mbar_arrive(full);
        }
        __syncwarp();
        if (id >= 0) {
          if constexpr (F8) {  // the raw codes into the stage's upper half
            tma_load_4d(area + s * T::TILE + T::HALF + lane * BS * 128, map, full, 0, U.hk, 0, id, policy);
          } else {
            const uint32_t dst = area + s * T::TILE + lane * BS * 128;
            tma_load_4d(dst, map, full, 0, U.hk, 0, id, policy);
            tma_load_4d(dst + T::HALF, map, full, 64, U.hk, 0, id, policy);
          }
        }
        id = j + 1 < U.nt ? tile_block(U, j + 1) : -1;
      }
    }
    // drain (bounded): the copies of the last stages (and the last Q) have landed before exit
    if (lane == 0) {
      if (is_k && ku > 0) mbar_wait_sleep(q_full, (ku - 1) & 1, p.status);
      for (int i = max(0, g - ns); i < g; ++i)
        mbar_wait_sleep(is_k ? k_full(i % ns) : v_full(i % ns), (i / ns) & 1, p.status);
    }
  } else if (F8 && (warp == T::W_KWIDEN || warp == T::W_VWIDEN)) {  // ---- fp8: widen the landed tiles ----
    const bool is_k = warp == T::W_KWIDEN;
    const int ns = is_k ? T::NSK : T::NSV;
    const int area = is_k ? T::K_OFF : T::V_OFF;
    int g = 0;
    bool ok = true;
    for (int k = 0; ok && k < n_units; ++k) {
      const MqUnit U = unit_at(k);
      if (U.kind != kRun) continue;
      // blocks of the unit with a bad id: their V rows are zeroed
      bool any_bad = false;
      if (!is_k) {
        for (int i = lane; i < U.nb; i += 32) any_bad |= block_id(U, i) < 0;
        any_bad = __any_sync(kFullMask, any_bad);
      }
      for (int j = 0; j < U.nt; ++j, ++g) {
        const int st = g % ns;
        if (!(ok = warp_wait_bounded(is_k ? k_full(st) : v_full(st), (g / ns) & 1, p.status))) break;
        uint8_t* stage = data + area + st * T::TILE;
        const int tile0 = U.tok_begin + j * T::TOK;
        if (is_k) {  // scores of rows that are not loaded are masked, whatever these rows hold
          widen_e4m3_tile_in_place(stage, lane, [](int) { return false; });
        } else {     // V rows that must not contribute (past tok_end, bad blocks) are zeroed
          widen_e4m3_tile_in_place(stage, lane, [&](int t) {
            return tile0 + t >= U.tok_end || (any_bad && block_id(U, (tile0 + t - U.tok_begin) / BS) < 0);
          });
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(is_k ? k_ready(st) : v_ready(st));
      }
    }
  } else if (warp == T::W_MMA || warp == T::W_PV) {  // ---------------- MMA issuers ----------------------
    // bf16 caches: warp 11 issues the S MMAs and warp 9 the P . V MMAs, each with its own waits and
    // commits, so one thread's barrier work overlaps the other's MMAs in the tensor pipe (the two
    // streams touch disjoint TMEM columns; their order is set by the barriers alone).  fp8 caches:
    // warp 9 the S MMAs and warp 13 the P . V MMAs.
    if (lane == 0) {
      constexpr uint32_t idesc_s = F8 ? idesc_f16_f32(128, 128, 0) : idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = F8 ? idesc_f16_f32(128, 128, 1) : idesc_bf16_f32(128, 128, 1);
      const uint64_t qd0 = smem_desc_sw128(base + T::Q_OFF, 16, 1024);         // K-major Q (and K, offset)
      const uint64_t vdb = smem_desc_sw128(base + T::V_OFF, T::HALF, 1024);     // N-major V
      const bool do_s = warp == T::W_MMA;  // else the P . V issuer
      // S of tile j of the unit (tile gj of the CTA)
      auto issue_s = [&](const MqUnit& U, int j, int gj) -> bool {
        const int sk = gj % T::NSK;
        if (!mbar_wait_bounded(F8 ? k_ready(sk) : k_full(sk), (gj / T::NSK) & 1, p.status)) return false;
        if (gj > 0 && !mbar_wait_bounded(s_free, (gj - 1) & 1, p.status)) return false;
        tc_fence_after();
        // descriptors differ only in the start-address field (address >> 4 in the low bits, all
        // addresses below 256 KB): the base descriptors plus offsets
        const uint64_t kd0 = qd0 + ((T::K_OFF - T::Q_OFF + sk * T::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = ((kk >> 2) * T::HALF + (kk & 3) * 32) >> 4;
          tc_mma_bf16(tmem_s, qd0 + off, kd0 + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        tc_commit(k_empty(sk));
        if (j == U.nt - 1) tc_commit(q_empty);  // the unit's S MMAs are its only readers of Q
        return true;
      };
      // P . V of tile jj of unit ku (tile gjj of the CTA); half1_past: every token of the tile's second half
      // lies past the unit's tokens (a unit's last tile, not its first: O_1 is already written), so its
      // P . V would add zeros and is left out
      auto issue_pv = [&](int jj, int gjj, int ku, bool half1_past) -> bool {
        const int sv = gjj % T::NSV;
        const uint64_t vd0 = vdb + ((sv * T::TILE) >> 4);
        // the V tile (bf16: landed; fp8: widened)
        if (!mbar_wait_bounded(F8 ? v_ready(sv) : v_full(sv), (gjj / T::NSV) & 1, p.status)) return false;
        // the unit's first P . V overwrites O: the previous unit's epilogue must have read it
        if (jj == 0 && ku > 0 && !mbar_wait_bounded(o_free, (ku - 1) & 1, p.status)) return false;
        if (!mbar_wait_bounded(p_full(gjj), (gjj >> 1) & 1, p.status)) return false;
        tc_fence_after();
        // O_h += P_h(jj) . V_h(jj); the branch is taken once, before the MMAs (a branch between MMAs
        // costs the issuing thread)
        auto pv_half = [&](int h) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // 16 tokens = 8 packed TMEM columns of P per k-step
            const uint64_t vdesc = vd0 + (((64 * h + 16 * kk) * 128) >> 4);
            tc_mma_bf16_tmem_a(tmem_o(h), tmem_p(h, gjj) + 8 * kk, vdesc, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
            if constexpr (!F8 && !STACK) tc_mma_bf16_tmem_a(tmem_o(h), tmem_plo(h) + 8 * kk, vdesc, idesc_pv, 1u);
          }
        };
        if (half1_past) {
          pv_half(0);
        } else {
          pv_half(0);
          pv_half(1);
        }
        tc_commit(pv_done(gjj));
        tc_commit(v_empty(sv));
        return true;
      };
      int g = 0, ku = 0;  // tiles of the CTA so far; units
      bool ok = true;
      for (int k = 0; ok && k < n_units; ++k) {
        const MqUnit U = unit_at(k);
        if (U.kind != kRun) continue;
        if (do_s && !(ok = mbar_wait_bounded(F8 || STACK ? q_ready : q_full, ku & 1, p.status))) break;
        // tile j's second half lies past the unit's tokens (only a last tile can; never the first)
        auto half1_past = [&](int j) { return j > 0 && U.tok_begin + j * T::TOK + 64 >= U.tok_end; };
        if (do_s) {
          for (int j = 0; ok && j < U.nt; ++j) ok = issue_s(U, j, g + j);
        } else {
          for (int j = 0; ok && j < U.nt; ++j) ok = issue_pv(j, g + j, ku, half1_past(j));
        }
        g += U.nt;
        ++ku;
      }
      // drain (bounded): no MMA of this thread may still read shared memory or write TMEM at exit
      tc_commit(mma_done);
      mbar_wait_bounded(mma_done, 0, p.status);
    }
  } else if (warp < 8) {  // ---------------- softmax warps 0-7 --------------------------------------
    const int quarter = warp & 3, h = warp >> 2;  // TMEM lane quarter, token half of each tile
    const int tl = 32 * quarter + lane;           // this thread's TMEM lane
    // its row of a unit; stacked: lanes 64-127 repeat rows 0-63 and write the residual part of P
    const bool lo_part = STACK && quarter >= 2;
    const int r = STACK ? (tl & 63) : tl;
    const uint32_t lane_off = static_cast<uint32_t>(32 * quarter) << 16;
    const float qk = p.q_scale;
    const int pair_bar = 5 + 2 * (quarter & 1) + h;  // stacked: named barrier of the two warps of a row
    // After a timed-out wait the warp stops waiting (every later wait fails at
    // once) but still runs every unit and iteration, so the two warps of a pair
    // meet at the epilogue's named barriers; the status bit reports the failure.
    bool ok = true;
    auto wait = [&](uint32_t bar, uint32_t parity) {
      if (ok) ok = warp_wait_bounded(bar, parity, p.status);
      return ok;
    };
    // fp8 caches with at most 64 rows per (sequence, KV head) (grouped verification): lane quarters 2
    // and 3 have no rows in any unit, so their warps take no part, and the warp of lane quarter 0 of
    // each token half arrives for them on q_ready, s_free, p_full and o_free (8 arrivals each) -- those
    // barriers never wait for warps that would only wake to arrive.  (It holds for every unit of the
    // launch, so no warp runs ahead of the barrier phases.  bf16 caches: such warps zero their share of
    // V rows, and with at most 64 rows the stacked tile fills every quarter.)
    const bool skip_q23 = F8 && p.max_q_len * G <= 64;
    const uint32_t arrive_n = skip_q23 && quarter == 0 ? 3u : 1u;
    int g = 0, ku = 0;  // tiles consumed; units
    for (int k = 0; k < (skip_q23 && quarter >= 2 ? 0 : n_units); ++k) {
      const MqUnit U = unit_at(k);
      if (U.kind == kBadQuery) {
        if (threadIdx.x == 0) set_status(p.status, PKV_STATUS_BAD_QUERY_LOC);
        continue;
      }
      if (U.kind == kZero) {  // nothing to attend: zero rows
        if (warp < 4) {
          const int row = U.qt * T::ROWS + tl;
          if (row < U.rows_total) {
            const int64_t orow = static_cast<int64_t>(U.q0 + row / G) * Hq + U.hk * G + row % G;
            for (int d = 0; d < D; d += 8)
              *reinterpret_cast<uint4*>(out + orow * D + d) = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
      if (U.kind != kRun) continue;
      const int tok_begin = U.tok_begin, tok_end = U.tok_end, nt = U.nt, nb = U.nb;
      const int row = U.qt * T::ROWS + r;
      const bool valid = row < U.rows_total;
      // an invalid row (its output is never written) sees what the unit's last row sees, so that it
      // takes the same path as its warp's valid rows (a row that saw nothing would take the masking
      // path alone and hold the warp on it every tile); its P only feeds its own accumulator row
      const int pos = U.base_pos + (valid ? row : U.row_last) / G;
      float m = -INFINITY, l = 0.f;  // this half's running reference max (log2 units) and row sum
      if constexpr (F8) {  // this thread's Q row half to fp16, in place (exact for |q| in [2^-14, 65504])
        wait(q_full, ku & 1);
        uint4* qrow = reinterpret_cast<uint4*>(data + T::Q_OFF + h * T::HALF + r * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = qrow[c];
          qrow[c] = make_uint4(bf16x2_to_f16x2(w.x), bf16x2_to_f16x2(w.y), bf16x2_to_f16x2(w.z), bf16x2_to_f16x2(w.w));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(q_ready, arrive_n);
      }
      if constexpr (STACK) {  // Q rows 0-63 (this warp's 64-dim half) copied below themselves, same phase
        if (lo_part) {
          wait(q_full, ku & 1);
          const int i = 32 * (quarter - 2) + lane;  // 64 threads x 8 x 16 bytes of the half
          const uint4* src = reinterpret_cast<const uint4*>(data + T::Q_OFF + h * T::HALF);
          uint4* dst = reinterpret_cast<uint4*>(data + T::Q_OFF + h * T::HALF + 64 * 128);
#pragma unroll
          for (int c = 0; c < 8; ++c) dst[i + 64 * c] = src[i + 64 * c];
          fence_proxy_async_smem();  // these writes before the MMA's reads (async proxy)
          __syncwarp();
          if (lane == 0) mbar_arrive(q_ready);
        }
      }
      // blocks of the unit with a bad id (reported by the K producer): masked, their V rows zeroed
      bool any_bad = false;
      for (int i = lane; i < nb; i += 32) any_bad |= block_id(U, i) < 0;
      any_bad = __any_sync(kFullMask, any_bad);
      // bf16 caches: V rows of tokens that must not contribute (past tok_end, bad blocks) are zeroed:
      // 0 * NaN would poison O.  The 64 rows of this half: thread (quarter, lane) takes row
      // 16 quarter + lane / 2, dims half lane & 1.  (fp8 caches: the widening warp zeroed them.)
      auto zero_v_rows = [&](int j, bool bad) {
        const int gj = g + j;
        wait(v_full(gj % T::NSV), (gj / T::NSV) & 1);
        const int vr = 64 * h + 16 * quarter + (lane >> 1);
        const int t = tok_begin + j * T::TOK + vr;
        if (t >= tok_end || (bad && block_id(U, (t - tok_begin) / BS) < 0)) {
          uint8_t* vrow = data + T::V_OFF + (gj % T::NSV) * T::TILE + (lane & 1) * T::HALF + vr * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(vrow + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();  // the zeroed rows before the MMA reads them
      };
      // bit k set: block k of the half tile starting at token t0 has a bad id (t0 - tok_begin is a
      // multiple of 64, so the half tile holds 64 / BS whole blocks)
      auto half_tile_bad = [&](int t0) {
        unsigned bad = 0u;
        if (any_bad) {
          const int i0 = (t0 - tok_begin) / BS;
          for (int kb = 0; kb < 64 / BS && i0 + kb < nb; ++kb)
            if (block_id(U, i0 + kb) < 0) bad |= 1u << kb;
        }
        return bad;
      };
      // P of tile t goes into a buffer last read by the P . V of tile t - NPB: that one must be complete
      // (and so the warp never arrives on p_full ahead of the phase)
      auto wait_p_buffer = [&](int t) {
        const int tw = t - T::NPB;
        if (tw >= 0) wait(pv_done(tw), (tw >> 1) & 1);
      };
      // A warp whose 32 rows all lie past the unit's query rows (grouped verification uses 40 of 128)
      // computes nothing: it keeps every barrier step -- including the wait for the P buffer -- and its
      // share of the V-row zeroing (that share is by token, not by query row).  Its P rows stay stale:
      // they only feed output rows nobody writes.
      if (U.qt * T::ROWS + 32 * (STACK ? (quarter & 1) : quarter) >= U.rows_total) {
        for (int j = 0; j < nt; ++j) {
          const int t0 = tok_begin + j * T::TOK + 64 * h;
          wait(s_full, (g + j) & 1);
          tc_fence_after();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free);
          const bool bad = half_tile_bad(t0) != 0u;
          wait_p_buffer(g + j);
          if (!F8 && (t0 + 64 > tok_end || bad)) zero_v_rows(j, bad);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full(g + j));
        }
      } else
      for (int j = 0; j < nt; ++j) {
        const int t0 = tok_begin + j * T::TOK + 64 * h;  // first token of this half of the tile
        wait(s_full, (g + j) & 1);
        tc_fence_after();
        float sv[64];
        {
          uint32_t u[2][32];
          tmem_ld32(tmem_s + lane_off + 64 * h, u[0]);
          tmem_ld32(tmem_s + lane_off + 64 * h + 32, u[1]);
          tmem_ld_wait(u[0]);
          tmem_ld_wait(u[1]);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[e] = __uint_as_float(u[0][e]);
            sv[32 + e] = __uint_as_float(u[1][e]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(s_free, arrive_n);

        // blocks of this half tile with a bad id (their tokens are masked, their V rows zeroed)
        const unsigned bad_blocks = half_tile_bad(t0);
        const bool bad = bad_blocks != 0u;
        const bool ragged = t0 + 64 > tok_end;  // tokens at or past tok_end in this half tile
        // row max of the raw scores (q_scale > 0 commutes with the max); masked scores -> -inf.
        // Eight independent partial maxima / sums: instruction-level parallelism hides latency.
        float mx8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx8[e] = -INFINITY;
        if (t0 + 63 > pos || ragged || bad) {
          if (bad) {  // scores of blocks that were not loaded (stale tiles) never reach the max
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if ((bad_blocks >> (c / BS)) & 1u) sv[c] = -INFINITY;
          }
          // column c is visible iff c <= last (causal position and the end of what is loaded)
          const int last = min(pos, tok_end - 1) - t0;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            sv[c] = c > last ? -INFINITY : sv[c];
            mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; c += 2) mx8[(c >> 1) & 7] = fmax3f(mx8[(c >> 1) & 7], sv[c], sv[c + 1]);
        }
        const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                               fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * qk;
        // reference max: move it (and rescale) only when a score passes it by more than 8 (log2 units)
        float alpha = 1.f;
        if (mx > m + 8.f) {
          alpha = m == -INFINITY ? 0.f : fast_exp2(m - mx);
          l *= alpha;
          m = mx;
        }
        const float neg_m = m == -INFINITY ? 0.f : -m;  // m = -inf: every score is -inf, p = 0
        // p = 2^(s * q_scale - m), pairs of values through the packed fp32x2 FMA / add, and at once the
        // row's half of P as packed pairs (tokens 2k, 2k+1 in word k).  bf16 caches: a high part (the
        // top 16 bits of the fp32 value: truncation) and the residual (exact in fp32, then truncated to
        // its top 16 bits), ~16 significant bits per probability, with integer ops only.  fp8 caches:
        // one fp16 value (round to nearest; p <= 2^8).  One loop, so the special-function unit (ex2)
        // and the integer / FMA pipes (packing) work side by side; the stores to TMEM wait below.
        const float2 qk2 = make_float2(qk, qk), nm2 = make_float2(neg_m, neg_m);
        float2 sum4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) sum4[e] = make_float2(0.f, 0.f);
        uint32_t ph[32], plo[32];
        if constexpr (STACK) {
          // The row's two warps hold the same scores: the high-part warp takes token pairs 0-15 of the
          // half tile, the residual warp pairs 16-31; each sends the other the part it stores (the
          // residuals of pairs 0-15, the high parts of pairs 16-31) and keeps its share of the row sum.
          uint32_t own[16], send[16], recv[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float x0 = lo_part ? sv[32 + 2 * k] : sv[2 * k], x1 = lo_part ? sv[33 + 2 * k] : sv[2 * k + 1];
            const float2 x = __ffma2_rn(make_float2(x0, x1), qk2, nm2);
            const float a = fast_exp2(x.x), bb = fast_exp2(x.y);
            sum4[k & 3] = __fadd2_rn(sum4[k & 3], make_float2(a, bb));
            const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(bb);
            const float2 rr = __fadd2_rn(make_float2(a, bb),
                                         make_float2(__uint_as_float((ua & 0xFFFF0000u) ^ 0x80000000u),
                                                     __uint_as_float((ub & 0xFFFF0000u) ^ 0x80000000u)));
            const uint32_t hi = __byte_perm(ua, ub, 0x7632);
            const uint32_t lo = __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
            own[k] = lo_part ? lo : hi;
            send[k] = lo_part ? hi : lo;
          }
          // thread (warp, lane) and its partner (warp ^ 2, lane): word group c of thread i at c * 256 + i
          uint4* xs = reinterpret_cast<uint4*>(data + T::XCH_OFF + ((g + j) & 1) * T::XCH_TILE);
          const int me = warp * 32 + lane, other = (warp ^ 2) * 32 + lane;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            xs[c * 256 + me] = make_uint4(send[4 * c], send[4 * c + 1], send[4 * c + 2], send[4 * c + 3]);
          asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = xs[c * 256 + other];
            recv[4 * c] = v.x;
            recv[4 * c + 1] = v.y;
            recv[4 * c + 2] = v.z;
            recv[4 * c + 3] = v.w;
          }
#pragma unroll
          for (int k = 0; k < 16; ++k) {  // high parts for the high-part warp, residuals for the other
            ph[k] = own[k];
            ph[16 + k] = recv[k];
            plo[k] = recv[k];
            plo[16 + k] = own[k];
          }
        } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float2 x = __ffma2_rn(make_float2(sv[2 * k], sv[2 * k + 1]), qk2, nm2);
          const float a = fast_exp2(x.x), bb = fast_exp2(x.y);
          sum4[k & 3] = __fadd2_rn(sum4[k & 3], make_float2(a, bb));
          if constexpr (F8) {
            const __half2 hp = __floats2half2_rn(a, bb);  // token 2k in the low half
            ph[k] = *reinterpret_cast<const uint32_t*>(&hp);
            plo[k] = 0u;
          } else {
            const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(bb);
            // residual = value - its truncation (the negated truncation is one logic op)
            const float2 rr = __fadd2_rn(make_float2(a, bb),
                                         make_float2(__uint_as_float((ua & 0xFFFF0000u) ^ 0x80000000u),
                                                     __uint_as_float((ub & 0xFFFF0000u) ^ 0x80000000u)));
            ph[k] = __byte_perm(ua, ub, 0x7632);  // {b.hi16, a.hi16}: token 2k in the low half
            plo[k] = __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
          }
        }
        }
        const float2 s2 = __fadd2_rn(__fadd2_rn(sum4[0], sum4[1]), __fadd2_rn(sum4[2], sum4[3]));
        l += s2.x + s2.y;
        // the P buffer of this tile must be free; O_h is rescaled (rarely) once the previous tile's
        // P . V is complete
        wait_p_buffer(g + j);
        tc_fence_after();
        if (j > 0) {
          if (__any_sync(kFullMask, alpha != 1.f)) {  // a moved reference: rescale this row of O_h
            if constexpr (T::NPB == 2) {
              wait(pv_done(g + j - 1), ((g + j - 1) >> 1) & 1);
              tc_fence_after();
            }
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t u[32];
              const uint32_t oa = tmem_o(h) + lane_off + 32 * c;
              tmem_ld32(oa, u);
              tmem_ld_wait(u);
#pragma unroll
              for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * alpha);
              tmem_st32(oa, u);
            }
          }
        }
        if (!F8 && (ragged || bad)) zero_v_rows(j, bad);
        // this half of row r of P into TMEM lane r: the stacked tile's one part in a 32-column store
        // (measured +0.9%); elsewhere 16 columns at a time (32-column stores measured -1.9% on prefill,
        // and spill with fp8 caches)
        if constexpr (STACK) {
          if (lo_part)
            tmem_st32(tmem_p(h, g + j) + lane_off, plo);
          else
            tmem_st32(tmem_p(h, g + j) + lane_off, ph);
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pw[16], lw[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              pw[k] = ph[16 * c + k];
              lw[k] = plo[16 * c + k];
            }
            tmem_st16(tmem_p(h, g + j) + lane_off + 16 * c, pw);
            if constexpr (!F8) tmem_st16(tmem_plo(h) + lane_off + 16 * c, lw);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cnt(p_full(g + j), arrive_n);
      }
      g += nt;
      wait(pv_done(g - 1), ((g - 1) >> 1) & 1);  // (and so every earlier P . V)
      tc_fence_after();
      if constexpr (STACK) {  // the row sum: this warp's share plus its partner's (high-part share first)
        float* lx = reinterpret_cast<float*>(data + T::XCH_OFF + 2 * T::XCH_TILE);
        lx[warp * 32 + lane] = l;
        asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        const float lp = lx[(warp ^ 2) * 32 + lane];
        l = lo_part ? lp + l : l + lp;
      }
      // ---- epilogue: merge the two halves' (m, l, O_h); this warp writes output dims 64h .. 64h+63 ---
      // (m, l) of this half go to the partner warp through TMEM columns of P_h (its P . V is done)
      {
        uint32_t w[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = 0u;
        w[0] = __float_as_uint(m);
        w[1] = __float_as_uint(l);
        tmem_st16(tmem_p(h, 0) + lane_off, w);
        tmem_st_wait();
      }
      tc_fence_before();
      asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");  // the two warps of this lane quarter
      tc_fence_after();
      float m_o, l_o;
      {
        uint32_t x[32];
        tmem_ld32(tmem_p(h ^ 1, 0) + lane_off, x);
        tmem_ld_wait(x);
        m_o = __uint_as_float(x[0]);
        l_o = __uint_as_float(x[1]);
      }
      const float M = fmaxf(l > 0.f ? m : -INFINITY, l_o > 0.f ? m_o : -INFINITY);
      const float w_self = l > 0.f ? fast_exp2(m - M) : 0.f, w_oth = l_o > 0.f ? fast_exp2(m_o - M) : 0.f;
      const float lsum = l * w_self + l_o * w_oth;
      const float inv = lsum > 0.f ? p.out_scale / lsum : 0.f;
      const float w0 = (h == 0 ? w_self : w_oth) * inv, w1 = (h == 0 ? w_oth : w_self) * inv;  // O_0, O_1 weights
      const int64_t orow = static_cast<int64_t>(U.q0 + row / G) * Hq + U.hk * G + row % G;
      // stacked: the residual's share of this row's output (accumulator rows 64-127) goes from the warp
      // of lanes 64-127 to the warp of the same row and half through the P exchange buffers (the
      // unit's last exchange was read before the row-sum barrier above), so the next unit's Q can
      // load while this epilogue runs
      float* xo = reinterpret_cast<float*>(data + T::XCH_OFF);  // [64 rows][128 dims]
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        const int d0 = 64 * h + 32 * c;
        uint32_t u0[32], u1[32];
        tmem_ld32(tmem_o(0) + lane_off + d0, u0);
        tmem_ld32(tmem_o(1) + lane_off + d0, u1);
        tmem_ld_wait(u0);
        tmem_ld_wait(u1);
        // (the high-part warp's first accumulator reads overlap the residual warp's writes)
        if (STACK && !lo_part && c == 0) asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        if (!valid || !ok) continue;
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(u0[e]) * w0 + __uint_as_float(u1[e]) * w1;
        if constexpr (STACK) {
          float4* x4 = reinterpret_cast<float4*>(xo + r * 128 + d0);
          if (lo_part) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) x4[e / 4] = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
            continue;
          }
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 v = x4[e / 4];
            o[e] += v.x;
            o[e + 1] += v.y;
            o[e + 2] += v.z;
            o[e + 3] += v.w;
          }
        }
        // Each lane writes its own row: 32-byte stores (whole sectors, half the store transactions of
        // 16-byte ones) where the base allows, 16-byte ones otherwise.
        if (U.nparts == 1) {
          __nv_bfloat16* dst = out + orow * D + d0;
          uint32_t w[2][8];
#pragma unroll
          for (int kq = 0; kq < 16; ++kq) {
            __nv_bfloat162 hv = __floats2bfloat162_rn(o[2 * kq], o[2 * kq + 1]);
            w[kq >> 3][kq & 7] = *reinterpret_cast<uint32_t*>(&hv);
          }
          if (out_v8) {
            st_global_v8(dst, w[0]);
            st_global_v8(dst + 16, w[1]);
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              *reinterpret_cast<uint4*>(dst + 8 * e) =
                  make_uint4(w[e >> 1][4 * (e & 1)], w[e >> 1][4 * (e & 1) + 1], w[e >> 1][4 * (e & 1) + 2],
                             w[e >> 1][4 * (e & 1) + 3]);
          }
        } else {
          float* dst = p.ws_o + (orow * p.max_partitions + U.part) * D + d0;
          if (ws_v8) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint32_t w8[8];
#pragma unroll
              for (int q = 0; q < 8; ++q) w8[q] = __float_as_uint(o[e + q]);
              st_global_v8(dst + e, w8);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dst + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
          }
        }
      }
      if constexpr (STACK) {
        // the residual warp's writes are complete (its arrival pairs with the wait before the loop);
        // then both wait until the high-part warp has read them: the next unit's exchanges reuse the
        // buffers
        if (lo_part) asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      }
      if (valid && ok && U.nparts > 1 && h == 0 && !lo_part) {
        const int64_t srow = orow * p.max_partitions + U.part;
        p.ws_ml[srow * 2] = lsum > 0.f ? M * kLn2 : 0.f;
        p.ws_ml[srow * 2 + 1] = lsum;
      }
      // both warps of the pair have read the exchanged (m, l) before either writes the next unit's P,
      // and every softmax warp has read O before the next unit's first P . V overwrites it
      tc_fence_before();
      asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
      if (lane == 0) mbar_arrive_cnt(o_free, arrive_n);
      ++ku;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == T::W_K) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, T::TMEM_COLS);
  }
}

}  // namespace pkv

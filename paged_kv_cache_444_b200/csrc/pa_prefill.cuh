// pa_prefill.cuh -- paged (chunked) prefill attention on the sm_100a tensor
// cores (tcgen05, accumulators in tensor memory).
//
// "vLLM PagedAttention 原理与源码深度解析" §8.1 (Chunked Prefill): a long prompt
// is processed a chunk of tokens per step, so a step holds sequences with
// several new query tokens at the end of their context.  Query token i of
// sequence s (q_len new tokens, context_lens[s] tokens in all, their K/V
// already in the paged cache) sits at position ctx - q_len + i and attends
// causally to tokens 0..pos.
//
// Work item: (sequence, KV head, pair of query tiles A and B).  A tile is
// 128/G consecutive query tokens x the G query heads of the KV head,
// token-major: 128 rows, the M of one MMA.  Both tiles walk the same keys in
// blocks of 128 (8 pages of 16), so every K/V block gathered into shared
// memory feeds 256 query rows.  Per tile t and block j:
//   S_t  = Q_t K_j^T    128 x 128 fp32 in tensor memory; Q and K from shared
//   P_t  = 2^(S_t*scale*log2 e - m)   by the tile's softmax warpgroup (thread
//                       r = row r), written back over S_t as 16-bit pairs
//   O_t += P_t V_j      128 x D fp32 in tensor memory; P from tensor memory,
//                       V from shared memory
// One warp issues every MMA in the order S_A(j), P_B(j-1) V, S_B(j), P_A(j) V,
// so each warpgroup's softmax overlaps the other tile's MMAs.  MMAs from one
// thread run in issue order: S_t(j+1) may overwrite P_t(j) as soon as it is
// issued after the P V that reads it, and the commit that reports S_t(j+1)
// also reports that P V done (the softmax may then rescale O_t).  Another warp
// loads each item's Q and the K and V pages with TMA through rings of NST
// stages.
//
// The grid is persistent, one CTA per SM: each CTA walks its share of the
// items (ordered longest first, see below) with every ring and phase running
// on from item to item, and hands items over with three barriers (Q free: the
// item's S products are done; O full / O free per tile: its last P V is done,
// its epilogue has read O), so an item's epilogue and Q load overlap the
// neighbouring item's products.
//
// The causal mask is a per-row key limit (pos + 1) applied to S; blocks past
// the pair's last key are never loaded, and V rows past the context are
// zeroed before use (never written, they may hold anything).  O is rescaled
// only when a row's running maximum grows by more than 2^8 (the reference
// maximum may lag the true one by that much: P <= 2^8 stays exact in the
// 16-bit operand and the final 1/l uses the same reference).  bf16 P enters
// P V as a hi + lo pair of bf16 products (at least 14 bits of P, split by
// bit truncation so the conversion unit stays free for 2^x); fp16 P is
// rounded once and l sums the fp32 p.  With bf16 caches the default
// build rewrites each V block as fp16 in shared memory (six converter warps)
// and takes the fp16 P path instead (PA_PREFILL_V_FP16, below).
#pragma once

#include "pa_decode.cuh"
#include "pa_umma.cuh"

namespace pa {

constexpr unsigned kErrQuery = 7;
constexpr int kPrefillRows = 128;                   // query rows per tile = MMA M
constexpr int kPrefillKeys = 128;                   // keys per block = S tile N
constexpr int kPrefillPages = kPrefillKeys / kPage; // 8 pages per block
constexpr int kWarpMma = 8;                         // issues every MMA, owns tensor memory
constexpr int kWarpTma = 9;                         // Q, K and V loads
constexpr int kPrefillThreads = 10 * 32;            // + two softmax warpgroups (warps 0-7)
constexpr int kWarpConv = 10;                       // V converters: warps 10-15 (convert mode)
constexpr int kConvWarps = 6;
constexpr unsigned kErrValue = 8;
constexpr int kRankMaxSeqs = 256;     // batches ranked longest-first by every CTA: sequences,
constexpr int kRankMaxUnits = 2048;   // units (sequence, tile pair),
constexpr int kRankMaxWork = 16384;   // and units x sequences counted

// bf16 caches: rewrite each landed V block as fp16 in shared memory (warps
// 10-13, once per block for both tiles), so that P enters P V once, as fp16
// (11 bits), instead of as a bf16 hi + lo pair.  fp16 holds every bf16 value
// of magnitude below 65 520 exactly, apart from the tiny ones below 2^-14,
// which lose at most 2^-25 each; larger values saturate to +-65 504 and are
// reported (PA_CHECK_VALUE).
#ifndef PA_PREFILL_V_FP16
#define PA_PREFILL_V_FP16 1
#endif
template <bool BF16>
struct PrefillRoles {
  static constexpr bool kConvert = BF16 && PA_PREFILL_V_FP16 != 0;
  // convert mode: four whole warpgroups (setmaxnreg works per warpgroup):
  // softmax 0-7, then MMA, TMA and converters 10-15
  static constexpr int kThreads = kConvert ? 16 * 32 : kPrefillThreads;
  static constexpr bool kPHiLo = BF16 && !kConvert;   // P as a bf16 hi + lo pair
};

// Register split of convert mode: 512 threads launched at 128 registers each
// (65 536, the whole file); the two softmax warpgroups take 184, the other two
// give up to 72: 2 x 128 x 184 + 2 x 128 x 72 = 65 536.
constexpr uint32_t kRegsSoftmax = 184, kRegsOther = 72;
__device__ __forceinline__ void regs_increase() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
}
__device__ __forceinline__ void regs_decrease() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsOther));
}
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                      // O_t: columns [128 t, 128 t + D)
constexpr uint32_t kTmemS = 256;                    // S_t / P_t: [256 + 128 t, +128)
constexpr float kRescaleSlack = 8.f;                // log2 units

struct PrefillArgs {
  uint16_t* out;                // [T, H, D]
  const int32_t* block_tables;  // [S, MB]
  const int32_t* context_lens;  // [S]
  const int32_t* query_starts;  // [S + 1]
  float scale_log2;
  int num_seqs;
  int num_tokens;               // T
  int num_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int tile_tokens;              // query tokens per tile (128 / group, rounded down)
};

template <int D, bool BF16>
struct PrefillSmem {
  static constexpr int NST = D == 64 ? 4 : 2;       // K (and V) blocks in flight
  static constexpr int kSlabs = D / 64;             // 64-element column slabs
  static constexpr int kSlab = 128 * 128;           // 128 rows x 128 B
  static constexpr int kQTile = kSlabs * kSlab;     // one tile of Q
  static constexpr int kQ = 0;                      // Q_A, then Q_B
  static constexpr int kStage = kSlabs * kSlab;     // one block of K (or V)
  static constexpr int kK = kQ + 2 * kQTile;
  static constexpr int kV = kK + NST * kStage;
  static constexpr int kBarQ = kV + NST * kStage;
  static constexpr int kBarKFull = kBarQ + 8;
  static constexpr int kBarKEmpty = kBarKFull + 8 * NST;
  static constexpr int kBarVFull = kBarKEmpty + 8 * NST;
  static constexpr int kBarVEmpty = kBarVFull + 8 * NST;
  static constexpr int kBarVConv = kBarVEmpty + 8 * NST;  // V block rewritten as fp16 (convert mode)
  static constexpr int kBarS = kBarVConv + 8 * NST;    // per tile: S_t(j) (and P_t(j-1) V) done
  static constexpr int kBarP = kBarS + 16;             // per tile: P_t(j) written
  static constexpr int kBarO = kBarP + 16;             // every MMA done
  static constexpr int kBarQFree = kBarO + 8;          // an item's S products done: Q replaceable
  static constexpr int kBarOFull = kBarQFree + 8;      // per tile: an item's last P V done
  static constexpr int kBarOFree = kBarOFull + 16;     // per tile: O read by the epilogue
  static constexpr int kTmemSlot = kBarOFree + 16;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kSched = kAbort + 4;            // unit count and per-warp sums (32 ints)
  static constexpr int kSeqs = (kSched + 128 + 15) & ~15;  // int4 per sequence while ranking
  static constexpr int kList = kSeqs + 16 * kRankMaxSeqs;  // unit of each rank
  static constexpr int kBytes = kList + 4 * kRankMaxUnits;
  static constexpr int kAlloc = kBytes + 1024;
};

// max(a, b, c) in one instruction.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Bounded barrier wait that also gives up as soon as another role of the CTA
// has given up (the shared abort flag); the first to time out records it.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      record_error(kErrWaitTimeout, blockIdx.x);
      return false;
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// Work items and their order.  An item is (sequence s, tile pair p, KV head);
// a unit is (s, p), and item i is unit i / Hk with KV head i % Hk.  The grid
// is persistent (one CTA per SM, G = gridDim.x): CTA b takes the items
//   k G + b  (k even)   and   k G + G - 1 - b  (k odd),   k = 0, 1, ...
// of a list ordered by descending cost, so each CTA gets a mix of long and
// short items.  A unit's cost grows with the keys its last query token sees,
// hist + min(T2 (p + 1), q_len) (hist = context - q_len, T2 = query tokens
// of a tile pair).  For up to kRankMaxSeqs sequences and small unit counts,
// every CTA ranks the units itself: descending key count, ties by sequence
// then pair (a sequence's own pairs all differ in key count); each thread
// counts the units ranked before one unit.  Other batches take the units
// sequence-major, only those that exist (prefill_order_units).
// ---------------------------------------------------------------------------

// floor(x / d) for x >= 0 and d >= 2 from a float reciprocal: below 2^24 both
// are exact floats and the quotient (< 2^23) comes out within 1 of its floor,
// which one correction step fixes.
__device__ __forceinline__ int div_floor(int x, int d, float inv_d) {
  if (x >= (1 << 24)) return x / d;
  int q = __float2int_rz(__int2float_rn(x) * inv_d);
  if (q * d > x) --q;
  else if ((q + 1) * d <= x) ++q;
  return q;
}

// Pairs of a sequence (hist, q_len, pairs) whose key count exceeds K.
__device__ __forceinline__ int pairs_above_of(int hist, int q_len, int pairs, int t2,
                                              float inv_t2, int K) {
  if (q_len <= 0) return 0;
  const int x = K - hist;
  if (x >= q_len) return 0;
  return x < 0 ? pairs : pairs - div_floor(x, t2, inv_t2);  // T2 (p + 1) <= x fall short
}

// The k-th item of CTA b of g, snake order, or -1 past the last.
__device__ __forceinline__ int prefill_item_index(int k, int total, int b, int g) {
  const long long i = static_cast<long long>(k) * g + ((k & 1) ? g - 1 - b : b);
  return i < total ? static_cast<int>(i) : -1;
}

struct PrefillItem {
  int s, kvh, q0, q_len, ctx, tile_a, n_pages, nkb;
  bool has_b;
};

// Tile pairs (units) of sequence s: ceil(q_len / span), or -1 for an invalid
// sequence (outside the query rows, longer than its context, or a context
// past the block table), which has none.
__device__ __forceinline__ int prefill_units_of(const PrefillArgs& a, int s, int span) {
  const int q0 = a.query_starts[s], len = a.query_starts[s + 1] - q0;
  const int ctx = a.context_lens[s];
  if (q0 < 0 || len < 0 || q0 > a.num_tokens - len || len > ctx ||
      ctx > a.max_blocks_per_seq * kPage)
    return -1;
  return len / span + (len % span != 0);
}

// Item i (unit i / Hk, KV head i % Hk); false when it has no work.  The unit
// comes from the ranked list, or, sequence-major, from the per-thread chunk
// sums (`list`, see prefill_order_units).  A tile pair covers `span` query
// tokens, tile A the first half and tile B the second.
__device__ __forceinline__ bool prefill_item(const PrefillArgs& a, const int* list, bool ranked,
                                             int i, int span, PrefillItem& it) {
  const int u = i / a.num_kv_heads;
  it.kvh = i - u * a.num_kv_heads;
  int p;
  if (ranked) {
    const int e = list[u];
    it.s = e & 0xffff;
    p = e >> 16;
  } else {
    // the chunk holding u: the last one whose first unit is <= u; then its
    // sequences one by one
    const int n = static_cast<int>(blockDim.x);
    const int chunk = (a.num_seqs + n - 1) / n;
    int lo = 0, hi = n;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (list[mid] <= u) lo = mid;
      else hi = mid;
    }
    int first = list[lo], s = lo * chunk;
    const int s_end = min(a.num_seqs, s + chunk);
    for (; s < s_end; ++s) {
      const int units = max(0, prefill_units_of(a, s, span));
      if (u < first + units) break;
      first += units;
    }
    if (s >= s_end) return false;   // not reached: u is below the unit count
    it.s = s;
    p = u - first;
  }
  it.q0 = a.query_starts[it.s];
  it.q_len = a.query_starts[it.s + 1] - it.q0;
  it.ctx = a.context_lens[it.s];
  if (it.q0 < 0 || it.q_len < 0 || it.q0 > a.num_tokens - it.q_len || it.q_len > it.ctx ||
      it.ctx > a.max_blocks_per_seq * kPage)
    return false;                   // not reached: an invalid sequence has no units
  it.tile_a = p * span;
  if (it.tile_a >= it.q_len) return false;
  const int half = span / 2;
  const int tile_b = it.tile_a + half;
  it.has_b = tile_b < it.q_len;
  const int last_tok = min((it.has_b ? tile_b : it.tile_a) + half, it.q_len);
  const int lim_max = it.ctx - it.q_len + last_tok;   // keys the pair's last token sees
  it.n_pages = (lim_max + kPage - 1) / kPage;
  it.nkb = (it.n_pages + kPrefillPages - 1) / kPrefillPages;
  return true;
}

// One 128-key block of a tile's online softmax, thread = row (tensor-memory
// lane): S of keys j*128 .. j*128 + 127 (fp32, in p) -> P written over S in
// tensor memory as 16-bit (for PHiLo, bf16 hi + lo in two column halves),
// l and the reference maximum m_ref updated, O_t rescaled in tensor memory
// when m_ref moves.  lim = keys this row sees.
template <bool PHiLo, int D>
__device__ __forceinline__ void prefill_softmax_block(float (&p)[kPrefillKeys], int j, int lim,
                                                      float sl2, float& m_ref, float& l,
                                                      uint32_t t_lane, uint32_t s_col,
                                                      uint32_t o_col) {
  // keys at or past this row's limit are -inf
  const int kbase = j * kPrefillKeys;
  if (kbase + kPrefillKeys > lim) {
#pragma unroll
    for (int c = 0; c < kPrefillKeys; ++c) p[c] = kbase + c < lim ? p[c] : -INFINITY;
  }
  // the block's largest logit in log2 units: for scale > 0 the maximum of
  // the raw S (three-input max), scaled once; otherwise S is scaled first
  float mul = sl2;
  if (!(sl2 > 0.f)) {
#pragma unroll
    for (int c = 0; c < kPrefillKeys; ++c) p[c] = p[c] == -INFINITY ? -INFINITY : p[c] * sl2;
    mul = 1.f;
  }
  float mx8[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) mx8[q] = p[q];
  static_assert((kPrefillKeys - 8) % 16 == 8, "the key loop below leaves 8 keys for the tail");
#pragma unroll
  for (int c = 8; c + 16 <= kPrefillKeys; c += 16) {   // keys 8 .. 119
#pragma unroll
    for (int q = 0; q < 8; ++q) mx8[q] = fmax3(mx8[q], p[c + q], p[c + 8 + q]);
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) mx8[q] = fmaxf(mx8[q], p[kPrefillKeys - 8 + q]);   // 120 .. 127
  const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                         fmaxf(mx8[6], mx8[7])) * mul;
  const float m_new = fmaxf(m_ref, mx);
  const bool need = m_new > m_ref + kRescaleSlack;
  float alpha = 1.f;
  if (need) {
    alpha = ex2(m_ref - m_new);   // 0 when m_ref is still -inf
    m_ref = m_new;
  }
  l *= alpha;
  const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
  const float2 negm = make_float2(-m_use, -m_use), mul2 = make_float2(mul, mul);
#pragma unroll
  for (int c = 0; c < kPrefillKeys; c += 2) {
    const float2 x = ffma2(make_float2(p[c], p[c + 1]), mul2, negm);   // S * scale - m
    p[c] = ex2(x.x);
    p[c + 1] = ex2(x.y);
  }
  // P (and l) over S_t: keys 2i, 2i+1 packed in column i (hi); for bf16 the
  // remainder p - hi in column 64 + i (lo)
  float2 lsum[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) lsum[q] = make_float2(0.f, 0.f);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t h[32], lo[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const float x0 = p[64 * half + 2 * q], x1 = p[64 * half + 2 * q + 1];
      if constexpr (PHiLo) {
        // hi = the top 16 bits of p (p truncated to bf16, remainder below
        // 2^-7 p), lo = the exact fp32 remainder p - hi >= 0 truncated the
        // same way: P keeps at least 14 significant bits (error < 2^-14 p),
        // with no rounding arithmetic and no conversion-unit work
        const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
        h[q] = __byte_perm(b0, b1, 0x7632);
        const float2 r = ffma2(make_float2(__uint_as_float(b0 & 0xffff0000u),
                                           __uint_as_float(b1 & 0xffff0000u)),
                               make_float2(-1.f, -1.f), make_float2(x0, x1));
        lo[q] = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
        lsum[q & 3] = ffma2(make_float2(x0, x1), make_float2(1.f, 1.f), lsum[q & 3]);
      } else {
        // l sums the fp32 p (P.V takes them rounded to fp16: O / l is off
        // by at most 2^-11 relative, summed over keys with random signs)
        h[q] = pack2<false>(x0, x1);
        lsum[q & 3] = ffma2(make_float2(x0, x1), make_float2(1.f, 1.f), lsum[q & 3]);
      }
    }
    tmem_st32u(t_lane + s_col + 32 * half, h);
    if constexpr (PHiLo) tmem_st32u(t_lane + s_col + 64 + 32 * half, lo);
  }
  l += ((lsum[0].x + lsum[0].y) + (lsum[1].x + lsum[1].y)) +
       ((lsum[2].x + lsum[2].y) + (lsum[3].x + lsum[3].y));
  if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(t_lane + o_col + 32 * c, o);
#pragma unroll
      for (int q = 0; q < 32; ++q) o[q] *= alpha;
      tmem_st32(t_lane + o_col + 32 * c, o);
    }
  }
}

// The epilogue of a tile, thread = row: O_t / l from tensor memory as the
// output dtype, for rows below nrows (row r = token t_begin + r / G, head
// kvh * G + r % G of the query rows starting at q0).
template <bool BF16, int D>
__device__ __forceinline__ void prefill_store_rows(const PrefillArgs& a, uint32_t t_lane,
                                                   uint32_t o_col, float l, int row, int nrows,
                                                   int q0, int t_begin, int kvh) {
  const int G = a.group;
  tmem_fence_after_sync();
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint16_t* o_row = a.out + (static_cast<size_t>(q0 + t_begin + row / G) * a.num_heads +
                             kvh * G + row % G) * D;
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    float o[32];
    tmem_ld32(t_lane + o_col + 32 * c, o);
    if (row < nrows) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack2<BF16>(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
        v.y = pack2<BF16>(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
        v.z = pack2<BF16>(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
        v.w = pack2<BF16>(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
        *reinterpret_cast<uint4*>(o_row + 32 * c + 8 * q) = v;
      }
    }
  }
}

// The unit order, the same in every CTA; every thread of the CTA calls it and
// gets the number of units.  t2 = query tokens per unit.  Invalid sequences
// have no units and are reported here (each by one CTA).
//  - Up to kRankMaxSeqs sequences and small unit counts (`ranked`): list[rank]
//    = s | p << 16, longest first.
//  - Otherwise sequence-major: thread t takes a chunk of ceil(S / blockDim)
//    sequences and list[t] = the first unit of its chunk (prefix sums), so
//    only units that exist are walked (prefill_item finds one by a binary
//    search over the chunks and a scan of one chunk).
__device__ __forceinline__ int prefill_order_units(const PrefillArgs& a, int t2, int* sched,
                                                   int4* seqs, int* list, int warp, int lane,
                                                   bool& ranked) {
  const int t = threadIdx.x;
  const bool table = a.num_seqs <= kRankMaxSeqs;
  ranked = false;
  if (table) {
    int hist = 0, ql = -1, np = 0;
    if (t < a.num_seqs) {
      const int q0 = a.query_starts[t], len = a.query_starts[t + 1] - q0;
      const int ctx = a.context_lens[t];
      if (q0 < 0 || len < 0 || q0 > a.num_tokens - len || len > ctx ||
          ctx > a.max_blocks_per_seq * kPage) {
        if (t % gridDim.x == blockIdx.x) record_error(kErrQuery, t);  // one CTA reports it
      } else {
        hist = ctx - len;
        ql = len;
        np = len / t2 + (len % t2 != 0);
      }
    }
    int first = np;  // inclusive scan over the warp's sequences
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, first, d);
      if (lane >= d) first += v;
    }
    if (lane == 31) sched[4 + warp] = first;
    __syncthreads();
    if (t < a.num_seqs) {
      for (int w = 0; w < warp; ++w) first += sched[4 + w];
      seqs[t] = make_int4(hist, ql, np, first - np);
      if (t == a.num_seqs - 1) sched[0] = first;
    }
    __syncthreads();
    const int n_units = sched[0];
    ranked = n_units <= kRankMaxUnits &&
             static_cast<long long>(n_units) * a.num_seqs <= kRankMaxWork;
    if (ranked) {
      const float inv_t2 = 1.f / static_cast<float>(t2);
      for (int u = t; u < n_units; u += blockDim.x) {
        int lo = 0, hi = a.num_seqs;  // the owner: the last sequence whose first unit is <= u
        while (hi - lo > 1) {
          const int mid = (lo + hi) >> 1;
          if (seqs[mid].w <= u) lo = mid;
          else hi = mid;
        }
        const int4 me = seqs[lo];
        const int p = u - me.w;
        const int K = me.x + min(t2 * (p + 1), me.y);
        int rank = 0;
        for (int i = 0; i < a.num_seqs; ++i) {
          const int4 o = seqs[i];
          const int gt = pairs_above_of(o.x, o.y, o.z, t2, inv_t2, K);
          rank += gt;
          if (i < lo) rank += pairs_above_of(o.x, o.y, o.z, t2, inv_t2, K - 1) - gt;
        }
        list[rank] = lo | (p << 16);
      }
      __syncthreads();
      return n_units;
    }
  }
  // sequence-major: this thread's chunk of sequences and its unit count
  const int n = static_cast<int>(blockDim.x);
  const int chunk = (a.num_seqs + n - 1) / n;
  int mine = 0;
  for (int s = t * chunk; s < min(a.num_seqs, (t + 1) * chunk); ++s) {
    const int units = prefill_units_of(a, s, t2);
    if (units < 0) {
      if (!table && s % gridDim.x == blockIdx.x) record_error(kErrQuery, s);  // one CTA reports it
    } else {
      mine += units;
    }
  }
  int first = mine;  // inclusive scan over the warp
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, first, d);
    if (lane >= d) first += v;
  }
  __syncthreads();   // sched and list are reused from the ranked form
  if (lane == 31) sched[4 + warp] = first;
  __syncthreads();
  for (int w = 0; w < warp; ++w) first += sched[4 + w];
  list[t] = first - mine;
  if (t == n - 1) sched[0] = first;
  __syncthreads();
  return sched[0];
}

template <int D, bool BF16>
__global__ void __launch_bounds__(PrefillRoles<BF16>::kThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using L = PrefillSmem<D, BF16>;
  using R = PrefillRoles<BF16>;
  constexpr int NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kWarpTma && lane == 0) {
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  pdl_launch_dependents();
  pdl_wait();

  // ---- the unit order (every CTA derives the same one) ----
  const int G = a.group;
  const int t2 = 2 * a.tile_tokens;
  int* sched = reinterpret_cast<int*>(smem + L::kSched);   // [0] units, [4 + w] per-warp sums
  int4* seqs = reinterpret_cast<int4*>(smem + L::kSeqs);   // hist, q_len, pairs, first unit
  int* list = reinterpret_cast<int*>(smem + L::kList);     // unit of each rank: s | p << 16
  bool ranked;
  const int total = prefill_order_units(a, t2, sched, seqs, list, warp, lane, ranked) *
                    a.num_kv_heads;
  if (prefill_item_index(0, total, blockIdx.x, gridDim.x) < 0) return;   // more CTAs than items
  const int q_rows = a.tile_tokens * G;           // rows a Q box fills

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  if (threadIdx.x == 0) {
    mbar_init(sb + L::kBarQ, 1);
    mbar_init(sb + L::kBarQFree, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(sb + L::kBarKFull + 8 * i, 1);
      mbar_init(sb + L::kBarKEmpty + 8 * i, 1);
      mbar_init(sb + L::kBarVFull + 8 * i, 1);
      mbar_init(sb + L::kBarVEmpty + 8 * i, 1);
      if constexpr (R::kConvert) mbar_init(sb + L::kBarVConv + 8 * i, kConvWarps * 32);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(sb + L::kBarS + 8 * t, 1);
      mbar_init(sb + L::kBarP + 8 * t, 4 * 32);
      mbar_init(sb + L::kBarOFull + 8 * t, 1);
      mbar_init(sb + L::kBarOFree + 8 * t, 4 * 32);
    }
    mbar_init(sb + L::kBarO, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) tmem_alloc(sb + L::kTmemSlot, kTmemCols);
  if (warp < 8 && q_rows < kPrefillRows) {
    // rows no Q box covers are zero (they are masked, but must not be NaN)
    const int t = warp >> 2, chunks = (kPrefillRows - q_rows) * 8;
    for (int i = threadIdx.x & 127; i < chunks * L::kSlabs; i += 128) {
      const int b = i / chunks, c = i % chunks;
      sts128(sb + L::kQ + t * L::kQTile + b * L::kSlab + q_rows * 128 + c * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);
  // the warpgroup index, made visibly warp-uniform for the register split
  const int wgroup = __shfl_sync(0xffffffffu, static_cast<int>(threadIdx.x) / 128, 0);
  if (wgroup >= 2) {
  // warpgroups 2 and 3: MMA issuer, TMA producer, V converters
  if constexpr (R::kConvert) regs_decrease();
  if (warp == kWarpTma) {
    // ================= TMA producer =================
    // Blocks of K and V go through the rings in one running count g over all
    // of the CTA's items; Q is replaced once the previous item's S products
    // are done.
    int n_q = 0, k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = prefill_item_index(k, total, blockIdx.x, gridDim.x);
      if (i < 0) break;
      PrefillItem it;
      if (!prefill_item(a, list, ranked, i, t2, it)) continue;
      if (n_q > 0 && !(ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarQFree,
                                                                  (n_q - 1) & 1, abort_flag))))
        break;
      if (lane == 0) {
        const int tiles = it.has_b ? 2 : 1;
        mbar_arrive_expect_tx(sb + L::kBarQ, tiles * L::kSlabs * q_rows * 128);
        for (int t = 0; t < tiles; ++t) {
#pragma unroll
          for (int b = 0; b < L::kSlabs; ++b)
            tma_load_4d(sb + L::kQ + t * L::kQTile + b * L::kSlab, &qmap, sb + L::kBarQ, 0, b,
                        it.kvh * G, it.q0 + it.tile_a + t * a.tile_tokens);
        }
      }
      ++n_q;
      const int32_t* bt = a.block_tables + static_cast<size_t>(it.s) * a.max_blocks_per_seq;
      for (int j = 0; j < it.nkb; ++j) {
        const int g = k_issued;
        const int st = g % NST;
        const uint32_t par = ((g / NST) & 1) ^ 1;
        int id = -1;
        if (lane < kPrefillPages) {
          const int pg = j * kPrefillPages + lane;
          if (pg < it.n_pages) {
            id = bt[pg];
            if (id < 0 || id >= a.num_blocks) {
              record_error(kErrBlockId, static_cast<long long>(it.s) * a.max_blocks_per_seq + pg);
              id = -1;   // a fully out-of-range box: zeros
            }
          }
        }
        if (g >= NST && !(ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarKEmpty + 8 * st,
                                                                     par, abort_flag))))
          break;
        const uint32_t kst = sb + L::kK + st * L::kStage;
        if (lane == 0) mbar_arrive_expect_tx(sb + L::kBarKFull + 8 * st, L::kStage);
        // lane 0 registers the stage's bytes first; then lane p issues page p's boxes, which
        // measured faster than lane 0 issuing all of them
        __syncwarp();
        if (lane < kPrefillPages) {
#pragma unroll
          for (int b = 0; b < L::kSlabs; ++b)
            tma_load_4d(kst + b * L::kSlab + lane * 2048, &kmap, sb + L::kBarKFull + 8 * st, 0, b,
                        it.kvh, id * kPage);
        }
        k_issued = g + 1;
        if (g >= NST && !(ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarVEmpty + 8 * st,
                                                                     par, abort_flag))))
          break;
        const uint32_t vst = sb + L::kV + st * L::kStage;
        if (lane == 0) mbar_arrive_expect_tx(sb + L::kBarVFull + 8 * st, L::kStage);
        __syncwarp();
        if (lane < kPrefillPages) {
#pragma unroll
          for (int b = 0; b < L::kSlabs; ++b)
            tma_load_4d(vst + b * L::kSlab + lane * 2048, &vmap, sb + L::kBarVFull + 8 * st, 0, b,
                        it.kvh, id * kPage);
        }
        v_issued = g + 1;
      }
    }
    // every load issued lands before the CTA can exit (after an abort some were
    // never consumed); in the normal path these phases have long completed
    if (n_q > 0 && !mbar_wait_bounded(sb + L::kBarQ, (n_q - 1) & 1) && lane == 0)
      record_error(kErrWaitTimeout, blockIdx.x);
    for (int g = max(0, k_issued - NST); g < k_issued; ++g)
      mbar_wait_bounded(sb + L::kBarKFull + 8 * (g % NST), (g / NST) & 1);
    for (int g = max(0, v_issued - NST); g < v_issued; ++g)
      mbar_wait_bounded(sb + L::kBarVFull + 8 * (g % NST), (g / NST) & 1);
  } else if (warp == kWarpMma) {
    // ================= MMA issuer =================
    constexpr uint32_t kIdS = umma_idesc_f16(BF16, kPrefillRows, kPrefillKeys, false);
    constexpr uint32_t kIdO = umma_idesc_f16(R::kPHiLo, kPrefillRows, D, true);
    auto issue_s = [&](int t, int g) {   // S_t = Q_t K_g^T, then report it
      const uint32_t kst = sb + L::kK + (g % NST) * L::kStage;
      const uint32_t qt = sb + L::kQ + t * L::kQTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kSlab + (kk & 3) * 32;
        umma_f16_ss(tmem + kTmemS + 128 * t, umma_desc_sw128(qt + off, 16, 1024),
                    umma_desc_sw128(kst + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
      }
      umma_commit(sb + L::kBarS + 8 * t);
    };
    // O_t (+)= P_t V_g over the pages of block j of an item with n_pages pages
    auto issue_pv = [&](int t, int g, int j, int n_pages) {
      const uint32_t vst = sb + L::kV + (g % NST) * L::kStage;
      const uint32_t pcol = tmem + kTmemS + 128 * t;  // hi in 64 columns, lo in the next 64
      const int pages_here = min(kPrefillPages, n_pages - j * kPrefillPages);
      for (int k = 0; k < pages_here; ++k) {
        const uint64_t bd = umma_desc_sw128(vst + k * 2048, L::kSlab, 1024);
        umma_f16_ts(tmem + kTmemO + 128 * t, pcol + 8 * k, bd, kIdO, (j > 0 || k > 0) ? 1u : 0u);
        if constexpr (R::kPHiLo)
          umma_f16_ts(tmem + kTmemO + 128 * t, pcol + 64 + 8 * k, bd, kIdO, 1u);
      }
    };
    // whole-warp waits; lane 0 issues
    auto wait = [&](uint32_t bar, uint32_t parity) {
      const bool r = __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort_flag));
      tmem_fence_after_sync();
      return r;
    };
    // V of running block g (block j of item `it`) landed; rows past the context cleared
    auto v_ready = [&](int g, int j, const PrefillItem& it) {
      if constexpr (R::kConvert)   // the converters rewrote it (and cleared those rows)
        return wait(sb + L::kBarVConv + 8 * (g % NST), (g / NST) & 1);
      if (!wait(sb + L::kBarVFull + 8 * (g % NST), (g / NST) & 1)) return false;
      const int lp = (it.ctx - 1) / kPage - j * kPrefillPages;
      const int tail_row = it.ctx % kPage;     // first row past the context in the last page
      if (tail_row != 0 && lp >= 0 && lp < kPrefillPages) {
        const uint32_t vst = sb + L::kV + (g % NST) * L::kStage;
        const int chunks = (kPage - tail_row) * 8;
        for (int i = lane; i < chunks * L::kSlabs; i += 32) {
          const int b = i / chunks, c = i % chunks;
          sts128(vst + b * L::kSlab + lp * 2048 + tail_row * 128 + c * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      return true;
    };
    // Per item the issue order is S_A(j), P_B(j-1) V, S_B(j), P_A(j) V, so each
    // tile's softmax overlaps the other tile's MMAs.  Running counts: g0 blocks
    // before this item, done[t] S/P rounds and items[t] items of tile t.
    int n_q = 0, g0 = 0, done[2] = {0, 0}, items[2] = {0, 0};
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = prefill_item_index(k, total, blockIdx.x, gridDim.x);
      if (i < 0) break;
      PrefillItem it;
      if (!prefill_item(a, list, ranked, i, t2, it)) continue;
      const bool hb = it.has_b;
      const int nkb = it.nkb;
      // before the first P_t V of an item: the epilogue has read O_t of the last one
      auto o_free = [&](int t) {
        return items[t] == 0 || wait(sb + L::kBarOFree + 8 * t, (items[t] - 1) & 1);
      };
      if (!(ok = wait(sb + L::kBarQ, n_q & 1))) break;
      ++n_q;
      for (int j = 0; j < nkb; ++j) {
        const int g = g0 + j;
        if (!(ok = wait(sb + L::kBarKFull + 8 * (g % NST), (g / NST) & 1))) break;
        if (lane == 0) issue_s(0, g);                    // after P_A(j-1) V in issue order
        __syncwarp();
        if (j > 0 && hb) {
          if (!(ok = (j > 1 || o_free(1)) && wait(sb + L::kBarP + 8, (done[1] + j - 1) & 1))) break;
          if (lane == 0) issue_pv(1, g - 1, j - 1, it.n_pages);
          __syncwarp();
        }
        if (lane == 0) {
          if (j > 0) umma_commit(sb + L::kBarVEmpty + 8 * ((g - 1) % NST));  // V used by both tiles
          if (hb) issue_s(1, g);
          umma_commit(sb + L::kBarKEmpty + 8 * (g % NST));                  // K used by both tiles
          if (j == nkb - 1) umma_commit(sb + L::kBarQFree);                 // the item's last S
        }
        __syncwarp();
        if (!(ok = (j > 0 || o_free(0)) && v_ready(g, j, it) &&
                   wait(sb + L::kBarP, (done[0] + j) & 1)))
          break;
        if (lane == 0) issue_pv(0, g, j, it.n_pages);
        __syncwarp();
      }
      if (!ok) break;
      const int gl = g0 + nkb - 1;
      if (hb) {
        if (!(ok = (nkb > 1 || o_free(1)) && wait(sb + L::kBarP + 8, (done[1] + nkb - 1) & 1)))
          break;
        if (lane == 0) issue_pv(1, gl, nkb - 1, it.n_pages);
        __syncwarp();
      }
      if (lane == 0) {
        umma_commit(sb + L::kBarVEmpty + 8 * (gl % NST));
        umma_commit(sb + L::kBarOFull);
        if (hb) umma_commit(sb + L::kBarOFull + 8);
      }
      __syncwarp();
      g0 += nkb;
      done[0] += nkb;
      ++items[0];
      if (hb) {
        done[1] += nkb;
        ++items[1];
      }
    }
    // every MMA issued has completed before tensor memory is freed (also
    // after an abort)
    if (lane == 0) umma_commit(sb + L::kBarO);
    __syncwarp();
    if (!mbar_wait_bounded(sb + L::kBarO, 0) && lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
  } else if (R::kConvert && warp >= kWarpConv && warp < kWarpConv + kConvWarps) {
    // ================= V converters (convert mode) =================
    // Each landed V block (bf16, 128 keys x D, two or one 128-byte-swizzled
    // slabs) is rewritten in place as fp16, element for element (the swizzle
    // moves whole 16-byte chunks, so chunk positions are unchanged), and rows
    // past the context in the sequence's last page are cleared.
    const int ct = threadIdx.x - kWarpConv * 32;   // 0 .. kConvWarps * 32 - 1
    int g0 = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int i = prefill_item_index(k, total, blockIdx.x, gridDim.x);
      if (i < 0) break;
      PrefillItem it;
      if (!prefill_item(a, list, ranked, i, t2, it)) continue;
      const int last_page = (it.ctx - 1) / kPage;
      const int tail_row = it.ctx % kPage;
      uint32_t hmax = 0;   // per-half maximum of |fp16| written
      for (int j = 0; j < it.nkb; ++j) {
        const int g = g0 + j, st = g % NST;
        if (!(ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarVFull + 8 * st,
                                                         (g / NST) & 1, abort_flag))))
          break;
        const uint32_t vst = sb + L::kV + st * L::kStage;
        const int lp = last_page - j * kPrefillPages;  // this block's page holding the end, if any
        const bool tail_block = tail_row != 0 && lp >= 0 && lp < kPrefillPages;
        for (int c = ct; c < L::kStage / 16; c += kConvWarps * 32) {
          const int row = (c >> 3) & (kPrefillKeys - 1);   // key within the block
          const uint32_t addr = vst + c * 16;
          uint32_t w[4];
          if (tail_block && (row >> 4) == lp && (row & 15) >= tail_row) {
            w[0] = w[1] = w[2] = w[3] = 0u;
          } else {
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float lo = __uint_as_float(w[q] << 16), hi = __uint_as_float(w[q] & 0xffff0000u);
              uint32_t h;
              asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hi), "f"(lo));
              hmax = __vmaxu2(hmax, h & 0x7fff7fffu);
              w[q] = h;
            }
          }
          sts128(addr, w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(sb + L::kBarVConv + 8 * st);
      }
      // no bf16 value is 65 504, so a half of magnitude 65 504 was clipped
      if (__any_sync(0xffffffffu, __vcmpeq2(hmax, 0x7bff7bffu) != 0) && lane == 0)
        record_error(kErrValue, it.s);
      g0 += it.nkb;
    }
  }
  } else {
  // warpgroups 0 and 1: the softmax of tiles A and B
  if constexpr (R::kConvert) regs_increase();
  // ================= softmax: tile t = warp / 4, row = TMEM lane =================
  const int t = warp >> 2;
  const int row = threadIdx.x & 127;
  const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t s_col = kTmemS + 128 * t, o_col = kTmemO + 128 * t;
  const float sl2 = a.scale_log2;
  int done = 0, items = 0;   // S/P rounds and items of this tile so far
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int i = prefill_item_index(k, total, blockIdx.x, gridDim.x);
    if (i < 0) break;
    PrefillItem it;
    if (!prefill_item(a, list, ranked, i, t2, it)) continue;
    if (t == 1 && !it.has_b) continue;
    const int t_begin = it.tile_a + t * a.tile_tokens;
    const int nrows = (min(t_begin + a.tile_tokens, it.q_len) - t_begin) * G;
    const int lim = row < nrows ? it.ctx - it.q_len + t_begin + row / G + 1 : 0;
    float m_ref = -INFINITY, l = 0.f;
    for (int j = 0; j < it.nkb; ++j) {
      // S_t(j) is in, and with it every earlier P_t V: O_t is current
      ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarS + 8 * t, (done + j) & 1,
                                                 abort_flag));
      if (!ok) break;
      tmem_fence_after_sync();
      float p[kPrefillKeys];
      if constexpr (R::kConvert) tmem_ld128_x32(t_lane + s_col, p);
      else tmem_ld128(t_lane + s_col, p);
      prefill_softmax_block<R::kPHiLo, D>(p, j, lim, sl2, m_ref, l, t_lane, s_col, o_col);
      tmem_fence_before_sync();
      mbar_arrive(sb + L::kBarP + 8 * t);
    }
    if (!ok) break;
    done += it.nkb;
    // the item's last P_t V is done: O_t is final
    ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarOFull + 8 * t, items & 1, abort_flag));
    if (!ok) break;
    prefill_store_rows<BF16, D>(a, t_lane, o_col, l, row, nrows, it.q0, t_begin, it.kvh);
    tmem_fence_before_sync();
    mbar_arrive(sb + L::kBarOFree + 8 * t);   // O_t may be overwritten
    ++items;
  }
  }

  tmem_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tmem_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pa

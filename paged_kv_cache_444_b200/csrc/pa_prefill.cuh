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
// loads Q once and the K and V pages with TMA through rings of NST stages.
//
// The causal mask is a per-row key limit (pos + 1) applied to S; blocks past
// the pair's last key are never loaded, and V rows past the context are
// zeroed before use (never written, they may hold anything).  O is rescaled
// only when a row's running maximum grows by more than 2^8 (the reference
// maximum may lag the true one by that much: P <= 2^8 stays exact in the
// 16-bit operand and the final 1/l uses the same reference).  bf16 P enters
// P V as a hi + lo pair of bf16 products (at least 14 bits of P, split by
// bit truncation so the conversion unit stays free for 2^x); fp16 P is
// rounded once and l sums the rounded values.  With bf16 caches the default
// build rewrites each V block as fp16 in shared memory (four converter warps)
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
constexpr int kWarpConv = 10;                       // V converters: warps 10-13 (convert mode)
constexpr unsigned kErrValue = 8;

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
  // softmax 0-7, then MMA, TMA, converters 10-13 and two idle warps
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
  int pairs_per_seq;            // ceil(ceil(max_query_len / tile_tokens) / 2)
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
  static constexpr int kTmemSlot = kBarO + 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
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
// Longest-first item order.  A unit is (sequence, tile pair); its cost grows
// with the keys its last query token sees, hist + min(T2 (p + 1), q_len)
// (hist = context - q_len, T2 = query tokens of a tile pair).  CTAs start in
// grid order, so handing out units by descending key count (ties by
// sequence, then pair) starts the long ones first and fills the tail with
// short ones; the K/V a sequence's pairs share is read again from L2.
// ---------------------------------------------------------------------------
constexpr int kLptSeqsPerLane = 8;  // one warp ranks up to 256 sequences

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

// One sequence as the ranking sees it: hist = context - q_len, its tile
// pairs, and q_len (-1 marks an invalid sequence, which has no units).
struct LptSeq {
  int hist[kLptSeqsPerLane], q_len[kLptSeqsPerLane], pairs[kLptSeqsPerLane];
};

// Pairs of sequence i whose key count exceeds K.
__device__ __forceinline__ int pairs_above(const LptSeq& q, int i, int t2, float inv_t2, int K) {
  if (q.q_len[i] <= 0) return 0;
  const int x = K - q.hist[i];
  if (x >= q.q_len[i]) return 0;
  return x < 0 ? q.pairs[i] : q.pairs[i] - div_floor(x, t2, inv_t2);  // T2 (p + 1) <= x fall short
}

// The unit of rank j (0 = most keys), found by one warp: a binary search for
// its key count K (the least K with at most j units above it), then its place
// among the units with exactly K keys in (sequence, pair) order.  Returns
// false when fewer than j + 1 units exist.
__device__ __forceinline__ bool prefill_unit_of_rank(const LptSeq& q, int max_keys, int t2, int j,
                                                     int lane, int& s_out, int& p_out) {
  const float inv_t2 = 1.f / static_cast<float>(t2);
  auto above = [&](int K) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < kLptSeqsPerLane; ++i) c += pairs_above(q, i, t2, inv_t2, K);
    return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
  };
  if (above(-1) <= j) return false;
  int lo = -1, hi = max_keys;  // above(lo) > j >= above(hi) = 0
  while (hi - lo > 1) {
    const int mid = lo + (hi - lo) / 2;
    if (above(mid) <= j) hi = mid;
    else lo = mid;
  }
  const int K = hi;
  int t = j - above(K);  // index among the units with exactly K keys
  bool found = false;
#pragma unroll
  for (int i = 0; i < kLptSeqsPerLane; ++i) {
    const int below = pairs_above(q, i, t2, inv_t2, K - 1);
    const int e = below - pairs_above(q, i, t2, inv_t2, K);
    int inc = e;  // inclusive scan over the lanes (sequences i*32 + lane)
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += v;
    }
    const int total = __shfl_sync(0xffffffffu, inc, 31);
    if (!found && t < total) {
      const int src = __ffs(__ballot_sync(0xffffffffu, t < inc)) - 1;
      const int before = __shfl_sync(0xffffffffu, inc - e, src);
      // the pairs with exactly K keys follow the pairs - below with fewer
      const int first = __shfl_sync(0xffffffffu, q.pairs[i] - below, src);
      s_out = i * 32 + src;
      p_out = first + (t - before);
      found = true;
    }
    if (!found) t -= total;
  }
  return found;
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

  // ---- work item ----
  const int cap = a.max_blocks_per_seq * kPage;
  auto seq_valid = [&](int q0, int q_len, int ctx) {
    return !(q0 < 0 || q_len < 0 || q0 > a.num_tokens - q_len || q_len > ctx || ctx > cap);
  };
  const int G = a.group;
  int s, pair, kvh;
  if (a.num_seqs <= 32 * kLptSeqsPerLane) {
    // longest first: CTA b takes unit b / Hk, KV head b % Hk
    int* slot = reinterpret_cast<int*>(smem);  // stage area, not in use yet
    if (warp == 0) {
      LptSeq q;
      int max_keys = 0;
      const int t2 = 2 * a.tile_tokens;
#pragma unroll
      for (int i = 0; i < kLptSeqsPerLane; ++i) {
        const int t = i * 32 + lane;
        q.hist[i] = 0;
        q.q_len[i] = -1;
        q.pairs[i] = 0;
        if (t < a.num_seqs) {
          const int q0 = a.query_starts[t], ql = a.query_starts[t + 1] - q0;
          const int ctx = a.context_lens[t];
          if (seq_valid(q0, ql, ctx)) {
            q.hist[i] = ctx - ql;
            q.q_len[i] = ql;
            q.pairs[i] = ql / t2 + (ql % t2 != 0);
            max_keys = max(max_keys, ctx);
          } else if (t == static_cast<int>(blockIdx.x)) {
            record_error(kErrQuery, t);  // each sequence is checked by one CTA
          }
        }
      }
      max_keys = static_cast<int>(__reduce_max_sync(0xffffffffu, static_cast<unsigned>(max_keys)));
      int us = -1, up = 0;
      const bool found = prefill_unit_of_rank(
          q, max_keys, t2, static_cast<int>(blockIdx.x) / a.num_kv_heads, lane, us, up);
      if (lane == 0) {
        slot[0] = found ? us : -1;
        slot[1] = up;
      }
    }
    __syncthreads();
    s = slot[0];
    pair = slot[1];
    kvh = static_cast<int>(blockIdx.x) % a.num_kv_heads;
    fence_proxy_async_smem();  // generic writes to the stage area before TMA writes to it
    __syncthreads();  // the stage area is about to be reused
    if (s < 0) return;  // more CTAs than units: nothing to do
  } else {
    // the last tile pairs of every sequence (most keys) first
    const int per_pair = a.num_seqs * a.num_kv_heads;
    int item = blockIdx.x;
    pair = a.pairs_per_seq - 1 - item / per_pair;
    item %= per_pair;
    kvh = item % a.num_kv_heads;
    s = item / a.num_kv_heads;
  }

  const int q0 = a.query_starts[s];
  const int q_len = a.query_starts[s + 1] - q0;
  const int ctx = a.context_lens[s];
  if (!seq_valid(q0, q_len, ctx)) {
    if (threadIdx.x == 0 && kvh == 0 && pair == 0) record_error(kErrQuery, s);
    return;
  }
  const int tile_a = 2 * pair * a.tile_tokens, tile_b = tile_a + a.tile_tokens;
  if (tile_a >= q_len) return;
  const bool has_b = tile_b < q_len;
  const int last_tok = min((has_b ? tile_b : tile_a) + a.tile_tokens, q_len);  // exclusive
  const int lim_max = ctx - q_len + last_tok;      // keys the pair's last token sees
  const int n_pages = (lim_max + kPage - 1) / kPage;
  const int nkb = (n_pages + kPrefillPages - 1) / kPrefillPages;
  const int q_rows = a.tile_tokens * G;           // rows a Q box fills

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  if (threadIdx.x == 0) {
    mbar_init(sb + L::kBarQ, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(sb + L::kBarKFull + 8 * i, 1);
      mbar_init(sb + L::kBarKEmpty + 8 * i, 1);
      mbar_init(sb + L::kBarVFull + 8 * i, 1);
      mbar_init(sb + L::kBarVEmpty + 8 * i, 1);
      if constexpr (R::kConvert) mbar_init(sb + L::kBarVConv + 8 * i, 128);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(sb + L::kBarS + 8 * t, 1);
      mbar_init(sb + L::kBarP + 8 * t, 4 * 32);
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
  // warpgroups 2 and 3: MMA issuer, TMA producer, V converters, idle warps
  if constexpr (R::kConvert) regs_decrease();
  if (warp == kWarpTma) {
    // ================= TMA producer =================
    if (lane == 0) {
      const int tiles = has_b ? 2 : 1;
      mbar_arrive_expect_tx(sb + L::kBarQ, tiles * L::kSlabs * q_rows * 128);
      for (int t = 0; t < tiles; ++t) {
#pragma unroll
        for (int b = 0; b < L::kSlabs; ++b)
          tma_load_4d(sb + L::kQ + t * L::kQTile + b * L::kSlab, &qmap, sb + L::kBarQ, 0, b,
                      kvh * G, q0 + (t == 0 ? tile_a : tile_b));
      }
    }
    const int32_t* bt = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq;
    int k_issued = 0, v_issued = 0;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      const int st = j % NST;
      const uint32_t par = ((j / NST) & 1) ^ 1;
      int id = -1;
      if (lane < kPrefillPages) {
        const int pg = j * kPrefillPages + lane;
        if (pg < n_pages) {
          id = bt[pg];
          if (id < 0 || id >= a.num_blocks) {
            record_error(kErrBlockId, static_cast<long long>(s) * a.max_blocks_per_seq + pg);
            id = -1;   // a fully out-of-range box: zeros
          }
        }
      }
      if (j >= NST) ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarKEmpty + 8 * st, par,
                                                               abort_flag));
      if (!ok) break;
      const uint32_t kst = sb + L::kK + st * L::kStage;
      if (lane == 0) mbar_arrive_expect_tx(sb + L::kBarKFull + 8 * st, L::kStage);
#pragma unroll
      for (int p = 0; p < kPrefillPages; ++p) {
        const int idp = __shfl_sync(0xffffffffu, id, p);
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < L::kSlabs; ++b)
            tma_load_4d(kst + b * L::kSlab + p * 2048, &kmap, sb + L::kBarKFull + 8 * st, 0, b,
                        kvh, idp * kPage);
        }
      }
      k_issued = j + 1;
      if (j >= NST) ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarVEmpty + 8 * st, par,
                                                               abort_flag));
      if (!ok) break;
      const uint32_t vst = sb + L::kV + st * L::kStage;
      if (lane == 0) mbar_arrive_expect_tx(sb + L::kBarVFull + 8 * st, L::kStage);
#pragma unroll
      for (int p = 0; p < kPrefillPages; ++p) {
        const int idp = __shfl_sync(0xffffffffu, id, p);
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < L::kSlabs; ++b)
            tma_load_4d(vst + b * L::kSlab + p * 2048, &vmap, sb + L::kBarVFull + 8 * st, 0, b,
                        kvh, idp * kPage);
        }
      }
      v_issued = j + 1;
    }
    // every load issued lands before the CTA can exit (after an abort some were
    // never consumed); in the normal path these phases have long completed
    if (!mbar_wait_bounded(sb + L::kBarQ, 0) && lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
    for (int j = max(0, k_issued - NST); j < k_issued; ++j)
      mbar_wait_bounded(sb + L::kBarKFull + 8 * (j % NST), (j / NST) & 1);
    for (int j = max(0, v_issued - NST); j < v_issued; ++j)
      mbar_wait_bounded(sb + L::kBarVFull + 8 * (j % NST), (j / NST) & 1);
  } else if (warp == kWarpMma) {
    // ================= MMA issuer =================
    constexpr uint32_t kIdS = umma_idesc_f16(BF16, kPrefillRows, kPrefillKeys, false);
    constexpr uint32_t kIdO = umma_idesc_f16(R::kPHiLo, kPrefillRows, D, true);
    auto issue_s = [&](int t, int j) {   // S_t(j) = Q_t K_j^T, then report it
      const uint32_t kst = sb + L::kK + (j % NST) * L::kStage;
      const uint32_t qt = sb + L::kQ + t * L::kQTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kSlab + (kk & 3) * 32;
        umma_f16_ss(tmem + kTmemS + 128 * t, umma_desc_sw128(qt + off, 16, 1024),
                    umma_desc_sw128(kst + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
      }
      umma_commit(sb + L::kBarS + 8 * t);
    };
    auto issue_pv = [&](int t, int j) {  // O_t += P_t(j) V_j over the block's pages
      const uint32_t vst = sb + L::kV + (j % NST) * L::kStage;
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
    const int last_page = (ctx - 1) / kPage;
    const int tail_row = ctx % kPage;          // first row past the context in the last page
    auto v_ready = [&](int j) {                // V_j landed; clear its rows past the context
      if constexpr (R::kConvert)   // the converters rewrote it (and cleared those rows)
        return wait(sb + L::kBarVConv + 8 * (j % NST), (j / NST) & 1);
      if (!wait(sb + L::kBarVFull + 8 * (j % NST), (j / NST) & 1)) return false;
      const int lp = last_page - j * kPrefillPages;
      if (tail_row != 0 && lp >= 0 && lp < kPrefillPages) {
        const uint32_t vst = sb + L::kV + (j % NST) * L::kStage;
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
    bool ok = wait(sb + L::kBarQ, 0) && wait(sb + L::kBarKFull, 0);
    if (ok) {
      if (lane == 0) {
        issue_s(0, 0);
        if (has_b) issue_s(1, 0);
        umma_commit(sb + L::kBarKEmpty);
      }
      __syncwarp();
      ok = v_ready(0) && wait(sb + L::kBarP, 0);
      if (ok && lane == 0) issue_pv(0, 0);
      __syncwarp();
    }
    for (int j = 1; ok && j < nkb; ++j) {
      const int st = j % NST;
      if (!(ok = wait(sb + L::kBarKFull + 8 * st, (j / NST) & 1))) break;
      if (lane == 0) issue_s(0, j);                      // after P_A(j-1) V in issue order
      __syncwarp();
      if (has_b) {
        if (!(ok = wait(sb + L::kBarP + 8, (j - 1) & 1))) break;
        if (lane == 0) issue_pv(1, j - 1);
        __syncwarp();
      }
      if (lane == 0) {
        umma_commit(sb + L::kBarVEmpty + 8 * ((j - 1) % NST));   // V_{j-1} used by both tiles
        if (has_b) issue_s(1, j);
        umma_commit(sb + L::kBarKEmpty + 8 * st);                 // K_j used by both tiles
      }
      __syncwarp();
      if (!(ok = v_ready(j) && wait(sb + L::kBarP, j & 1))) break;
      if (lane == 0) issue_pv(0, j);
      __syncwarp();
    }
    if (ok && has_b) {
      ok = wait(sb + L::kBarP + 8, (nkb - 1) & 1);
      if (ok && lane == 0) issue_pv(1, nkb - 1);
      __syncwarp();
    }
    // every MMA issued has completed before the epilogue reads O and before
    // tensor memory is freed (also after an abort)
    if (lane == 0) umma_commit(sb + L::kBarO);
    __syncwarp();
    if (!mbar_wait_bounded(sb + L::kBarO, 0) && lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
  } else if (R::kConvert && warp >= kWarpConv && warp < kWarpConv + 4) {
    // ================= V converters (convert mode) =================
    // Each landed V block (bf16, 128 keys x D, two or one 128-byte-swizzled
    // slabs) is rewritten in place as fp16, element for element (the swizzle
    // moves whole 16-byte chunks, so chunk positions are unchanged), and rows
    // past the context in the sequence's last page are cleared.
    const int ct = threadIdx.x - kWarpConv * 32;   // 0 .. 127
    const int last_page = (ctx - 1) / kPage;
    const int tail_row = ctx % kPage;
    uint32_t clipped = 0;
    for (int j = 0; j < nkb; ++j) {
      const int st = j % NST;
      if (!__all_sync(0xffffffffu, wait_or_abort(sb + L::kBarVFull + 8 * st, (j / NST) & 1,
                                                 abort_flag)))
        break;
      const uint32_t vst = sb + L::kV + st * L::kStage;
      const int lp = last_page - j * kPrefillPages;  // this block's page holding the end, if any
      for (int c = ct; c < L::kStage / 16; c += 128) {
        const int row = (c >> 3) & (kPrefillKeys - 1);   // key within the block
        const uint32_t addr = vst + c * 16;
        uint32_t w[4];
        if (tail_row != 0 && (row >> 4) == lp && (row & 15) >= tail_row) {
          w[0] = w[1] = w[2] = w[3] = 0u;
        } else {
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float lo = __uint_as_float(w[i] << 16), hi = __uint_as_float(w[i] & 0xffff0000u);
            uint32_t h;
            asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(h) : "f"(hi), "f"(lo));
            // no bf16 value is 65 504, so a half of magnitude 65 504 was clipped
            clipped |= __vcmpeq2(h & 0x7fff7fffu, 0x7bff7bffu);
            w[i] = h;
          }
        }
        sts128(addr, w[0], w[1], w[2], w[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(sb + L::kBarVConv + 8 * st);
    }
    if (__any_sync(0xffffffffu, clipped != 0) && lane == 0) record_error(kErrValue, s);
  }
  } else {
  // warpgroups 0 and 1: the softmax of tiles A and B
  if constexpr (R::kConvert) regs_increase();
  if (warp < 4 || has_b) {
    // ================= softmax: tile t = warp / 4, row = TMEM lane =================
    const int t = warp >> 2;
    const int row = threadIdx.x & 127;
    const int t_begin = t == 0 ? tile_a : tile_b;
    const int nrows = (min(t_begin + a.tile_tokens, q_len) - t_begin) * G;
    const int lim = row < nrows ? ctx - q_len + t_begin + row / G + 1 : 0;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = kTmemS + 128 * t, o_col = kTmemO + 128 * t;
    const float sl2 = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      // S_t(j) is in, and with it every earlier P_t V: O_t is current
      ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarS + 8 * t, j & 1, abort_flag));
      if (!ok) break;
      tmem_fence_after_sync();
      float p[kPrefillKeys];
      if constexpr (R::kConvert) tmem_ld128_x32(t_lane + s_col, p);
      else tmem_ld128(t_lane + s_col, p);
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
      for (int i = 0; i < 8; ++i) mx8[i] = p[i];
      static_assert((kPrefillKeys - 8) % 16 == 8, "the key loop below leaves 8 keys for the tail");
#pragma unroll
      for (int c = 8; c + 16 <= kPrefillKeys; c += 16) {   // keys 8 .. 119
#pragma unroll
        for (int i = 0; i < 8; ++i) mx8[i] = fmax3(mx8[i], p[c + i], p[c + 8 + i]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = fmaxf(mx8[i], p[kPrefillKeys - 8 + i]);   // 120 .. 127
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
      for (int i = 0; i < 4; ++i) lsum[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h[32], lo[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = p[64 * half + 2 * i], x1 = p[64 * half + 2 * i + 1];
          if constexpr (R::kPHiLo) {
            // hi = the top 16 bits of p (p truncated to bf16, remainder below
            // 2^-7 p), lo = the exact fp32 remainder p - hi >= 0 truncated the
            // same way: P keeps at least 14 significant bits (error < 2^-14 p),
            // with no rounding arithmetic and no conversion-unit work
            const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
            h[i] = __byte_perm(b0, b1, 0x7632);
            const float2 r = ffma2(make_float2(__uint_as_float(b0 & 0xffff0000u),
                                               __uint_as_float(b1 & 0xffff0000u)),
                                   make_float2(-1.f, -1.f), make_float2(x0, x1));
            lo[i] = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x7632);
            lsum[i & 3] = ffma2(make_float2(x0, x1), make_float2(1.f, 1.f), lsum[i & 3]);
          } else {
            h[i] = pack2<false>(x0, x1);
            lsum[i & 3] = ffma2(unpack2<false>(h[i]), make_float2(1.f, 1.f), lsum[i & 3]);
          }
        }
        tmem_st32u(t_lane + s_col + 32 * half, h);
        if constexpr (R::kPHiLo) tmem_st32u(t_lane + s_col + 64 + 32 * half, lo);
      }
      l += ((lsum[0].x + lsum[0].y) + (lsum[1].x + lsum[1].y)) +
           ((lsum[2].x + lsum[2].y) + (lsum[3].x + lsum[3].y));
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float o[32];
          tmem_ld32(t_lane + o_col + 32 * c, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= alpha;
          tmem_st32(t_lane + o_col + 32 * c, o);
        }
      }
      tmem_fence_before_sync();
      mbar_arrive(sb + L::kBarP + 8 * t);
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarO, 0, abort_flag));
    if (ok) {
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

// pa_decode.cuh -- paged decode attention on sm_100a.
//
// What it computes ("vLLM PagedAttention 原理与源码深度解析" §5.3; "vllm源码分析"
// §第三讲): for one query token per sequence, out = softmax(scale * q K^T) V
// over the sequence's first context_lens[s] tokens, whose K/V rows live in
// 16-token physical blocks named by the sequence's block table ("vllm源码剖析"
// §一.2: cache [num_blocks, block_size, num_kv_heads, head_dim]).
//
// Work decomposition.  One CTA owns one (sequence, KV head, partition) item:
// the whole sequence for pa_decode, `partition_size` tokens for
// pa_decode_split.  The CTA's four warps take the item's pages round-robin;
// each warp streams its pages through its own ring of NST shared-memory
// stages, keeps its own online-softmax state, and the four states are merged
// through shared memory at the end (the log-sum-exp identity, exact up to
// rounding).  No warp ever waits for another until that merge.
//
// Gather.  A page of one KV head is 16 rows of head_dim 16-bit values,
// num_kv_heads*head_dim elements apart.  One TMA tensor-tile load moves a
// 16 x 64-element box (2 KB) of it into shared memory, 128-byte swizzled so
// that the 8-row ldmatrix reads of the page step are bank-conflict free.  Lane 0 of the warp
// issues the loads for a page NST pages ahead, right after the page that last
// used the stage has been consumed.  The block id of every page comes from a
// window of 32 ids held one per lane (a second window is prefetched).
//
// Math.  fp32 throughout.  The G query heads of a KV head (1 for MHA, up to
// 16 for GQA) form a small dense contraction on mma.sync m16n8k16 with fp32
// accumulators (P in the cache dtype for the second product, bf16 as a hi +
// lo pair).  Groups of up to 8 heads run both products transposed (MmaWarpT:
// S^T = K Q^T, O^T = V^T P^T, tokens and head dims as the mma's 16 rows, the
// heads as its 8 columns); groups of 9 to 16 run a 16-row query tile
// (MmaWarp), which the shared-prefix kernel also uses.  Even for one head the
// tensor cores take the products off the issue path, which measured faster
// than packed fp32 FMA on the CUDA cores.  The softmax is online, in base 2
// with scale*log2(e) folded into the logits, with warp-shuffle max reductions;
// in the transposed steps the reference max may trail the true one by 2^8, so
// O is rescaled only when a row outgrows that, and the partials are restated
// against the true max at the end.
#pragma once

#include "pa_device.cuh"

namespace pa {

constexpr int kPage = 16;       // tokens per physical block (block_size)
constexpr int kWarps = 4;       // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kBoxBytes = kPage * 128;  // one 16 x 64-element TMA box
constexpr int kMaxCluster = 8;          // CTAs per item at most (portable cluster size)
constexpr int kLptMaxSeqs = 256;        // longest-first ordering for batches up to this size

struct DecodeArgs {
  const uint16_t* query;      // [S, H, D]
  uint16_t* out;              // [S, H, D]            (single-pass mode)
  float* tmp_out;             // [S, H, P, D]         (split mode, else null)
  float* max_logits;          // [S, H, P]
  float* exp_sums;            // [S, H, P]
  const int32_t* block_tables;  // [S, MB]
  const int32_t* context_lens;  // [S]
  float scale_log2;           // scale * log2(e) (* k_scale for an fp8 cache)
  float v_scale;              // multiplies every output (1, or v_scale for an fp8 cache)
  int num_heads;
  int num_kv_heads;
  int group;                  // num_heads / num_kv_heads
  int max_blocks_per_seq;
  int num_blocks;
  int partition_size;         // tokens per item in split mode (multiple of 16)
  int parts_per_head;         // grid items per (seq, kv head): max_partitions or 1
  int max_partitions;
  int cluster_pages;          // an item with more pages than this is spread over its cluster
  int num_seqs;
  int longest_first;          // order single-pass items by descending context length
  int persistent;             // split mode: CTAs loop over a dense list of the items that exist
};


template <int D, int NST, int EB = 2>   // EB: bytes per cache element (2, or 1 for fp8)
struct DecodeSmem {
  static constexpr int kPageBytes = kPage * D * EB;      // one tensor, one page, one head
  static constexpr int kBoxesPerRow = D * EB / 128;       // 128-byte TMA boxes per row
  static constexpr int kStageBytes = 2 * kPageBytes;      // K page + V page
  static constexpr int kStagesBytes = kWarps * NST * kStageBytes;
  static constexpr int kBarOffset = kStagesBytes;
  static constexpr int kRedMOffset = kBarOffset + kWarps * NST * 8;
  static constexpr int kRedLOffset = kRedMOffset + kWarps * 16 * 4;
  static constexpr int kPartMOffset = kRedLOffset + kWarps * 16 * 4;
  static constexpr int kPartLOffset = kPartMOffset + 16 * 4;
  // persistent split mode (outside the stage area: kept across items): up to
  // kLptMaxSeqs sequences, every context and the partitions before each
  // sequence; beyond, the partitions before each thread's chunk of
  // sequences and per-warp sums
  static constexpr int kSeqOffset = kPartLOffset + 16 * 4;
  static constexpr int kSeqBytes = (2 * kLptMaxSeqs + 1) * 4 > (kThreads + 1 + kWarps) * 4
                                       ? (2 * kLptMaxSeqs + 1) * 4
                                       : (kThreads + 1 + kWarps) * 4;
  static constexpr int kBytes = kSeqOffset + kSeqBytes;
  static constexpr int kAlloc = kBytes + 1024;            // + alignment slack
  // the merge buffers reuse the stage area: per-warp rows (kWarps x group x D
  // floats) and, for an item spread over a cluster, this CTA's merged rows
  static constexpr int kPartAccOffset = kWarps * 16 * D * 4;
  static_assert(kPartAccOffset + 16 * D * 4 <= kStagesBytes, "merge buffers must fit in the stages");
  static_assert((D * EB) % 128 == 0, "a cache row must be a whole number of 128-byte boxes");
};

// Address of 16-byte chunk `c` (0 .. D/8-1) of row `r` in a swizzled page.
template <int D>
__device__ __forceinline__ uint32_t page_chunk(uint32_t base, int r, int c) {
  return base + (c >> 3) * kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

// ---------------------------------------------------------------------------
// Per-warp state and page step with a 16-row query tile (groups of 9 to 16,
// and the shared-prefix kernel's member rows)
// ---------------------------------------------------------------------------
template <int D, bool BF16>
struct MmaWarp {
  static constexpr int KSTEPS = D / 16;  // k-steps of 16 over head_dim
  static constexpr int NTILES = D / 8;   // 8-wide n-tiles of the output
  static constexpr int kMinBlocks = 0;   // single pass: no register cap
  uint32_t qa[KSTEPS][4];                // Q as mma A fragments (rows = query heads of the group)
  float acc[NTILES][4];                  // O fragments (rows r0 / r1)
  float m[2], l[2];                      // running max (log2 domain) and lane-partial sums

  __device__ __forceinline__ void init(const uint16_t* q_group, int group, int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8, tig = lane & 3;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int klo = kk * 16 + tig * 2, khi = klo + 8;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q_group + r0 * D);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q_group + r1 * D);
      qa[kk][0] = r0 < group ? q0[klo >> 1] : 0u;
      qa[kk][1] = r1 < group ? q1[klo >> 1] : 0u;
      qa[kk][2] = r0 < group ? q0[khi >> 1] : 0u;
      qa[kk][3] = r1 < group ? q1[khi >> 1] : 0u;
    }
#pragma unroll
    for (int n = 0; n < NTILES; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  __device__ __forceinline__ void page(uint32_t kbase, uint32_t vbase, int tok0, int t_end,
                                       float scale_log2, int lane) {
    page_rows(kbase, vbase, tok0, t_end, t_end, scale_log2, lane);
  }

  // One page with a token limit per row: row r0 (lane/4) sees tokens < lim0,
  // row r1 (lane/4 + 8) tokens < lim1.  A row whose tokens are all masked so
  // far keeps m = -inf, l = 0, O = 0 (exp of -inf against a zero reference).
  __device__ __forceinline__ void page_rows(uint32_t kbase, uint32_t vbase, int tok0, int lim0,
                                            int lim1, float scale_log2, int lane) {
    const int tig = lane & 3;
    // ---- S = Q K^T for the page's 16 tokens (two 8-token n-tiles) ----
    float sc[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[0][i] = sc[1][i] = 0.f;
    const int ktok = ((lane >> 4) << 3) + (lane & 7);
    const int kchk = (lane >> 3) & 1;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(page_chunk<D>(kbase, ktok, kk * 2 + kchk), b0, b1, b2, b3);
      mma_16816<BF16>(sc[0], qa[kk], b0, b1);
      mma_16816<BF16>(sc[1], qa[kk], b2, b3);
    }
    // ---- scale, mask the tail, row max over the page ----
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tok0 + nt * 8 + tig * 2 + (i & 1);
        const float x = t < (i < 2 ? lim0 : lim1) ? sc[nt][i] * scale_log2 : -INFINITY;
        sc[nt][i] = x;
        if (i < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    // reference max: the running max, or 0 while a row has seen no token
    // (then every exponent below is of -inf and gives 0, never NaN)
    const float mn0r = fmaxf(m[0], mx0), mn1r = fmaxf(m[1], mx1);
    const float mn0 = mn0r == -INFINITY ? 0.f : mn0r;
    const float mn1 = mn1r == -INFINITY ? 0.f : mn1r;
    const float al0 = ex2(m[0] - mn0), al1 = ex2(m[1] - mn1);
    m[0] = mn0r;
    m[1] = mn1r;
    // ---- P = 2^(x - m) as the A operand of P V.  bf16 keeps 8 mantissa
    // bits, so P goes in as a hi + lo pair of bf16 (about 16 bits, two mma
    // per tile) and l sums the unrounded fp32 p; fp16 (11 bits) goes in once
    // and l sums the rounded values, so that O / l stays a convex combination.
    float p0[4], p1[4];
    p0[0] = ex2(sc[0][0] - mn0); p0[1] = ex2(sc[0][1] - mn0);
    p0[2] = ex2(sc[1][0] - mn0); p0[3] = ex2(sc[1][1] - mn0);
    p1[0] = ex2(sc[0][2] - mn1); p1[1] = ex2(sc[0][3] - mn1);
    p1[2] = ex2(sc[1][2] - mn1); p1[3] = ex2(sc[1][3] - mn1);
    uint32_t pa[4], pl[4];
    pa[0] = pack2<BF16>(p0[0], p0[1]);
    pa[2] = pack2<BF16>(p0[2], p0[3]);
    pa[1] = pack2<BF16>(p1[0], p1[1]);
    pa[3] = pack2<BF16>(p1[2], p1[3]);
    if constexpr (BF16) {
      const float2 h0 = unpack2<BF16>(pa[0]), h2 = unpack2<BF16>(pa[2]);
      const float2 h1 = unpack2<BF16>(pa[1]), h3 = unpack2<BF16>(pa[3]);
      pl[0] = pack2<BF16>(p0[0] - h0.x, p0[1] - h0.y);
      pl[2] = pack2<BF16>(p0[2] - h2.x, p0[3] - h2.y);
      pl[1] = pack2<BF16>(p1[0] - h1.x, p1[1] - h1.y);
      pl[3] = pack2<BF16>(p1[2] - h3.x, p1[3] - h3.y);
      l[0] = l[0] * al0 + ((p0[0] + p0[1]) + (p0[2] + p0[3]));
      l[1] = l[1] * al1 + ((p1[0] + p1[1]) + (p1[2] + p1[3]));
    } else {
      const float2 u = unpack2<BF16>(pa[0]), v = unpack2<BF16>(pa[2]);
      const float2 w = unpack2<BF16>(pa[1]), z = unpack2<BF16>(pa[3]);
      l[0] = l[0] * al0 + ((u.x + u.y) + (v.x + v.y));
      l[1] = l[1] * al1 + ((w.x + w.y) + (z.x + z.y));
    }
    // ---- rescale O, then O += P V ----
#pragma unroll
    for (int n = 0; n < NTILES; ++n) {
      acc[n][0] *= al0;
      acc[n][1] *= al0;
      acc[n][2] *= al1;
      acc[n][3] *= al1;
    }
    const int vtok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int vchk = lane >> 4;
#pragma unroll
    for (int j = 0; j < D / 16; ++j) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_trans(page_chunk<D>(vbase, vtok, 2 * j + vchk), b0, b1, b2, b3);
      mma_16816<BF16>(acc[2 * j], pa, b0, b1);
      mma_16816<BF16>(acc[2 * j + 1], pa, b2, b3);
      if constexpr (BF16) {
        mma_16816<BF16>(acc[2 * j], pl, b0, b1);
        mma_16816<BF16>(acc[2 * j + 1], pl, b2, b3);
      }
    }
  }

  // Write this warp's (m, l, O) rows < group into the merge buffers.
  __device__ __forceinline__ void publish(float* red_acc, float* red_m, float* red_l, int group,
                                          int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8, tig = lane & 3;
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (r0 < group) {
#pragma unroll
      for (int n = 0; n < NTILES; ++n)
        *reinterpret_cast<float2*>(red_acc + r0 * D + n * 8 + tig * 2) =
            make_float2(acc[n][0], acc[n][1]);
      if (tig == 0) {
        red_m[r0] = m[0];
        red_l[r0] = l0;
      }
    }
    if (r1 < group) {
#pragma unroll
      for (int n = 0; n < NTILES; ++n)
        *reinterpret_cast<float2*>(red_acc + r1 * D + n * 8 + tig * 2) =
            make_float2(acc[n][2], acc[n][3]);
      if (tig == 0) {
        red_m[r1] = m[1];
        red_l[r1] = l1;
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Page step with both products transposed, for groups of up to 8 query heads:
// S^T = K Q^T and O^T = V^T P^T, with the page's 16 tokens (first product)
// and 16-dim slices of the head (second) as the mma's M = 16 rows and the
// group's query heads as its N = 8 columns.  K comes in as A fragments
// through the plain ldmatrix, V^T through the transposed one, and the S^T
// accumulator (token, query row) becomes the B operand of the second product
// by one movmatrix transpose per 8 tokens.  bf16 P goes in as a hi + lo pair.
// ---------------------------------------------------------------------------
template <int D, bool BF16>
struct MmaWarpT {
  static constexpr int kMinBlocks = 0;
  static constexpr int KSTEPS = D / 16;
  static constexpr int MTILES = D / 16;
  static constexpr float kSlack = 8.f;  // log2 units the reference max may trail by
  uint32_t qb[KSTEPS][2];  // Q^T B fragments of query row lane / 4
  float acc[MTILES][4];    // O^T: (dim 16c + g, rows 2t, 2t+1), (dim 16c + 8 + g, ...)
  float m[2], l[2];        // query rows 2t, 2t+1: reference max (log2), lane-partial sum
  float mt[2];             // and their true running max

  __device__ __forceinline__ void init(const uint16_t* q_group, int group, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const uint32_t* q = reinterpret_cast<const uint32_t*>(q_group + g * D);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qb[kk][0] = g < group ? q[(kk * 16 + 2 * t) >> 1] : 0u;
      qb[kk][1] = g < group ? q[(kk * 16 + 8 + 2 * t) >> 1] : 0u;
    }
#pragma unroll
    for (int i = 0; i < MTILES; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    m[0] = m[1] = mt[0] = mt[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  __device__ __forceinline__ void page(uint32_t kbase, uint32_t vbase, int tok0, int t_end,
                                       float scale_log2, int lane) {
    const int g = lane >> 2;
    // ---- S^T = K Q^T ----
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
    const int ktok = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int kchk = lane >> 4;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a[4];  // (tok 0-7, chunk 2kk) (8-15, 2kk) (0-7, 2kk+1) (8-15, 2kk+1)
      ldsm_x4(page_chunk<D>(kbase, ktok, 2 * kk + kchk), a[0], a[1], a[2], a[3]);
      if (kk & 1) mma_16816<BF16>(s1, a, qb[kk][0], qb[kk][1]);
      else        mma_16816<BF16>(s0, a, qb[kk][0], qb[kk][1]);
    }
    // ---- scale, mask the tail, row maxima over the page's 16 tokens ----
    const int lim = t_end - tok0;
    const bool lo_live = g < lim, hi_live = g + 8 < lim;
    const float x0 = lo_live ? (s0[0] + s1[0]) * scale_log2 : -INFINITY;  // token g, row 2t
    const float x1 = lo_live ? (s0[1] + s1[1]) * scale_log2 : -INFINITY;  // token g, row 2t+1
    const float x2 = hi_live ? (s0[2] + s1[2]) * scale_log2 : -INFINITY;  // token g+8, row 2t
    const float x3 = hi_live ? (s0[3] + s1[3]) * scale_log2 : -INFINITY;
    // lanes of equal t hold the same two rows; each reduces one of them over
    // the 8 lanes and the other comes back from the neighbour of opposite g
    // parity (token 0 of the page is always live, so the maxima are finite)
    const bool odd = g & 1;
    float keep = odd ? fmaxf(x1, x3) : fmaxf(x0, x2);
    const float send = odd ? fmaxf(x0, x2) : fmaxf(x1, x3);
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, keep, 8));
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, keep, 16));
    const float other = __shfl_xor_sync(0xffffffffu, keep, 4);
    mt[0] = fmaxf(mt[0], odd ? other : keep);
    mt[1] = fmaxf(mt[1], odd ? keep : other);
    // The reference max m trails the true one by at most 2^kSlack, so P stays
    // at most 2^8; O and l are rescaled only when some row of the warp
    // outgrows that, a branch the whole warp takes.
    if (__any_sync(0xffffffffu, (mt[0] > m[0] + kSlack) | (mt[1] > m[1] + kSlack))) {
      const float al0 = ex2(m[0] - mt[0]), al1 = ex2(m[1] - mt[1]);
      m[0] = mt[0];
      m[1] = mt[1];
      l[0] *= al0;
      l[1] *= al1;
#pragma unroll
      for (int i = 0; i < MTILES; ++i) {
        acc[i][0] *= al0;
        acc[i][1] *= al1;
        acc[i][2] *= al0;
        acc[i][3] *= al1;
      }
    }
    // ---- P in the cache dtype as the B operand of the second product: fp16 P
    // once (l sums the rounded values), bf16 P as a hi + lo pair (l sums the
    // fp32 p) ----
    const float p0 = ex2(x0 - m[0]), p1 = ex2(x1 - m[1]), p2 = ex2(x2 - m[0]), p3 = ex2(x3 - m[1]);
    const uint32_t h_lo = pack2<BF16>(p0, p1), h_hi = pack2<BF16>(p2, p3);
    uint32_t pb[4];
    pb[0] = movmatrix_trans(h_lo);
    pb[1] = movmatrix_trans(h_hi);
    if constexpr (BF16) {
      const float2 u = unpack2<true>(h_lo), w = unpack2<true>(h_hi);
      pb[2] = movmatrix_trans(pack2<true>(p0 - u.x, p1 - u.y));
      pb[3] = movmatrix_trans(pack2<true>(p2 - w.x, p3 - w.y));
      l[0] += p0 + p2;
      l[1] += p1 + p3;
    } else {
      const float2 u = unpack2<false>(h_lo), w = unpack2<false>(h_hi);
      l[0] += u.x + w.x;
      l[1] += u.y + w.y;
    }
    // ---- O^T += V^T P^T ----
    const int vtok = (lane & 7) + (lane >> 4) * 8;
    const int vchk = (lane >> 3) & 1;
#pragma unroll
    for (int c = 0; c < MTILES; ++c) {
      uint32_t a[4];  // (tok 0-7, chunk 2c) (0-7, 2c+1) (8-15, 2c) (8-15, 2c+1), transposed
      ldsm_x4_trans(page_chunk<D>(vbase, vtok, 2 * c + vchk), a[0], a[1], a[2], a[3]);
      mma_16816<BF16>(acc[c], a, pb[0], pb[1]);
      if constexpr (BF16) mma_16816<BF16>(acc[c], a, pb[2], pb[3]);
    }
  }

  // The partials are restated against the true max (a factor <= 1).
  __device__ __forceinline__ void publish(float* red_acc, float* red_m, float* red_l, int group,
                                          int lane) {
    const int g = lane >> 2, t = lane & 3;
    float f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) f[h] = mt[h] > -INFINITY ? ex2(m[h] - mt[h]) : 1.f;
    float l0 = l[0] * f[0], l1 = l[1] * f[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = 2 * t + h;
      if (row < group) {
#pragma unroll
        for (int c = 0; c < MTILES; ++c) {
          red_acc[row * D + 16 * c + g] = acc[c][h] * f[h];
          red_acc[row * D + 16 * c + 8 + g] = acc[c][2 + h] * f[h];
        }
        if (g == 0) {
          red_m[row] = mt[h];
          red_l[row] = h ? l1 : l0;
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// End of an item: merge the four warps' rows (already published into the
// red_* buffers) and, for an item spread over a cluster, the CTAs' rows
// through distributed shared memory.  emit(row, d, o0, o1, m, l) receives
// each finished pair of output dims: the unnormalised sums o0, o1, the row
// max m (log2 domain) and the row sum l.  With `spread`, every CTA of the
// cluster must call this (it holds two cluster barriers); each emits a slice.
// ---------------------------------------------------------------------------
template <int D, int NST, int EB = 2, class Emit>
__device__ __forceinline__ void merge_and_emit(uint8_t* smem, int nrows, bool spread, int ctas,
                                               int crank, Emit&& emit) {
  using L = DecodeSmem<D, NST, EB>;
  const float* red_acc = reinterpret_cast<const float*>(smem);
  const float* red_m = reinterpret_cast<const float*>(smem + L::kRedMOffset);
  const float* red_l = reinterpret_cast<const float*>(smem + L::kRedLOffset);
  float* part_acc = reinterpret_cast<float*>(smem + L::kPartAccOffset);
  float* part_m = reinterpret_cast<float*>(smem + L::kPartMOffset);
  float* part_l = reinterpret_cast<float*>(smem + L::kPartLOffset);
  for (int o = threadIdx.x * 2; o < nrows * D; o += kThreads * 2) {
    const int g = o / D, d = o % D;
    float mw[kWarps];
    float big_m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      mw[w] = red_m[w * 16 + g];
      big_m = fmaxf(big_m, mw[w]);
    }
    float big_l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float e = (mw[w] == -INFINITY) ? 0.f : ex2(mw[w] - big_m);
      big_l += e * red_l[w * 16 + g];
      if (e != 0.f) {
        const float2 v = *reinterpret_cast<const float2*>(red_acc + (w * nrows + g) * D + d);
        o0 += e * v.x;
        o1 += e * v.y;
      }
    }
    if (spread) {
      *reinterpret_cast<float2*>(part_acc + g * D + d) = make_float2(o0, o1);
      if (d == 0) {
        part_m[g] = big_m;
        part_l[g] = big_l;
      }
    } else {
      emit(g, d, o0, o1, big_m, big_l);
    }
  }
  if (!spread) return;

  cluster_sync();  // every CTA's part_* rows are complete and visible
  const int pairs = nrows * D / 2;
  const int per = (pairs + ctas - 1) / ctas;
  const int lo = crank * per, hi = min(pairs, lo + per);
  const uint32_t acc_base = smem_addr(part_acc), m_base = smem_addr(part_m),
                 l_base = smem_addr(part_l);
  for (int pr = lo + static_cast<int>(threadIdx.x); pr < hi; pr += kThreads) {
    const int o = pr * 2, g = o / D, d = o % D;
    float mc[kMaxCluster];
    float big_m = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) {
      mc[c] = c < ctas ? ld_cluster_f32(map_cluster(m_base + g * 4, c)) : -INFINITY;
      big_m = fmaxf(big_m, mc[c]);
    }
    float big_l = 0.f, o0 = 0.f, o1 = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) {
      const float e = (mc[c] == -INFINITY) ? 0.f : ex2(mc[c] - big_m);
      if (e != 0.f) {
        big_l += e * ld_cluster_f32(map_cluster(l_base + g * 4, c));
        const float2 v = ld_cluster_f32x2(map_cluster(acc_base + (g * D + d) * 4, c));
        o0 += e * v.x;
        o1 += e * v.y;
      }
    }
    emit(g, d, o0, o1, big_m, big_l);
  }
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

// ---------------------------------------------------------------------------
// After a warp's page loop: true when none of its TMA loads is still in
// flight.  A loop that ended normally (ok) consumed every page it issued.  One
// that gave up at page k_stop has issued pages k_stop .. min(k_stop + NST,
// n_pages) - 1 (at most one per stage) and not consumed them; each is waited
// for with the bounded wait.  Whole warp.
// ---------------------------------------------------------------------------
template <int NST>
__device__ __forceinline__ bool drain_stages(bool ok, int k_stop, int n_pages, uint32_t bar0,
                                             int kbase = 0) {
  if (ok) return true;
  bool landed = true;
  const int k_end = min(k_stop + NST, n_pages);
  for (int k = k_stop; k < k_end; ++k)
    landed &= __all_sync(~0u, mbar_wait_bounded(bar0 + ((kbase + k) % NST) * 8,
                                                 ((kbase + k) / NST) & 1));
  return landed;
}

// ---------------------------------------------------------------------------
// The kernel: one (sequence, KV head, partition) item per cluster.
//
// Launched without a cluster attribute, every CTA is a cluster of one and
// owns one item.  Launched with clusters of C CTAs (pa_decode only), an item
// longer than cluster_pages pages is spread over all C CTAs of its cluster
// (page i goes to CTA i % C, then to warp (i / C) % 4); each CTA merges its
// four warps in shared memory, then the CTAs merge their partial rows through
// distributed shared memory, each CTA finishing a slice of the outputs.  A
// shorter item stays on CTA 0 and the other CTAs of its cluster exit at once;
// the choice depends only on the item's length, so every CTA of a cluster
// takes the same branch and either all of them reach both cluster barriers
// or none does.
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Each warp's ring of NST stages, one mbarrier per stage.  The barriers are
// initialised once per CTA; a CTA that takes several items carries each
// warp's count of pages through the ring (kbase) from item to item, so that
// page k of an item uses stage (kbase + k) % NST with phase parity
// ((kbase + k) / NST) & 1.  Whole warp.
// ---------------------------------------------------------------------------
template <int NST>
__device__ __forceinline__ void init_ring(uint32_t bar0, int lane) {
  if (lane == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(bar0 + i * 8, 1);
    fence_barrier_init();
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// One (sequence, KV head, partition) item, whole CTA (and, spread, whole
// cluster): the page loop of every warp, the merge, the output or partials.
// ctx is the sequence's validated context length; the warps' rings are
// initialised and kbase (per warp) counts the pages they already took.
// Returns false when a wait gave up on this item (after draining what it
// can): the ring's count is then no longer known, and the CTA must end.
// ---------------------------------------------------------------------------
template <int D, int NST, bool BF16, class Warp, int EB>
__device__ __forceinline__ bool decode_item(const CUtensorMap& kmap, const CUtensorMap& vmap,
                                            const DecodeArgs& a, uint8_t* smem, int s, int kvh,
                                            int part, int ctx, int csize, int crank, int& kbase) {
  using L = DecodeSmem<D, NST, EB>;
  // ---- this item's token range ----
  const int group = a.group;
  const bool split = a.tmp_out != nullptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int t_begin = 0, t_end = ctx;
  if (split) {
    t_begin = part * a.partition_size;
    t_end = min(t_begin + a.partition_size, ctx);
    if (t_begin >= t_end) return true;  // partition past the end: nothing to write
  } else if (ctx == 0) {
    // empty sequence: zero output rows
    if (crank == 0) {
      uint16_t* o = a.out + (static_cast<size_t>(s) * a.num_heads + kvh * group) * D;
      for (int i = threadIdx.x; i < group * D; i += kThreads) o[i] = 0;
    }
    return true;
  }

  const int first_page = t_begin / kPage;
  const int n_pages = (t_end - first_page * kPage + kPage - 1) / kPage;
  const bool spread = csize > 1 && n_pages > a.cluster_pages;
  if (csize > 1 && !spread && crank != 0) return true;  // short item: CTA 0 alone
  const int ctas = spread ? csize : 1;             // CTAs sharing this item
  const int page0 = (spread ? crank : 0) + ctas * warp;  // this warp's first page
  const int pstride = ctas * kWarps;                      // and its page stride
  const int my_pages = n_pages > page0 ? (n_pages - page0 + pstride - 1) / pstride : 0;
  const int32_t* bt = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq + first_page;

  const uint32_t stage0 = smem_addr(smem) + warp * NST * L::kStageBytes;
  const uint32_t bar0 = smem_addr(smem + L::kBarOffset) + warp * NST * 8;

  // ---- block ids: lane j holds the id of this warp's page (win*32 + j) ----
  const size_t row_base = static_cast<size_t>(s) * a.max_blocks_per_seq + first_page;
  auto load_ids = [&](int win) -> int {
    const int k = win * 32 + lane;
    if (k >= my_pages) return -1;
    const int idx = page0 + k * pstride;
    int id = bt[idx];
    if (id < 0 || id >= a.num_blocks) {
      record_error(kErrBlockId, static_cast<long long>(row_base + idx));
      id = -1;  // TMA zero-fills a box at a negative row: no out-of-range read
    }
    return id;
  };
  int win = 0;
  int ids_cur = load_ids(0);
  int ids_next = my_pages > 32 ? load_ids(1) : -1;

  auto issue = [&](int k) {  // whole warp; lane 0 issues the TMA for page k
    const int src = ((k >> 5) == win) ? ids_cur : ids_next;
    const int id = __shfl_sync(0xffffffffu, src, k & 31);
    if (lane == 0) {
      const int st = (kbase + k) % NST;
      const uint32_t bar = bar0 + st * 8;
      const uint32_t dk = stage0 + st * L::kStageBytes;
      const uint32_t dv = dk + L::kPageBytes;
      const int row = id * kPage;
      mbar_arrive_expect_tx(bar, L::kStageBytes);
#pragma unroll
      for (int b = 0; b < L::kBoxesPerRow; ++b)
        tma_load_4d(dk + b * kBoxBytes, &kmap, bar, 0, b, kvh, row);
#pragma unroll
      for (int b = 0; b < L::kBoxesPerRow; ++b)
        tma_load_4d(dv + b * kBoxBytes, &vmap, bar, 0, b, kvh, row);
    }
  };

  const int pre = my_pages < NST ? my_pages : NST;
  for (int k = 0; k < pre; ++k) issue(k);

  // ---- this warp's query rows ----
  Warp st;
  const uint16_t* q_group =
      a.query + (static_cast<size_t>(s) * a.num_heads + static_cast<size_t>(kvh) * group) * D;
  st.init(q_group, group, lane);

  // ---- main loop over this warp's pages ----
  bool ok = true;
  int k_stop = my_pages;  // first page not consumed
  for (int k = 0; k < my_pages; ++k) {
    if (k > 0 && (k & 31) == 0) {
      ++win;
      ids_cur = ids_next;
      ids_next = my_pages > (win + 1) * 32 ? load_ids(win + 1) : -1;
    }
    const int stg = (kbase + k) % NST;
    // the whole warp takes the same branch, whatever each lane's wait saw
    if (!__all_sync(~0u, mbar_wait_bounded(bar0 + stg * 8, ((kbase + k) / NST) & 1))) {
      if (lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
      ok = false;
      k_stop = k;
      break;
    }
    const uint32_t kb = stage0 + stg * L::kStageBytes;
    const int tok0 = (first_page + page0 + k * pstride) * kPage;
    if (tok0 + kPage > ctx) zero_page_tail<L::kBoxesPerRow>(kb + L::kPageBytes, ctx - tok0, lane);
    st.page(kb, kb + L::kPageBytes, tok0, t_end, a.scale_log2, lane);
    __syncwarp();
    if (k + NST < my_pages) issue(k + NST);
  }

  // ---- merge the four warps (the stage area is reused as the merge buffer).
  // A warp that gave up on a wait still has its loads for pages k_stop ..
  // k_stop + NST - 1 in flight: wait for them (bounded) first.  If one never
  // lands, the stage area is left alone and the CTA ends without writing. ----
  if (!__syncthreads_and(drain_stages<NST>(ok, k_stop, my_pages, bar0, kbase))) {
    if (spread) {  // still meet the cluster's two merge barriers
      cluster_sync();
      cluster_sync();
    }
    return false;
  }
  float* red_acc = reinterpret_cast<float*>(smem);
  float* red_m = reinterpret_cast<float*>(smem + L::kRedMOffset);
  float* red_l = reinterpret_cast<float*>(smem + L::kRedLOffset);
  if (ok) {
    st.publish(red_acc + warp * group * D, red_m + warp * 16, red_l + warp * 16, group, lane);
  } else {
    for (int g = lane; g < group; g += 32) {
      red_m[warp * 16 + g] = -INFINITY;
      red_l[warp * 16 + g] = 0.f;
    }
  }
  __syncthreads();

  const size_t hrow0 = static_cast<size_t>(s) * a.num_heads + static_cast<size_t>(kvh) * group;
  merge_and_emit<D, NST, EB>(smem, group, spread, ctas, crank,
                             [&](int g, int d, float o0, float o1, float big_m, float big_l) {
    const size_t hrow = hrow0 + g;
    o0 *= a.v_scale;
    o1 *= a.v_scale;
    if (split) {
      const size_t pidx = hrow * a.max_partitions + part;
      *reinterpret_cast<float2*>(a.tmp_out + pidx * D + d) = make_float2(o0, o1);
      if (d == 0) {
        a.max_logits[pidx] = big_m * kLn2;
        a.exp_sums[pidx] = big_l;
      }
    } else {
      const float inv = big_l > 0.f ? 1.f / big_l : 0.f;
      *reinterpret_cast<uint32_t*>(a.out + hrow * D + d) = pack2<BF16>(o0 * inv, o1 * inv);
    }
  });
  // the merge buffers were written through the generic proxy: order those
  // writes before a later item's TMA loads into the same stage area
  fence_proxy_async_smem();
  kbase += my_pages;
  return __syncthreads_and(ok);
}

template <int D, int NST, bool BF16, class Warp, int EB = 2>
__global__ void __launch_bounds__(kThreads, Warp::kMinBlocks)
    paged_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  using L = DecodeSmem<D, NST, EB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int csize = static_cast<int>(cluster_nctarank());
  const int crank = static_cast<int>(cluster_ctarank());
  prefetch_tensormap(&kmap);
  prefetch_tensormap(&vmap);
  pdl_launch_dependents();
  pdl_wait();  // inputs may come from the previous kernel of the stream

  int item = blockIdx.x / csize;
  const int part = item % a.parts_per_head;
  item /= a.parts_per_head;
  const int kvh = item % a.num_kv_heads;
  int s = item / a.num_kv_heads;
  const bool split = a.tmp_out != nullptr;
  const bool reporter = threadIdx.x == 0 && crank == 0 && part == 0 && kvh == 0;
  const int cap = a.max_blocks_per_seq * kPage;

  // ---- longest-first order: grid slot s takes the s-th longest sequence
  // (ties by index), so that long items start first and short ones fill the
  // tail.  The rank of every sequence is counted against all others, on keys
  // (length << 8 | 255 - index) that order both at once. ----
  if (a.longest_first) {
    unsigned* keys = reinterpret_cast<unsigned*>(smem);  // stage area, not in use yet
    int* chosen = reinterpret_cast<int*>(keys + kLptMaxSeqs);
    const int n4 = (a.num_seqs + 3) >> 2;
    const unsigned lcap = static_cast<unsigned>(min(cap, (1 << 24) - 1));
    for (int i = threadIdx.x; i < n4 * 4; i += kThreads) {
      unsigned key = 0u;  // pads: below every sequence's key, never counted
      if (i < a.num_seqs)
        key = (min(static_cast<unsigned>(max(a.context_lens[i], 0)), lcap) << 8) |
              static_cast<unsigned>(255 - i);
      keys[i] = key;
    }
    __syncthreads();
    const uint4* keys4 = reinterpret_cast<const uint4*>(keys);
    for (int t = threadIdx.x; t < a.num_seqs; t += kThreads) {
      const unsigned kt = keys[t];
      int rank = 0;
      for (int j4 = 0; j4 < n4; ++j4) {
        const uint4 v = keys4[j4];
        rank += (v.x > kt) + (v.y > kt) + (v.z > kt) + (v.w > kt);
      }
      if (rank == s) *chosen = t;
    }
    __syncthreads();
    s = *chosen;
    fence_proxy_async_smem();  // generic writes to the stage area before TMA writes to it
    __syncthreads();  // the stage area is about to be reused
  }

  // ---- context length ----
  int ctx = a.context_lens[s];
  if (ctx < 0 || ctx > cap) {
    if (reporter) record_error(kErrContextLen, s);
    ctx = ctx < 0 ? 0 : cap;
  }
  if (split && reporter && (ctx + a.partition_size - 1) / a.partition_size > a.max_partitions)
    record_error(kErrPartitions, s);
  init_ring<NST>(smem_addr(smem + L::kBarOffset) + (threadIdx.x >> 5) * NST * 8, threadIdx.x & 31);
  int kbase = 0;
  decode_item<D, NST, BF16, Warp, EB>(kmap, vmap, a, smem, s, kvh, part, ctx, csize, crank,
                                      kbase);
}


// ---------------------------------------------------------------------------
// Split mode, persistent: the items that exist -- partition p of sequence s
// for p < ceil(ctx_s / partition_size), every KV head -- in a dense order that
// every CTA derives from the context lengths.  Up to kLptMaxSeqs sequences
// every context and the partitions before each sequence sit in shared
// memory, and an item's sequence is a binary search away.  Beyond, thread t
// counts the partitions of a chunk of ceil(S / kThreads) sequences, a block
// scan gives each chunk's first partition, and an item's sequence is found by
// a binary search over the chunks and a scan of one chunk.  The grid is one
// wave (SMs x resident CTAs); CTA b takes items b, b + gridDim.x, ..., so no
// CTA is launched for a partition past its sequence's end.  Each warp's ring
// runs on from item to item.
// ---------------------------------------------------------------------------

// Partitions of sequence s (clamped as the kernels clamp: a context outside
// [0, cap] to the range, a count past max_partitions to it), its clamped
// context in ctx; the clamps are reported when `report`.
__device__ __forceinline__ int split_partitions(const DecodeArgs& a, int s, int cap, bool report,
                                                int& ctx) {
  int c = a.context_lens[s];
  if (c < 0 || c > cap) {
    if (report) record_error(kErrContextLen, s);
    c = c < 0 ? 0 : cap;
  }
  int np = (c + a.partition_size - 1) / a.partition_size;
  if (np > a.max_partitions) {
    if (report) record_error(kErrPartitions, s);
    np = a.max_partitions;
  }
  ctx = c;
  return np;
}

template <int D, int NST, bool BF16, class Warp, int EB = 2>
// at least three CTAs per SM (at most 168 registers), more where the page step allows
__global__ void __launch_bounds__(kThreads, Warp::kMinBlocks > 3 ? Warp::kMinBlocks : 3)
    paged_decode_persistent_kernel(const __grid_constant__ CUtensorMap kmap,
                                   const __grid_constant__ CUtensorMap vmap, const DecodeArgs a) {
  using L = DecodeSmem<D, NST, EB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  prefetch_tensormap(&kmap);
  prefetch_tensormap(&vmap);
  pdl_launch_dependents();
  pdl_wait();  // inputs may come from the previous kernel of the stream
  const int cap = a.max_blocks_per_seq * kPage;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const bool small = a.num_seqs <= kLptMaxSeqs;
  int* ctxs = reinterpret_cast<int*>(smem + L::kSeqOffset);   // small: [S] contexts
  int* cum = ctxs + kLptMaxSeqs;                              // small: [S + 1] partitions before
  int* chunk_first = ctxs;                                    // else: [kThreads + 1]
  int* warp_sum = ctxs + kThreads + 1;                        // else: [kWarps]
  const int chunk = (a.num_seqs + kThreads - 1) / kThreads;
  const int t = threadIdx.x;
  int total;
  if (small) {
    for (int s = t; s < a.num_seqs; s += kThreads)
      cum[s + 1] = split_partitions(a, s, cap, blockIdx.x == 0, ctxs[s]);   // one CTA reports
    __syncthreads();
    if (t == 0) {  // running count
      int acc = 0;
      cum[0] = 0;
      for (int s = 0; s < a.num_seqs; ++s) cum[s + 1] = (acc += cum[s + 1]);
    }
    __syncthreads();
    total = cum[a.num_seqs];
  } else {
    int mine = 0;
    for (int s = t * chunk; s < min(a.num_seqs, (t + 1) * chunk); ++s) {
      int c;
      mine += split_partitions(a, s, cap, blockIdx.x == 0, c);   // one CTA reports
    }
    int incl = mine;  // block scan of the chunk counts
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += v;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    for (int w = 0; w < warp; ++w) incl += warp_sum[w];
    chunk_first[t] = incl - mine;
    if (t == kThreads - 1) chunk_first[kThreads] = incl;
    __syncthreads();
    total = chunk_first[kThreads];
  }
  const int items = total * a.num_kv_heads;
  init_ring<NST>(smem_addr(smem + L::kBarOffset) + warp * NST * 8, lane);
  int kbase = 0;  // this warp's pages through its ring so far
  for (int u = blockIdx.x; u < items; u += gridDim.x) {
    const int kv = u % a.num_kv_heads, su = u / a.num_kv_heads;
    int s, first, ctx = 0;
    if (small) {
      int lo = 0, hi = a.num_seqs;  // the sequence with cum[s] <= su < cum[s + 1]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= su) lo = mid; else hi = mid;
      }
      s = lo;
      first = cum[lo];
      ctx = ctxs[lo];
    } else {
      int lo = 0, hi = kThreads;  // the chunk: the last one whose first partition is <= su
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (chunk_first[mid] <= su) lo = mid; else hi = mid;
      }
      first = chunk_first[lo];
      s = lo * chunk;
      for (const int s_end = min(a.num_seqs, s + chunk); s < s_end; ++s) {
        const int np = split_partitions(a, s, cap, false, ctx);
        if (su < first + np) break;
        first += np;
      }
    }
    // (decode_item ends with a CTA barrier: the merge buffers, in the stage
    // area, are free for the next item's pages)
    if (!decode_item<D, NST, BF16, Warp, EB>(kmap, vmap, a, smem, s, kv, su - first, ctx, 1, 0,
                                             kbase))
      return;
  }
}

}  // namespace pa

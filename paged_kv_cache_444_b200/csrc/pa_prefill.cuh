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
// Work item: (sequence, KV head, tile of 128/G query tokens).  Its 128 rows are
// the tile's tokens x the G query heads of the KV head, token-major -- the M of
// one 128-row MMA.  Keys go in blocks of 128 (8 pages of 16):
//   S  = Q K^T      128 x 128 fp32 in tensor memory (three buffers), Q and K
//                   from shared memory
//   P  = 2^(S*scale*log2 e - m)   by four softmax warps, thread r = row r,
//                   written back over S in tensor memory as 16-bit pairs
//   O += P V        128 x D fp32 in tensor memory, P from tensor memory and V
//                   from shared memory
// Keeping P in tensor memory leaves shared-memory bandwidth to the K and V
// operands.  Warp roles: warps 0-3 softmax and epilogue, warp 4 TMA (Q once;
// the K and V pages of each block through rings of NST stages), warp 5 issues
// the MMAs.  The causal mask is a per-row key limit (pos + 1) applied to S;
// blocks past the tile's last key are never loaded.  O is rescaled only when
// a row's running maximum grows by more than 2^8 (the reference maximum may
// lag the true one by that much: P <= 2^8 stays exact in the 16-bit operand
// and the final 1/l uses the same reference).  bf16 P enters P V as a hi + lo
// pair of bf16 products (16 bits of P); fp16 P is rounded once and l sums the
// rounded values.
#pragma once

#include "pa_decode.cuh"
#include "pa_umma.cuh"

namespace pa {

constexpr unsigned kErrQuery = 7;
constexpr int kPrefillRows = 128;                   // query rows per CTA = MMA M
constexpr int kPrefillKeys = 128;                   // keys per block = S tile N
constexpr int kPrefillPages = kPrefillKeys / kPage; // 8 pages per block
constexpr int kPrefillThreads = 192;                // 4 softmax warps, TMA warp, MMA warp
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 0;                      // O: columns [0, D)
constexpr uint32_t kTmemS = 128;                    // S / P buffers at 128, 256, 384
constexpr int kSBufs = 3;
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
  int tile_tokens;              // query tokens per CTA (128 / group, rounded down)
  int tiles_per_seq;            // ceil(max_query_len / tile_tokens)
};

template <int D, bool BF16>
struct PrefillSmem {
  static constexpr int NST = D == 64 ? 4 : 3;       // K (and V) blocks in flight
  static constexpr int kSlabs = D / 64;             // 64-element column slabs
  static constexpr int kSlab = 128 * 128;           // 128 rows x 128 B
  static constexpr int kQ = 0;
  static constexpr int kStage = kSlabs * kSlab;     // one block of K (or V)
  static constexpr int kK = kQ + kSlabs * kSlab;
  static constexpr int kV = kK + NST * kStage;
  static constexpr int kBarQ = kV + NST * kStage;
  static constexpr int kBarKFull = kBarQ + 8;
  static constexpr int kBarKEmpty = kBarKFull + 8 * NST;
  static constexpr int kBarVFull = kBarKEmpty + 8 * NST;
  static constexpr int kBarVEmpty = kBarVFull + 8 * NST;
  static constexpr int kBarS = kBarVEmpty + 8 * NST;   // one per S / P buffer
  static constexpr int kBarP = kBarS + 8 * kSBufs;
  static constexpr int kBarO = kBarP + 8;
  static constexpr int kBarDrain = kBarO + 8;
  static constexpr int kTmemSlot = kBarDrain + 8;
  static constexpr int kAbort = kTmemSlot + 4;
  static constexpr int kBytes = kAbort + 4;
  static constexpr int kAlloc = kBytes + 1024;
};

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

template <int D, bool BF16>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap qmap,
                         const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using L = PrefillSmem<D, BF16>;
  constexpr int NST = L::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_addr(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&qmap);
    prefetch_tensormap(&kmap);
    prefetch_tensormap(&vmap);
  }
  pdl_launch_dependents();
  pdl_wait();

  // ---- work item: the last tiles of every sequence (most keys) start first ----
  const int per_tile = a.num_seqs * a.num_kv_heads;
  int item = blockIdx.x;
  const int tile = a.tiles_per_seq - 1 - item / per_tile;
  item %= per_tile;
  const int kvh = item % a.num_kv_heads;
  const int s = item / a.num_kv_heads;
  const int G = a.group;

  const int q0 = a.query_starts[s];
  const int q_len = a.query_starts[s + 1] - q0;
  const int ctx = a.context_lens[s];
  const int cap = a.max_blocks_per_seq * kPage;
  if (q0 < 0 || q_len < 0 || q0 > a.num_tokens - q_len || q_len > ctx || ctx > cap) {
    if (threadIdx.x == 0 && kvh == 0 && tile == 0) record_error(kErrQuery, s);
    return;
  }
  const int t_begin = tile * a.tile_tokens;
  if (t_begin >= q_len) return;
  const int t_end = min(t_begin + a.tile_tokens, q_len);
  const int nrows = (t_end - t_begin) * G;
  const int pos_base = ctx - q_len + t_begin;     // position of the tile's first token
  const int lim_max = pos_base + (t_end - t_begin);
  const int n_pages = (lim_max + kPage - 1) / kPage;
  const int nkb = (n_pages + kPrefillPages - 1) / kPrefillPages;
  const int q_rows = a.tile_tokens * G;           // rows the Q box fills

  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbort);
  if (threadIdx.x == 0) {
    mbar_init(sb + L::kBarQ, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(sb + L::kBarKFull + 8 * i, 1);
      mbar_init(sb + L::kBarKEmpty + 8 * i, 1);
      mbar_init(sb + L::kBarVFull + 8 * i, 1);
      mbar_init(sb + L::kBarVEmpty + 8 * i, 1);
    }
    for (int i = 0; i < kSBufs; ++i) mbar_init(sb + L::kBarS + 8 * i, 1);
    mbar_init(sb + L::kBarP, 4 * 32);
    mbar_init(sb + L::kBarO, 1);
    mbar_init(sb + L::kBarDrain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) tmem_alloc(sb + L::kTmemSlot, kTmemCols);
  if (warp < 4 && q_rows < kPrefillRows) {
    // rows no Q box covers are zero (they are masked, but must not be NaN)
    const int chunks = (kPrefillRows - q_rows) * 8;
    for (int i = threadIdx.x; i < chunks * L::kSlabs; i += 128) {
      const int b = i / chunks, c = i % chunks;
      sts128(sb + L::kQ + b * L::kSlab + q_rows * 128 + c * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlot);

  if (warp == 4) {
    // ================= TMA producer =================
    if (lane == 0) {
      mbar_arrive_expect_tx(sb + L::kBarQ, L::kSlabs * q_rows * 128);
#pragma unroll
      for (int b = 0; b < L::kSlabs; ++b)
        tma_load_4d(sb + L::kQ + b * L::kSlab, &qmap, sb + L::kBarQ, 0, b, kvh * G,
                    q0 + t_begin);
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
  } else if (warp == 5) {
    // ================= MMA issuer =================
    constexpr uint32_t kIdS = umma_idesc_f16(BF16, kPrefillRows, kPrefillKeys, false);
    constexpr uint32_t kIdO = umma_idesc_f16(BF16, kPrefillRows, D, true);
    auto issue_s = [&](int j) {   // S_j = Q K_j^T into buffer j % 3
      const uint32_t kst = sb + L::kK + (j % NST) * L::kStage;
      const uint32_t d = tmem + kTmemS + static_cast<uint32_t>(j % kSBufs) * kPrefillKeys;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * L::kSlab + (kk & 3) * 32;
        umma_f16_ss(d, umma_desc_sw128(sb + L::kQ + off, 16, 1024),
                    umma_desc_sw128(kst + off, 16, 1024), kIdS, kk > 0 ? 1u : 0u);
      }
      umma_commit(sb + L::kBarS + 8 * (j % kSBufs));
      umma_commit(sb + L::kBarKEmpty + 8 * (j % NST));
    };
    bool ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarQ, 0, abort_flag));
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarKFull, 0, abort_flag));
    if (ok) {
      tmem_fence_after_sync();
      if (lane == 0) issue_s(0);
      __syncwarp();
    }
    const int last_page = (ctx - 1) / kPage;
    const int tail_row = ctx % kPage;          // first row past the context in the last page
    for (int j = 0; ok && j < nkb; ++j) {
      if (j + 1 < nkb) {
        const int st1 = (j + 1) % NST;
        ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarKFull + 8 * st1,
                                                   ((j + 1) / NST) & 1, abort_flag));
        if (!ok) break;
        tmem_fence_after_sync();
        if (lane == 0) issue_s(j + 1);
        __syncwarp();
      }
      const int st = j % NST;
      ok = __all_sync(0xffffffffu,
                      wait_or_abort(sb + L::kBarVFull + 8 * st, (j / NST) & 1, abort_flag));
      if (!ok) break;
      const uint32_t vst = sb + L::kV + st * L::kStage;
      const int pages_here = min(kPrefillPages, n_pages - j * kPrefillPages);
      const int lp = last_page - j * kPrefillPages;
      if (tail_row != 0 && lp >= 0 && lp < pages_here) {
        // V rows past the context may hold anything; P is 0 there, and 0 * NaN
        // must not reach O
        const int chunks = (kPage - tail_row) * 8;
        for (int i = lane; i < chunks * L::kSlabs; i += 32) {
          const int b = i / chunks, c = i % chunks;
          sts128(vst + b * L::kSlab + lp * 2048 + tail_row * 128 + c * 16, 0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarP, j & 1, abort_flag));
      if (!ok) break;
      tmem_fence_after_sync();
      if (lane == 0) {
        // P_j sits in S_j's buffer: hi in its first 64 columns, lo in the next 64
        const uint32_t pcol = tmem + kTmemS + static_cast<uint32_t>(j % kSBufs) * kPrefillKeys;
        for (int k = 0; k < pages_here; ++k) {
          const uint64_t bd = umma_desc_sw128(vst + k * 2048, L::kSlab, 1024);
          umma_f16_ts(tmem + kTmemO, pcol + 8 * k, bd, kIdO, (j > 0 || k > 0) ? 1u : 0u);
          if constexpr (BF16) umma_f16_ts(tmem + kTmemO, pcol + 64 + 8 * k, bd, kIdO, 1u);
        }
        umma_commit(sb + L::kBarO);
        umma_commit(sb + L::kBarVEmpty + 8 * st);
      }
      __syncwarp();
    }
    // every MMA issued has completed before tensor memory is freed
    if (lane == 0) umma_commit(sb + L::kBarDrain);
    __syncwarp();
    if (!mbar_wait_bounded(sb + L::kBarDrain, 0) && lane == 0)
      record_error(kErrWaitTimeout, blockIdx.x);
  } else {
    // ================= softmax (row = threadIdx.x = TMEM lane) =================
    const int row = threadIdx.x;
    const int lim = row < nrows ? pos_base + row / G + 1 : 0;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkb; ++j) {
      const uint32_t buf = kTmemS + static_cast<uint32_t>(j % kSBufs) * kPrefillKeys;
      ok = __all_sync(0xffffffffu,
                      wait_or_abort(sb + L::kBarS + 8 * (j % kSBufs), (j / kSBufs) & 1, abort_flag));
      if (!ok) break;
      tmem_fence_after_sync();
      float p[kPrefillKeys];
      tmem_ld128(t_lane + buf, p);
      // logits in log2 units; keys at or past this row's limit are -inf
      const int kbase = j * kPrefillKeys;
      const float2 sl2x2 = make_float2(sl2, sl2);
      if (kbase + kPrefillKeys <= lim) {
#pragma unroll
        for (int c = 0; c < kPrefillKeys; c += 2) {
          const float2 x = fmul2(make_float2(p[c], p[c + 1]), sl2x2);
          p[c] = x.x;
          p[c + 1] = x.y;
        }
      } else {
#pragma unroll
        for (int c = 0; c < kPrefillKeys; ++c) p[c] = kbase + c < lim ? p[c] * sl2 : -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx8[i] = p[i];
#pragma unroll
      for (int c = 8; c < kPrefillKeys; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], p[c]);
      const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const float m_new = fmaxf(m_ref, mx);
      const bool need = m_new > m_ref + kRescaleSlack;
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m_ref - m_new);   // 0 when m_ref is still -inf
        m_ref = m_new;
      }
      l *= alpha;
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      const float2 negm = make_float2(-m_use, -m_use), one2 = make_float2(1.f, 1.f);
#pragma unroll
      for (int c = 0; c < kPrefillKeys; c += 2) {
        const float2 x = ffma2(make_float2(p[c], p[c + 1]), one2, negm);
        p[c] = ex2(x.x);
        p[c + 1] = ex2(x.y);
      }

      if (j > 0) {
        // P V of the previous block is done: O holds it and the P buffers are free
        ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarO, (j - 1) & 1, abort_flag));
        if (!ok) break;
        tmem_fence_after_sync();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float o[32];
            tmem_ld32(t_lane + kTmemO + 32 * c, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(t_lane + kTmemO + 32 * c, o);
          }
        }
      }
      // P (and l) -> this S buffer: keys 2i, 2i+1 packed in column i (hi), and
      // for bf16 the remainder p - hi in column 64 + i (lo)
      float2 lsum[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) lsum[i] = make_float2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t h[32], lo[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x0 = p[64 * half + 2 * i], x1 = p[64 * half + 2 * i + 1];
          h[i] = pack2<BF16>(x0, x1);
          const float2 hf = unpack2<BF16>(h[i]);
          if constexpr (BF16) {
            const float2 r = ffma2(hf, make_float2(-1.f, -1.f), make_float2(x0, x1));
            lo[i] = pack2<true>(r.x, r.y);
            lsum[i & 3].x += x0;
            lsum[i & 3].y += x1;
          } else {
            lsum[i & 3].x += hf.x;
            lsum[i & 3].y += hf.y;
          }
        }
        tmem_st32u(t_lane + buf + 32 * half, h);
        if constexpr (BF16) tmem_st32u(t_lane + buf + 64 + 32 * half, lo);
      }
      l += ((lsum[0].x + lsum[0].y) + (lsum[1].x + lsum[1].y)) +
           ((lsum[2].x + lsum[2].y) + (lsum[3].x + lsum[3].y));
      tmem_fence_before_sync();
      mbar_arrive(sb + L::kBarP);
    }
    if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(sb + L::kBarO, (nkb - 1) & 1, abort_flag));
    if (ok) {
      tmem_fence_after_sync();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      uint16_t* o_row = a.out + (static_cast<size_t>(q0 + t_begin + row / G) * a.num_heads +
                                 kvh * G + row % G) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(t_lane + kTmemO + 32 * c, o);
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

  tmem_fence_before_sync();
  __syncthreads();
  if (warp == 5) {
    tmem_fence_after_sync();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pa

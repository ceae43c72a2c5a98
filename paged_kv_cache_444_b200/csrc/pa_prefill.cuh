// pa_prefill.cuh -- paged (chunked) prefill attention on sm_100a.
//
// "vLLM PagedAttention 原理与源码深度解析" §8.1 (Chunked Prefill): a long prompt
// is processed a chunk of tokens per step, so a step holds sequences with
// several new query tokens at the end of their context.  Query token i of
// sequence s (q_len new tokens, context_lens[s] tokens in all, their K/V
// already in the paged cache) sits at position ctx - q_len + i and attends
// causally to tokens 0..pos.
//
// Work item: (sequence, KV head, tile of query tokens).  Its rows are the
// tile's tokens x the G query heads of the KV head, token-major, at most 64:
// warp w owns rows 16w..16w+15 as one mma tile, so -- unlike decode -- every
// warp reads every page and no merge between warps is needed.  The pages go
// through one ring of NST stages shared by the CTA: warp 0 holds the block
// ids (32 per window, one per lane) and its lane 0 issues the TMA loads; each
// page is released by a CTA barrier once all warps have used it.  The page
// step is the GQA tensor-core step with a token limit per row (pos + 1), so
// the causal mask costs nothing extra; a warp skips pages past all its rows.
#pragma once

#include "pa_decode.cuh"

namespace pa {

constexpr unsigned kErrQuery = 7;

struct PrefillArgs {
  const uint16_t* query;        // [T, H, D]
  uint16_t* out;                // [T, H, D]
  const int32_t* block_tables;  // [S, MB]
  const int32_t* context_lens;  // [S]
  const int32_t* query_starts;  // [S + 1]
  float scale_log2;
  int num_heads;
  int num_kv_heads;
  int group;
  int max_blocks_per_seq;
  int num_blocks;
  int tile_tokens;              // query tokens per CTA (64 / group)
  int tiles_per_seq;            // ceil(max_query_len / tile_tokens)
};

template <int D, int NST>
struct PrefillSmem {
  static constexpr int kPageBytes = kPage * D * 2;
  static constexpr int kStageBytes = 2 * kPageBytes;
  static constexpr int kBoxesPerRow = D * 2 / 128;
  static constexpr int kBarOffset = NST * kStageBytes;
  static constexpr int kBytes = kBarOffset + NST * 8;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D, int NST, bool BF16>
__global__ void __launch_bounds__(kThreads)
    paged_prefill_kernel(const __grid_constant__ CUtensorMap kmap,
                         const __grid_constant__ CUtensorMap vmap, const PrefillArgs a) {
  using L = PrefillSmem<D, NST>;
  using Warp = MmaWarp<D, BF16, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  prefetch_tensormap(&kmap);
  prefetch_tensormap(&vmap);
  pdl_launch_dependents();
  pdl_wait();

  int item = blockIdx.x;
  const int tile = item % a.tiles_per_seq;
  item /= a.tiles_per_seq;
  const int kvh = item % a.num_kv_heads;
  const int s = item / a.num_kv_heads;
  const int G = a.group;

  const int q0 = a.query_starts[s];
  const int q_len = a.query_starts[s + 1] - q0;
  int ctx = a.context_lens[s];
  const int cap = a.max_blocks_per_seq * kPage;
  if (q_len < 0 || q_len > ctx || ctx > cap) {
    if (threadIdx.x == 0 && kvh == 0 && tile == 0) record_error(kErrQuery, s);
    return;
  }
  const int t_begin = tile * a.tile_tokens;
  if (t_begin >= q_len) return;
  const int t_end = min(t_begin + a.tile_tokens, q_len);
  const int nrows = (t_end - t_begin) * G;
  const int pos_base = ctx - q_len + t_begin;   // position of the tile's first token
  const int n_pages = (pos_base + (t_end - t_begin) - 1) / kPage + 1;

  const uint32_t stage0 = smem_addr(smem);
  const uint32_t bar0 = smem_addr(smem + L::kBarOffset);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(bar0 + i * 8, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ---- block ids (warp 0): lane j holds page win*32 + j ----
  const int32_t* bt = a.block_tables + static_cast<size_t>(s) * a.max_blocks_per_seq;
  auto load_ids = [&](int w) -> int {
    const int k = w * 32 + lane;
    if (k >= n_pages) return -1;
    int id = bt[k];
    if (id < 0 || id >= a.num_blocks) {
      record_error(kErrBlockId, static_cast<long long>(s) * a.max_blocks_per_seq + k);
      id = -1;
    }
    return id;
  };
  int win = 0, ids_cur = -1, ids_next = -1;
  auto issue = [&](int k) {  // warp 0 only
    const int src = ((k >> 5) == win) ? ids_cur : ids_next;
    const int id = __shfl_sync(0xffffffffu, src, k & 31);
    if (lane == 0) {
      const int st = k % NST;
      const uint32_t bar = bar0 + st * 8;
      const uint32_t dk = stage0 + st * L::kStageBytes;
      const uint32_t dv = dk + L::kPageBytes;
      mbar_arrive_expect_tx(bar, L::kStageBytes);
#pragma unroll
      for (int b = 0; b < L::kBoxesPerRow; ++b)
        tma_load_4d(dk + b * kBoxBytes, &kmap, bar, 0, b, kvh, id * kPage);
#pragma unroll
      for (int b = 0; b < L::kBoxesPerRow; ++b)
        tma_load_4d(dv + b * kBoxBytes, &vmap, bar, 0, b, kvh, id * kPage);
    }
  };
  if (warp == 0) {
    ids_cur = load_ids(0);
    ids_next = n_pages > 32 ? load_ids(1) : -1;
    const int pre = n_pages < NST ? n_pages : NST;
    for (int k = 0; k < pre; ++k) issue(k);
  }

  // ---- this warp's rows: r = token * G + head; lane rows r0, r1 = r0 + 8 ----
  Warp st;
  const int r0 = warp * 16 + (lane >> 2), r1 = r0 + 8, tig = lane & 3;
  {
    const uint16_t* qa0 = a.query + (static_cast<size_t>(q0 + t_begin + r0 / G) * a.num_heads +
                                     kvh * G + r0 % G) * D;
    const uint16_t* qa1 = a.query + (static_cast<size_t>(q0 + t_begin + r1 / G) * a.num_heads +
                                     kvh * G + r1 % G) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int klo = kk * 16 + tig * 2, khi = klo + 8;
      st.qa[kk][0] = r0 < nrows ? *reinterpret_cast<const uint32_t*>(qa0 + klo) : 0u;
      st.qa[kk][1] = r1 < nrows ? *reinterpret_cast<const uint32_t*>(qa1 + klo) : 0u;
      st.qa[kk][2] = r0 < nrows ? *reinterpret_cast<const uint32_t*>(qa0 + khi) : 0u;
      st.qa[kk][3] = r1 < nrows ? *reinterpret_cast<const uint32_t*>(qa1 + khi) : 0u;
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) st.acc[n][0] = st.acc[n][1] = st.acc[n][2] = st.acc[n][3] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
  }
  // keys j < lim take part: lim = position + 1 (0 for a padding row)
  const int lim0 = r0 < nrows ? pos_base + r0 / G + 1 : 0;
  const int lim1 = r1 < nrows ? pos_base + r1 / G + 1 : 0;
  int warp_lim = max(lim0, lim1);
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) warp_lim = max(warp_lim, __shfl_xor_sync(0xffffffffu, warp_lim, o));

  // ---- every warp walks every page ----
  bool ok = true;
  for (int k = 0; k < n_pages; ++k) {
    const int stg = k % NST;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar0 + stg * 8, (k / NST) & 1))) {
      if (lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
      ok = false;
    }
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;  // every thread leaves the loop together
    }
    if (k * kPage < warp_lim) {
      const uint32_t kb = stage0 + stg * L::kStageBytes;
      st.page_rows(kb, kb + L::kPageBytes, k * kPage, lim0, lim1, a.scale_log2, lane);
    }
    __syncthreads();  // the stage is free again
    if (warp == 0 && k + NST < n_pages) {
      const int nk = k + NST;
      if ((nk & 31) == 0 && (nk >> 5) != win) {
        ++win;
        ids_cur = ids_next;
        ids_next = n_pages > (win + 1) * 32 ? load_ids(win + 1) : -1;
      }
      issue(nk);
    }
  }

  // ---- finish this warp's rows ----
  float l0 = st.l[0], l1 = st.l[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = (ok && l0 > 0.f) ? 1.f / l0 : 0.f;
  const float inv1 = (ok && l1 > 0.f) ? 1.f / l1 : 0.f;
  if (r0 < nrows) {
    uint16_t* o = a.out + (static_cast<size_t>(q0 + t_begin + r0 / G) * a.num_heads + kvh * G +
                           r0 % G) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<uint32_t*>(o + n * 8 + tig * 2) =
          pack2<BF16>(st.acc[n][0] * inv0, st.acc[n][1] * inv0);
  }
  if (r1 < nrows) {
    uint16_t* o = a.out + (static_cast<size_t>(q0 + t_begin + r1 / G) * a.num_heads + kvh * G +
                           r1 % G) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
      *reinterpret_cast<uint32_t*>(o + n * 8 + tig * 2) =
          pack2<BF16>(st.acc[n][2] * inv1, st.acc[n][3] * inv1);
  }
}

}  // namespace pa

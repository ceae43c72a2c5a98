// pa_shared_prefix.cuh -- decode attention for groups of sequences that share
// a prefix of physical blocks (beam candidates, prompts with a common system
// prefix): each shared page is read from HBM once per group.
//
// The pages describe the sharing ("vLLM PagedAttention 原理与源码深度解析" §3.3:
// beams share prefix blocks through ref_count, copy-on-write before a write;
// "读一个真实 serving 系统 · vLLM 架构巡礼" §2: KVCacheBlock.ref_cnt) but not a
// kernel that exploits it.  The result is the same softmax(scale q K^T) V per
// sequence and head as pa_decode; only the order of the work changes.
//
// Work item: (group, KV head, chunk of members).  Its rows are the chunk's
// members x the G query heads of the KV head -- at most 16, one mma tile.  Its
// pages are the group's shared prefix pages, on which every row is live, and
// then each member's private tail pages, on which only that member's rows are
// live (the others see a zero token limit and stay unchanged).  The pages are
// spread over the CTAs of a cluster and their warps exactly as in
// paged_decode_kernel, and merged the same way.
#pragma once

#include "pa_decode.cuh"

namespace pa {

constexpr unsigned kErrGroup = 6;

struct SharedPrefixArgs {
  const uint16_t* query;          // [S, H, D]
  uint16_t* out;                  // [S, H, D]
  const int32_t* block_tables;    // [S, MB]
  const int32_t* context_lens;    // [S]
  const int32_t* group_starts;    // [num_groups + 1]: members of g are [starts[g], starts[g+1])
  const int32_t* prefix_blocks;   // [num_groups]: table entries shared by all members of g
  float scale_log2;
  int num_seqs;
  int num_heads;
  int num_kv_heads;
  int group;                      // query heads per KV head (G)
  int max_blocks_per_seq;
  int num_blocks;
  int num_groups;
  int members_per_chunk;          // 16 / G
  int chunks_per_group;           // ceil(max_group_size / members_per_chunk)
  int cluster_pages;              // items with more pages are spread over the cluster
  int longest_first;              // order (group, chunk) slots by descending page count
};

template <int D, int NST, bool BF16>
__global__ void __launch_bounds__(kThreads)
    shared_prefix_decode_kernel(const __grid_constant__ CUtensorMap kmap,
                                const __grid_constant__ CUtensorMap vmap,
                                const SharedPrefixArgs a) {
  using L = DecodeSmem<D, NST>;
  using Warp = MmaWarp<D, BF16>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int csize = static_cast<int>(cluster_nctarank());
  const int crank = static_cast<int>(cluster_ctarank());
  prefetch_tensormap(&kmap);
  prefetch_tensormap(&vmap);
  pdl_launch_dependents();
  pdl_wait();

  // grid slot -> (group, chunk) and KV head; KV heads of one slot are adjacent
  const int item = blockIdx.x / csize;
  const int kvh = item % a.num_kv_heads;
  int slot = item / a.num_kv_heads;
  const int G = a.group;
  if (a.longest_first) {
    // rank every (group, chunk) slot by its page count, longest first (ties
    // by index), and take the one whose rank is this grid slot
    const int U = a.num_groups * a.chunks_per_group;
    int* pages = reinterpret_cast<int*>(smem);       // stage area, not in use yet
    int* chosen = pages + kLptMaxSeqs;
    for (int u = threadIdx.x; u < U; u += kThreads) {
      const int g = u / a.chunks_per_group, c = u % a.chunks_per_group;
      const int b0 = a.group_starts[g], b1 = a.group_starts[g + 1];
      const int p = a.prefix_blocks[g];
      int tail = 0, most = 0;
      const int first_m = b0 + c * a.members_per_chunk;
      const int last_m = min(b1, first_m + a.members_per_chunk);
      if (b0 >= 0 && b1 <= a.num_seqs && p >= 0) {
        for (int sq = first_m; sq < last_m; ++sq) {
          const int np = (max(a.context_lens[sq], 0) + kPage - 1) / kPage;
          most = max(most, np);
          tail += max(0, np - p);
        }
      }
      pages[u] = min(p, most) + tail;
    }
    __syncthreads();
    for (int u = threadIdx.x; u < U; u += kThreads) {
      const int pu = pages[u];
      int rank = 0;
      for (int v = 0; v < U; ++v) {
        const int pv = pages[v];
        rank += (pv > pu) | ((pv == pu) & (v < u));
      }
      if (rank == slot) *chosen = u;
    }
    __syncthreads();
    slot = *chosen;
    fence_proxy_async_smem();  // generic writes to the stage area before TMA writes to it
    __syncthreads();  // the stage area is about to be reused
  }
  const int chunk = slot % a.chunks_per_group;
  const int grp = slot / a.chunks_per_group;
  const bool reporter = threadIdx.x == 0 && crank == 0 && kvh == 0 && chunk == 0;

  // ---- the group and this chunk's members ----
  int s_begin = a.group_starts[grp], s_end = a.group_starts[grp + 1];
  if (s_begin < 0 || s_end < s_begin || s_end > a.num_seqs) {
    if (reporter) record_error(kErrGroup, grp);
    return;  // same decision in every CTA of the cluster
  }
  if (s_end - s_begin > a.chunks_per_group * a.members_per_chunk) {
    if (reporter) record_error(kErrGroup, grp);
    s_end = s_begin + a.chunks_per_group * a.members_per_chunk;
  }
  const int first = s_begin + chunk * a.members_per_chunk;
  const int members = min(a.members_per_chunk, s_end - first);
  if (members <= 0) return;
  const int nrows = members * G;
  int P = a.prefix_blocks[grp];
  if (P < 0 || P > a.max_blocks_per_seq) {
    if (reporter) record_error(kErrGroup, grp);
    P = P < 0 ? 0 : a.max_blocks_per_seq;
  }

  // lane j < members describes member j: its sequence, context length, and
  // the pages of its private tail (table entries P .. P+tail-1)
  const int cap = a.max_blocks_per_seq * kPage;
  int my_ctx = 0;
  if (lane < members) {
    my_ctx = a.context_lens[first + lane];
    if (my_ctx < 0 || my_ctx > cap) {
      if (crank == 0 && kvh == 0) record_error(kErrContextLen, first + lane);
      my_ctx = my_ctx < 0 ? 0 : cap;
    }
  }
  const int my_pages = (my_ctx + kPage - 1) / kPage;
  int most_pages = my_pages;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) most_pages = max(most_pages, __shfl_xor_sync(~0u, most_pages, o));
  int most_ctx = my_ctx;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) most_ctx = max(most_ctx, __shfl_xor_sync(~0u, most_ctx, o));
  const int Pn = min(P, most_pages);                 // prefix pages anyone needs
  const int my_tail = lane < members ? max(0, my_pages - P) : 0;
  int incl = my_tail;                                // inclusive prefix sum of tails
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(~0u, incl, o);
    if (lane >= o) incl += t;
  }
  const int my_off = Pn + incl - my_tail;            // first virtual page of my tail
  const int n_pages = Pn + __shfl_sync(~0u, incl, 31);

  if (n_pages == 0) {  // every member has an empty context
    if (crank == 0) {
      for (int i = threadIdx.x; i < nrows * D; i += kThreads) {
        const int r = i / D;
        a.out[(static_cast<size_t>(first + r / G) * a.num_heads + kvh * G + r % G) * D + i % D] = 0;
      }
    }
    return;
  }

  const bool spread = csize > 1 && n_pages > a.cluster_pages;
  if (csize > 1 && !spread && crank != 0) return;
  const int ctas = spread ? csize : 1;
  const int page0 = (spread ? crank : 0) + ctas * warp;
  const int pstride = ctas * kWarps;
  const int my_count = n_pages > page0 ? (n_pages - page0 + pstride - 1) / pstride : 0;

  // virtual page v -> (member owning it or -1 for the shared prefix, table
  // entry).  Every lane of the warp must call this (the shuffles are
  // warp-wide); v may differ from lane to lane.  The owner of a tail page is
  // the last member whose tail starts at or before it (members with an empty
  // tail share the next member's start and are skipped that way).
  auto locate = [&](int v, int& member, int& entry) {
    int owner = -1, start = Pn;
    for (int j = 0; j < members; ++j) {              // members is warp-uniform
      const int off_j = __shfl_sync(~0u, my_off, j);
      if (off_j <= v) {
        owner = j;
        start = off_j;
      }
    }
    if (v < Pn) {
      member = -1;
      entry = v;
    } else {
      member = owner;
      entry = P + (v - start);
    }
  };

  const uint32_t stage0 = smem_addr(smem) + warp * NST * L::kStageBytes;
  const uint32_t bar0 = smem_addr(smem + L::kBarOffset) + warp * NST * 8;
  if (lane == 0) {
    for (int i = 0; i < NST; ++i) mbar_init(bar0 + i * 8, 1);
    fence_barrier_init();
  }
  __syncwarp();

  // ---- block ids, 32 pages per window, one per lane ----
  auto load_ids = [&](int win) -> int {
    int member, entry;
    const int k = win * 32 + lane;
    const int v = page0 + k * pstride;
    locate(min(v, n_pages - 1), member, entry);      // whole warp takes part
    if (k >= my_count) return -1;
    const int seq = first + (member < 0 ? 0 : member);
    const size_t idx = static_cast<size_t>(seq) * a.max_blocks_per_seq + entry;
    int id = a.block_tables[idx];
    if (id < 0 || id >= a.num_blocks) {
      record_error(kErrBlockId, static_cast<long long>(idx));
      id = -1;
    }
    return id;
  };
  int win = 0;
  int ids_cur = load_ids(0);
  int ids_next = my_count > 32 ? load_ids(1) : -1;

  auto issue = [&](int k) {
    const int src = ((k >> 5) == win) ? ids_cur : ids_next;
    const int id = __shfl_sync(~0u, src, k & 31);
    if (lane == 0) {
      const int st = k % NST;
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
  const int pre = my_count < NST ? my_count : NST;
  for (int k = 0; k < pre; ++k) issue(k);

  // ---- rows: r = member * G + head; lane holds rows r0 = lane/4, r1 = r0 + 8 ----
  Warp st;
  {
    const int r0 = lane >> 2, r1 = r0 + 8, tig = lane & 3;
    const uint16_t* q0 = a.query + (static_cast<size_t>(first + r0 / G) * a.num_heads +
                                    kvh * G + r0 % G) * D;
    const uint16_t* q1 = a.query + (static_cast<size_t>(first + r1 / G) * a.num_heads +
                                    kvh * G + r1 % G) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const int klo = kk * 16 + tig * 2, khi = klo + 8;
      st.qa[kk][0] = r0 < nrows ? *reinterpret_cast<const uint32_t*>(q0 + klo) : 0u;
      st.qa[kk][1] = r1 < nrows ? *reinterpret_cast<const uint32_t*>(q1 + klo) : 0u;
      st.qa[kk][2] = r0 < nrows ? *reinterpret_cast<const uint32_t*>(q0 + khi) : 0u;
      st.qa[kk][3] = r1 < nrows ? *reinterpret_cast<const uint32_t*>(q1 + khi) : 0u;
    }
#pragma unroll
    for (int n = 0; n < D / 8; ++n) st.acc[n][0] = st.acc[n][1] = st.acc[n][2] = st.acc[n][3] = 0.f;
    st.m[0] = st.m[1] = -INFINITY;
    st.l[0] = st.l[1] = 0.f;
  }
  const int mem0 = (lane >> 2) / G, mem1 = ((lane >> 2) + 8) / G;
  const int ctx0 = __shfl_sync(~0u, my_ctx, min(mem0, 31));
  const int ctx1 = __shfl_sync(~0u, my_ctx, min(mem1, 31));
  const bool live0 = (lane >> 2) < nrows, live1 = ((lane >> 2) + 8) < nrows;

  // ---- main loop ----
  bool ok = true;
  int k_stop = my_count;  // first page not consumed
  for (int k = 0; k < my_count; ++k) {
    if (k > 0 && (k & 31) == 0) {
      ++win;
      ids_cur = ids_next;
      ids_next = my_count > (win + 1) * 32 ? load_ids(win + 1) : -1;
    }
    int member, entry;
    locate(page0 + k * pstride, member, entry);
    const int stg = k % NST;
    // the whole warp takes the same branch, whatever each lane's wait saw
    if (!__all_sync(~0u, mbar_wait_bounded(bar0 + stg * 8, (k / NST) & 1))) {
      if (lane == 0) record_error(kErrWaitTimeout, blockIdx.x);
      ok = false;
      k_stop = k;
      break;
    }
    const int lim0 = (live0 && (member < 0 || member == mem0)) ? ctx0 : 0;
    const int lim1 = (live1 && (member < 0 || member == mem1)) ? ctx1 : 0;
    const uint32_t kb = stage0 + stg * L::kStageBytes;
    // rows of this page no row of the item reads: past the owner's context
    // (a tail page) or past every member's (the prefix)
    const int page_lim = member >= 0 ? __shfl_sync(~0u, my_ctx, member) : most_ctx;
    if (entry * kPage + kPage > page_lim && page_lim > entry * kPage)
      zero_page_tail<L::kBoxesPerRow>(kb + L::kPageBytes, page_lim - entry * kPage, lane);
    st.page_rows(kb, kb + L::kPageBytes, entry * kPage, lim0, lim1, a.scale_log2, lane);
    __syncwarp();
    if (k + NST < my_count) issue(k + NST);
  }

  // ---- merge warps (and the cluster's CTAs) and write the rows; loads left
  // in flight by a wait that gave up are drained first (see drain_stages) ----
  if (!__syncthreads_and(drain_stages<NST>(ok, k_stop, my_count, bar0))) {
    if (spread) {
      cluster_sync();
      cluster_sync();
    }
    return;
  }
  float* red_acc = reinterpret_cast<float*>(smem);
  float* red_m = reinterpret_cast<float*>(smem + L::kRedMOffset);
  float* red_l = reinterpret_cast<float*>(smem + L::kRedLOffset);
  if (ok) {
    st.publish(red_acc + warp * nrows * D, red_m + warp * 16, red_l + warp * 16, nrows, lane);
  } else {
    for (int g = lane; g < nrows; g += 32) {
      red_m[warp * 16 + g] = -INFINITY;
      red_l[warp * 16 + g] = 0.f;
    }
  }
  __syncthreads();
  merge_and_emit<D, NST>(smem, nrows, spread, ctas, crank,
                         [&](int r, int d, float o0, float o1, float, float big_l) {
    const size_t hrow = static_cast<size_t>(first + r / G) * a.num_heads + kvh * G + r % G;
    const float inv = big_l > 0.f ? 1.f / big_l : 0.f;
    *reinterpret_cast<uint32_t*>(a.out + hrow * D + d) = pack2<BF16>(o0 * inv, o1 * inv);
  });
}

}  // namespace pa

// pa_cache_reduce.cuh -- the paged cache write and the split-partition merge.
#pragma once

#include "pa_device.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// Cache write ("vllm源码剖析" §一.2 / §一.3): every new token's K and V row
// goes to flat slot slot_mapping[t] of the [num_blocks*block_size, Hk, D]
// view.  One thread moves one 16-byte chunk of K and the same chunk of V;
// consecutive threads walk a token row, so loads and stores are coalesced.
// A pure bit copy.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    reshape_and_cache_kernel(const uint16_t* __restrict__ key, const uint16_t* __restrict__ value,
                             long long key_stride, long long value_stride,
                             uint16_t* __restrict__ key_cache, uint16_t* __restrict__ value_cache,
                             const int64_t* __restrict__ slot_mapping, long long num_tokens,
                             int chunks_per_token, long long num_slots) {
  pdl_launch_dependents();
  pdl_wait();
  const long long total = num_tokens * chunks_per_token;
  const long long row = static_cast<long long>(chunks_per_token) * 8;  // elements per token row
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / chunks_per_token;
    const int c = static_cast<int>(i - t * chunks_per_token);
    const long long slot = slot_mapping[t];
    if (slot < 0) continue;  // padding token
    if (slot >= num_slots) {
      if (c == 0) record_error(kErrSlot, t);
      continue;
    }
    const uint4 k = *reinterpret_cast<const uint4*>(key + t * key_stride + c * 8);
    const uint4 v = *reinterpret_cast<const uint4*>(value + t * value_stride + c * 8);
    *reinterpret_cast<uint4*>(key_cache + slot * row + c * 8) = k;
    *reinterpret_cast<uint4*>(value_cache + slot * row + c * 8) = v;
  }
}

// ---------------------------------------------------------------------------
// Block copy for copy-on-write ("vllm源码分析" 第一讲, "vLLM PagedAttention
// 原理与源码深度解析" §3.3): before a sequence writes into a block it shares,
// the block is copied to a private one.  Pair i copies block mapping[2i] onto
// block mapping[2i+1] in both caches; one thread moves one 16-byte unit of K
// and the same unit of V, consecutive threads walk a block.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ key_cache, uint4* __restrict__ value_cache,
                       const int64_t* __restrict__ mapping, long long num_pairs,
                       long long units_per_block, long long num_blocks) {
  pdl_launch_dependents();
  pdl_wait();
  const long long total = num_pairs * units_per_block;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long pair = i / units_per_block;
    const long long u = i - pair * units_per_block;
    const long long src = mapping[2 * pair], dst = mapping[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
      if (u == 0) record_error(kErrBlockId, pair);
      continue;
    }
    key_cache[dst * units_per_block + u] = key_cache[src * units_per_block + u];
    value_cache[dst * units_per_block + u] = value_cache[src * units_per_block + u];
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of split partitions.  One CTA per (sequence, query head):
//   M = max_p m_p;  w_p = exp(m_p - M);  out = sum_p w_p acc_p / sum_p w_p l_p.
// Single pass: thread t owns the float4 column t % (D/4) of every
// (threads/(D/4))-th partition and merges them online (running max, with the
// partial sum and accumulator rescaled when the max grows), loading
// kReduceBatch partitions before using any so that the loads overlap.  The
// partition groups are then merged through shared memory the same way.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 256;
constexpr int kReduceBatch = 8;

template <bool BF16>
__global__ void __launch_bounds__(kReduceThreads)
    lse_reduce_kernel(uint16_t* __restrict__ out, const float* __restrict__ tmp_out,
                      const float* __restrict__ max_logits, const float* __restrict__ exp_sums,
                      const int32_t* __restrict__ context_lens, int num_heads, int head_dim,
                      int partition_size, int max_partitions) {
  __shared__ float4 acc_sh[kReduceThreads];
  __shared__ float m_sh[kReduceThreads];
  __shared__ float l_sh[kReduceThreads];
  pdl_launch_dependents();
  pdl_wait();
  const int sh = blockIdx.x;  // s * num_heads + h
  const int s = sh / num_heads;
  const int tid = threadIdx.x;

  int ctx = context_lens[s];
  if (ctx < 0) ctx = 0;
  int nparts = (ctx + partition_size - 1) / partition_size;
  if (nparts > max_partitions) nparts = max_partitions;  // flagged by the split kernel
  const size_t base = static_cast<size_t>(sh) * max_partitions;
  uint16_t* o = out + static_cast<size_t>(sh) * head_dim;
  if (nparts == 0) {
    for (int d = tid * 2; d < head_dim; d += kReduceThreads * 2)
      *reinterpret_cast<uint32_t*>(o + d) = 0u;
    return;
  }

  const int quads = head_dim >> 2;                 // float4 columns per row
  const int groups = kReduceThreads / quads;       // partition groups (head_dim <= 4*threads)
  const int q = tid % quads, grp = tid / quads;
  float m = -INFINITY, l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (grp < groups) {
    const float4* rows = reinterpret_cast<const float4*>(tmp_out + base * head_dim) + q;
    for (int p0 = grp; p0 < nparts; p0 += groups * kReduceBatch) {
      float mp[kReduceBatch], lp[kReduceBatch];
      float4 v[kReduceBatch];
#pragma unroll
      for (int u = 0; u < kReduceBatch; ++u) {
        const int p = p0 + u * groups;
        if (p < nparts) {
          mp[u] = __ldg(max_logits + base + p);
          lp[u] = __ldg(exp_sums + base + p);
          v[u] = __ldg(rows + static_cast<size_t>(p) * quads);
        }
      }
#pragma unroll
      for (int u = 0; u < kReduceBatch; ++u) {
        if (p0 + u * groups < nparts) {
          const float mn = fmaxf(m, mp[u]);
          const float sc = ex2((m - mn) * kLog2e);     // 0 while m is still -inf
          const float e = ex2((mp[u] - mn) * kLog2e);
          acc.x = acc.x * sc + e * v[u].x;
          acc.y = acc.y * sc + e * v[u].y;
          acc.z = acc.z * sc + e * v[u].z;
          acc.w = acc.w * sc + e * v[u].w;
          l = l * sc + e * lp[u];
          m = mn;
        }
      }
    }
  }
  acc_sh[tid] = acc;
  m_sh[tid] = m;
  l_sh[tid] = l;
  __syncthreads();
  if (tid < quads) {
    float big_m = -INFINITY;
    for (int g = 0; g < groups; ++g) big_m = fmaxf(big_m, m_sh[g * quads + tid]);
    float big_l = 0.f;
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g = 0; g < groups; ++g) {
      const float mg = m_sh[g * quads + tid];
      if (mg == -INFINITY) continue;                 // a group without partitions
      const float e = ex2((mg - big_m) * kLog2e);
      const float4 u = acc_sh[g * quads + tid];
      t.x += e * u.x; t.y += e * u.y; t.z += e * u.z; t.w += e * u.w;
      big_l += e * l_sh[g * quads + tid];
    }
    const float inv = big_l > 0.f ? 1.f / big_l : 0.f;
    uint2 packed;
    packed.x = pack2<BF16>(t.x * inv, t.y * inv);
    packed.y = pack2<BF16>(t.z * inv, t.w * inv);
    *reinterpret_cast<uint2*>(o + tid * 4) = packed;
  }
}

}  // namespace pa

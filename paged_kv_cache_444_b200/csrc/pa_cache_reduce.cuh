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
// Log-sum-exp merge of split partitions.  One CTA per (sequence, query head):
//   M = max_p m_p;  w_p = exp(m_p - M);  out = sum_p w_p acc_p / sum_p w_p l_p.
// The weights go to shared memory (kReduceChunk partitions at a time).  The
// partial accumulators are read as float4: thread t owns dims 4*(t % (D/4))
// of every kReduceThreads/(D/4)-th partition, with kReduceUnroll independent
// loads in flight, and the partition groups are summed through shared memory.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 128;
constexpr int kReduceChunk = 1024;
constexpr int kReduceUnroll = 4;

template <bool BF16>
__global__ void __launch_bounds__(kReduceThreads)
    lse_reduce_kernel(uint16_t* __restrict__ out, const float* __restrict__ tmp_out,
                      const float* __restrict__ max_logits, const float* __restrict__ exp_sums,
                      const int32_t* __restrict__ context_lens, int num_heads, int head_dim,
                      int partition_size, int max_partitions) {
  __shared__ float w_sh[kReduceChunk];
  __shared__ float red[kReduceThreads / 32];
  __shared__ float4 part_sh[kReduceThreads];
  const int sh = blockIdx.x;  // s * num_heads + h
  const int s = sh / num_heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

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

  // M = max over partitions
  float mloc = -INFINITY;
  for (int p = tid; p < nparts; p += kReduceThreads) mloc = fmaxf(mloc, max_logits[base + p]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, off));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  float big_m = red[0];
#pragma unroll
  for (int w = 1; w < kReduceThreads / 32; ++w) big_m = fmaxf(big_m, red[w]);
  __syncthreads();

  const int quads = head_dim >> 2;                 // float4 columns per row
  const int groups = kReduceThreads / quads;       // partition groups (head_dim <= 4*threads)
  const int q = tid % quads, grp = tid / quads;
  const bool active = grp < groups;
  float lsum = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = 0; c0 < nparts; c0 += kReduceChunk) {
    const int n = min(kReduceChunk, nparts - c0);
    for (int p = tid; p < n; p += kReduceThreads) {
      const float w = ex2((max_logits[base + c0 + p] - big_m) * kLog2e);
      w_sh[p] = w;
      lsum += w * exp_sums[base + c0 + p];
    }
    __syncthreads();
    if (active) {
      const float4* src = reinterpret_cast<const float4*>(tmp_out + (base + c0) * head_dim) + q;
      int p = grp;
      for (; p + (kReduceUnroll - 1) * groups < n; p += kReduceUnroll * groups) {
        float4 v[kReduceUnroll];
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u)
          v[u] = __ldg(src + static_cast<size_t>(p + u * groups) * quads);
#pragma unroll
        for (int u = 0; u < kReduceUnroll; ++u) {
          const float w = w_sh[p + u * groups];
          acc.x += w * v[u].x; acc.y += w * v[u].y; acc.z += w * v[u].z; acc.w += w * v[u].w;
        }
      }
      for (; p < n; p += groups) {
        const float4 v = __ldg(src + static_cast<size_t>(p) * quads);
        const float w = w_sh[p];
        acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  if (lane == 0) red[warp] = lsum;
  part_sh[tid] = acc;
  __syncthreads();
  float big_l = 0.f;
#pragma unroll
  for (int w = 0; w < kReduceThreads / 32; ++w) big_l += red[w];
  const float inv = big_l > 0.f ? 1.f / big_l : 0.f;
  if (tid < quads) {
    float4 t = part_sh[tid];
    for (int g = 1; g < groups; ++g) {
      const float4 u = part_sh[g * quads + tid];
      t.x += u.x; t.y += u.y; t.z += u.z; t.w += u.w;
    }
    uint2 packed;
    packed.x = pack2<BF16>(t.x * inv, t.y * inv);
    packed.y = pack2<BF16>(t.z * inv, t.w * inv);
    *reinterpret_cast<uint2*>(o + tid * 4) = packed;
  }
}

}  // namespace pa

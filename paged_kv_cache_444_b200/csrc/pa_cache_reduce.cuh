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
// The weights are computed once per partition into shared memory (in chunks
// of kReduceChunk partitions); each thread then owns two output dims and
// walks the partitions with coalesced loads.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 128;
constexpr int kReduceChunk = 1024;

template <bool BF16>
__global__ void __launch_bounds__(kReduceThreads)
    lse_reduce_kernel(uint16_t* __restrict__ out, const float* __restrict__ tmp_out,
                      const float* __restrict__ max_logits, const float* __restrict__ exp_sums,
                      const int32_t* __restrict__ context_lens, int num_heads, int head_dim,
                      int partition_size, int max_partitions) {
  __shared__ float w_sh[kReduceChunk];
  __shared__ float red[kReduceThreads / 32];
  const int sh = blockIdx.x;  // s * num_heads + h
  const int s = sh / num_heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  int ctx = context_lens[s];
  if (ctx < 0) ctx = 0;
  int nparts = (ctx + partition_size - 1) / partition_size;
  if (nparts > max_partitions) nparts = max_partitions;  // flagged by the split kernel
  const size_t base = static_cast<size_t>(sh) * max_partitions;
  uint16_t* o = out + static_cast<size_t>(sh) * head_dim;
  const int d = tid * 2;
  if (nparts == 0) {
    if (d < head_dim) *reinterpret_cast<uint32_t*>(o + d) = 0u;
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

  float lsum = 0.f;
  float2 acc = make_float2(0.f, 0.f);
  for (int c0 = 0; c0 < nparts; c0 += kReduceChunk) {
    const int n = min(kReduceChunk, nparts - c0);
    for (int p = tid; p < n; p += kReduceThreads) {
      const float w = ex2((max_logits[base + c0 + p] - big_m) * kLog2e);
      w_sh[p] = w;
      lsum += w * exp_sums[base + c0 + p];
    }
    __syncthreads();
    if (d < head_dim) {
      const float* src = tmp_out + (base + c0) * head_dim + d;
      for (int p = 0; p < n; ++p) {
        const float2 v = *reinterpret_cast<const float2*>(src + static_cast<size_t>(p) * head_dim);
        acc.x += w_sh[p] * v.x;
        acc.y += w_sh[p] * v.y;
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  if (lane == 0) red[warp] = lsum;
  __syncthreads();
  float big_l = 0.f;
#pragma unroll
  for (int w = 0; w < kReduceThreads / 32; ++w) big_l += red[w];
  if (d < head_dim) {
    const float inv = big_l > 0.f ? 1.f / big_l : 0.f;
    *reinterpret_cast<uint32_t*>(o + d) = pack2<BF16>(acc.x * inv, acc.y * inv);
  }
}

}  // namespace pa

// pa_device.cuh -- device-side building blocks for the sm_100a paged-attention
// kernels: the per-device error word, shared-memory barriers, TMA tile loads,
// ldmatrix / mma.sync wrappers and 16-bit <-> fp32 conversions.
//
// Everything here is inline PTX or CUDA intrinsics written for this library.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// ---------------------------------------------------------------------------
// Error word: the first out-of-range index a kernel meets, per device.
// (code << 56) | index; 0 = clean.  Read and cleared by pa_check_error.
// ---------------------------------------------------------------------------
__device__ unsigned long long g_error_word;

__device__ __forceinline__ void record_error(unsigned code, long long index) {
  const unsigned long long v = (static_cast<unsigned long long>(code) << 56) |
                               (static_cast<unsigned long long>(index) & ((1ull << 56) - 1));
  atomicCAS(&g_error_word, 0ull, v);
}

constexpr unsigned kErrSlot = 1, kErrBlockId = 2, kErrContextLen = 3, kErrPartitions = 4,
                   kErrWaitTimeout = 5;

// A barrier wait gives up after this long (no legitimate wait comes close).
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// mbarrier (shared-memory transaction barrier)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(bar), "r"(bytes) : "memory");
}

// Plain arrival (one count) on a barrier.
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of the barrier; false if it did not complete within
// kWaitLimitNs (the caller records the error and stops using the stage).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA: 4-D tiled tensor load global -> shared, completion on an mbarrier.
// No multicast.  Out-of-range boxes are zero-filled by the hardware.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA, tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Zero rows [row0, 16) of a staged page (BOXES boxes of 16 rows x 128 B, whole
// warp).  Cache rows past a sequence's context were never written and may
// hold anything; their probability is 0, and 0 * NaN must not reach O.  The
// proxy fence orders these writes before a later TMA refill of the stage.
template <int BOXES>
__device__ __forceinline__ void zero_page_tail(uint32_t page, int row0, int lane) {
  const int chunks = (16 - row0) * 8;
  for (int i = lane; i < chunks * BOXES; i += 32) {
    const int b = i / chunks, c = i % chunks;
    sts128(page + b * 2048 + row0 * 128 + c * 16, 0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  __syncwarp();
}

// ---------------------------------------------------------------------------
// Shared-memory loads
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Transpose of an 8 x 8 matrix of 16-bit elements held in the mma fragment
// layout (lane l: row l / 4, elements 2(l % 4) and 2(l % 4) + 1).  Whole warp.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ---------------------------------------------------------------------------
// mma.sync m16n8k16, fp32 accumulate, A row-major / B column-major.
// ---------------------------------------------------------------------------
template <bool BF16>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialisation may start while the previous kernel of its stream is still
// running; pdl_wait() blocks until that kernel has completed and its writes
// are visible (a no-op for a normal launch).  Every kernel here calls it
// before its first read of any input, and calls pdl_launch_dependents() early
// so that the next kernel can be scheduled during its own tail.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, size, barrier, distributed shared memory.
// Without a cluster launch a CTA is a cluster of one (rank 0, size 1).
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned cluster_ctarank() {
  unsigned r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ unsigned cluster_nctarank() {
  unsigned n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}

// Every thread of every CTA in the cluster must call this (same count).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-memory address `addr` of this CTA, mapped into CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_cluster(uint32_t addr, unsigned rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float2 ld_cluster_f32x2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared::cluster.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// Arithmetic helpers
// ---------------------------------------------------------------------------
// 2^x with the hardware approximation (relative error ~2^-22); 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  return __ffma2_rn(a, b, make_float2(0.f, 0.f));
}

// Two packed 16-bit values (low half first) -> two floats, exactly.
template <bool BF16>
__device__ __forceinline__ float2 unpack2(uint32_t u) {
  if constexpr (BF16) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
  } else {
    __half2 h = *reinterpret_cast<__half2*>(&u);
    return __half22float2(h);
  }
}

// Two floats -> two packed 16-bit values (low half = lo), round to nearest even.
template <bool BF16>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (BF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

// Two E4M3 values (low byte first) -> half2, exactly (E4M3 is a subset of fp16).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t pair16) {
  uint32_t h;
  const unsigned short p = static_cast<unsigned short>(pair16 & 0xffffu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(p));
  return h;
}

// Two E4M3 values -> the packed 16-bit operand type of the mma (fp16 or bf16),
// exactly: E4M3 -> fp16 is exact, and fp16 values of E4M3 range are exact in bf16.
template <bool BF16>
__device__ __forceinline__ uint32_t e4m3x2_to_op2(uint32_t pair16) {
  const uint32_t h = e4m3x2_to_h2(pair16);
  if constexpr (BF16) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<uint32_t*>(&b);
  } else {
    return h;
  }
}

// Two E4M3 values -> two floats, exactly.
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t pair16) {
  const uint32_t h = e4m3x2_to_h2(pair16);
  return __half22float2(*reinterpret_cast<const __half2*>(&h));
}

// Two floats -> two E4M3 (low byte = lo), nearest even, saturating to +-448.
__device__ __forceinline__ uint32_t f2_to_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace pa

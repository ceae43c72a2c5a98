// pa_api.cu -- the extern "C" entry points of libpa (declared in include/pa.h):
// host-side argument validation, TMA tensor-map encoding, kernel selection
// and launch on the caller's stream.  The library allocates nothing and keeps
// no state beyond the per-device error word and per-device kernel attributes.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <map>
#include <mutex>
#include <utility>

#include "pa.h"
#include "pa_cache_reduce.cuh"
#include "pa_decode.cuh"
#include "pa_decode_fp8.cuh"

namespace {

using namespace pa;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// cuTensorMapEncodeTiled, fetched once through the runtime (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 4-D view of a cache [num_blocks, 16, Hk, D] for 16 x 64-element page boxes:
//   dim0: 64 elements (128 B, contiguous)
//   dim1: D/64 column boxes of a row      stride 128 B
//   dim2: Hk KV heads                      stride D*2 B
//   dim3: num_blocks*16 token rows         stride Hk*D*2 B
// box {64, 1, 1, 16}, 128-byte swizzle, zero fill out of range.
bool encode_cache_map(CUtensorMap* map, const void* cache, pa_dtype dtype, int64_t num_blocks,
                      int64_t num_kv_heads, int64_t head_dim, int elem_bytes = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t per_box = 128 / elem_bytes;   // elements in one 128-byte box row
  const cuuint64_t dims[4] = {per_box, static_cast<cuuint64_t>(head_dim * elem_bytes / 128),
                              static_cast<cuuint64_t>(num_kv_heads),
                              static_cast<cuuint64_t>(num_blocks * kPage)};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(head_dim * elem_bytes),
                                 static_cast<cuuint64_t>(num_kv_heads * head_dim * elem_bytes)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(per_box), 1, 1, kPage};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType type = elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                      : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  const CUresult r = fn(map, type,
                        4, const_cast<void*>(cache), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <class K>
bool ensure_smem(K kernel, int bytes, std::atomic<uint64_t>* done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  const uint64_t bit = 1ull << dev;
  if (done_mask->load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done_mask->fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Launch as clusters of `cluster` CTAs along x when cluster > 1; a plain
// launch otherwise, with programmatic stream serialisation if `programmatic`
// (the kernel may start while the previous kernel of the stream drains; every
// kernel here waits for it with griddepcontrol.wait before reading inputs).
template <class K, class... Args>
pa_status launch_cfg(K kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                     int cluster, bool programmatic, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int n = 0;
  if (cluster > 1) {
    attrs[n].id = cudaLaunchAttributeClusterDimension;
    attrs[n].val.clusterDim.x = cluster;
    attrs[n].val.clusterDim.y = 1;
    attrs[n].val.clusterDim.z = 1;
    ++n;
  } else if (programmatic) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
    cudaGetLastError();
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <class K, class... Args>
pa_status launch_ex(K kernel, unsigned grid, unsigned block, size_t smem, cudaStream_t stream,
                    int cluster, Args... args) {
  return launch_cfg(kernel, grid, block, smem, stream, cluster, true, args...);
}

// Pipeline depth per head_dim: stages of (K page + V page) per warp.
#ifndef PA_STAGES_D128
#define PA_STAGES_D128 2
#endif
#ifndef PA_STAGES_D64
#define PA_STAGES_D64 4
#endif
#ifndef PA_STAGES_FP8
#define PA_STAGES_FP8 4  // fp8 pages are half the bytes: twice the stages in the same space
#endif
#ifndef PA_STAGES_FP8_T
#define PA_STAGES_FP8_T 3  // transposed fp8 page step: four CTAs per SM share the space
#endif
template <int D>
struct Stages { static constexpr int value = D == 64 ? PA_STAGES_D64 : PA_STAGES_D128; };

// 16-bit split launches go persistent past this many waves of resident CTAs
constexpr long long kPersistWaves = 64;

#ifndef PA_SPLIT_PERSISTENT
#define PA_SPLIT_PERSISTENT 1  // fp8 split launches: one wave of CTAs over the items that exist
#endif
#ifndef PA_CLUSTER_PAGES
#define PA_CLUSTER_PAGES 256  // an item with more pages is spread over its cluster
#endif
#ifndef PA_CLUSTER_TABLE_PAGES
#define PA_CLUSTER_TABLE_PAGES 512  // clusters only when a table can hold more pages
#endif
#ifndef PA_CLUSTER_FILL_PAGES
#define PA_CLUSTER_FILL_PAGES 32  // pairs fit in the resident slots: spread items longer than this
#endif

// Cluster size for a single-pass launch.  Clusters are used only when the
// block table admits very long sequences (more than PA_CLUSTER_TABLE_PAGES
// pages): then every item longer than PA_CLUSTER_PAGES pages is spread so that
// the longest possible one gives each CTA about PA_CLUSTER_TABLE_PAGES pages.
// (launch_decode_t also asks for pairs when twice the grid fits in the
// resident CTA slots.)  A power of two, at most kMaxCluster, and no more than the device can
// co-schedule for this kernel.
template <class K>
int pick_cluster(K kernel, int smem_bytes, int64_t max_pages, std::atomic<int>* cache) {
  int want = 1;
  while (want < kMaxCluster && static_cast<int64_t>(want) * PA_CLUSTER_TABLE_PAGES < max_pages)
    want *= 2;
  int dev = 0;
  if (want == 1 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  int known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {  // largest schedulable cluster size for this kernel on this device
    int best = 1;
    for (int c = kMaxCluster; c > 1; c /= 2) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem_bytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = c;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) == cudaSuccess && n > 0) {
        best = c;
        break;
      }
      cudaGetLastError();
    }
    cache[dev].store(best, std::memory_order_relaxed);  // every thread finds the same value
    known = best;
  }
  return want < known ? want : known;
}

// CTAs of `kernel` that fit on the device at once (SMs x resident CTAs per SM),
// looked up once per device; 0 if the query fails.
template <class K>
long long resident_ctas(K kernel, int smem_bytes, std::atomic<long long>* cache) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  long long known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem_bytes) !=
            cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    known = static_cast<long long>(per_sm) * sms;
    cache[dev].store(known, std::memory_order_relaxed);
  }
  return known;
}

template <int D, bool BF16, class Warp, int EB = 2,
          int NST = (EB == 1 ? PA_STAGES_FP8 : Stages<D>::value)>
pa_status launch_decode_t(const CUtensorMap& km, const CUtensorMap& vm, DecodeArgs a,
                          long long grid, int64_t max_pages, cudaStream_t stream) {
  using L = DecodeSmem<D, NST, EB>;
  auto kernel = paged_decode_kernel<D, NST, BF16, Warp, EB>;
  static std::atomic<uint64_t> done{0};
  static std::atomic<int> cluster_cache[kMaxDevices] = {};
  const bool split = a.tmp_out != nullptr;
  {
    static std::atomic<uint64_t> done_persist{0};
    static std::atomic<long long> resident_cache[kMaxDevices] = {};
    auto kernel_persist = paged_decode_persistent_kernel<D, NST, BF16, Warp, EB>;
    if (split && a.persistent) {
      // one wave of CTAs loops over the items that exist (at most `grid`):
      // always for the fp8 pages; for 16-bit pages only when the grid over
      // every possible partition would run past kPersistWaves waves (a long
      // table, where most of those CTAs would find their partition empty)
      if (!ensure_smem(kernel_persist, L::kAlloc, &done_persist)) return PA_ERR_CUDA;
      const long long resident = resident_ctas(kernel_persist, L::kAlloc, resident_cache);
      if (resident > 0 && (EB == 1 || grid > kPersistWaves * resident)) {
        if (grid > resident) grid = resident;
        // in stream order, not programmatically: a persistent grid wants all
        // its CTAs resident together, and an early launch lets its first CTAs
        // take the slots the previous kernel leaves while the rest wait (the
        // fp8 long-context split + reduce, back to back: 324 us, against 245)
        return launch_cfg(kernel_persist, static_cast<unsigned>(grid), kThreads, L::kAlloc,
                          stream, 1, false, km, vm, a);
      }
      a.persistent = 0;
    }
  }
  if (!ensure_smem(kernel, L::kAlloc, &done)) return PA_ERR_CUDA;
  int c = split ? 1 : pick_cluster(kernel, L::kAlloc, max_pages, cluster_cache);
  a.cluster_pages = PA_CLUSTER_PAGES;
  if (!split && c == 1 && max_pages > PA_CLUSTER_FILL_PAGES) {
    // a grid whose CTA pairs all fit in the resident slots leaves half of
    // them idle: the items longer than PA_CLUSTER_FILL_PAGES are spread over
    // pairs so that they use them (32 fp8 sequences x 8 KV heads on 592
    // slots: 51.2 -> 40.6 us).  With more items some pairs would wait for a
    // second wave, which measured up to 39 % slower on uniform batches
    static std::atomic<long long> fill_resident[kMaxDevices] = {};
    const long long resident = resident_ctas(kernel, L::kAlloc, fill_resident);
    if (resident > 0 && 2 * grid <= resident) {
      c = pick_cluster(kernel, L::kAlloc, 2 * static_cast<int64_t>(PA_CLUSTER_TABLE_PAGES),
                       cluster_cache);
      a.cluster_pages = PA_CLUSTER_FILL_PAGES;
    }
  }
  if (grid * c > INT32_MAX) return PA_ERR_SHAPE;
  return launch_ex(kernel, static_cast<unsigned>(grid * c), kThreads, L::kAlloc, stream, c, km,
                   vm, a);
}

template <int D, bool BF16>
pa_status launch_decode_d(const CUtensorMap& km, const CUtensorMap& vm, const DecodeArgs& a,
                          long long grid, int64_t max_pages, cudaStream_t stream) {
  if (a.group <= 8)
    return launch_decode_t<D, BF16, MmaWarpT<D, BF16>>(km, vm, a, grid, max_pages, stream);
  return launch_decode_t<D, BF16, MmaWarp<D, BF16>>(km, vm, a, grid, max_pages, stream);
}

// Shared validation of the attention arguments (host only, no CUDA calls).
pa_status check_attention_args(const void* query, const void* key_cache, const void* value_cache,
                               const int32_t* block_tables, const int32_t* context_lens,
                               float scale, int64_t num_seqs, int64_t num_heads,
                               int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                               int64_t block_size, int64_t max_blocks_per_seq, pa_dtype dtype) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
      block_size <= 0 || max_blocks_per_seq <= 0)
    return PA_ERR_SHAPE;
  if (num_heads % num_kv_heads != 0) return PA_ERR_SHAPE;
  if (!std::isfinite(scale)) return PA_ERR_SHAPE;
  if (num_seqs > 0 && (!query || !key_cache || !value_cache || !block_tables || !context_lens))
    return PA_ERR_NULL;
  if (head_dim % 8 != 0) return PA_ERR_ALIGN;
  if (num_seqs > 0 && (!aligned16(query) || !aligned16(key_cache) || !aligned16(value_cache)))
    return PA_ERR_ALIGN;
  if (num_seqs > 0 && ((reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
                        (reinterpret_cast<uintptr_t>(context_lens) & 3u)))
    return PA_ERR_ALIGN;
  if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (block_size != kPage) return PA_ERR_UNSUPPORTED;
  if (num_heads / num_kv_heads > 16) return PA_ERR_UNSUPPORTED;
  // index ranges the kernels address with 32-bit ints
  if (num_blocks * kPage > INT32_MAX || max_blocks_per_seq * kPage > INT32_MAX ||
      num_heads > 65535 || num_seqs * num_heads > INT32_MAX)
    return PA_ERR_SHAPE;
  return PA_OK;
}

pa_status run_decode(DecodeArgs a, const void* key_cache, const void* value_cache,
                     int64_t num_seqs, int64_t head_dim, int64_t num_blocks, pa_dtype dtype,
                     cudaStream_t stream) {
  CUtensorMap km, vm;
  if (!encode_cache_map(&km, key_cache, dtype, num_blocks, a.num_kv_heads, head_dim) ||
      !encode_cache_map(&vm, value_cache, dtype, num_blocks, a.num_kv_heads, head_dim))
    return PA_ERR_CUDA;
  const long long grid = num_seqs * a.num_kv_heads * static_cast<long long>(a.parts_per_head);
  if (grid > INT32_MAX) return PA_ERR_SHAPE;
  // 16-bit split launches keep the grid over every possible partition unless
  // it runs past kPersistWaves waves: the persistent form measured 3-4 %
  // slower on full tables, and 3.3x faster on a skewed one (one 128K-token
  // sequence among 255 of 1K, 524 288 possible partitions)
  a.num_seqs = static_cast<int>(num_seqs);
  a.persistent = PA_SPLIT_PERSISTENT && a.tmp_out != nullptr;
  const bool bf16 = dtype == PA_BF16;
  const int64_t max_pages = a.max_blocks_per_seq;  // block_size == 16 == one page
  if (head_dim == 64)
    return bf16 ? launch_decode_d<64, true>(km, vm, a, grid, max_pages, stream)
                : launch_decode_d<64, false>(km, vm, a, grid, max_pages, stream);
  return bf16 ? launch_decode_d<128, true>(km, vm, a, grid, max_pages, stream)
              : launch_decode_d<128, false>(km, vm, a, grid, max_pages, stream);
}

// >>> fp8 KV cache launch: decode over E4M3 caches (head_dim 128), same
// kernel, fp8 page steps.
pa_status run_decode_fp8(DecodeArgs a, const void* key_cache, const void* value_cache,
                         int64_t num_seqs, int64_t num_blocks, pa_dtype dtype,
                         cudaStream_t stream) {
  CUtensorMap km, vm;
  if (!encode_cache_map(&km, key_cache, dtype, num_blocks, a.num_kv_heads, 128, 1) ||
      !encode_cache_map(&vm, value_cache, dtype, num_blocks, a.num_kv_heads, 128, 1))
    return PA_ERR_CUDA;
  const long long grid = num_seqs * a.num_kv_heads * static_cast<long long>(a.parts_per_head);
  if (grid > INT32_MAX) return PA_ERR_SHAPE;
  // fp8 split launches: one persistent wave of CTAs over the partitions that
  // exist (measured 2.5-7 % faster than the grid over every possible
  // partition; the fp8 items are short)
  a.num_seqs = static_cast<int>(num_seqs);
  a.persistent = PA_SPLIT_PERSISTENT && a.tmp_out != nullptr;
  const int64_t max_pages = a.max_blocks_per_seq;
  if (dtype == PA_BF16) {
    if (a.group <= 8)
      return launch_decode_t<128, true, MmaFp8WarpT<128, true>, 1, PA_STAGES_FP8_T>(
          km, vm, a, grid, max_pages, stream);
    return launch_decode_t<128, true, MmaFp8Warp<128, true>, 1>(km, vm, a, grid, max_pages,
                                                                     stream);
  }
  if (a.group <= 8)
    return launch_decode_t<128, false, MmaFp8WarpT<128, false>, 1, PA_STAGES_FP8_T>(
        km, vm, a, grid, max_pages, stream);
  return launch_decode_t<128, false, MmaFp8Warp<128, false>, 1>(km, vm, a, grid, max_pages,
                                                                     stream);
}
// <<< fp8 KV cache launch

pa_status check_fp8_scales(float k_scale, float v_scale) {
  if (!std::isfinite(k_scale) || !std::isfinite(v_scale) || !(k_scale > 0.f) || !(v_scale > 0.f))
    return PA_ERR_SHAPE;
  return PA_OK;
}

DecodeArgs make_args(const void* query, const int32_t* block_tables, const int32_t* context_lens,
                     float scale, int64_t num_heads, int64_t num_kv_heads,
                     int64_t max_blocks_per_seq, int64_t num_blocks) {
  DecodeArgs a{};
  a.query = static_cast<const uint16_t*>(query);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.scale_log2 = scale * kLog2e;
  a.v_scale = 1.0f;
  a.num_heads = static_cast<int>(num_heads);
  a.num_kv_heads = static_cast<int>(num_kv_heads);
  a.group = static_cast<int>(num_heads / num_kv_heads);
  a.max_blocks_per_seq = static_cast<int>(max_blocks_per_seq);
  a.num_blocks = static_cast<int>(num_blocks);
  a.partition_size = 0;
  a.parts_per_head = 1;
  a.max_partitions = 1;
  a.num_seqs = 0;
  a.longest_first = 0;
  return a;
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status status) {
  switch (status) {
    case PA_OK: return "ok";
    case PA_ERR_NULL: return "null pointer";
    case PA_ERR_SHAPE: return "bad shape or size";
    case PA_ERR_DTYPE: return "unknown dtype";
    case PA_ERR_ALIGN: return "misaligned pointer or stride";
    case PA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PA_ERR_CUDA: return "CUDA error";
    case PA_ERR_BOUNDS: return "out-of-range index met on the device";
  }
  return "unknown status";
}

int32_t pa_abi_version(void) { return (1 << 16) | 0; }

pa_status pa_reshape_and_cache(const void* key, const void* value, int64_t key_stride,
                               int64_t value_stride, void* key_cache, void* value_cache,
                               const int64_t* slot_mapping, int64_t num_tokens,
                               int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                               int64_t block_size, pa_dtype dtype, void* stream) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
    return PA_ERR_SHAPE;
  const int64_t row = num_kv_heads * head_dim;
  if (key_stride < row || value_stride < row) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
  if (head_dim % 8 != 0 || key_stride % 8 != 0 || value_stride % 8 != 0) return PA_ERR_ALIGN;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_ALIGN;
  const int64_t chunks = row / 8;
  if (chunks > INT32_MAX) return PA_ERR_SHAPE;
  const int64_t total = num_tokens * chunks;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;  // grid-stride beyond 32 CTAs per SM
  return launch_ex(reshape_and_cache_kernel, static_cast<unsigned>(blocks), threads, 0,
                   as_stream(stream), 1, static_cast<const uint16_t*>(key),
                   static_cast<const uint16_t*>(value), static_cast<long long>(key_stride),
                   static_cast<long long>(value_stride), static_cast<uint16_t*>(key_cache),
                   static_cast<uint16_t*>(value_cache), slot_mapping,
                   static_cast<long long>(num_tokens), static_cast<int>(chunks),
                   static_cast<long long>(num_blocks * block_size));
}

pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_mapping,
                         int64_t num_pairs, int64_t num_blocks, int64_t block_size,
                         int64_t num_kv_heads, int64_t head_dim, int64_t elem_bytes,
                         void* stream) {
  if (num_pairs < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || (elem_bytes != 1 && elem_bytes != 2))
    return PA_ERR_SHAPE;
  if (num_pairs == 0) return PA_OK;
  if (!key_cache || !value_cache || !block_mapping) return PA_ERR_NULL;
  const int64_t block_bytes = block_size * num_kv_heads * head_dim * elem_bytes;
  if (block_bytes % 16 != 0 || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
    return PA_ERR_ALIGN;
  const int64_t units = block_bytes / 16;
  const int64_t total = num_pairs * units;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  return launch_ex(copy_blocks_kernel, static_cast<unsigned>(blocks), threads, 0,
                   as_stream(stream), 1, static_cast<uint4*>(key_cache),
                   static_cast<uint4*>(value_cache), block_mapping,
                   static_cast<long long>(num_pairs), static_cast<long long>(units),
                   static_cast<long long>(num_blocks));
}

pa_status pa_decode(void* out, const void* query, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, const int32_t* context_lens, float scale,
                    int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads, int64_t head_dim,
                    int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq,
                    pa_dtype dtype, void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if (num_seqs == 0) return PA_OK;
  if (!out) return PA_ERR_NULL;
  if (!aligned16(out)) return PA_ERR_ALIGN;
  DecodeArgs a = make_args(query, block_tables, context_lens, scale, num_heads, num_kv_heads,
                           max_blocks_per_seq, num_blocks);
  a.out = static_cast<uint16_t*>(out);
  a.num_seqs = static_cast<int>(num_seqs);
  a.longest_first = num_seqs > 1 && num_seqs <= kLptMaxSeqs;
  return run_decode(a, key_cache, value_cache, num_seqs, head_dim, num_blocks, dtype,
                    as_stream(stream));
}

pa_status pa_decode_split(float* tmp_out, float* max_logits, float* exp_sums, const void* query,
                          const void* key_cache, const void* value_cache,
                          const int32_t* block_tables, const int32_t* context_lens, float scale,
                          int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                          int64_t head_dim, int64_t num_blocks, int64_t block_size,
                          int64_t max_blocks_per_seq, int64_t partition_size,
                          int64_t max_partitions, pa_dtype dtype, void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if (partition_size <= 0 || max_partitions <= 0) return PA_ERR_SHAPE;
  if (partition_size % kPage != 0) return PA_ERR_UNSUPPORTED;
  if (partition_size > INT32_MAX || max_partitions > INT32_MAX) return PA_ERR_SHAPE;
  if (num_seqs == 0) return PA_OK;
  if (!tmp_out || !max_logits || !exp_sums) return PA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(tmp_out) & 7u) || (reinterpret_cast<uintptr_t>(max_logits) & 3u) ||
      (reinterpret_cast<uintptr_t>(exp_sums) & 3u))
    return PA_ERR_ALIGN;
  DecodeArgs a = make_args(query, block_tables, context_lens, scale, num_heads, num_kv_heads,
                           max_blocks_per_seq, num_blocks);
  a.tmp_out = tmp_out;
  a.max_logits = max_logits;
  a.exp_sums = exp_sums;
  a.partition_size = static_cast<int>(partition_size);
  a.parts_per_head = static_cast<int>(max_partitions);
  a.max_partitions = static_cast<int>(max_partitions);
  return run_decode(a, key_cache, value_cache, num_seqs, head_dim, num_blocks, dtype,
                    as_stream(stream));
}

pa_status pa_reduce(void* out, const float* tmp_out, const float* max_logits,
                    const float* exp_sums, const int32_t* context_lens, int64_t num_seqs,
                    int64_t num_heads, int64_t head_dim, int64_t partition_size,
                    int64_t max_partitions, pa_dtype dtype, void* stream) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_seqs < 0 || num_heads <= 0 || head_dim <= 0 || partition_size <= 0 ||
      max_partitions <= 0)
    return PA_ERR_SHAPE;
  if (num_seqs == 0) return PA_OK;
  if (!out || !tmp_out || !max_logits || !exp_sums || !context_lens) return PA_ERR_NULL;
  if (head_dim % 4 != 0 || head_dim > 4 * kReduceThreads) return PA_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(out) & 7u) || (reinterpret_cast<uintptr_t>(tmp_out) & 15u))
    return PA_ERR_ALIGN;
  if (num_seqs * num_heads > INT32_MAX || partition_size > INT32_MAX ||
      max_partitions > INT32_MAX)
    return PA_ERR_SHAPE;
  const unsigned grid = static_cast<unsigned>(num_seqs * num_heads);
  auto kernel = dtype == PA_BF16 ? lse_reduce_kernel<true> : lse_reduce_kernel<false>;
  return launch_ex(kernel, grid, kReduceThreads, 0, as_stream(stream), 1,
                   static_cast<uint16_t*>(out), tmp_out, max_logits, exp_sums, context_lens,
                   static_cast<int>(num_heads), static_cast<int>(head_dim),
                   static_cast<int>(partition_size), static_cast<int>(max_partitions));
}

// >>> fp8 KV cache entry points
pa_status pa_reshape_and_cache_fp8(const void* key, const void* value, int64_t key_stride,
                                   int64_t value_stride, void* key_cache, void* value_cache,
                                   const int64_t* slot_mapping, int64_t num_tokens,
                                   int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                   int64_t block_size, float k_scale, float v_scale,
                                   pa_dtype dtype, void* stream) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || block_size <= 0)
    return PA_ERR_SHAPE;
  pa_status st = check_fp8_scales(k_scale, v_scale);
  if (st != PA_OK) return st;
  const int64_t row = num_kv_heads * head_dim;
  if (key_stride < row || value_stride < row) return PA_ERR_SHAPE;
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_NULL;
  if (head_dim % 16 != 0 || key_stride % 8 != 0 || value_stride % 8 != 0) return PA_ERR_ALIGN;
  if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PA_ERR_ALIGN;
  const int64_t chunks = row / 16;
  if (chunks > INT32_MAX) return PA_ERR_SHAPE;
  const int64_t total = num_tokens * chunks;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 32) blocks = 148 * 32;
  const float inv_k = 1.0f / k_scale, inv_v = 1.0f / v_scale;
  auto kernel = dtype == PA_BF16 ? reshape_and_cache_fp8_kernel<true>
                                 : reshape_and_cache_fp8_kernel<false>;
  return launch_ex(kernel, static_cast<unsigned>(blocks), threads, 0, as_stream(stream), 1,
                   static_cast<const uint16_t*>(key), static_cast<const uint16_t*>(value),
                   static_cast<long long>(key_stride), static_cast<long long>(value_stride),
                   static_cast<uint8_t*>(key_cache), static_cast<uint8_t*>(value_cache),
                   slot_mapping, static_cast<long long>(num_tokens), static_cast<int>(chunks),
                   static_cast<long long>(num_blocks * block_size), inv_k, inv_v);
}

pa_status pa_decode_fp8(void* out, const void* query, const void* key_cache,
                        const void* value_cache, const int32_t* block_tables,
                        const int32_t* context_lens, float scale, float k_scale, float v_scale,
                        int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                        int64_t head_dim, int64_t num_blocks, int64_t block_size,
                        int64_t max_blocks_per_seq, pa_dtype dtype, void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if ((st = check_fp8_scales(k_scale, v_scale)) != PA_OK) return st;
  if (head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out) return PA_ERR_NULL;
  if (!aligned16(out)) return PA_ERR_ALIGN;
  DecodeArgs a = make_args(query, block_tables, context_lens, scale * k_scale, num_heads,
                           num_kv_heads, max_blocks_per_seq, num_blocks);
  a.v_scale = v_scale;
  a.out = static_cast<uint16_t*>(out);
  a.num_seqs = static_cast<int>(num_seqs);
  a.longest_first = num_seqs > 1 && num_seqs <= kLptMaxSeqs;
  return run_decode_fp8(a, key_cache, value_cache, num_seqs, num_blocks, dtype,
                        as_stream(stream));
}

pa_status pa_decode_split_fp8(float* tmp_out, float* max_logits, float* exp_sums,
                              const void* query, const void* key_cache, const void* value_cache,
                              const int32_t* block_tables, const int32_t* context_lens,
                              float scale, float k_scale, float v_scale, int64_t num_seqs,
                              int64_t num_heads, int64_t num_kv_heads, int64_t head_dim,
                              int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq,
                              int64_t partition_size, int64_t max_partitions, pa_dtype dtype,
                              void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if ((st = check_fp8_scales(k_scale, v_scale)) != PA_OK) return st;
  if (head_dim != 128) return PA_ERR_UNSUPPORTED;
  if (partition_size <= 0 || max_partitions <= 0) return PA_ERR_SHAPE;
  if (partition_size % kPage != 0) return PA_ERR_UNSUPPORTED;
  if (partition_size > INT32_MAX || max_partitions > INT32_MAX) return PA_ERR_SHAPE;
  if (num_seqs == 0) return PA_OK;
  if (!tmp_out || !max_logits || !exp_sums) return PA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(tmp_out) & 7u) || (reinterpret_cast<uintptr_t>(max_logits) & 3u) ||
      (reinterpret_cast<uintptr_t>(exp_sums) & 3u))
    return PA_ERR_ALIGN;
  DecodeArgs a = make_args(query, block_tables, context_lens, scale * k_scale, num_heads,
                           num_kv_heads, max_blocks_per_seq, num_blocks);
  a.v_scale = v_scale;
  a.tmp_out = tmp_out;
  a.max_logits = max_logits;
  a.exp_sums = exp_sums;
  a.partition_size = static_cast<int>(partition_size);
  a.parts_per_head = static_cast<int>(max_partitions);
  a.max_partitions = static_cast<int>(max_partitions);
  return run_decode_fp8(a, key_cache, value_cache, num_seqs, num_blocks, dtype,
                        as_stream(stream));
}
// <<< fp8 KV cache entry points

// >>> host-buffer step (pa_decode_step_host): one decode step from host
// buffers.  Workspace layout (each part 256-byte aligned): key, value,
// slot_mapping, query, block_tables, context_lens, out, then for the split
// path tmp_out, max_logits, exp_sums.
namespace {
struct StepLayout {
  int64_t off[10];
  int64_t total;
};

int64_t align256(int64_t x) { return (x + 255) & ~static_cast<int64_t>(255); }

StepLayout step_layout(int64_t S, int64_t H, int64_t Hk, int64_t D, int64_t MB, int64_t bs,
                       int64_t partition_size) {
  const int64_t parts = partition_size > 0 ? (MB * bs + partition_size - 1) / partition_size : 0;
  // key, value, slot_mapping (what the cache write needs), then query,
  // block_tables, context_lens, then out and the split partials
  const int64_t sizes[10] = {S * Hk * D * 2, S * Hk * D * 2, S * 8, S * H * D * 2, S * MB * 4,
                             S * 4, S * H * D * 2, S * H * parts * D * 4, S * H * parts * 4,
                             S * H * parts * 4};
  StepLayout l{};
  int64_t at = 0;
  for (int i = 0; i < 10; ++i) {
    l.off[i] = at;
    at = align256(at + sizes[i]);
  }
  l.total = at;
  return l;
}

// A side stream and two events per (device, caller stream): the step's query
// and table copies run on the side stream while the cache write runs on the
// caller's stream (fork after the caller's earlier work, join before the
// attention).  Created once; calls on one stream are ordered, so reusing the
// events is safe.
struct StepFork {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

const StepFork* step_fork(cudaStream_t s) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, StepFork> forks;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  auto it = forks.find({dev, s});
  if (it != forks.end()) return &it->second;
  StepFork f;
  if (cudaStreamCreateWithFlags(&f.side, cudaStreamNonBlocking) != cudaSuccess ||
      cudaEventCreateWithFlags(&f.fork, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&f.join, cudaEventDisableTiming) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return &forks.emplace(std::make_pair(dev, s), f).first->second;
}

// The device address of `bytes` bytes of page-locked host memory at p that
// the GPU can read and write directly, or nullptr.  Both the first and the
// last byte must lie in page-locked memory, and the last byte's device
// address must follow from the first's: a range that runs past the end of
// its page-locked allocation (into pageable memory or another allocation) is
// not addressable as one piece and takes the copy path instead.
void* device_view_of_host(const void* p, int64_t bytes) {
  if (bytes <= 0) return nullptr;
  auto view = [](const void* q) -> void* {
    cudaPointerAttributes attr{};
    if (cudaPointerGetAttributes(&attr, q) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return attr.type == cudaMemoryTypeHost ? attr.devicePointer : nullptr;
  };
  void* first = view(p);
  if (!first) return nullptr;
  const void* last_host = static_cast<const uint8_t*>(p) + (bytes - 1);
  void* last = view(last_host);
  if (last != static_cast<void*>(static_cast<uint8_t*>(first) + (bytes - 1))) return nullptr;
  return first;
}
}  // namespace

int64_t pa_decode_step_host_workspace_bytes(int64_t num_seqs, int64_t num_heads,
                                            int64_t num_kv_heads, int64_t head_dim,
                                            int64_t max_blocks_per_seq, int64_t block_size,
                                            int64_t partition_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      max_blocks_per_seq <= 0 || block_size <= 0 || partition_size < 0)
    return -1;
  return step_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                     block_size, partition_size)
      .total;
}

pa_status pa_decode_step_host(void* out_host, const void* query_host, const void* key_host,
                              const void* value_host, const int64_t* slot_mapping_host,
                              const int32_t* block_tables_host,
                              const int32_t* context_lens_host, void* key_cache,
                              void* value_cache, void* workspace, int64_t workspace_bytes,
                              float scale, int64_t num_seqs, int64_t num_heads,
                              int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                              int64_t block_size, int64_t max_blocks_per_seq,
                              int64_t partition_size, pa_dtype dtype, void* stream) {
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_DTYPE;
  if (num_seqs < 0 || partition_size < 0) return PA_ERR_SHAPE;
  if (num_seqs == 0) return PA_OK;
  // value and slot_mapping: both given, or both NULL to say they follow
  // key_host in one buffer at the workspace's offsets; the same for
  // block_tables and context_lens after query_host
  if (!out_host || !query_host || !key_host || !key_cache || !value_cache || !workspace ||
      (!value_host != !slot_mapping_host) || (!block_tables_host != !context_lens_host))
    return PA_ERR_NULL;
  const int64_t need = pa_decode_step_host_workspace_bytes(num_seqs, num_heads, num_kv_heads,
                                                           head_dim, max_blocks_per_seq,
                                                           block_size, partition_size);
  if (need < 0) return PA_ERR_SHAPE;
  if (workspace_bytes < need) return PA_ERR_SHAPE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PA_ERR_ALIGN;
  const StepLayout l = step_layout(num_seqs, num_heads, num_kv_heads, head_dim,
                                   max_blocks_per_seq, block_size, partition_size);
  uint8_t* w = static_cast<uint8_t*>(workspace);
  void* d_key = w + l.off[0];
  void* d_value = w + l.off[1];
  int64_t* d_slots = reinterpret_cast<int64_t*>(w + l.off[2]);
  void* d_query = w + l.off[3];
  int32_t* d_tables = reinterpret_cast<int32_t*>(w + l.off[4]);
  int32_t* d_lens = reinterpret_cast<int32_t*>(w + l.off[5]);
  cudaStream_t s = as_stream(stream);
  const StepFork* fork = step_fork(s);
  if (!fork) return PA_ERR_CUDA;
  const int64_t q_bytes = num_seqs * num_heads * head_dim * 2;
  const int64_t kv_bytes = num_seqs * num_kv_heads * head_dim * 2;
  struct Copy { void* dst; const void* src; int64_t bytes; };
  // A stage whose later parts the caller marked as packed (NULL) goes over in
  // one copy from its first part's address, else one copy per part.
  auto copy_in = [&](const Copy* c, int n, int first, cudaStream_t on) {
    if (!c[1].src) {
      const int64_t bytes = l.off[first + n - 1] - l.off[first] + c[n - 1].bytes;
      return cudaMemcpyAsync(c[0].dst, c[0].src, static_cast<size_t>(bytes),
                             cudaMemcpyHostToDevice, on) == cudaSuccess;
    }
    for (int i = 0; i < n; ++i)
      if (cudaMemcpyAsync(c[i].dst, c[i].src, static_cast<size_t>(c[i].bytes),
                          cudaMemcpyHostToDevice, on) != cudaSuccess)
        return false;
    return true;
  };
  const Copy write_in[3] = {{d_key, key_host, kv_bytes}, {d_value, value_host, kv_bytes},
                            {d_slots, slot_mapping_host, num_seqs * 8}};
  const Copy attend_in[3] = {{d_query, query_host, q_bytes},
                             {d_tables, block_tables_host, num_seqs * max_blocks_per_seq * 4},
                             {d_lens, context_lens_host, num_seqs * 4}};
  // The cache write reads the new rows straight from host memory when all
  // three parts are page-locked memory the device can address: its reads then
  // share the link with the side stream's copy of the query and tables, and
  // nothing waits for a separate copy of the rows.  Otherwise the rows are
  // copied into the workspace first, and the side stream forks after that copy.
  const void* src_key = nullptr;
  const void* src_value = nullptr;
  const void* src_slots = nullptr;
  if (value_host) {
    src_key = device_view_of_host(key_host, kv_bytes);
    if (src_key) {
      src_value = device_view_of_host(value_host, kv_bytes);
      src_slots = device_view_of_host(slot_mapping_host, num_seqs * 8);
    }
  } else {  // packed after key_host, at the workspace's offsets: the whole stage
    src_key = device_view_of_host(key_host, l.off[2] - l.off[0] + num_seqs * 8);
    if (src_key) {
      src_value = static_cast<const uint8_t*>(src_key) + (l.off[1] - l.off[0]);
      src_slots = static_cast<const uint8_t*>(src_key) + (l.off[2] - l.off[0]);
    }
  }
  const bool read_direct = src_key && src_value && src_slots && aligned16(src_key) &&
                           aligned16(src_value) &&
                           (reinterpret_cast<uintptr_t>(src_slots) & 7u) == 0;
  // The fork comes after all earlier work on this stream, so nothing still
  // reads the workspace the side stream overwrites.
  if ((!read_direct && !copy_in(write_in, 3, 0, s)) ||
      cudaEventRecord(fork->fork, s) != cudaSuccess ||
      cudaStreamWaitEvent(fork->side, fork->fork, 0) != cudaSuccess ||
      !copy_in(attend_in, 3, 3, fork->side) ||
      cudaEventRecord(fork->join, fork->side) != cudaSuccess)
    return PA_ERR_CUDA;
  pa_status st = pa_reshape_and_cache(
      read_direct ? src_key : d_key, read_direct ? src_value : d_value, num_kv_heads * head_dim,
      num_kv_heads * head_dim, key_cache, value_cache,
      read_direct ? static_cast<const int64_t*>(src_slots) : d_slots, num_seqs, num_kv_heads,
      head_dim, num_blocks, block_size, dtype, stream);
  if (st != PA_OK) return st;
  // join, then attend; the output goes straight into out_host when that is
  // page-locked memory the device can address, else through the workspace
  if (cudaStreamWaitEvent(s, fork->join, 0) != cudaSuccess) return PA_ERR_CUDA;
  void* direct = device_view_of_host(out_host, q_bytes);
  if (direct && !aligned16(direct)) direct = nullptr;
  void* d_out = direct ? direct : static_cast<void*>(w + l.off[6]);
  if (partition_size > 0) {
    const int64_t parts = (max_blocks_per_seq * block_size + partition_size - 1) / partition_size;
    float* tmp = reinterpret_cast<float*>(w + l.off[7]);
    float* mx = reinterpret_cast<float*>(w + l.off[8]);
    float* es = reinterpret_cast<float*>(w + l.off[9]);
    st = pa_decode_split(tmp, mx, es, d_query, key_cache, value_cache, d_tables, d_lens, scale,
                         num_seqs, num_heads, num_kv_heads, head_dim, num_blocks, block_size,
                         max_blocks_per_seq, partition_size, parts, dtype, stream);
    if (st != PA_OK) return st;
    st = pa_reduce(d_out, tmp, mx, es, d_lens, num_seqs, num_heads, head_dim, partition_size,
                   parts, dtype, stream);
  } else {
    st = pa_decode(d_out, d_query, key_cache, value_cache, d_tables, d_lens, scale, num_seqs,
                   num_heads, num_kv_heads, head_dim, num_blocks, block_size, max_blocks_per_seq,
                   dtype, stream);
  }
  if (st != PA_OK) return st;
  if (!direct && cudaMemcpyAsync(out_host, d_out, static_cast<size_t>(q_bytes),
                                 cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PA_ERR_CUDA;
  return PA_OK;
}
// <<< host-buffer step

pa_status pa_check_error(void* stream, int64_t* detail) {
  cudaStream_t s = as_stream(stream);
  unsigned long long word = 0;
  const unsigned long long zero = 0;
  if (cudaMemcpyFromSymbolAsync(&word, pa::g_error_word, sizeof word, 0, cudaMemcpyDeviceToHost,
                                s) != cudaSuccess)
    return PA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
  if (word != 0) {
    if (cudaMemcpyToSymbolAsync(pa::g_error_word, &zero, sizeof zero, 0, cudaMemcpyHostToDevice,
                                s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return PA_ERR_CUDA;
  }
  if (detail) *detail = static_cast<int64_t>(word);
  return word ? PA_ERR_BOUNDS : PA_OK;
}

}  // extern "C"
// >>> self-test of the bounded barrier wait (pa_selftest_wait_timeout): one
// CTA waits, with the kernels' own bounded wait, on an mbarrier that nothing
// completes, and records the timeout the way every kernel does.
namespace {
__global__ void wait_timeout_selftest_kernel() {
  __shared__ alignas(8) uint64_t bar;
  const uint32_t b = pa::smem_addr(&bar);
  if (threadIdx.x == 0) {
    pa::mbar_init(b, 1);   // one arrival completes phase 0; none is made
    pa::fence_barrier_init();
  }
  __syncthreads();
  const bool landed = pa::mbar_wait_bounded(b, 0);
  if (!__all_sync(0xffffffffu, landed) && threadIdx.x == 0)
    pa::record_error(pa::kErrWaitTimeout, blockIdx.x);
}
}  // namespace

extern "C" pa_status pa_selftest_wait_timeout(void* stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
// <<< self-test of the bounded barrier wait

// >>> no-allocation entry point (pa_decode_noalloc): split decode + merge
// with the partition scratch in a fixed device array of this file (declared
// in pa.h).  Host code must not use the array's name as a device address; the
// address is looked up once per device below and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set up on the
// first call per device, with that device current).
pa_status noalloc_scratch(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *ptr = g_noalloc_ptr[dev];
  return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* query, const void* key_cache,
                                       const void* value_cache, const int32_t* block_tables,
                                       const int32_t* context_lens, float scale,
                                       int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                                       int64_t head_dim, int64_t num_blocks, int64_t block_size,
                                       int64_t max_blocks_per_seq, int64_t partition_size,
                                       pa_dtype dtype, void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if (partition_size <= 0 || partition_size > INT32_MAX) return PA_ERR_SHAPE;
  if (partition_size % kPage != 0) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!out) return PA_ERR_NULL;
  if (!aligned16(out)) return PA_ERR_ALIGN;
  const int64_t parts = (max_blocks_per_seq * block_size + partition_size - 1) / partition_size;
  const int64_t rows = num_seqs * num_heads * parts;         // (seq, head, partition) entries
  const int64_t acc_bytes = rows * head_dim * 4;
  const int64_t need = acc_bytes + 2 * rows * 4;
  if (parts > INT32_MAX || need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_SHAPE;

  void* base = nullptr;
  if ((st = noalloc_scratch(&base)) != PA_OK) return st;
  float* tmp_out = static_cast<float*>(base);
  float* max_logits = tmp_out + rows * head_dim;
  float* exp_sums = max_logits + rows;

  DecodeArgs a = make_args(query, block_tables, context_lens, scale, num_heads, num_kv_heads,
                           max_blocks_per_seq, num_blocks);
  a.tmp_out = tmp_out;
  a.max_logits = max_logits;
  a.exp_sums = exp_sums;
  a.partition_size = static_cast<int>(partition_size);
  a.parts_per_head = static_cast<int>(parts);
  a.max_partitions = static_cast<int>(parts);
  cudaStream_t s = as_stream(stream);
  if ((st = run_decode(a, key_cache, value_cache, num_seqs, head_dim, num_blocks, dtype, s)) !=
      PA_OK)
    return st;
  const unsigned grid = static_cast<unsigned>(num_seqs * num_heads);
  auto kernel = dtype == PA_BF16 ? lse_reduce_kernel<true> : lse_reduce_kernel<false>;
  return launch_ex(kernel, grid, kReduceThreads, 0, s, 1, static_cast<uint16_t*>(out), tmp_out,
                   max_logits, exp_sums, context_lens, static_cast<int>(num_heads),
                   static_cast<int>(head_dim), static_cast<int>(partition_size),
                   static_cast<int>(parts));
}
// <<< no-allocation entry point


// >>> shared-prefix decode (pa_decode_shared_prefix): host side, one region.
#include "pa_shared_prefix.cuh"

namespace {
#ifndef PA_SHARED_CLUSTER
#define PA_SHARED_CLUSTER 4        // CTAs per shared-prefix item (2: 69.6 µs, 4: 63.5, 8: 75.7 on the beam batch)
#endif
#ifndef PA_SHARED_CLUSTER_PAGES
#define PA_SHARED_CLUSTER_PAGES 64  // items with more pages are spread over the cluster
#endif

template <int D, bool BF16>
pa_status launch_shared_prefix_t(const CUtensorMap& km, const CUtensorMap& vm,
                                 SharedPrefixArgs a, long long items, cudaStream_t stream) {
  constexpr int NST = Stages<D>::value;
  using L = DecodeSmem<D, NST>;
  auto kernel = shared_prefix_decode_kernel<D, NST, BF16>;
  static std::atomic<uint64_t> done{0};
  static std::atomic<int> cluster_cache[kMaxDevices] = {};
  if (!ensure_smem(kernel, L::kAlloc, &done)) return PA_ERR_CUDA;
  // one cluster size for the launch: as large as PA_SHARED_CLUSTER if the
  // device can co-schedule it, and 1 when no item can exceed the threshold
  const int64_t max_item_pages =
      static_cast<int64_t>(a.members_per_chunk) * a.max_blocks_per_seq;
  int c = 1;
  if (max_item_pages > PA_SHARED_CLUSTER_PAGES) {
    c = pick_cluster(kernel, L::kAlloc, static_cast<int64_t>(PA_SHARED_CLUSTER) *
                                            PA_CLUSTER_TABLE_PAGES, cluster_cache);
    if (c > PA_SHARED_CLUSTER) c = PA_SHARED_CLUSTER;
  }
  a.cluster_pages = PA_SHARED_CLUSTER_PAGES;
  if (items * c > INT32_MAX) return PA_ERR_SHAPE;
  return launch_ex(kernel, static_cast<unsigned>(items * c), kThreads, L::kAlloc, stream, c, km,
                   vm, a);
}

}  // namespace

extern "C" pa_status pa_decode_shared_prefix(void* out, const void* query, const void* key_cache,
                                  const void* value_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, const int32_t* group_starts,
                                  const int32_t* prefix_blocks, float scale, int64_t num_seqs,
                                  int64_t num_groups, int64_t max_group_size, int64_t num_heads,
                                  int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                  int64_t block_size, int64_t max_blocks_per_seq, pa_dtype dtype,
                                  void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if (num_groups < 0 || max_group_size <= 0) return PA_ERR_SHAPE;
  if (num_seqs == 0 || num_groups == 0) return PA_OK;
  if (!out || !group_starts || !prefix_blocks) return PA_ERR_NULL;
  if (!aligned16(out) || (reinterpret_cast<uintptr_t>(group_starts) & 3u) ||
      (reinterpret_cast<uintptr_t>(prefix_blocks) & 3u))
    return PA_ERR_ALIGN;
  const int64_t G = num_heads / num_kv_heads;
  const int64_t per_chunk = 16 / G;                       // G <= 16 checked above
  const int64_t chunks = (max_group_size + per_chunk - 1) / per_chunk;
  const int64_t items = num_groups * num_kv_heads * chunks;
  if (num_groups > INT32_MAX || chunks > INT32_MAX || items > INT32_MAX) return PA_ERR_SHAPE;
  CUtensorMap km, vm;
  if (!encode_cache_map(&km, key_cache, dtype, num_blocks, num_kv_heads, head_dim) ||
      !encode_cache_map(&vm, value_cache, dtype, num_blocks, num_kv_heads, head_dim))
    return PA_ERR_CUDA;
  SharedPrefixArgs a{};
  a.query = static_cast<const uint16_t*>(query);
  a.out = static_cast<uint16_t*>(out);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.group_starts = group_starts;
  a.prefix_blocks = prefix_blocks;
  a.scale_log2 = scale * kLog2e;
  a.num_seqs = static_cast<int>(num_seqs);
  a.num_heads = static_cast<int>(num_heads);
  a.num_kv_heads = static_cast<int>(num_kv_heads);
  a.group = static_cast<int>(G);
  a.max_blocks_per_seq = static_cast<int>(max_blocks_per_seq);
  a.num_blocks = static_cast<int>(num_blocks);
  a.num_groups = static_cast<int>(num_groups);
  a.members_per_chunk = static_cast<int>(per_chunk);
  a.chunks_per_group = static_cast<int>(chunks);
  a.longest_first = num_groups * chunks <= kLptMaxSeqs;
  cudaStream_t s = as_stream(stream);
  const bool bf16 = dtype == PA_BF16;
  if (head_dim == 64)
    return bf16 ? launch_shared_prefix_t<64, true>(km, vm, a, items, s)
                : launch_shared_prefix_t<64, false>(km, vm, a, items, s);
  return bf16 ? launch_shared_prefix_t<128, true>(km, vm, a, items, s)
              : launch_shared_prefix_t<128, false>(km, vm, a, items, s);
}
// <<< shared-prefix decode

// >>> chunked prefill (pa_prefill): host side.  Kept in one region, apart from
// the decode path's code, so that the two can be versioned separately.
#include "pa_prefill.cuh"

namespace {
// 4-D view of the query [T, H, D] for boxes of G heads x tile tokens x 64
// elements (128-byte swizzle): rows land token-major, row = token * G + head.
bool encode_query_map(CUtensorMap* map, const void* query, pa_dtype dtype, int64_t num_tokens,
                      int64_t num_heads, int64_t head_dim, int64_t group, int64_t tile_tokens) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {64, static_cast<cuuint64_t>(head_dim / 64),
                              static_cast<cuuint64_t>(num_heads),
                              static_cast<cuuint64_t>(num_tokens)};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(head_dim * 2),
                                 static_cast<cuuint64_t>(num_heads * head_dim * 2)};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(group),
                             static_cast<cuuint32_t>(tile_tokens)};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        4, const_cast<void*>(query), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device, looked up once per device
// (0 if the query fails).
long long sm_count() {
  static std::atomic<long long> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  long long known = cache[dev].load(std::memory_order_relaxed);
  if (known == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    known = sms;
    cache[dev].store(known, std::memory_order_relaxed);
  }
  return known;
}

// The prefill grid is persistent: one CTA per SM (its shared memory admits
// no second one), each walking its share of the items.
template <int D, bool BF16>
pa_status launch_prefill_t(const CUtensorMap& qm, const CUtensorMap& km, const CUtensorMap& vm,
                           const PrefillArgs& a, long long items, cudaStream_t stream) {
  using L = PrefillSmem<D, BF16>;
  auto kernel = paged_prefill_kernel<D, BF16>;
  static std::atomic<uint64_t> done{0};
  if (!ensure_smem(kernel, L::kAlloc, &done)) return PA_ERR_CUDA;
  const long long sms = sm_count();
  if (sms <= 0) return PA_ERR_CUDA;
  const long long grid = items < sms ? items : sms;
  return launch_ex(kernel, static_cast<unsigned>(grid), PrefillRoles<BF16>::kThreads, L::kAlloc,
                   stream, 1, qm, km, vm, a);
}


}  // namespace

extern "C" pa_status pa_prefill(void* out, const void* query, const void* key_cache, const void* value_cache,
                     const int32_t* block_tables, const int32_t* context_lens,
                     const int32_t* query_starts, float scale, int64_t num_seqs,
                     int64_t num_query_tokens, int64_t max_query_len, int64_t num_heads,
                     int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                     int64_t block_size, int64_t max_blocks_per_seq, pa_dtype dtype,
                     void* stream) {
  pa_status st = check_attention_args(query, key_cache, value_cache, block_tables, context_lens,
                                      scale, num_seqs, num_heads, num_kv_heads, head_dim,
                                      num_blocks, block_size, max_blocks_per_seq, dtype);
  if (st != PA_OK) return st;
  if (num_query_tokens < 0 || max_query_len < 0) return PA_ERR_SHAPE;
  if (num_seqs == 0 || num_query_tokens == 0 || max_query_len == 0) return PA_OK;
  if (!out || !query_starts) return PA_ERR_NULL;
  if (!aligned16(out) || (reinterpret_cast<uintptr_t>(query_starts) & 3u)) return PA_ERR_ALIGN;
  if (num_query_tokens * num_heads > INT32_MAX || max_query_len > INT32_MAX) return PA_ERR_SHAPE;
  const int64_t G = num_heads / num_kv_heads;
  const int64_t tile = kPrefillRows / G;                  // G <= 16 checked above
  const int64_t span = 2 * tile;                          // two query tiles per CTA
  const int64_t pairs = (max_query_len + span - 1) / span;
  const long long items = num_seqs * num_kv_heads * pairs;   // (sequence, KV head, tile pair)
  if (items > INT32_MAX) return PA_ERR_SHAPE;
  CUtensorMap qm, km, vm;
  if (!encode_query_map(&qm, query, dtype, num_query_tokens, num_heads, head_dim, G, tile) ||
      !encode_cache_map(&km, key_cache, dtype, num_blocks, num_kv_heads, head_dim) ||
      !encode_cache_map(&vm, value_cache, dtype, num_blocks, num_kv_heads, head_dim))
    return PA_ERR_CUDA;
  PrefillArgs a{};
  a.out = static_cast<uint16_t*>(out);
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.query_starts = query_starts;
  a.scale_log2 = scale * kLog2e;
  a.num_seqs = static_cast<int>(num_seqs);
  a.num_tokens = static_cast<int>(num_query_tokens);
  a.num_heads = static_cast<int>(num_heads);
  a.num_kv_heads = static_cast<int>(num_kv_heads);
  a.group = static_cast<int>(G);
  a.max_blocks_per_seq = static_cast<int>(max_blocks_per_seq);
  a.num_blocks = static_cast<int>(num_blocks);
  a.tile_tokens = static_cast<int>(tile);
  cudaStream_t s = as_stream(stream);
  const bool bf16 = dtype == PA_BF16;
  if (head_dim == 64)
    return bf16 ? launch_prefill_t<64, true>(qm, km, vm, a, items, s)
                : launch_prefill_t<64, false>(qm, km, vm, a, items, s);
  return bf16 ? launch_prefill_t<128, true>(qm, km, vm, a, items, s)
              : launch_prefill_t<128, false>(qm, km, vm, a, items, s);
}
// <<< chunked prefill

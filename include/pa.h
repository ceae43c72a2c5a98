/*
 * pa.h -- C ABI of libpa, the B200 (sm_100a) paged decode-attention library.
 *
 * The operations follow the pages on vLLM's PagedAttention:
 *  - "vllm源码剖析" (jsqmd.com/news/690568) §一.2 "为什么要reshape": the KV
 *    cache is [num_blocks, block_size, num_kv_heads, head_size], addressed per
 *    token through the flat view [num_blocks*block_size, num_kv_heads,
 *    head_size]; §一.3 "token和请求块的映射": a token's slot is its block id
 *    times block_size plus its offset (index mod block_size).
 *  - "vLLM PagedAttention 原理与源码深度解析" (toukenai.cn) §3.1: a per-sequence
 *    block table maps logical blocks to physical blocks; §5.3 "注意力计算":
 *    forward(q, kv_cache, block_tables, context_lens) gathers K/V through the
 *    block tables and returns softmax(q.k * scale) . v per query head.
 *  - "vllm源码分析：…PagedAttention核心实现" (vergex.cn/9743.html) §第三讲:
 *    logical block i of a sequence is read from physical block block_table[i].
 *
 * Conventions shared by every entry point:
 *  - Every buffer argument is a DEVICE pointer owned by the caller.  The
 *    library allocates no memory, never synchronises (except
 *    pa_check_error), and keeps no per-call state (pa_decode_step_host,
 *    which takes host buffers, keeps a side stream and two events per
 *    device and stream; see there).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; the returned status covers argument
 *    validation and launch errors only.
 *  - 16-bit element type `dtype`: PA_F16 (IEEE binary16) or PA_BF16.  Query,
 *    caches, new K/V and the output all share it.
 *  - All tensors are dense row-major with the layouts stated per call; every
 *    pointer to 16-bit data must be 16-byte aligned and head_dim a multiple of 8.
 *  - Query head h reads KV head h / (num_heads / num_kv_heads) (consecutive
 *    grouping, as in Llama-style GQA).
 *  - context_lens[s] counts the tokens sequence s attends to, including a
 *    token written this step by pa_reshape_and_cache (call it first, on the
 *    same stream).  context_lens[s] == 0 yields an all-zero output row.
 *  - Only block_tables[s][0 .. ceil(context_lens[s]/block_size)-1] are read.
 *  - Kernels check every block id, slot and context length they read.  An
 *    out-of-range value never causes an out-of-bounds access: the access is
 *    skipped (reads return zeros), and the first such event is recorded in a
 *    per-device error word that pa_check_error reports.
 */
#ifndef PA_H_
#define PA_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_NULL = 1,        /* a required pointer is NULL */
    PA_ERR_SHAPE = 2,       /* a size is out of range or sizes disagree */
    PA_ERR_DTYPE = 3,       /* unknown element type */
    PA_ERR_ALIGN = 4,       /* a pointer or row stride is not 16-byte aligned */
    PA_ERR_UNSUPPORTED = 5, /* valid, but not built: head_dim, block_size, partition size */
    PA_ERR_CUDA = 6,        /* a CUDA call failed (no device, launch, tensor map) */
    PA_ERR_BOUNDS = 7       /* pa_check_error: a kernel met an out-of-range index */
} pa_status;

typedef enum pa_dtype { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Codes stored in the top 8 bits of the detail word of pa_check_error;
 * the low 56 bits hold the offending index (see each code). */
enum {
    PA_CHECK_SLOT = 1,          /* slot_mapping[t] >= num_blocks*block_size; index = t */
    PA_CHECK_BLOCK_ID = 2,      /* block id outside [0, num_blocks); index = s*max_blocks_per_seq + i */
    PA_CHECK_CONTEXT_LEN = 3,   /* context_lens[s] < 0 or > max_blocks_per_seq*block_size; index = s */
    PA_CHECK_PARTITIONS = 4,    /* ceil(context_lens[s]/partition_size) > max_partitions; index = s */
    PA_CHECK_WAIT_TIMEOUT = 5,  /* a shared-memory barrier wait gave up; index = CTA id */
    PA_CHECK_GROUP = 6,         /* malformed group bounds or prefix length; index = group */
    PA_CHECK_QUERY = 7,         /* prefill: q_len < 0, q_len > context_lens[s] or context too long; index = s */
    PA_CHECK_VALUE = 8          /* prefill, bf16: a V value beyond the fp16 range was clamped to +-65504; index = s */
};

/* Short English name of a status code (static string, never NULL). */
const char *pa_status_string(pa_status status);

/* ABI version of this header: (major << 16) | minor. */
int32_t pa_abi_version(void);

/*
 * pa_reshape_and_cache -- write this step's new K/V rows into the paged caches.
 * ("vllm源码剖析" §一.2 and §一.3.)
 *   key, value     [num_tokens, num_kv_heads, head_dim], consecutive tokens
 *                  key_stride / value_stride ELEMENTS apart (>= num_kv_heads*head_dim,
 *                  a multiple of 8); inside a token row the layout is dense.
 *   key_cache, value_cache
 *                  [num_blocks, block_size, num_kv_heads, head_dim] (dense).
 *   slot_mapping   [num_tokens] int64: flat slot = block_id*block_size + offset;
 *                  a negative slot marks a padding token and is skipped.
 * For every token t with slot >= 0: key_cache_flat[slot] = key[t] and
 * value_cache_flat[slot] = value[t], bit for bit.  Slots must be distinct.
 * block_size may be any positive value here.  num_tokens == 0 is a no-op.
 */
pa_status pa_reshape_and_cache(const void *key, const void *value,
                               int64_t key_stride, int64_t value_stride,
                               void *key_cache, void *value_cache,
                               const int64_t *slot_mapping, int64_t num_tokens,
                               int64_t num_kv_heads, int64_t head_dim,
                               int64_t num_blocks, int64_t block_size,
                               pa_dtype dtype, void *stream);

/*
 * pa_copy_blocks -- the device half of copy-on-write: before a sequence
 * writes into a block it shares with others (ref_count > 1), the block is
 * copied to a private one ("vllm源码分析" 第一讲; "vLLM PagedAttention 原理与源码
 * 深度解析" §3.3).
 *   key_cache, value_cache  [num_blocks, block_size, num_kv_heads, head_dim],
 *                           elem_bytes per element (2 for fp16/bf16, 1 for fp8)
 *   block_mapping           [num_pairs, 2] int64 (device): (source, destination)
 * Copies every byte of block source onto block destination, in both caches.
 * Destinations must be distinct and must not be the source of another pair in
 * the same call.  An id outside [0, num_blocks) skips its pair and is reported
 * by pa_check_error (PA_CHECK_BLOCK_ID, index = pair).  A block must be a
 * multiple of 16 bytes and both caches 16-byte aligned.
 */
pa_status pa_copy_blocks(void *key_cache, void *value_cache, const int64_t *block_mapping,
                         int64_t num_pairs, int64_t num_blocks, int64_t block_size,
                         int64_t num_kv_heads, int64_t head_dim, int64_t elem_bytes,
                         void *stream);

/*
 * pa_decode -- single-pass paged decode attention, one query token per sequence.
 * ("vLLM PagedAttention 原理与源码深度解析" §5.3.)
 *   out            [num_seqs, num_heads, head_dim]       (written)
 *   query          [num_seqs, num_heads, head_dim]
 *   key_cache, value_cache  [num_blocks, block_size, num_kv_heads, head_dim]
 *   block_tables   [num_seqs, max_blocks_per_seq] int32
 *   context_lens   [num_seqs] int32
 *   scale          multiplies q.k before the softmax (1/sqrt(head_dim) on the page)
 * out[s,h,:] = sum_j softmax_j(scale * q[s,h,:] . k_j) v_j over the first
 * context_lens[s] tokens of sequence s, computed with fp32 accumulation and
 * rounded to dtype (nearest even).
 * Built for head_dim in {64, 128}, block_size == 16, num_heads % num_kv_heads == 0.
 */
pa_status pa_decode(void *out, const void *query,
                    const void *key_cache, const void *value_cache,
                    const int32_t *block_tables, const int32_t *context_lens,
                    float scale, int64_t num_seqs, int64_t num_heads,
                    int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                    int64_t block_size, int64_t max_blocks_per_seq,
                    pa_dtype dtype, void *stream);

/*
 * pa_decode_split -- the same attention cut into partitions of partition_size
 * logical tokens (partition p covers tokens [p*P, (p+1)*P) of [0, ctx)), for
 * long contexts.  The pages do not describe this split; its merge is the
 * log-sum-exp identity applied by pa_reduce.
 *   tmp_out     [num_seqs, num_heads, max_partitions, head_dim] fp32 (written)
 *   max_logits  [num_seqs, num_heads, max_partitions] fp32 (written)
 *   exp_sums    [num_seqs, num_heads, max_partitions] fp32 (written)
 * For every partition p < ceil(ctx/partition_size), with z_j = scale*q.k_j:
 *   max_logits = max_j z_j,  exp_sums = sum_j exp(z_j - max),
 *   tmp_out    = sum_j exp(z_j - max) v_j        (not normalised).
 * Entries of partitions >= ceil(ctx/partition_size) are not written.
 * partition_size must be a positive multiple of block_size; the caller
 * guarantees ceil(ctx/partition_size) <= max_partitions (checked on device).
 * The three fp32 buffers are caller-owned scratch that pa_reduce consumes.
 */
pa_status pa_decode_split(float *tmp_out, float *max_logits, float *exp_sums,
                          const void *query, const void *key_cache,
                          const void *value_cache, const int32_t *block_tables,
                          const int32_t *context_lens, float scale,
                          int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                          int64_t head_dim, int64_t num_blocks, int64_t block_size,
                          int64_t max_blocks_per_seq, int64_t partition_size,
                          int64_t max_partitions, pa_dtype dtype, void *stream);

/*
 * pa_reduce -- merge the partitions written by pa_decode_split:
 *   M = max_p max_logits[p],  w_p = exp(max_logits[p] - M),
 *   out = (sum_p w_p tmp_out[p]) / (sum_p w_p exp_sums[p])
 * over p < ceil(context_lens[s]/partition_size); ctx == 0 gives zeros.
 *   out  [num_seqs, num_heads, head_dim] dtype (written)
 */
pa_status pa_reduce(void *out, const float *tmp_out, const float *max_logits,
                    const float *exp_sums, const int32_t *context_lens,
                    int64_t num_seqs, int64_t num_heads, int64_t head_dim,
                    int64_t partition_size, int64_t max_partitions,
                    pa_dtype dtype, void *stream);

/*
 * pa_decode_shared_prefix -- pa_decode for a batch whose sequences come in
 * groups that share the first blocks of their tables (beam candidates, a
 * common prompt prefix): "vLLM PagedAttention 原理与源码深度解析" §3.3 (beams
 * share prefix blocks through ref_count) and "读一个真实 serving 系统 · vLLM
 * 架构巡礼" §2 (KVCacheBlock.ref_cnt).  The output equals pa_decode's (same
 * formula, fp32 accumulation, another summation order), but each shared
 * page is read once per group instead of once per member.
 *   group_starts   [num_groups + 1] int32: group g is sequences
 *                  [group_starts[g], group_starts[g+1]); 0 = starts[0] <= ... <= starts[G] = num_seqs
 *   prefix_blocks  [num_groups] int32: entries 0 .. prefix_blocks[g]-1 of every
 *                  member's block table are the same ids (read from the first member)
 *   max_group_size host-side upper bound of any group's size
 * Other arguments and layouts as pa_decode.  A group larger than
 * max_group_size or malformed group bounds are reported by pa_check_error
 * (PA_CHECK_GROUP).  Members are processed 16 / (num_heads/num_kv_heads) at a
 * time, so a group wider than that re-reads its prefix once per chunk.
 */
pa_status pa_decode_shared_prefix(void *out, const void *query, const void *key_cache,
                                  const void *value_cache, const int32_t *block_tables,
                                  const int32_t *context_lens, const int32_t *group_starts,
                                  const int32_t *prefix_blocks, float scale, int64_t num_seqs,
                                  int64_t num_groups, int64_t max_group_size, int64_t num_heads,
                                  int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                                  int64_t block_size, int64_t max_blocks_per_seq,
                                  pa_dtype dtype, void *stream);

/*
 * FP8 KV cache ("vLLM PagedAttention 原理与源码深度解析" §8.4: --kv-cache-dtype
 * fp8).  The caches hold one byte per element, an OCP E4M3 code c; with one
 * scale per cache tensor, c stands for c * k_scale in the key cache and
 * c * v_scale in the value cache (k_scale, v_scale finite and > 0).  Query,
 * new K/V rows and outputs stay 16-bit (dtype).  head_dim must be 128 for the
 * decode calls.
 *
 * pa_reshape_and_cache_fp8 -- as pa_reshape_and_cache, but element x of key
 * (value) is stored as E4M3(x * (1.0f / k_scale)) (resp. v_scale): the
 * reciprocal and the product in float, then nearest-even to E4M3 with
 * saturation to +-448 (NaN stays NaN).  Caches are [num_blocks, block_size,
 * num_kv_heads, head_dim] bytes; head_dim must be a multiple of 16.
 */
pa_status pa_reshape_and_cache_fp8(const void *key, const void *value,
                                   int64_t key_stride, int64_t value_stride,
                                   void *key_cache, void *value_cache,
                                   const int64_t *slot_mapping, int64_t num_tokens,
                                   int64_t num_kv_heads, int64_t head_dim,
                                   int64_t num_blocks, int64_t block_size,
                                   float k_scale, float v_scale, pa_dtype dtype,
                                   void *stream);

/* pa_decode over E4M3 caches: out = softmax(scale * q . (c_k * k_scale)) . (c_v * v_scale). */
pa_status pa_decode_fp8(void *out, const void *query, const void *key_cache,
                        const void *value_cache, const int32_t *block_tables,
                        const int32_t *context_lens, float scale, float k_scale,
                        float v_scale, int64_t num_seqs, int64_t num_heads,
                        int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                        int64_t block_size, int64_t max_blocks_per_seq, pa_dtype dtype,
                        void *stream);

/* pa_decode_split over E4M3 caches (partials as pa_decode_split, in dequantised
 * units); merge them with pa_reduce. */
pa_status pa_decode_split_fp8(float *tmp_out, float *max_logits, float *exp_sums,
                              const void *query, const void *key_cache,
                              const void *value_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, float k_scale,
                              float v_scale, int64_t num_seqs, int64_t num_heads,
                              int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                              int64_t block_size, int64_t max_blocks_per_seq,
                              int64_t partition_size, int64_t max_partitions,
                              pa_dtype dtype, void *stream);

/*
 * pa_decode_step_host -- one whole decode step of one attention layer for a
 * caller whose per-step inputs are in HOST memory (pinned memory makes the
 * copies asynchronous; pageable memory works but the copies then block).
 * Enqueues on `stream`: the cache write (pa_reshape_and_cache) of key and
 * value [S,Hk,D] (one new token per sequence) at slot_mapping [S] int64,
 * while query [S,H,D], block_tables [S,MB] int32 and context_lens [S] int32
 * are copied into `workspace` on a library-owned side stream (forked from and
 * joined back to `stream` with events).  When key, value and slot_mapping are
 * all page-locked memory the device can address (16-, 16- and 8-byte
 * aligned), the cache write reads them there, over the host link; otherwise
 * they are first copied into `workspace` and the side stream forks after that
 * copy.  Then attention (pa_decode, or pa_decode_split + pa_reduce when
 * partition_size > 0); and the output [S,H,D]: written by the attention
 * kernel straight into out_host when out_host is page-locked memory the
 * device can address, else copied back.
 * Returns without waiting: the host inputs must stay unchanged, and out_host
 * is valid, once the stream has reached this point.  Calls on one stream are
 * ordered; the workspace is reused per call.
 * State: unlike the other entry points, this one keeps state across calls.
 * The first call for a (device, stream) pair creates a side stream and two
 * events (cudaStreamCreateWithFlags, cudaEventCreateWithFlags) and keeps them
 * in a process-wide table until exit; later calls on that pair reuse them.
 * It allocates no device memory.
 * A part is read (or the output written) in place only when its first and
 * last byte both lie in one page-locked range the device can address; a part
 * that runs past the end of its page-locked allocation is copied instead.
 *   key_cache, value_cache   device caches as for pa_decode (stay resident)
 *   workspace                caller-owned device memory, 256-byte aligned, of
 *                            pa_decode_step_host_workspace_bytes(...) bytes
 * Packed inputs: pass value_host = slot_mapping_host = NULL when value and
 * slot_mapping follow key_host in one host buffer at the workspace's relative
 * offsets (key, value, slot_mapping, each part starting 256-byte aligned after
 * the previous one); the three then go over in one transfer (or are read in
 * place).  Likewise
 * block_tables_host = context_lens_host = NULL for query, block_tables,
 * context_lens packed after query_host.  Otherwise every part is copied on
 * its own (parts that merely happen to be adjacent are never merged).
 * PA_ERR_NULL if exactly one pointer of such a pair is NULL.
 * Errors as for the calls it makes; PA_ERR_SHAPE if the workspace is small.
 */
int64_t pa_decode_step_host_workspace_bytes(int64_t num_seqs, int64_t num_heads,
                                            int64_t num_kv_heads, int64_t head_dim,
                                            int64_t max_blocks_per_seq, int64_t block_size,
                                            int64_t partition_size);

pa_status pa_decode_step_host(void *out_host, const void *query_host, const void *key_host,
                              const void *value_host, const int64_t *slot_mapping_host,
                              const int32_t *block_tables_host,
                              const int32_t *context_lens_host, void *key_cache,
                              void *value_cache, void *workspace, int64_t workspace_bytes,
                              float scale, int64_t num_seqs, int64_t num_heads,
                              int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                              int64_t block_size, int64_t max_blocks_per_seq,
                              int64_t partition_size, pa_dtype dtype, void *stream);

/*
 * pa_prefill -- paged (chunked) prefill attention ("vLLM PagedAttention 原理与
 * 源码深度解析" §8.1 Chunked Prefill: a prompt is processed a chunk of tokens
 * per step).  Sequence s has q_len = query_starts[s+1] - query_starts[s] new
 * query tokens, the LAST q_len of its context_lens[s] tokens, whose K/V are
 * already in the caches (pa_reshape_and_cache first, on the same stream).
 * Query token i (row query_starts[s] + i) sits at position
 * pos = context_lens[s] - q_len + i and attends causally to tokens 0..pos:
 *   out[t,h,:] = sum_{j<=pos} softmax_j(scale * q[t,h,:] . k_j) v_j.
 *   query, out     [num_query_tokens, num_heads, head_dim], rows grouped by sequence
 *   query_starts   [num_seqs + 1] int32, query_starts[0] = 0, nondecreasing,
 *                  query_starts[num_seqs] = num_query_tokens
 *   max_query_len  host-side upper bound of every q_len (bounds the work list; the
 *                  grid is persistent, at most one CTA per SM)
 * Other arguments as pa_decode.  A sequence with q_len > context_lens[s] is
 * skipped and reported (PA_CHECK_QUERY).  fp32 accumulation.  P enters the
 * P.V product as fp16 (11 bits).  With bf16 caches each V block is first
 * rewritten as fp16 in shared memory: exact for every bf16 value below
 * 65 520 in magnitude (values below 2^-14 lose at most 2^-25 each); a V value
 * beyond the fp16 range saturates to +-65504 and is reported
 * (PA_CHECK_VALUE, index = the sequence).
 */
pa_status pa_prefill(void *out, const void *query, const void *key_cache,
                     const void *value_cache, const int32_t *block_tables,
                     const int32_t *context_lens, const int32_t *query_starts, float scale,
                     int64_t num_seqs, int64_t num_query_tokens, int64_t max_query_len,
                     int64_t num_heads, int64_t num_kv_heads, int64_t head_dim,
                     int64_t num_blocks, int64_t block_size, int64_t max_blocks_per_seq,
                     pa_dtype dtype, void *stream);

/*
 * pa_check_error -- synchronise `stream`, read and clear the current device's
 * error word.  Returns PA_OK if no kernel recorded a problem since the last
 * call, PA_ERR_BOUNDS otherwise (then *detail, if not NULL, receives
 * (code << 56) | index with a PA_CHECK_* code), or PA_ERR_CUDA.
 */
pa_status pa_check_error(void *stream, int64_t *detail);

/*
 * pa_selftest_wait_timeout -- the failure path of every kernel's shared-memory
 * barrier waits, exercised on purpose: one CTA waits on an mbarrier that
 * nothing completes, with the kernels' own bounded wait (2 s of %globaltimer),
 * then records PA_CHECK_WAIT_TIMEOUT (index 0) and returns.  No memory is
 * touched and the device context stays usable; pa_check_error then reports
 * the timeout.  Asynchronous on `stream` like every launch.
 */
pa_status pa_selftest_wait_timeout(void *stream);

/*
 * pa_decode_noalloc -- the long-context decode of pa_decode_split followed by
 * pa_reduce, for callers that cannot allocate device memory when they call.
 * The pages have no counterpart of this entry point: it exists for
 * integration.  Some callers cannot call cudaMalloc (or any allocator) at
 * this point: runtimes that hand all device memory to their own pool at
 * start-up and forbid later allocations, plugin hosts that give a plugin no
 * allocator, and latency-critical paths that cannot afford an allocation's
 * implicit synchronisation.  They still pass every input and the output
 * (same layouts as pa_decode); the partition scratch lives in a fixed
 * device array inside this library instead of caller-owned buffers.
 *
 * Limits and behaviour:
 *  - The scratch is PA_NOALLOC_SCRATCH_BYTES (64 MiB).  A call needs
 *    num_seqs*num_heads*P*(head_dim+2)*4 bytes with
 *    P = ceil(max_blocks_per_seq*block_size / partition_size); a larger call
 *    is rejected with PA_ERR_SHAPE before anything is launched.
 *  - Every GPU that loads the library holds the 64 MiB until the process exits.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and caches it; make that first call before any
 *    stream capture.
 *  - All calls share the one array and it keeps the last call's contents;
 *    every partition entry the merge reads is written earlier in the same
 *    call, so nothing needs clearing.  Calls whose work overlaps on the GPU
 *    (other streams, other host threads) race on the array: serialise them.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Other preconditions are those of pa_decode_split (partition_size a positive
 * multiple of block_size) and pa_decode.
 */
#define PA_NOALLOC_SCRATCH_BYTES (64ll * 1024 * 1024)

pa_status pa_decode_noalloc(void *out, const void *query, const void *key_cache,
                            const void *value_cache, const int32_t *block_tables,
                            const int32_t *context_lens, float scale, int64_t num_seqs,
                            int64_t num_heads, int64_t num_kv_heads, int64_t head_dim,
                            int64_t num_blocks, int64_t block_size,
                            int64_t max_blocks_per_seq, int64_t partition_size,
                            pa_dtype dtype, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */

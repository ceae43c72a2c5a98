/*
 * pa_oracle.c -- plain, slow, single-threaded fp64 reference for the paged
 * decode path.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * CPU-baseline leg of the benchmark load it; the product library never does,
 * and this file shares no code, header or table with the CUDA path.
 *
 * Sources (web pages on vLLM's PagedAttention):
 *  [P1] "vllm源码分析：我是如何一步步读懂PagedAttention核心实现的？", §第三讲
 *       PagedAttention内核 (pseudo code: key_cache[num_blocks, block_size,
 *       num_heads, head_dim], logical block i -> block_table[i]).
 *  [P2] "vLLM PagedAttention 原理与源码深度解析", §2.1 (KV bytes per token),
 *       §3.1 (block table: logical block -> physical block), §5.3
 *       (PagedAttention.forward: gather K/V through block_tables and
 *       context_lens, softmax(q.k / sqrt(head_dim)) . v).
 *  [P5] "vllm源码剖析", §一.2 "为什么要reshape" (cache [num_blocks,
 *       block_size, num_kv_heads, head_size] viewed as [num_blocks*block_size,
 *       num_kv_heads, head_size]), §一.3 "token和请求块的映射 / 怎么求token的
 *       offset" (block = index div block_size, offset = index mod block_size),
 *       §一.6 "显存块" (page_size, num_blocks sizing).
 *
 * Everything is computed in double.  16-bit inputs are decoded exactly from
 * their bit patterns (IEEE-754 binary16; bfloat16 = upper half of binary32).
 * No blocking, no online softmax, no reordering: each sequence's K/V is first
 * materialised contiguously from its block table, then attention is the plain
 * two-pass softmax of the definition.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - only tokens j < context_lens[s] take part (the pseudo code of [P1] scores
 *    whole blocks; [P2] §5.3 passes context_lens);
 *  - query head h reads KV head h / (H / Hk) (consecutive grouping);
 *  - a negative slot in slot_mapping marks a padding token that is skipped;
 *  - context_lens[s] == 0 gives an all-zero output row;
 *  - split partition p covers logical tokens [p*P, (p+1)*P) intersected with
 *    [0, ctx) and the partitions are merged with log-sum-exp weights.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* element type codes (same numbering as the public header, kept separate) */
#define ORACLE_F16 0
#define ORACLE_BF16 1

/* return codes */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_BLOCK 2
#define ORACLE_BAD_SLOT 3
#define ORACLE_NO_MEMORY 4

/* ------------------------------------------------------------------------ */
/* 16-bit float <-> double, from the format definitions                      */
/* ------------------------------------------------------------------------ */

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_f64(uint16_t bits)
{
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)frac, -24); /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(1024 + frac), expo - 25); /* (1 + frac/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

/* bfloat16: the upper 16 bits of an IEEE-754 binary32 value. */
double oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/*
 * Round a double to the nearest value of a binary format with `mant_bits`
 * stored fraction bits and minimum normal exponent `emin`, ties to even.
 * The quantum (spacing of representable values) at |x| is
 * 2^(max(floor(log2|x|), emin) - mant_bits); x / quantum is exact, and
 * nearbyint() in the default rounding mode rounds half to even.
 */
static double round_to_format(double x, int mant_bits, int emin)
{
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    int e;
    frexp(fabs(x), &e);      /* |x| = f * 2^e, f in [0.5, 1) -> floor(log2|x|) = e - 1 */
    int ex = e - 1;
    if (ex < emin) ex = emin;
    double quantum = ldexp(1.0, ex - mant_bits);
    return nearbyint(x / quantum) * quantum;
}

/* double -> binary16 bits, round to nearest even, overflow to infinity. */
uint16_t oracle_f64_to_f16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return 0x7e00;
    double r = round_to_format(x, 10, -14);
    double a = fabs(r);
    if (a >= 65536.0 || isinf(a)) return sign | 0x7c00; /* max finite is 65504 */
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -14)) {                           /* subnormal */
        return sign | (uint16_t)(a / ldexp(1.0, -24));
    }
    int e;
    double f = frexp(a, &e);                             /* a = f * 2^e */
    int biased = e - 1 + 15;
    uint16_t frac = (uint16_t)((f * 2.0 - 1.0) * 1024.0);
    return sign | (uint16_t)(biased << 10) | frac;
}

/* double -> bfloat16 bits, round to nearest even, overflow to infinity. */
uint16_t oracle_f64_to_bf16(double x)
{
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    if (isnan(x)) return 0x7fc0;
    double r = round_to_format(x, 7, -126);
    double a = fabs(r);
    if (a >= ldexp(1.0, 128) || isinf(a)) return sign | 0x7f80;
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -126)) {                          /* subnormal */
        return sign | (uint16_t)(a / ldexp(1.0, -133));
    }
    int e;
    double f = frexp(a, &e);
    int biased = e - 1 + 127;
    uint16_t frac = (uint16_t)((f * 2.0 - 1.0) * 128.0);
    return sign | (uint16_t)(biased << 7) | frac;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3
 * fraction bits, no infinities; S.1111.111 is NaN; max finite 448. */
double oracle_e4m3_to_f64(uint8_t bits)
{
    int sign = (bits >> 7) & 1;
    int expo = (bits >> 3) & 0xf;
    int frac = bits & 0x7;
    double mag;
    if (expo == 0xf && frac == 0x7) {
        mag = NAN;
    } else if (expo == 0) {
        mag = ldexp((double)frac, -9);                 /* subnormal: frac/8 * 2^-6 */
    } else {
        mag = ldexp((double)(8 + frac), expo - 10);    /* (1 + frac/8) * 2^(e-7) */
    }
    return sign ? -mag : mag;
}

/* double -> E4M3, round to nearest even, saturating finite values to +-448. */
uint8_t oracle_f64_to_e4m3(double x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0;
    if (isnan(x)) return 0x7f;
    double r = round_to_format(x, 3, -6);
    double a = fabs(r);
    if (a > 448.0 || isinf(a)) a = 448.0;              /* saturate */
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -6)) {                          /* subnormal */
        return sign | (uint8_t)(a / ldexp(1.0, -9));
    }
    int e;
    double f = frexp(a, &e);
    int biased = e - 1 + 7;
    uint8_t frac = (uint8_t)((f * 2.0 - 1.0) * 8.0);
    return sign | (uint8_t)(biased << 3) | frac;
}

static double decode16(uint16_t bits, int dtype)
{
    return dtype == ORACLE_BF16 ? oracle_bf16_to_f64(bits) : oracle_f16_to_f64(bits);
}

/* ------------------------------------------------------------------------ */
/* Sizes: [P2] §2.1 and [P5] §一.6                                          */
/* ------------------------------------------------------------------------ */

/* Bytes of K plus V that one token occupies over all layers ([P2] §2.1):
 * 2 (K and V) * layers * kv_heads * head_dim * element bytes. */
int64_t oracle_kv_bytes_per_token(int64_t num_layers, int64_t num_kv_heads,
                                  int64_t head_dim, int64_t elem_bytes)
{
    return 2 * num_layers * num_kv_heads * head_dim * elem_bytes;
}

/* [P5] §一.6: one block (page) holds block_size tokens of K and V for one
 * layer: page_size = kv_heads * head_dim * elem_bytes * block_size * 2. */
int64_t oracle_page_size_bytes(int64_t num_kv_heads, int64_t head_dim,
                               int64_t elem_bytes, int64_t block_size)
{
    return num_kv_heads * head_dim * elem_bytes * block_size * 2;
}

/* [P5] §一.6: num_blocks = available_memory / (page_size * num_layers). */
int64_t oracle_num_blocks(int64_t available_bytes, int64_t page_size_bytes,
                          int64_t num_layers)
{
    if (page_size_bytes <= 0 || num_layers <= 0) return -1;
    return available_bytes / (page_size_bytes * num_layers);
}

/* ------------------------------------------------------------------------ */
/* Slot of a logical position: [P5] §一.3                                    */
/* ------------------------------------------------------------------------ */

/* The token at logical (0-based) position pos of a sequence lives in logical
 * block pos div block_size at offset pos mod block_size; its flat slot in the
 * [num_blocks*block_size, ...] view is block_table[block] * block_size + offset. */
int64_t oracle_slot(const int32_t *block_table, int64_t pos, int64_t block_size)
{
    int64_t logical_block = pos / block_size;
    int64_t offset = pos % block_size;
    return (int64_t)block_table[logical_block] * block_size + offset;
}

/* ------------------------------------------------------------------------ */
/* Cache write: [P5] §一.2 (the flat slot view) and §一.3 (slot mapping)      */
/* ------------------------------------------------------------------------ */

/*
 * For every new token t with slot = slot_mapping[t] >= 0, copy the bytes of
 * key[t, :, :] into key_cache_flat[slot, :, :] and value[t] into
 * value_cache_flat[slot].  key/value rows are `key_stride` / `value_stride`
 * elements apart (a row holds num_kv_heads*head_dim elements).  A pure byte
 * copy: the result must match the GPU cache bit for bit.
 * Returns ORACLE_BAD_SLOT (after skipping the token) if a slot is out of range.
 */
int oracle_reshape_and_cache(const uint16_t *key, const uint16_t *value,
                             uint16_t *key_cache, uint16_t *value_cache,
                             const int64_t *slot_mapping, int64_t num_tokens,
                             int64_t num_kv_heads, int64_t head_dim,
                             int64_t num_blocks, int64_t block_size,
                             int64_t key_stride, int64_t value_stride)
{
    int rc = ORACLE_OK;
    int64_t row = num_kv_heads * head_dim;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;                       /* padding token */
        if (slot >= num_blocks * block_size) { rc = ORACLE_BAD_SLOT; continue; }
        memcpy(key_cache + slot * row, key + t * key_stride, (size_t)row * 2);
        memcpy(value_cache + slot * row, value + t * value_stride, (size_t)row * 2);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Block copy for copy-on-write: [P1] §第一讲, [P2] §3.3                      */
/* ------------------------------------------------------------------------ */

/*
 * Copy-on-write: before a sequence writes into a block it shares (ref_count
 * > 1), the block is copied to a private one.  For each pair i, copy the whole
 * block block_mapping[2i] (source) of both caches onto block block_mapping[2i+1]
 * (destination), byte for byte: block_size * num_kv_heads * head_dim
 * elements of elem_bytes each.  Pairs are applied in order.  Returns
 * ORACLE_BAD_BLOCK (after skipping the pair) if an id is out of range.
 */
int oracle_copy_blocks(uint8_t *key_cache, uint8_t *value_cache,
                       const int64_t *block_mapping, int64_t num_pairs,
                       int64_t num_blocks, int64_t block_size, int64_t num_kv_heads,
                       int64_t head_dim, int64_t elem_bytes)
{
    int rc = ORACLE_OK;
    size_t block_bytes = (size_t)(block_size * num_kv_heads * head_dim * elem_bytes);
    for (int64_t i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            rc = ORACLE_BAD_BLOCK;
            continue;
        }
        memmove(key_cache + dst * block_bytes, key_cache + src * block_bytes, block_bytes);
        memmove(value_cache + dst * block_bytes, value_cache + src * block_bytes, block_bytes);
    }
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Decode attention: [P2] §5.3 and [P1] §第三讲                              */
/* ------------------------------------------------------------------------ */

/*
 * Copy the first ctx tokens of one KV head of sequence s out of the paged
 * caches into contiguous [ctx, head_dim] double arrays.  Logical token j lives
 * in physical block block_table[j div bs] at row j mod bs; inside a block the
 * rows are [block_size, num_kv_heads, head_dim].
 */
static int gather_head(double *k_out, double *v_out,
                       const uint16_t *key_cache, const uint16_t *value_cache,
                       const int32_t *block_table, int64_t ctx, int64_t kv_head,
                       int64_t num_kv_heads, int64_t head_dim,
                       int64_t num_blocks, int64_t block_size, int dtype)
{
    for (int64_t j = 0; j < ctx; ++j) {
        int64_t block = block_table[j / block_size];
        int64_t r = j % block_size;
        if (block < 0 || block >= num_blocks) return ORACLE_BAD_BLOCK;
        int64_t base = ((block * block_size + r) * num_kv_heads + kv_head) * head_dim;
        for (int64_t d = 0; d < head_dim; ++d) {
            k_out[j * head_dim + d] = decode16(key_cache[base + d], dtype);
            v_out[j * head_dim + d] = decode16(value_cache[base + d], dtype);
        }
    }
    return ORACLE_OK;
}

/*
 * Attention of one query vector q[head_dim] over tokens [t0, t1) of one
 * contiguous KV head (k, v: [ctx, head_dim]):
 *   z_j = scale * sum_d q_d k_{j,d};  m = max_j z_j;  p_j = exp(z_j - m);
 *   l = sum_j p_j;  acc_d = sum_j p_j v_{j,d}.
 * Two plain passes (max first, then sums).  Writes m, l and acc (unnormalised).
 */
static void attend_range(const double *q, const double *k, const double *v,
                         int64_t head_dim, int64_t t0, int64_t t1,
                         double scale, double *z, double *m_out, double *l_out,
                         double *acc)
{
    double m = -INFINITY;
    for (int64_t j = t0; j < t1; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d) dot += q[d] * k[j * head_dim + d];
        z[j - t0] = scale * dot;
        if (z[j - t0] > m) m = z[j - t0];
    }
    double l = 0.0;
    for (int64_t d = 0; d < head_dim; ++d) acc[d] = 0.0;
    for (int64_t j = t0; j < t1; ++j) {
        double p = exp(z[j - t0] - m);
        l += p;
        for (int64_t d = 0; d < head_dim; ++d) acc[d] += p * v[j * head_dim + d];
    }
    *m_out = m;
    *l_out = l;
}

/*
 * out[s, h, :] = softmax_j(scale * q[s,h,:] . k_j) . v_j over the first
 * context_lens[s] tokens of sequence s, with query head h reading KV head
 * h / (num_heads / num_kv_heads).
 *   query         [num_seqs, num_heads, head_dim]          16-bit bits
 *   key_cache     [num_blocks, block_size, num_kv_heads, head_dim]
 *   value_cache   same
 *   block_tables  [num_seqs, max_blocks_per_seq] int32
 *   context_lens  [num_seqs] int32
 *   out           [num_seqs, num_heads, head_dim] double
 */
int oracle_decode(double *out, const uint16_t *query,
                  const uint16_t *key_cache, const uint16_t *value_cache,
                  const int32_t *block_tables, const int32_t *context_lens,
                  int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                  int64_t head_dim, int64_t num_blocks, int64_t block_size,
                  int64_t max_blocks_per_seq, double scale, int dtype)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || block_size <= 0)
        return ORACLE_BAD_ARG;
    int64_t group = num_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        double *o = out + s * num_heads * head_dim;
        if (ctx <= 0) {
            for (int64_t e = 0; e < num_heads * head_dim; ++e) o[e] = 0.0;
            continue;
        }
        if (ctx > max_blocks_per_seq * block_size) return ORACLE_BAD_ARG;
        double *kc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *vc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *z = malloc(sizeof(double) * (size_t)ctx);
        double *q = malloc(sizeof(double) * (size_t)head_dim);
        if (!kc || !vc || !z || !q) { free(kc); free(vc); free(z); free(q); return ORACLE_NO_MEMORY; }
        for (int64_t h = 0; h < num_heads; ++h) {
            int64_t kvh = h / group;
            if (h % group == 0) {
                int rc = gather_head(kc, vc, key_cache, value_cache,
                                     block_tables + s * max_blocks_per_seq, ctx, kvh,
                                     num_kv_heads, head_dim, num_blocks, block_size, dtype);
                if (rc != ORACLE_OK) { free(kc); free(vc); free(z); free(q); return rc; }
            }
            const uint16_t *qs = query + (s * num_heads + h) * head_dim;
            for (int64_t d = 0; d < head_dim; ++d) q[d] = decode16(qs[d], dtype);
            double m, l;
            double *acc = o + h * head_dim;
            attend_range(q, kc, vc, head_dim, 0, ctx, scale, z, &m, &l, acc);
            for (int64_t d = 0; d < head_dim; ++d) acc[d] /= l;
        }
        free(kc); free(vc); free(z); free(q);
    }
    return ORACLE_OK;
}

/*
 * Split form of the same attention: tokens of sequence s are cut into
 * partitions of `partition_size` logical tokens; for every partition
 * p < ceil(ctx / partition_size) this writes
 *   part_max[s,h,p] = max_j z_j,   part_sum[s,h,p] = sum_j exp(z_j - max),
 *   part_acc[s,h,p,:] = sum_j exp(z_j - max) v_j        (not normalised)
 * over the partition's tokens.  Arrays are [num_seqs, num_heads, max_partitions(, head_dim)].
 * Entries of partitions at or beyond ceil(ctx / partition_size) are left untouched.
 */
int oracle_decode_partitioned(double *part_acc, double *part_max, double *part_sum,
                              const uint16_t *query,
                              const uint16_t *key_cache, const uint16_t *value_cache,
                              const int32_t *block_tables, const int32_t *context_lens,
                              int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                              int64_t head_dim, int64_t num_blocks, int64_t block_size,
                              int64_t max_blocks_per_seq, double scale, int dtype,
                              int64_t partition_size, int64_t max_partitions)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || block_size <= 0 ||
        partition_size <= 0)
        return ORACLE_BAD_ARG;
    int64_t group = num_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        if (ctx <= 0) continue;
        if (ctx > max_blocks_per_seq * block_size) return ORACLE_BAD_ARG;
        int64_t nparts = (ctx + partition_size - 1) / partition_size;
        if (nparts > max_partitions) return ORACLE_BAD_ARG;
        double *kc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *vc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *z = malloc(sizeof(double) * (size_t)partition_size);
        double *q = malloc(sizeof(double) * (size_t)head_dim);
        if (!kc || !vc || !z || !q) { free(kc); free(vc); free(z); free(q); return ORACLE_NO_MEMORY; }
        for (int64_t h = 0; h < num_heads; ++h) {
            int64_t kvh = h / group;
            if (h % group == 0) {
                int rc = gather_head(kc, vc, key_cache, value_cache,
                                     block_tables + s * max_blocks_per_seq, ctx, kvh,
                                     num_kv_heads, head_dim, num_blocks, block_size, dtype);
                if (rc != ORACLE_OK) { free(kc); free(vc); free(z); free(q); return rc; }
            }
            const uint16_t *qs = query + (s * num_heads + h) * head_dim;
            for (int64_t d = 0; d < head_dim; ++d) q[d] = decode16(qs[d], dtype);
            for (int64_t p = 0; p < nparts; ++p) {
                int64_t t0 = p * partition_size;
                int64_t t1 = t0 + partition_size < ctx ? t0 + partition_size : ctx;
                int64_t idx = (s * num_heads + h) * max_partitions + p;
                attend_range(q, kc, vc, head_dim, t0, t1, scale, z,
                             &part_max[idx], &part_sum[idx], part_acc + idx * head_dim);
            }
        }
        free(kc); free(vc); free(z); free(q);
    }
    return ORACLE_OK;
}

/*
 * Log-sum-exp merge of the partitions of oracle_decode_partitioned:
 *   M = max_p m_p,  w_p = exp(m_p - M),  L = sum_p w_p l_p,
 *   out = (sum_p w_p acc_p) / L     over p < ceil(ctx / partition_size);
 * ctx == 0 gives zeros.
 */
int oracle_lse_merge(double *out, const double *part_acc, const double *part_max,
                     const double *part_sum, const int32_t *context_lens,
                     int64_t num_seqs, int64_t num_heads, int64_t head_dim,
                     int64_t partition_size, int64_t max_partitions)
{
    if (partition_size <= 0) return ORACLE_BAD_ARG;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        int64_t nparts = ctx > 0 ? (ctx + partition_size - 1) / partition_size : 0;
        if (nparts > max_partitions) return ORACLE_BAD_ARG;
        for (int64_t h = 0; h < num_heads; ++h) {
            double *o = out + (s * num_heads + h) * head_dim;
            int64_t base = (s * num_heads + h) * max_partitions;
            for (int64_t d = 0; d < head_dim; ++d) o[d] = 0.0;
            if (nparts == 0) continue;
            double big_m = -INFINITY;
            for (int64_t p = 0; p < nparts; ++p)
                if (part_max[base + p] > big_m) big_m = part_max[base + p];
            double big_l = 0.0;
            for (int64_t p = 0; p < nparts; ++p) {
                double w = exp(part_max[base + p] - big_m);
                big_l += w * part_sum[base + p];
                for (int64_t d = 0; d < head_dim; ++d)
                    o[d] += w * part_acc[(base + p) * head_dim + d];
            }
            for (int64_t d = 0; d < head_dim; ++d) o[d] /= big_l;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* FP8 KV cache ("vLLM PagedAttention 原理与源码深度解析" §8.4: --kv-cache-dtype fp8) */
/* ------------------------------------------------------------------------ */

/*
 * Quantising cache write: like oracle_reshape_and_cache, but each element x
 * of key (value) is stored as E4M3 of the float product x * inv_k (x * inv_v),
 * where inv = 1.0f / scale is computed in float and the product is a float
 * multiplication -- the same two roundings a GPU takes -- then rounded to
 * E4M3 nearest-even with saturation.  The stored code dequantises as
 * code * scale.
 */
int oracle_reshape_and_cache_fp8(const uint16_t *key, const uint16_t *value,
                                 uint8_t *key_cache, uint8_t *value_cache,
                                 const int64_t *slot_mapping, int64_t num_tokens,
                                 int64_t num_kv_heads, int64_t head_dim,
                                 int64_t num_blocks, int64_t block_size,
                                 int64_t key_stride, int64_t value_stride,
                                 float k_scale, float v_scale, int dtype)
{
    int rc = ORACLE_OK;
    int64_t row = num_kv_heads * head_dim;
    float inv_k = 1.0f / k_scale, inv_v = 1.0f / v_scale;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_blocks * block_size) { rc = ORACLE_BAD_SLOT; continue; }
        for (int64_t e = 0; e < row; ++e) {
            float kx = (float)decode16(key[t * key_stride + e], dtype);
            float vx = (float)decode16(value[t * value_stride + e], dtype);
            key_cache[slot * row + e] = oracle_f64_to_e4m3((double)(kx * inv_k));
            value_cache[slot * row + e] = oracle_f64_to_e4m3((double)(vx * inv_v));
        }
    }
    return rc;
}

/*
 * Decode over an E4M3 cache: exactly oracle_decode with every cached K (V)
 * element replaced by its dequantised value code * k_scale (code * v_scale),
 * in double.  query is 16-bit (dtype).
 */
int oracle_decode_fp8(double *out, const uint16_t *query,
                      const uint8_t *key_cache, const uint8_t *value_cache,
                      const int32_t *block_tables, const int32_t *context_lens,
                      int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads,
                      int64_t head_dim, int64_t num_blocks, int64_t block_size,
                      int64_t max_blocks_per_seq, double scale, double k_scale,
                      double v_scale, int dtype)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || block_size <= 0)
        return ORACLE_BAD_ARG;
    int64_t group = num_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        double *o = out + s * num_heads * head_dim;
        if (ctx <= 0) {
            for (int64_t e = 0; e < num_heads * head_dim; ++e) o[e] = 0.0;
            continue;
        }
        if (ctx > max_blocks_per_seq * block_size) return ORACLE_BAD_ARG;
        double *kc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *vc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *z = malloc(sizeof(double) * (size_t)ctx);
        double *q = malloc(sizeof(double) * (size_t)head_dim);
        if (!kc || !vc || !z || !q) { free(kc); free(vc); free(z); free(q); return ORACLE_NO_MEMORY; }
        const int32_t *bt = block_tables + s * max_blocks_per_seq;
        for (int64_t h = 0; h < num_heads; ++h) {
            int64_t kvh = h / group;
            if (h % group == 0) {
                for (int64_t j = 0; j < ctx; ++j) {
                    int64_t block = bt[j / block_size];
                    int64_t r = j % block_size;
                    if (block < 0 || block >= num_blocks) {
                        free(kc); free(vc); free(z); free(q);
                        return ORACLE_BAD_BLOCK;
                    }
                    int64_t base = ((block * block_size + r) * num_kv_heads + kvh) * head_dim;
                    for (int64_t d = 0; d < head_dim; ++d) {
                        kc[j * head_dim + d] = oracle_e4m3_to_f64(key_cache[base + d]) * k_scale;
                        vc[j * head_dim + d] = oracle_e4m3_to_f64(value_cache[base + d]) * v_scale;
                    }
                }
            }
            const uint16_t *qs = query + (s * num_heads + h) * head_dim;
            for (int64_t d = 0; d < head_dim; ++d) q[d] = decode16(qs[d], dtype);
            double m, l;
            double *acc = o + h * head_dim;
            attend_range(q, kc, vc, head_dim, 0, ctx, scale, z, &m, &l, acc);
            for (int64_t d = 0; d < head_dim; ++d) acc[d] /= l;
        }
        free(kc); free(vc); free(z); free(q);
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Paged (chunked) prefill: "vLLM PagedAttention 原理与源码深度解析" §8.1       */
/* (Chunked Prefill: a long prompt is processed a chunk of tokens at a time)  */
/* ------------------------------------------------------------------------ */

/*
 * Sequence s contributes q_len = query_starts[s+1] - query_starts[s] query
 * tokens: the LAST q_len positions of its context_lens[s] tokens (their K/V
 * already in the cache).  Query token i sits at position
 * pos = context_lens[s] - q_len + i and attends causally to tokens 0..pos:
 *   out[t, h, :] = softmax_j<=pos(scale * q[t,h,:] . k_j) . v_j,
 * t = query_starts[s] + i, query head h reading KV head h / (H / Hk).
 *   query, out  [T, num_heads, head_dim] (T = query_starts[num_seqs])
 * Requires q_len <= context_lens[s].
 */
int oracle_prefill(double *out, const uint16_t *query,
                   const uint16_t *key_cache, const uint16_t *value_cache,
                   const int32_t *block_tables, const int32_t *context_lens,
                   const int32_t *query_starts, int64_t num_seqs, int64_t num_heads,
                   int64_t num_kv_heads, int64_t head_dim, int64_t num_blocks,
                   int64_t block_size, int64_t max_blocks_per_seq, double scale, int dtype)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || block_size <= 0)
        return ORACLE_BAD_ARG;
    int64_t group = num_heads / num_kv_heads;
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        int64_t q0 = query_starts[s], q_len = query_starts[s + 1] - q0;
        if (q_len <= 0) continue;
        if (q_len > ctx || ctx > max_blocks_per_seq * block_size) return ORACLE_BAD_ARG;
        double *kc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *vc = malloc(sizeof(double) * (size_t)(ctx * head_dim));
        double *z = malloc(sizeof(double) * (size_t)ctx);
        double *q = malloc(sizeof(double) * (size_t)head_dim);
        if (!kc || !vc || !z || !q) { free(kc); free(vc); free(z); free(q); return ORACLE_NO_MEMORY; }
        for (int64_t h = 0; h < num_heads; ++h) {
            int64_t kvh = h / group;
            if (h % group == 0) {
                int rc = gather_head(kc, vc, key_cache, value_cache,
                                     block_tables + s * max_blocks_per_seq, ctx, kvh,
                                     num_kv_heads, head_dim, num_blocks, block_size, dtype);
                if (rc != ORACLE_OK) { free(kc); free(vc); free(z); free(q); return rc; }
            }
            for (int64_t i = 0; i < q_len; ++i) {
                int64_t t = q0 + i;
                int64_t pos = ctx - q_len + i;
                const uint16_t *qs = query + (t * num_heads + h) * head_dim;
                for (int64_t d = 0; d < head_dim; ++d) q[d] = decode16(qs[d], dtype);
                double m, l;
                double *acc = out + (t * num_heads + h) * head_dim;
                attend_range(q, kc, vc, head_dim, 0, pos + 1, scale, z, &m, &l, acc);
                for (int64_t d = 0; d < head_dim; ++d) acc[d] /= l;
            }
        }
        free(kc); free(vc); free(z); free(q);
    }
    return ORACLE_OK;
}

// pa_decode_fp8.cuh -- page steps of paged decode attention over an E4M3
// (fp8) KV cache ("vLLM PagedAttention 原理与源码深度解析" §8.4 names the
// --kv-cache-dtype fp8 option; the scheme here is one scale per cache tensor:
// a stored code c means c * k_scale for K and c * v_scale for V).
//
// A cached row of head_dim 128 is 128 bytes: one 128-byte-swizzled TMA box
// per page and tensor, so a page of one head is 2 KB instead of 4 KB.  The
// query stays 16-bit; k_scale is folded into the logit scale and v_scale into
// the output, so the page steps below work on the raw codes:
//  - MmaFp8WarpT (groups of up to 8 query heads, one included): both
//    products transposed, so that the page's tokens and the head's dims fill
//    the mma's 16 rows and the query heads its 8 columns.  Half the mma and
//    accumulators of MmaFp8Warp; 122 registers, four CTAs per SM.
//  - MmaFp8Warp (groups of 9 to 16: fp16 mma on a 16-row tile whose rows are
//    the group's heads; the same tile served every group size before the
//    transposed step, and for one head the tensor cores took the products
//    off the issue path, measured 7 % faster than packed fp32 FMA on CUDA
//    cores): the page is read with the same b16 ldmatrix as
//    the 16-bit path, which hands each lane 4 consecutive codes of a row
//    where the 16-bit fragment layout expects 2 + 2 codes 8 apart.  Inside
//    one 16-element k-step that is a fixed permutation of the head dims, so
//    Q's A fragments are loaded with the same permutation and S = Q K^T is
//    unchanged.  For P.V the transposed ldmatrix hands each lane 2 tokens x
//    2 dims; a byte permute splits them into the even-dim and odd-dim
//    fragments of two n-tiles, and the output dims are put back in order
//    when the warp publishes its rows.
#pragma once

#include "pa_decode.cuh"

namespace pa {

// ---------------------------------------------------------------------------
// Tensor-core path with a 16-row query tile (groups of 9 to 16), head_dim 128.
//
// Both products run as fp16 mma whatever the query dtype: E4M3 -> fp16 is one
// exact conversion, and P in fp16 keeps 11 bits.  A bf16 (or fp16) query row
// is brought into fp16 range exactly by a power of two 2^s chosen from its
// largest element (that element lands in [2^13, 2^14)); 2^-s is folded into
// the row's logit scale.  Only elements more than 2^27 below the row's
// largest can lose bits, and they cannot move a logit.
// ---------------------------------------------------------------------------
// 2^e as a float, e in [-126, 127].
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((e + 127) << 23); }

// The s for which 2^s brings a row whose largest |element| is mx into
// [2^13, 2^14) (0 for an all-zero row).
__device__ __forceinline__ int query_prescale_exp(float mx) {
  if (!(mx > 0.f)) return 0;
  const int e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xff) - 127;  // floor(log2 mx)
  return max(-100, min(100, 13 - e));
}

template <int D, bool BF16>
struct MmaFp8Warp {
  static_assert(D == 128, "fp8 tensor-core path is built for head_dim 128");
  static constexpr int kMinBlocks = 3;  // three CTAs per SM: at most 168 registers
  static constexpr int KSTEPS = D / 16;
  static constexpr int NTILES = D / 8;
  uint32_t qa[KSTEPS][4];   // fp16 Q fragments, head dims permuted as the fp8 K fragments
  float acc[NTILES][4];     // n-tile 2c: even dims of 16-dim chunk c; 2c+1: odd dims
  float m[2], l[2];
  float rs[2];              // 2^-s of rows r0, r1 (undo the query prescale)

  __device__ __forceinline__ void init(const uint16_t* q_group, int group, int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8, tig = lane & 3;
    float2 v0[KSTEPS][2], v1[KSTEPS][2];
    float mx0 = 0.f, mx1 = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      // k positions tig*2+{0,1} hold dims 4*tig+{0,1}; positions tig*2+8+{0,1}
      // hold dims 4*tig+{2,3} of this 16-dim step
      const int d0 = kk * 16 + tig * 4;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q_group + r0 * D);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q_group + r1 * D);
      v0[kk][0] = unpack2<BF16>(r0 < group ? q0[d0 >> 1] : 0u);
      v0[kk][1] = unpack2<BF16>(r0 < group ? q0[(d0 >> 1) + 1] : 0u);
      v1[kk][0] = unpack2<BF16>(r1 < group ? q1[d0 >> 1] : 0u);
      v1[kk][1] = unpack2<BF16>(r1 < group ? q1[(d0 >> 1) + 1] : 0u);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        mx0 = fmaxf(mx0, fmaxf(fabsf(v0[kk][h].x), fabsf(v0[kk][h].y)));
        mx1 = fmaxf(mx1, fmaxf(fabsf(v1[kk][h].x), fabsf(v1[kk][h].y)));
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const int s0 = query_prescale_exp(mx0), s1 = query_prescale_exp(mx1);
    const float f0 = pow2i(s0), f1 = pow2i(s1);
    rs[0] = pow2i(-s0);
    rs[1] = pow2i(-s1);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qa[kk][0] = pack2<false>(v0[kk][0].x * f0, v0[kk][0].y * f0);
      qa[kk][2] = pack2<false>(v0[kk][1].x * f0, v0[kk][1].y * f0);
      qa[kk][1] = pack2<false>(v1[kk][0].x * f1, v1[kk][0].y * f1);
      qa[kk][3] = pack2<false>(v1[kk][1].x * f1, v1[kk][1].y * f1);
    }
#pragma unroll
    for (int n = 0; n < NTILES; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    m[0] = m[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  __device__ __forceinline__ void page(uint32_t kbase, uint32_t vbase, int tok0, int t_end,
                                       float scale_log2, int lane) {
    const int tig = lane & 3;
    // ---- S = Q K^T: one x4 ldmatrix covers two k-steps for both 8-token n-tiles ----
    float sc[2][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) sc[0][i] = sc[1][i] = 0.f;
    const int mtok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int mchk = lane >> 4;
#pragma unroll
    for (int kp = 0; kp < KSTEPS / 2; ++kp) {
      const int c = 2 * kp + mchk;
      uint32_t r0, r1, r2, r3;  // (tok 0-7, chunk 2kp) (8-15, 2kp) (0-7, 2kp+1) (8-15, 2kp+1)
      ldsm_x4(kbase + mtok * 128 + ((c ^ (mtok & 7)) << 4), r0, r1, r2, r3);
      mma_16816<false>(sc[0], qa[2 * kp], e4m3x2_to_h2(r0), e4m3x2_to_h2(r0 >> 16));
      mma_16816<false>(sc[1], qa[2 * kp], e4m3x2_to_h2(r1), e4m3x2_to_h2(r1 >> 16));
      mma_16816<false>(sc[0], qa[2 * kp + 1], e4m3x2_to_h2(r2), e4m3x2_to_h2(r2 >> 16));
      mma_16816<false>(sc[1], qa[2 * kp + 1], e4m3x2_to_h2(r3), e4m3x2_to_h2(r3 >> 16));
    }
    // ---- scale (with each row's 2^-s), mask, online softmax ----
    const float sl0 = scale_log2 * rs[0], sl1 = scale_log2 * rs[1];
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = tok0 + nt * 8 + tig * 2 + (i & 1);
        const float x = t < t_end ? sc[nt][i] * (i < 2 ? sl0 : sl1) : -INFINITY;
        sc[nt][i] = x;
        if (i < 2) mx0 = fmaxf(mx0, x); else mx1 = fmaxf(mx1, x);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    // token 0 of the page is always live, so both maxima are finite
    const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);
    const float al0 = ex2(m[0] - mn0), al1 = ex2(m[1] - mn1);
    m[0] = mn0;
    m[1] = mn1;
    // ---- P in fp16; l sums the same rounded values ----
    uint32_t pa[4];
    pa[0] = pack2<false>(ex2(sc[0][0] - mn0), ex2(sc[0][1] - mn0));
    pa[2] = pack2<false>(ex2(sc[1][0] - mn0), ex2(sc[1][1] - mn0));
    pa[1] = pack2<false>(ex2(sc[0][2] - mn1), ex2(sc[0][3] - mn1));
    pa[3] = pack2<false>(ex2(sc[1][2] - mn1), ex2(sc[1][3] - mn1));
    {
      const float2 u = unpack2<false>(pa[0]), v = unpack2<false>(pa[2]);
      const float2 w = unpack2<false>(pa[1]), z = unpack2<false>(pa[3]);
      l[0] = l[0] * al0 + ((u.x + u.y) + (v.x + v.y));
      l[1] = l[1] * al1 + ((w.x + w.y) + (z.x + z.y));
    }
#pragma unroll
    for (int n = 0; n < NTILES; ++n) {
      acc[n][0] *= al0;
      acc[n][1] *= al0;
      acc[n][2] *= al1;
      acc[n][3] *= al1;
    }
    // ---- O += P V: one transposed x4 ldmatrix covers two 16-dim chunks.  Each
    // register holds codes [t0: d, d+1][t1: d, d+1] (t0 = 2*tig, d = 2*(lane/4));
    // bytes {0, 2} feed the even-dim n-tile, bytes {1, 3} the odd-dim one. ----
#pragma unroll
    for (int cp = 0; cp < D / 32; ++cp) {
      const int c = 2 * cp + mchk;
      uint32_t r0, r1, r2, r3;  // (tok 0-7, chunk 2cp) (8-15, 2cp) (0-7, 2cp+1) (8-15, 2cp+1)
      ldsm_x4_trans(vbase + mtok * 128 + ((c ^ (mtok & 7)) << 4), r0, r1, r2, r3);
      mma_16816<false>(acc[4 * cp + 0], pa, e4m3x2_to_h2(__byte_perm(r0, 0, 0x0020)),
                       e4m3x2_to_h2(__byte_perm(r1, 0, 0x0020)));
      mma_16816<false>(acc[4 * cp + 1], pa, e4m3x2_to_h2(__byte_perm(r0, 0, 0x0031)),
                       e4m3x2_to_h2(__byte_perm(r1, 0, 0x0031)));
      mma_16816<false>(acc[4 * cp + 2], pa, e4m3x2_to_h2(__byte_perm(r2, 0, 0x0020)),
                       e4m3x2_to_h2(__byte_perm(r3, 0, 0x0020)));
      mma_16816<false>(acc[4 * cp + 3], pa, e4m3x2_to_h2(__byte_perm(r2, 0, 0x0031)),
                       e4m3x2_to_h2(__byte_perm(r3, 0, 0x0031)));
    }
  }

  // Rows < group into the merge buffers, head dims back in order: chunk c's
  // dims 4*tig .. 4*tig+3 are (even c0, odd c0, even c1, odd c1).
  __device__ __forceinline__ void publish(float* red_acc, float* red_m, float* red_l, int group,
                                          int lane) {
    const int r0 = lane >> 2, r1 = r0 + 8, tig = lane & 3;
    float l0 = l[0], l1 = l[1];
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (r0 < group) {
#pragma unroll
      for (int c = 0; c < D / 16; ++c)
        *reinterpret_cast<float4*>(red_acc + r0 * D + c * 16 + tig * 4) =
            make_float4(acc[2 * c][0], acc[2 * c + 1][0], acc[2 * c][1], acc[2 * c + 1][1]);
      if (tig == 0) {
        red_m[r0] = m[0];
        red_l[r0] = l0;
      }
    }
    if (r1 < group) {
#pragma unroll
      for (int c = 0; c < D / 16; ++c)
        *reinterpret_cast<float4*>(red_acc + r1 * D + c * 16 + tig * 4) =
            make_float4(acc[2 * c][2], acc[2 * c + 1][2], acc[2 * c][3], acc[2 * c + 1][3]);
      if (tig == 0) {
        red_m[r1] = m[1];
        red_l[r1] = l1;
      }
    }
  }
};

// Four E4M3 codes -> two half2 (codes 0, 1 -> lo; codes 2, 3 -> hi), exactly.
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}


// ---------------------------------------------------------------------------
// Tensor-core path for groups of up to 8 query heads: both products
// transposed, S^T = K Q^T and O^T = V^T P^T.  The page's 16 tokens (first
// product) and 16-dim slices of the head (second) are the M = 16 rows of the
// mma, the group's query heads its N = 8 columns.  Against the 16-row query
// tile of MmaFp8Warp this halves the mma per page (8 + 8 instead of 16 + 16)
// and the accumulator registers: a small group no longer carries 8 or more
// padding rows.
//  - K: the b16 ldmatrix hands lane (g, t) codes 4t .. 4t+3 of token g (and
//    g + 8) in a 16-dim chunk.  The k-step takes dims 4t, 4t+1 at positions
//    2t, 2t+1 and dims 4t+2, 4t+3 at 2t+8, 2t+9; Q's B fragment is then the
//    same four consecutive dims of query row g.
//  - P: the S^T accumulator holds (token g or g + 8; query rows 2t, 2t+1),
//    and the B operand of the second product wants (tokens 2t, 2t+1; row g):
//    one movmatrix transpose per 8 tokens, after the fp16 packing.
//  - V: the transposed ldmatrix hands lane (g, t) tokens 2t, 2t+1 of dims
//    2g, 2g+1 of a chunk; one byte permute over two chunks gathers the
//    even-dim (or odd-dim) codes of two m-tile rows.  M-tile 2c holds the even
//    dims of chunks 2c, 2c+1 (row g: dim 32c + 2g; row g + 8: dim 32c + 16 +
//    2g), m-tile 2c + 1 the odd dims; publish puts them back in order.
// ---------------------------------------------------------------------------
template <int D, bool BF16>
struct MmaFp8WarpT {
  static_assert(D == 128, "fp8 tensor-core path is built for head_dim 128");
  static constexpr int kMinBlocks = 4;  // CTAs per SM the register budget is built for
  static constexpr int KSTEPS = D / 16;
  static constexpr int MTILES = D / 16;
  static constexpr float kSlack = 8.f;  // log2 units the reference max may trail by
  uint32_t qb[KSTEPS][2];  // fp16 Q^T fragments of query row lane / 4
  float acc[MTILES][4];    // O^T: (m-tile row g, query row 2t | 2t+1), (row g + 8, ...)
  float m[2], l[2];        // query rows 2t, 2t+1: reference max (log2), lane-partial sum
  float mt[2];             // and their true running max
  float rs[2];             // 2^-s of query rows 2t, 2t+1 (undo the query prescale)

  __device__ __forceinline__ void init(const uint16_t* q_group, int group, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float4 v[KSTEPS];
    float mx = 0.f;
    const uint16_t* qrow = q_group + g * D;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const uint2 w = g < group ? *reinterpret_cast<const uint2*>(qrow + kk * 16 + 4 * t)
                                : make_uint2(0u, 0u);
      const float2 x = unpack2<BF16>(w.x), y = unpack2<BF16>(w.y);
      v[kk] = make_float4(x.x, x.y, y.x, y.y);
      mx = fmaxf(mx, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(y.x), fabsf(y.y))));
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const int s = query_prescale_exp(mx);
    const float f = pow2i(s);
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qb[kk][0] = pack2<false>(v[kk].x * f, v[kk].y * f);
      qb[kk][1] = pack2<false>(v[kk].z * f, v[kk].w * f);
    }
    // the exponents of query rows 2t and 2t + 1 sit in lanes 8t and 8t + 4
    const int s0 = __shfl_sync(0xffffffffu, s, 8 * t), s1 = __shfl_sync(0xffffffffu, s, 8 * t + 4);
    rs[0] = pow2i(-s0);
    rs[1] = pow2i(-s1);
#pragma unroll
    for (int i = 0; i < MTILES; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    m[0] = m[1] = mt[0] = mt[1] = -INFINITY;
    l[0] = l[1] = 0.f;
  }

  __device__ __forceinline__ void page(uint32_t kbase, uint32_t vbase, int tok0, int t_end,
                                       float scale_log2, int lane) {
    const int g = lane >> 2;
    const int mtok = ((lane >> 3) & 1) * 8 + (lane & 7);
    const int mchk = lane >> 4;
    // ---- S^T = K Q^T: one x4 ldmatrix covers two k-steps (two accumulator chains) ----
    float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kp = 0; kp < KSTEPS / 2; ++kp) {
      const int c = 2 * kp + mchk;
      uint32_t r0, r1, r2, r3;  // (tok 0-7, chunk 2kp) (8-15, 2kp) (0-7, 2kp+1) (8-15, 2kp+1)
      ldsm_x4(kbase + mtok * 128 + ((c ^ (mtok & 7)) << 4), r0, r1, r2, r3);
      uint32_t a[4], b[4];
      e4m3x4_to_h2x2(r0, a[0], a[2]);
      e4m3x4_to_h2x2(r1, a[1], a[3]);
      e4m3x4_to_h2x2(r2, b[0], b[2]);
      e4m3x4_to_h2x2(r3, b[1], b[3]);
      mma_16816<false>(s0, a, qb[2 * kp][0], qb[2 * kp][1]);
      mma_16816<false>(s1, b, qb[2 * kp + 1][0], qb[2 * kp + 1][1]);
    }
    // ---- scale (with each row's 2^-s), mask, row maxima over the 16 tokens ----
    const float sl0 = scale_log2 * rs[0], sl1 = scale_log2 * rs[1];
    const int lim = t_end - tok0;
    const bool lo_live = g < lim, hi_live = g + 8 < lim;
    const float x0 = lo_live ? (s0[0] + s1[0]) * sl0 : -INFINITY;  // token g, row 2t
    const float x1 = lo_live ? (s0[1] + s1[1]) * sl1 : -INFINITY;  // token g, row 2t+1
    const float x2 = hi_live ? (s0[2] + s1[2]) * sl0 : -INFINITY;  // token g+8, row 2t
    const float x3 = hi_live ? (s0[3] + s1[3]) * sl1 : -INFINITY;  // token g+8, row 2t+1
    // lanes of equal t hold the same two rows; each reduces one of them over
    // the 8 lanes and the other comes back from the neighbour of opposite g parity
    const bool odd = g & 1;
    float keep = odd ? fmaxf(x1, x3) : fmaxf(x0, x2);
    const float send = odd ? fmaxf(x0, x2) : fmaxf(x1, x3);
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, keep, 8));
    keep = fmaxf(keep, __shfl_xor_sync(0xffffffffu, keep, 16));
    const float other = __shfl_xor_sync(0xffffffffu, keep, 4);
    mt[0] = fmaxf(mt[0], odd ? other : keep);
    mt[1] = fmaxf(mt[1], odd ? keep : other);
    // The reference max m trails the true one by at most 2^kSlack, so P stays
    // at most 2^8 (exact in fp16 up to its 11 bits); O and l are rescaled only
    // when some row of the warp outgrows that, a branch the whole warp takes.
    if (__any_sync(0xffffffffu, (mt[0] > m[0] + kSlack) | (mt[1] > m[1] + kSlack))) {
      const float al0 = ex2(m[0] - mt[0]), al1 = ex2(m[1] - mt[1]);
      m[0] = mt[0];
      m[1] = mt[1];
      l[0] *= al0;
      l[1] *= al1;
#pragma unroll
      for (int i = 0; i < MTILES; ++i) {
        acc[i][0] *= al0;
        acc[i][1] *= al1;
        acc[i][2] *= al0;
        acc[i][3] *= al1;
      }
    }
    // ---- P in fp16, l sums the same rounded values, then P^T as a B operand ----
    const uint32_t p_lo = pack2<false>(ex2(x0 - m[0]), ex2(x1 - m[1]));  // token g
    const uint32_t p_hi = pack2<false>(ex2(x2 - m[0]), ex2(x3 - m[1]));  // token g + 8
    {
      const float2 u = unpack2<false>(p_lo), w = unpack2<false>(p_hi);
      l[0] += u.x + w.x;
      l[1] += u.y + w.y;
    }
    const uint32_t pb0 = movmatrix_trans(p_lo);  // tokens 2t, 2t+1 of query row g
    const uint32_t pb1 = movmatrix_trans(p_hi);  // tokens 2t+8, 2t+9
    // ---- O^T += V^T P^T: one transposed x4 ldmatrix covers two 16-dim chunks ----
#pragma unroll
    for (int cp = 0; cp < D / 32; ++cp) {
      const int c = 2 * cp + mchk;
      uint32_t r0, r1, r2, r3;  // (tok 0-7, chunk 2cp) (8-15, 2cp) (0-7, 2cp+1) (8-15, 2cp+1)
      ldsm_x4_trans(vbase + mtok * 128 + ((c ^ (mtok & 7)) << 4), r0, r1, r2, r3);
      uint32_t ae[4], ao[4];  // rows g (chunk 2cp) and g + 8 (chunk 2cp+1); tokens 2t.. | 2t+8..
      e4m3x4_to_h2x2(__byte_perm(r0, r2, 0x6420), ae[0], ae[1]);
      e4m3x4_to_h2x2(__byte_perm(r1, r3, 0x6420), ae[2], ae[3]);
      e4m3x4_to_h2x2(__byte_perm(r0, r2, 0x7531), ao[0], ao[1]);
      e4m3x4_to_h2x2(__byte_perm(r1, r3, 0x7531), ao[2], ao[3]);
      mma_16816<false>(acc[2 * cp], ae, pb0, pb1);
      mma_16816<false>(acc[2 * cp + 1], ao, pb0, pb1);
    }
  }

  // Query rows < group into the merge buffers, head dims in order.
  // The partials are restated against the true max (a factor <= 1).
  __device__ __forceinline__ void publish(float* red_acc, float* red_m, float* red_l, int group,
                                          int lane) {
    const int g = lane >> 2, t = lane & 3;
    float f[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) f[h] = mt[h] > -INFINITY ? ex2(m[h] - mt[h]) : 1.f;
    float l0 = l[0] * f[0], l1 = l[1] * f[1];
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = 2 * t + h;
      if (row < group) {
#pragma unroll
        for (int cp = 0; cp < D / 32; ++cp) {
          float* o = red_acc + row * D + cp * 32 + 2 * g;
          *reinterpret_cast<float2*>(o) =
              make_float2(acc[2 * cp][h] * f[h], acc[2 * cp + 1][h] * f[h]);
          *reinterpret_cast<float2*>(o + 16) =
              make_float2(acc[2 * cp][2 + h] * f[h], acc[2 * cp + 1][2 + h] * f[h]);
        }
        if (g == 0) {
          red_m[row] = mt[h];
          red_l[row] = h ? l1 : l0;
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Quantising cache write: key/value rows (16-bit) -> E4M3 codes of x * inv_scale
// (float product, nearest even, saturating).  One thread makes one 16-byte
// chunk (16 elements) of K and the same chunk of V.
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256)
    reshape_and_cache_fp8_kernel(const uint16_t* __restrict__ key,
                                 const uint16_t* __restrict__ value, long long key_stride,
                                 long long value_stride, uint8_t* __restrict__ key_cache,
                                 uint8_t* __restrict__ value_cache,
                                 const int64_t* __restrict__ slot_mapping, long long num_tokens,
                                 int chunks_per_token, long long num_slots, float inv_k,
                                 float inv_v) {
  pdl_launch_dependents();
  pdl_wait();
  const long long total = num_tokens * chunks_per_token;
  const long long row = static_cast<long long>(chunks_per_token) * 16;  // bytes per cache row
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / chunks_per_token;
    const int c = static_cast<int>(i - t * chunks_per_token);
    const long long slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (c == 0) record_error(kErrSlot, t);
      continue;
    }
    auto quantise = [](const uint16_t* src, float inv) {
      const uint4 a = *reinterpret_cast<const uint4*>(src);
      const uint4 b = *reinterpret_cast<const uint4*>(src + 8);
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t out[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 u = unpack2<BF16>(w[2 * k]), v = unpack2<BF16>(w[2 * k + 1]);
        out[k] = f2_to_e4m3x2(u.x * inv, u.y * inv) | (f2_to_e4m3x2(v.x * inv, v.y * inv) << 16);
      }
      return make_uint4(out[0], out[1], out[2], out[3]);
    };
    *reinterpret_cast<uint4*>(key_cache + slot * row + c * 16) =
        quantise(key + t * key_stride + c * 16, inv_k);
    *reinterpret_cast<uint4*>(value_cache + slot * row + c * 16) =
        quantise(value + t * value_stride + c * 16, inv_v);
  }
}

}  // namespace pa

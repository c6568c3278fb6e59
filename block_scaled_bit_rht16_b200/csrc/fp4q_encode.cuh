// fp4q_encode.cuh -- per-block encoder shared by the row and dual-orientation kernels.
//
// Input: one 16-element block as P[8] = (v_i, v_{i+8}) after the butterfly (not yet times 1/4),
// the block's dequant multiplier s (0 marks an all-zero block) and its Divider. Output: the
// 8-byte code word pair, optional bf16 dequant, optional statistics.
//
// Rounding follows "蚂蚁集团揭秘…" (techwalker.com) section 二 (round to nearest, ties to even
// code) and "低精度量化技术：IF4…" (bxzpzcl.cn/news/2320061) section 6.1 (stochastic rounding
// floor(x) + (random() < frac), applied between adjacent grid points) and sections 3.1-3.2
// (IF4: FP4 candidate vs INT4 * 7/6 candidate, smaller squared error wins).
#pragma once
#include <cuda_fp16.h>

#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"

namespace fp4q {

struct EncCtx {
  float cinv;       // y = cinv * vraw
  uint64_t seedx;   // SR: seed ^ (stream << 63)
};

__device__ __forceinline__ uint32_t sign_bit(float x) { return __float_as_uint(x) >> 31; }

// Element e (0..15) of a block held as P[i] = (v_i, v_{i+8}).
__device__ __forceinline__ float elem_x(const float2* A, int e) { return e < 8 ? A[e].x : A[e - 8].y; }

// Small exact integer m (0..15) as a float.
__device__ __forceinline__ float small_int_f32(uint32_t m) {
  return __fadd_rn(__uint_as_float(0x4B000000u | m), -8388608.0f);
}

// Uniform grids (E1M2: step 1/2, qmax 3.5; INT4: step 1, qmax 7). Returns the nibble; val is
// the code's signed value in scaled units, mag the magnitude code.
template <int G, int R>
__device__ __forceinline__ uint32_t round_uniform(float q, float vraw, uint32_t rnd, float& val,
                                                  uint32_t& mag) {
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr float inv_step = (G == kE1M2) ? 2.0f : 1.0f;
  const float t = __fmul_rn(fminf(fabsf(q), qmax), inv_step);   // |v| in steps, exact
  uint32_t m;
  if constexpr (R == kRTNE) {
    m = __float_as_uint(__fadd_rn(t, 8388608.0f)) & 0xFu;        // round half to even
  } else {
    const float fl = floorf(t);
    const float frac = __fsub_rn(t, fl);                          // exact
    m = (__float_as_uint(__fadd_rn(fl, 8388608.0f)) & 0xFu) + (sr_up(rnd, frac) ? 1u : 0u);
  }
  const uint32_t neg = sign_bit(vraw);
  mag = m;
  if constexpr (G == kE1M2) {
    const float g = __fmul_rn(small_int_f32(m), 0.5f);
    val = __uint_as_float(__float_as_uint(g) | (neg << 31));      // -0 stays -0 (code 0x8)
    return m | (neg << 3);
  } else {
    const float g = small_int_f32(m);
    val = (neg && m) ? -g : g;                                    // two's complement has no -0
    return (neg ? (0u - m) : m) & 0xFu;
  }
}

// E2M1 stochastic rounding of one value: the chosen grid point, signed like vraw. qmax: 6, or
// the largest value of a range-restricted E2M1 table (4, 3, 2).
__device__ __forceinline__ float e2m1_sr_value(float q, float vraw, uint32_t rnd, float qmax = 6.0f) {
  const float a = fminf(fabsf(q), qmax);
  const bool lo = a < 2.0f, mid = a < 4.0f;
  const float inv_step = lo ? 2.0f : (mid ? 1.0f : 0.5f);
  const float step = lo ? 0.5f : (mid ? 1.0f : 2.0f);
  const float t = __fmul_rn(a, inv_step);   // exact
  const float fl = floorf(t);
  const float frac = __fsub_rn(t, fl);      // exact
  const float k = sr_up(rnd, frac) ? __fadd_rn(fl, 1.0f) : fl;
  const float g = __fmul_rn(k, step);       // exact: a grid point
  return __uint_as_float(__float_as_uint(g) | (__float_as_uint(vraw) & 0x80000000u));
}

__device__ __forceinline__ float with_sign_of(float q, float vraw) {
  return __uint_as_float((__float_as_uint(q) & 0x7FFFFFFFu) | (__float_as_uint(vraw) & 0x80000000u));
}

// ------------------------------------------------------------------ lean encoder (hot path)
//
// FP32 1x16 scale, round to nearest even, codes only.

// Exact RN(a / qmax) for the grid's compile-time qmax: one multiply and two FMAs (the same
// correction step as the element quotients, with the divisor's correctly rounded reciprocal
// folded at compile time), or the IEEE division outside the range where that step is exact.
template <int G>
__device__ __forceinline__ float div_qmax(float a) {
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr float r = 1.0f / qmax;
  if (a >= 0x1p-100f && a <= 0x1p+100f) {
    const float s0 = __fmul_rn(a, r);
    const float e = __fmaf_rn(-s0, qmax, a);
    return __fmaf_rn(e, r, s0);
  }
  return __fdiv_rn(a, qmax);
}

// Low nibbles of t[0..7] packed into one word, t[0] in bits 0..3 (bits above each nibble of
// t are ignored).
__device__ __forceinline__ uint32_t pack_low_nibbles(const uint32_t* t) {
  uint32_t w = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) w = __funnelshift_r(w, t[i], 4);
  return w;
}

// E1M2 codes of eight values given as quarters (e_k = v_k / 4, |e_k| <= 7/8), element k in
// nibble k: the FP6 E2M3 conversion of e, whose subnormal range below 1 has the uniform step 1/8,
// so each code byte is 00s00mmm with mmm = RNE(8 |e|) = RNE(2 |v|) (ties to even, the sign of
// zero kept). Even elements' bytes are converted into one word and odd elements' into another;
// each byte's sign moves to bit 3 (one shift and one three-input logic operation per word, bits
// 4..7 don't-care), and the two words interleave as low and high nibbles.
// fp4q_check_conversions runs it over every input in that range.
__device__ __forceinline__ uint32_t e1m2_word(const float* e) {
  const uint32_t E = cvt_e2m3x2(e[2], e[0]) | (cvt_e2m3x2(e[6], e[4]) << 16);   // e0 e2 e4 e6
  const uint32_t O = cvt_e2m3x2(e[3], e[1]) | (cvt_e2m3x2(e[7], e[5]) << 16);   // e1 e3 e5 e7
  const uint32_t NE = (E & 0x07070707u) | ((E >> 2) & 0xF8F8F8F8u);
  const uint32_t NO = (O & 0x07070707u) | ((O >> 2) & 0xF8F8F8F8u);
  return (NE & 0x0F0F0F0Fu) | ((NO << 4) & 0xF0F0F0F0u);
}

// Codes of one block on E1M2 / INT4 / E2M1 from the (rotated) raw values P, y = P / c with
// c = 4 under rotation and 1 without, and the block scale s. Returns the two code words.
//
// Signs: the element quotients carry the sign of P except for P = -0, where the correction step
// returns +0. Under rotation a butterfly output is -0 only when all sixteen inputs are zeros,
// i.e. in an all-zero block, which encodes as zeros anyway; without rotation the sign is copied
// from P explicitly.
//   E2M1: hardware round-to-nearest-even conversion of v (saturating at 6).
//   E1M2: the FP6 E2M3 conversion of v/4 (e1m2_word): |v/4| <= 7/8 lies in E2M3's subnormal
//         range, whose step 1/8 makes the code sign << 5 | RNE(2|v|) -- the E1M2 magnitude --
//         with ties to even and the sign of zero kept.
//   INT4: t = 1.5 * 2^23 + v rounds v half-to-even into t's low bits in two's complement.
// CLAMP: saturate |v| at qmax before rounding. The FP32 scale needs none (|v| <= qmax up to an
// ulp); E4M3 scales do (the rounded block scale, or a given tensor scale, can leave |v| > qmax).
// amax_raw (CLAMP only): max |P|. Its quotient bounds every element's (the quotient is
// monotonic in the numerator), so a block whose largest quotient stays below qmax + step/2
// rounds no element above qmax, and the clamp, which could not change a code, is skipped.
// The divisor of encode_lean's quotients: c * s, times 4 for E1M2 (whose codes come from v / 4).
template <int G, bool RHT>
constexpr float lean_divisor_factor() { return (RHT ? 4.0f : 1.0f) * (G == kE1M2 ? 4.0f : 1.0f); }

// encode_lean with the block's Divider of s * lean_divisor_factor<G, RHT>() given.
template <int G, bool RHT, bool CLAMP = false>
__device__ __forceinline__ uint2 encode_lean_dv(const float2* P, float s, const Divider& dv,
                                                float amax_raw = 0.0f) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr float kC = RHT ? 4.0f : 1.0f;
  constexpr float kVScale = (G == kE1M2) ? 4.0f : 1.0f;   // quotients of v / kVScale
  float2 Q[8];
  if (dv.fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) Q[i] = div2(dv, P[i]);
    if constexpr (CLAMP && !kIsE2M1<G>) {   // the E2M1 conversion saturates by itself
      constexpr float lim = qmax / kVScale;
      constexpr float half_above = (G == kE1M2 ? 3.75f : 7.5f) / kVScale;   // qmax + step / 2
      if (!(div2(dv, make_float2(amax_raw, amax_raw)).x < half_above)) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          Q[i] = make_float2(fminf(fmaxf(Q[i].x, -lim), lim), fminf(fmaxf(Q[i].y, -lim), lim));
      }
    }
  } else {
    // scale outside the exact range of the correction step (tiny or huge data): IEEE division,
    // then the saturation that the fast range never needs
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float qx = __fdiv_rn(__fmul_rn(P[i].x, 1.0f / kC), s);
      const float qy = __fdiv_rn(__fmul_rn(P[i].y, 1.0f / kC), s);
      Q[i] = make_float2(__fmul_rn(fminf(fmaxf(qx, -qmax), qmax), 1.0f / kVScale),
                         __fmul_rn(fminf(fmaxf(qy, -qmax), qmax), 1.0f / kVScale));
    }
  }
  if constexpr (!RHT && G != kINT4) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      Q[i] = make_float2(with_sign_of(Q[i].x, P[i].x), with_sign_of(Q[i].y, P[i].y));
  }
  uint32_t w[2];
  if constexpr (kIsE2M1<G>) {
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      uint32_t b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = l ? Q[2 * j].y : Q[2 * j].x, hi = l ? Q[2 * j + 1].y : Q[2 * j + 1].x;
        b[j] = cvt_e2m1x2(hi, lo);
      }
      w[l] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    }
  } else if constexpr (G == kE1M2) {
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      float e[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) e[k] = l ? Q[k].y : Q[k].x;
      w[l] = e1m2_word(e);
    }
  } else {
    const float2 c2 = make_float2(12582912.0f, 12582912.0f);   // 1.5 * 2^23
    uint32_t t0[8], t1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 t = __fadd2_rn(Q[i], c2);
      t0[i] = __float_as_uint(t.x);
      t1[i] = __float_as_uint(t.y);
    }
    w[0] = pack_low_nibbles(t0);
    w[1] = pack_low_nibbles(t1);
  }
  return make_uint2(w[0], w[1]);
}

// Round-to-nearest codes of a nonzero block from its exact quotients q[e] (v / 4 for E1M2, the
// divisor of lean_divisor_factor) and raw values raw[e] (for the signs without rotation): the
// code step of encode_lean_dv for the FP32 scale, on quotients computed elsewhere.
template <int G, bool RHT>
__device__ __forceinline__ uint2 lean_codes(const float* q, const float* raw) {
  float v[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = (!RHT && G != kINT4) ? with_sign_of(q[e], raw[e]) : q[e];
  uint32_t w[2];
  if constexpr (kIsE2M1<G>) {
#pragma unroll
    for (int l = 0; l < 2; ++l) {
      uint32_t b[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = cvt_e2m1x2(v[8 * l + 2 * j + 1], v[8 * l + 2 * j]);
      w[l] = b[0] | (b[1] << 8) | (b[2] << 16) | (b[3] << 24);
    }
  } else if constexpr (G == kE1M2) {
    w[0] = e1m2_word(v);
    w[1] = e1m2_word(v + 8);
  } else {
    uint32_t t0[8], t1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 t = __fadd2_rn(make_float2(v[i], v[i + 8]), make_float2(12582912.0f, 12582912.0f));
      t0[i] = __float_as_uint(t.x);
      t1[i] = __float_as_uint(t.y);
    }
    w[0] = pack_low_nibbles(t0);
    w[1] = pack_low_nibbles(t1);
  }
  return make_uint2(w[0], w[1]);
}

template <int G, bool RHT, bool CLAMP = false>
__device__ __forceinline__ uint2 encode_lean(const float2* P, float s, float amax_raw = 0.0f) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  return encode_lean_dv<G, RHT, CLAMP>(P, s, make_divider(s, lean_divisor_factor<G, RHT>()), amax_raw);
}

// Stochastic rounding, FP32 1x16 scale, codes only; runtime rotation factor c (4 or 1).
// Element e (0..15) of the block has logical index 4*quad0 + e and the 16-bit draw u_e.
//
// Per element, with a = min(|v|, qmax) and t = a / step in [0, 8) (exact), the rule "round up
// iff r < t - floor(t)" with r = u * 2^-16 picks k = floor(t) + [r < t - floor(t)] =
// ceil(t - r): t - r lies in (k-1, k]. Every k is read off K = 1.5 * 2^23 + k, exact in the
// unit-spaced binade [2^23, 2^24), whose bit pattern is 0x4B400000 + k. On E2M1, r is formed
// exactly as the float with bits 0x3F800000 + 128u (1 + u * 2^-16) minus 1, D = t - r rounded
// toward +inf stays in (k-1, k] (k is a float), and K = RU(D + 1.5 * 2^23); the step is 1/2, 1
// or 2 on [0, 2), [2, 4), [4, 6] and the code k, k + 2 or k + 4. The uniform grids fold the
// clamp at qmax into a saturating FMA (below). The decision runs on the floating-point pipe;
// the bit patterns of eight elements accumulate as sum(bits_j * 16^j), from which the constant
// part is subtracted once.
// Codes: sign-magnitude (E1M2, E2M1) takes the input's sign bit as bit 3; INT4 takes -k in
// two's complement for a negative input.

// Quotients v_e = RN(P_e / (c * s)) of a nonzero block, exact, with dv the Divider of c * s.
__device__ __forceinline__ void sr_quotients_dv(const float2* P, float s, float c, const Divider& dv,
                                                float* q) {
  const float cinv = __frcp_rn(c);   // exact: c is 4 or 1
  if (dv.fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float2 r = div2(dv, P[i]);
      q[i] = r.x;
      q[i + 8] = r.y;
    }
    // the correction step is exact for quotients of at least 2^-20; smaller nonzero ones (rare)
    // decide stochastic rounding through their exact value, so they take the IEEE division.
    // One block-wide minimum keeps the per-element test off the common path.
    float qmin = fabsf(q[0]);
#pragma unroll
    for (int e = 1; e < 15; e += 2) qmin = min3(qmin, fabsf(q[e]), fabsf(q[e + 1]));
    qmin = fminf(qmin, fabsf(q[15]));
    if (qmin < 0x1p-19f) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float pe = elem_x(P, e);
        if (fabsf(q[e]) < 0x1p-19f && pe != 0.0f) q[e] = __fdiv_rn(__fmul_rn(pe, cinv), s);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) q[e] = __fdiv_rn(__fmul_rn(elem_x(P, e), cinv), s);
  }
}

__device__ __forceinline__ void sr_quotients(const float2* P, float s, float c, float* q) {
  sr_quotients_dv(P, s, c, make_divider(s, c), q);
}

// Bit pattern 0x4B400000 + k of the stochastically rounded magnitude code k of one quotient q
// (element e of its block, draw words d from sr_words16).
template <int G>
__device__ __forceinline__ uint32_t sr_bits(float q, const uint32_t* d, int e) {
  constexpr float qmax = GridInfo<G>::qmax;
  float K;
  if constexpr (kIsE2M1<G>) {
    const float a = fminf(fabsf(q), qmax);
    const float r = __fmaf_rn(sr_one_plus(d, e), 128.0f, -128.0f);   // u * 2^-16, exact
    const bool lo = a < 2.0f, mid = a < 4.0f;
    const float inv_step = lo ? 2.0f : (mid ? 1.0f : 0.5f);
    const float base = lo ? 12582912.0f : (mid ? 12582914.0f : 12582916.0f);
    K = __fadd_ru(__fmaf_ru(a, inv_step, -r), base);
  } else {
    // uniform grids, t = |v| / step with qmax = 7 steps: F = 1 + u * 2^-23 (the draw in the
    // low mantissa bits, one byte permute of its word), c = 16.125 - 16 F = (1 - r) / 8 exactly;
    // w = min(RU((t - r + 1) / 8), 1) (the saturation is the clamp at qmax: t' = min(t, 7));
    // 8w = RU(t' - r + 1), whose ceiling is ceil(t' - r) + 1 (no integer up to 8 lies
    // between a real and its upward rounding), so K = RU(8w + 1.5 * 2^23 - 1) is
    // 1.5 * 2^23 + ceil(t' - r).
    const float F = sr_one_plus(d, e);
    const float c = __fmaf_rn(F, -16.0f, 16.125f);
    constexpr float inv8step = (G == kE1M2) ? 0.25f : 0.125f;
    float w;
    asm("fma.rp.sat.f32 %0, %1, %2, %3;" : "=f"(w) : "f"(fabsf(q)), "f"(inv8step), "f"(c));
    K = __fmaf_ru(w, 8.0f, 12582911.0f);
  }
  return __float_as_uint(K);
}

// sum over j = 0..7 of 0x4B400000 * 16^j, modulo 2^32
constexpr uint32_t kSrBias = 0x4B400000u + (0x4B400000u << 4) + (0x4B400000u << 8) +
                             (0x4B400000u << 12) + (0x4B400000u << 16) + (0x4B400000u << 20) +
                             (0x4B400000u << 24) + (0x4B400000u << 28);

// Appends element e's code to a word built from element 7 down to 0: mags accumulates
// sum bits_j * 16^j, signs the raw values' sign bits at bit 3 of each nibble (sign-magnitude
// grids); INT4 takes -k in two's complement for a negative raw value.
template <int G>
__device__ __forceinline__ void sr_append(uint32_t bits, float raw, uint32_t& mags, uint32_t& signs) {
  if constexpr (G == kINT4) {
    const uint32_t m = (uint32_t)((int32_t)__float_as_uint(raw) >> 31);
    mags = mags * 16u + (((bits ^ m) - m) & 0xFu);
  } else {
    mags = mags * 16u + bits;
    signs = __funnelshift_l(__float_as_uint(raw), signs, 4);
  }
}

template <int G>
__device__ __forceinline__ uint32_t sr_word(uint32_t mags, uint32_t signs) {
  if constexpr (G == kINT4) return mags;
  else return (mags - kSrBias) | (signs & 0x88888888u);
}

// Codes of a nonzero block from its quotients q, draw words d (sr_words16) and raw values raw
// (element e of the block, for the signs).
template <int G>
__device__ __forceinline__ uint2 sr_codes(const float* q, const uint32_t* d, const float* raw) {
  uint32_t w[2];
#pragma unroll
  for (int l = 0; l < 2; ++l) {
    uint32_t mags = 0u, signs = 0u;
#pragma unroll
    for (int j = 7; j >= 0; --j) sr_append<G>(sr_bits<G>(q[8 * l + j], d, 8 * l + j), raw[8 * l + j], mags, signs);
    w[l] = sr_word<G>(mags, signs);
  }
  return make_uint2(w[0], w[1]);
}

template <int G>
__device__ __forceinline__ uint2 encode_sr(const float2* P, float s, float c, uint64_t seedx,
                                          uint64_t quad0) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  float q[16], raw[16];
  sr_quotients(P, s, c, q);
#pragma unroll
  for (int e = 0; e < 16; ++e) raw[e] = elem_x(P, e);
  uint32_t d[8];
  sr_words16(seedx, quad0, d);
  return sr_codes<G>(q, d, raw);
}

// ------------------------------------------------------------------ two blocks at once
//
// Two blocks of one thread held as A[i] = (element i of block 0, element i of block 1),
// i = 0..15: every butterfly stage pairs A[i] with A[i+h] and runs as packed f32x2 operations
// (the same IEEE operations in the same stage order as fwht16, for both blocks at once), and the
// quotients of both blocks come from one packed correction step with a divisor per lane.

__device__ __forceinline__ void fwht16_pair(float2* A) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if ((i & h) == 0) {
        const float2 a = A[i], b = A[i + h];
        A[i] = add2(a, b);
        A[i + h] = sub2(a, b);
      }
    }
  }
}

__device__ __forceinline__ float2 absmax16_pair(const float2* A) {
  float m0 = max3(fabsf(A[0].x), fabsf(A[1].x), fabsf(A[2].x));
  float m1 = max3(fabsf(A[0].y), fabsf(A[1].y), fabsf(A[2].y));
#pragma unroll
  for (int i = 3; i < 15; i += 2) {
    m0 = max3(m0, fabsf(A[i].x), fabsf(A[i + 1].x));
    m1 = max3(m1, fabsf(A[i].y), fabsf(A[i + 1].y));
  }
  return make_float2(fmaxf(m0, fabsf(A[15].x)), fmaxf(m1, fabsf(A[15].y)));
}

// IF4 block, E4M3 block scale (NVFP4's), codes only: the E2M1 candidate (round to nearest even,
// saturating) and the INT4 candidate k = RNE(RN(v * RN(7/6))) clamped to +-7 with value
// RN(k * RN(6/7)); INT4 is kept iff its squared error, summed in FP32 over the balanced pairwise
// tree of elements 0..15, is strictly smaller ("低精度量化技术：IF4…", sections 3.1-3.2).
// Returns the code words; flag = 0x80 for an INT4 block.
// When even the largest |q| times RN(7/6) stays below 7.5, no INT4 candidate needs the clamp at
// +-7 (it could not change a code) and it is skipped.
// dv: the Divider of c * s (c = 4 with rotation, else 1).
template <bool RHT>
__device__ __forceinline__ uint2 encode_if4(const float2* P, float s, const Divider& dv, uint32_t& flag) {
  flag = 0u;
  if (s == 0.0f) return make_uint2(0u, 0u);
  float q[16];
  sr_quotients_dv(P, s, RHT ? 4.0f : 1.0f, dv, q);   // exact quotients, small ones included
  const float r76 = kR76, r67 = kR67;
  float qm = fabsf(q[0]);
#pragma unroll
  for (int e = 1; e < 15; e += 2) qm = max3(qm, fabsf(q[e]), fabsf(q[e + 1]));
  qm = fmaxf(qm, fabsf(q[15]));
  const bool clamp = !(__fmul_rn(qm, r76) < 7.5f);
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  // E2M1 candidate: codes from the signed quotients (-0 keeps its sign), decoded with signs.
  // Byte j of word l holds elements 8l + 2j (low nibble) and 8l + 2j + 1.
  uint32_t fw[2] = {0u, 0u};
  float g[16];
#pragma unroll
  for (int l = 0; l < 2; ++l) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = 8 * l + 2 * j;
      const float v0 = RHT ? q[e] : with_sign_of(q[e], elem_x(P, e));
      const float v1 = RHT ? q[e + 1] : with_sign_of(q[e + 1], elem_x(P, e + 1));
      const uint32_t b = cvt_e2m1x2(v1, v0);
      fw[l] |= b << (8 * j);
      const float2 d = e2m1x2_to_f32(b);
      g[e] = d.x;
      g[e + 1] = d.y;
    }
  }
  // INT4 candidate and both squared errors, two elements (i, i+8) per float2: w = RN(v * 7/6)
  // clamped to +-7 and rounded half-even by the 1.5 * 2^23 add (its low nibble is the two's
  // complement code), k back as an exact signed float. The errors are formed on signed values:
  // each candidate value has the sign of v (or is a zero), and RN is symmetric, so
  // RN(RN(k * 6/7) - v) and RN(g - v) have the magnitudes of the errors on magnitudes, and the
  // same squares.
  uint32_t t0[8], t1[8];
  float2 Sf[8], Si[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 q2 = make_float2(q[i], q[i + 8]);
    float2 w = __fmul2_rn(q2, make_float2(r76, r76));
    if (clamp) w = make_float2(fminf(fmaxf(w.x, -7.0f), 7.0f), fminf(fmaxf(w.y, -7.0f), 7.0f));
    const float2 tw = add2(w, make_float2(kMagic, kMagic));
    t0[i] = __float_as_uint(tw.x);
    t1[i] = __float_as_uint(tw.y);
    const float2 k = add2(tw, make_float2(-kMagic, -kMagic));   // exact
    const float2 vint = __fmul2_rn(k, make_float2(r67, r67));
    const float2 dint = sub2(vint, q2);
    const float2 dfp = sub2(make_float2(g[i], g[i + 8]), q2);
    Sf[i] = __fmul2_rn(dfp, dfp);
    Si[i] = __fmul2_rn(dint, dint);
  }
  // balanced tree over elements 0..15 with both halves at once: lanes (e_i, e_{i+8})
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; i += 2 * h) {
      Sf[i] = add2(Sf[i], Sf[i + h]);
      Si[i] = add2(Si[i], Si[i + h]);
    }
  }
  const float sse_fp = __fadd_rn(Sf[0].x, Sf[0].y), sse_int = __fadd_rn(Si[0].x, Si[0].y);
  if (sse_int < sse_fp) {
    flag = 0x80u;
    return make_uint2(pack_low_nibbles(t0), pack_low_nibbles(t1));
  }
  return make_uint2(fw[0], fw[1]);
}

// Round-to-nearest codes with a runtime rotation factor (signs always copied from the input).
template <int G>
__device__ __forceinline__ uint2 encode_rtne_rt(const float2* P, float s, bool rht) {
  return rht ? encode_lean<G, true>(P, s) : encode_lean<G, false>(P, s);
}

// ------------------------------------------------------------------ statistics accumulator

struct StatsAcc {
  double y2, err2, yx, blocks, if4_fp4;
  double* cell_err;    // shared [8][kThreads]
  uint32_t* cell_n;    // shared [8][kThreads]

  // cell error |val| - |q| is formed in FP64 (exact for two floats)
  __device__ __forceinline__ void element(float y, float xhat, uint32_t mag, float val, float q) {
    y2 += (double)y * (double)y;
    const double d = (double)y - (double)xhat;
    err2 += d * d;
    yx += (double)y * (double)xhat;
    cell_err[mag * kThreads + threadIdx.x] += fabs((double)val) - fabs((double)q);
    cell_n[mag * kThreads + threadIdx.x] += 1u;
  }
};


// Encodes one block. quad0 = (logical index of element 0) / 4 for the SR counter.
// Returns the IF4 flag (0x80 for an INT4 block, else 0).
template <int G, int R, bool STATS>
__device__ __forceinline__ uint32_t encode16(const EncCtx& ctx, const float2* P, uint64_t quad0,
                                             uint8_t* codes, uint16_t* deq, float s,
                                             const Divider& dv, StatsAcc* acc) {
  const bool zero = (s == 0.0f);
  constexpr bool kExactSmall = (R == kSR) || (G == kIF4);
  float2 Q[8];
  if (zero) {
#pragma unroll
    for (int i = 0; i < 8; ++i) Q[i] = make_float2(0.0f, 0.0f);
  } else if (dv.fast) {
#pragma unroll
    for (int i = 0; i < 8; ++i) Q[i] = div2(dv, P[i]);
    if constexpr (kExactSmall) {
      // the correction step is exact for quotients >= 2^-20; smaller nonzero ones (rare) are
      // recomputed with the IEEE division so stochastic rounding and IF4 errors stay exact
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (fabsf(Q[i].x) < 0x1p-19f && P[i].x != 0.0f) Q[i].x = __fdiv_rn(__fmul_rn(P[i].x, ctx.cinv), s);
        if (fabsf(Q[i].y) < 0x1p-19f && P[i].y != 0.0f) Q[i].y = __fdiv_rn(__fmul_rn(P[i].y, ctx.cinv), s);
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      Q[i] = make_float2(__fdiv_rn(__fmul_rn(P[i].x, ctx.cinv), s),
                         __fdiv_rn(__fmul_rn(P[i].y, ctx.cinv), s));
  }

  // one 16-bit draw per element
  uint32_t rnd[16];
  if constexpr (R == kSR) {
    sr_draws16(ctx.seedx, quad0, rnd);
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) rnd[j] = 0u;
  }

  const bool need_val = STATS || (deq != nullptr) || (G == kIF4);
  float val[16];
  uint32_t mag[16];
  uint32_t w0 = 0u, w1 = 0u, flag = 0u;

  if constexpr (G == kE1M2 || G == kINT4) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w0 |= round_uniform<G, R>(Q[i].x, P[i].x, rnd[i], val[i], mag[i]) << (4 * i);
      w1 |= round_uniform<G, R>(Q[i].y, P[i].y, rnd[i + 8], val[i + 8], mag[i + 8]) << (4 * i);
    }
  } else {  // E2M1 (and the FP4 candidate of IF4): hardware RNE conversion of signed values
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float e0, e1, f0, f1;   // elements 2j, 2j+1 (word 0) and 8+2j, 9+2j (word 1)
      if constexpr (R == kSR) {
        constexpr float qm = GridInfo<G>::qmax;
        e0 = e2m1_sr_value(Q[2 * j].x, P[2 * j].x, rnd[2 * j], qm);
        e1 = e2m1_sr_value(Q[2 * j + 1].x, P[2 * j + 1].x, rnd[2 * j + 1], qm);
        f0 = e2m1_sr_value(Q[2 * j].y, P[2 * j].y, rnd[2 * j + 8], qm);
        f1 = e2m1_sr_value(Q[2 * j + 1].y, P[2 * j + 1].y, rnd[2 * j + 9], qm);
      } else {
        e0 = with_sign_of(Q[2 * j].x, P[2 * j].x);
        e1 = with_sign_of(Q[2 * j + 1].x, P[2 * j + 1].x);
        f0 = with_sign_of(Q[2 * j].y, P[2 * j].y);
        f1 = with_sign_of(Q[2 * j + 1].y, P[2 * j + 1].y);
      }
      w0 |= cvt_e2m1x2(e1, e0) << (8 * j);
      w1 |= cvt_e2m1x2(f1, f0) << (8 * j);
    }
    if (need_val) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 d0 = e2m1x2_to_f32((w0 >> (8 * j)) & 0xFFu);
        const float2 d1 = e2m1x2_to_f32((w1 >> (8 * j)) & 0xFFu);
        val[2 * j] = d0.x;
        val[2 * j + 1] = d0.y;
        val[8 + 2 * j] = d1.x;
        val[9 + 2 * j] = d1.y;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        mag[e] = (w0 >> (4 * e)) & 7u;
        mag[e + 8] = (w1 >> (4 * e)) & 7u;
      }
    }
    if constexpr (G == kIF4) {
      const float r76 = kR76, r67 = kR67;
      float vint[16];
      uint32_t mint[16];
      uint32_t i0 = 0u, i1 = 0u;
      float2 Efp[8], Eint[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float d_fp[2], d_int[2];
#pragma unroll
        for (int l = 0; l < 2; ++l) {
          const int e = i + 8 * l;
          const float q = l ? Q[i].y : Q[i].x;
          const float w = __fmul_rn(q, r76);
          const uint32_t m = __float_as_uint(__fadd_rn(fminf(fabsf(w), 7.0f), 8388608.0f)) & 0xFu;
          const bool n = sign_bit(w) && m;
          const float k = small_int_f32(m);
          vint[e] = __fmul_rn(n ? -k : k, r67);
          mint[e] = m;
          const uint32_t nib = (n ? (0u - m) : m) & 0xFu;
          if (l) i1 |= nib << (4 * i); else i0 |= nib << (4 * i);
          d_fp[l] = __fsub_rn(val[e], q);
          d_int[l] = __fsub_rn(vint[e], q);
        }
        Efp[i] = make_float2(__fmul_rn(d_fp[0], d_fp[0]), __fmul_rn(d_fp[1], d_fp[1]));
        Eint[i] = make_float2(__fmul_rn(d_int[0], d_int[0]), __fmul_rn(d_int[1], d_int[1]));
      }
      // balanced pairwise sums over elements 0..15 ((e0+e1)+(e2+e3))..., both halves at once
#pragma unroll
      for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; i += 2 * h) {
          Efp[i] = add2(Efp[i], Efp[i + h]);
          Eint[i] = add2(Eint[i], Eint[i + h]);
        }
      }
      const float sse_fp = __fadd_rn(Efp[0].x, Efp[0].y);
      const float sse_int = __fadd_rn(Eint[0].x, Eint[0].y);
      if (!zero && sse_int < sse_fp) {
        flag = 0x80u;
        w0 = i0;
        w1 = i1;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          val[e] = vint[e];
          mag[e] = mint[e];
        }
      }
    }
  }
  if (zero) {
    w0 = 0u;
    w1 = 0u;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      val[e] = 0.0f;
      mag[e] = 0u;
    }
  }

  __stcs(reinterpret_cast<uint2*>(codes), make_uint2(w0, w1));

  if (deq != nullptr || STATS) {
    float xh[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) xh[e] = __fmul_rn(val[e], s);
    if (deq != nullptr) {
      uint4 o0, o1;
      o0.x = pack_bf16x2(xh[0], xh[1]);   o0.y = pack_bf16x2(xh[2], xh[3]);
      o0.z = pack_bf16x2(xh[4], xh[5]);   o0.w = pack_bf16x2(xh[6], xh[7]);
      o1.x = pack_bf16x2(xh[8], xh[9]);   o1.y = pack_bf16x2(xh[10], xh[11]);
      o1.z = pack_bf16x2(xh[12], xh[13]); o1.w = pack_bf16x2(xh[14], xh[15]);
      uint4* d = reinterpret_cast<uint4*>(deq);
      __stcs(d, o0);
      __stcs(d + 1, o1);
    }
    if constexpr (STATS) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float y = __fmul_rn(elem_x(P, e), ctx.cinv);
        acc->element(y, xh[e], mag[e], val[e], zero ? 0.0f : elem_x(Q, e));
      }
      acc->blocks += 1.0;
      if (G == kIF4 && flag == 0u) acc->if4_fp4 += 1.0;
    }
  }
  return flag;
}

}  // namespace fp4q

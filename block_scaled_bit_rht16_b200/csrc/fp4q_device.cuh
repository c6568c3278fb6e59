// fp4q_device.cuh -- device building blocks of the fused RHT16 + 4-bit quantizer (sm_100a).
//
// Layout of a 16-element block in registers: eight float2 P[i] = (v_i, v_{i+8}), i = 0..7.
// Butterfly stages h = 1, 2, 4 pair P[i] with P[i+h] and run as packed f32x2 adds (one
// instruction per two elements); stage h = 8 pairs the two lanes of each P[i] and runs scalar.
// Every operation is the same IEEE binary32 operation, in the same stage order, as the
// definition (butterfly stages 1, 2, 4, 8, each (a+b, a-b)), so the result is bit-identical.
//
// Sources: "蚂蚁集团揭秘：为什么给AI"降精度省电"会悄悄让它越来越笨？" (techwalker.com), section
// 六 Q5 (16-point rotation fused with the 16-element quantization block); "当你的 GPU 学不会算账"
// (zhichai.net/topic/178208020), sections "E2M1" and "UFP4" (grids, recipe table).
#pragma once
#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "fp4q_kernels.cuh"

namespace fp4q {


// ------------------------------------------------------------------ bf16 / packed helpers

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b as fma(b, -1, a): one rounding of the exact difference, like a plain subtraction.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// The two bf16 halves of a 32-bit word as floats, each negated when its flip (0 or 0x80000000) is
// set: the low half as w * 2^16 + flip (one integer multiply-add; adding 2^31 toggles the sign
// bit), the high half as (w & 0xFFFF0000) ^ flip (one three-input logic operation). Plain
// expressions, so that flips held in the kernel's parameters stay constant operands.
__device__ __forceinline__ float bf_lo_flip(uint32_t w, uint32_t flip) {
  return __uint_as_float(w * 65536u + flip);
}
__device__ __forceinline__ float bf_hi_flip(uint32_t w, uint32_t flip) {
  return __uint_as_float((w & 0xFFFF0000u) ^ flip);
}

// Load-side: eight 32-bit words (bf16 pairs) -> P[8], with the sign diagonal applied on the way
// (exact). flip_lo[k] / flip_hi[k] negate elements 2k / 2k+1 (bit 31).
__device__ __forceinline__ void unpack16(const uint4& lo, const uint4& hi, const uint32_t* flip_lo,
                                         const uint32_t* flip_hi, float2* P) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    P[2 * k] = make_float2(bf_lo_flip(w[k], flip_lo[k]), bf_lo_flip(w[k + 4], flip_lo[k + 4]));
    P[2 * k + 1] = make_float2(bf_hi_flip(w[k], flip_hi[k]), bf_hi_flip(w[k + 4], flip_hi[k + 4]));
  }
}

// Two blocks at once (words lo0/hi0 of block 0, lo1/hi1 of block 1) as A[i] = (element i of
// block 0, element i of block 1), with the same sign flips for both.
__device__ __forceinline__ void unpack16_pair(const uint4& lo0, const uint4& hi0, const uint4& lo1,
                                              const uint4& hi1, const uint32_t* flip_lo,
                                              const uint32_t* flip_hi, float2* A) {
  const uint32_t w0[8] = {lo0.x, lo0.y, lo0.z, lo0.w, hi0.x, hi0.y, hi0.z, hi0.w};
  const uint32_t w1[8] = {lo1.x, lo1.y, lo1.z, lo1.w, hi1.x, hi1.y, hi1.z, hi1.w};
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    A[2 * k] = make_float2(bf_lo_flip(w0[k], flip_lo[k]), bf_lo_flip(w1[k], flip_lo[k]));
    A[2 * k + 1] = make_float2(bf_hi_flip(w0[k], flip_hi[k]), bf_hi_flip(w1[k], flip_hi[k]));
  }
}

__device__ __forceinline__ uint4 ld_stream(const uint16_t* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

// 16 bf16 (32 bytes): one 256-bit load when the address is 32-byte aligned (callers pass vec32
// only when every block start is), else two 128-bit loads. Read-only, streamed past L1.
__device__ __forceinline__ void load16(const uint16_t* p, bool vec32, uint4& lo, uint4& hi) {
  if (vec32) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w),
                   "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
  } else {
    lo = ld_stream(p);
    hi = ld_stream(p + 8);
  }
}

// v <- H16 v in natural (Sylvester) order, stages h = 1, 2, 4, 8. No 1/4 here: callers fold the
// exact power-of-two normalisation into the scale.
__device__ __forceinline__ void fwht16(float2* P) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & h) == 0) {
        const float2 a = P[i], b = P[i + h];
        P[i] = add2(a, b);
        P[i + h] = sub2(a, b);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float a = P[i].x, b = P[i].y;
    P[i] = make_float2(__fadd_rn(a, b), __fsub_rn(a, b));
  }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// max_i |v_i| over the 16 elements (exact, order-free).
__device__ __forceinline__ float absmax16(const float2* P) {
  float m0 = max3(fabsf(P[0].x), fabsf(P[0].y), fabsf(P[1].x));
  float m1 = max3(fabsf(P[1].y), fabsf(P[2].x), fabsf(P[2].y));
  float m2 = max3(fabsf(P[3].x), fabsf(P[3].y), fabsf(P[4].x));
  float m3 = max3(fabsf(P[4].y), fabsf(P[5].x), fabsf(P[5].y));
  float m4 = max3(fabsf(P[6].x), fabsf(P[6].y), fabsf(P[7].x));
  float m5 = max3(m0, m1, fabsf(P[7].y));
  return max3(m2, m3, max3(m4, m5, 0.0f));
}

// ------------------------------------------------------------------ exact division
//
// v = RN(y / s) for a whole block, with y = c^-1 * vraw (c = 4 with rotation, 1 without; an
// exact power of two). The quotient is Markstein's correction step (P. Markstein, "Computation
// of elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// with R = RN(1/S) and q0 = RN(a R), the remainder r = a - q0 S is exact under an FMA and
// q1 = RN(q0 + r R) is the correctly rounded a/S. Here S = c*s and a = vraw, so a/S = y/s.
// With S in [2^-60, 2^90] (the fast range) the step is exact for every quotient of at least
// 2^-20: then |a| >= 2^-80, so the remainder is representable. Smaller quotients round to a
// zero code under round-to-nearest; stochastic rounding and IF4 recompute them with the IEEE
// division. Outside the fast range every quotient uses the IEEE division.
struct Divider {
  float2 R2, nS2;   // (R, R), (-S, -S)
  float S, R;
  bool fast;        // the block's S is in the range where the correction step is exact
};

// RN(1/S) for S in [2^-60, 2^90]: the hardware reciprocal approximation refined by one
// Newton-Raphson step in FMA form, r1 = r0 + r0 (1 - S r0) (Markstein 1990; Cornea, Golliver
// and Markstein, "Correctness proofs outline for Newton-Raphson based floating-point divide
// and square root algorithms", ARITH 1999). fp4q_check_division compares it with the IEEE
// reciprocal on every float of that range.
__device__ __forceinline__ float rcp_rn_fast(float S) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(S));
  return __fmaf_rn(__fmaf_rn(-S, r0, 1.0f), r0, r0);
}

__device__ __forceinline__ Divider make_divider(float s, float c) {
  Divider d;
  d.S = __fmul_rn(s, c);
  d.fast = (d.S >= 0x1p-60f) && (d.S <= 0x1p+90f);
  d.R = d.fast ? rcp_rn_fast(d.S) : 0.0f;
  d.R2 = make_float2(d.R, d.R);
  d.nS2 = make_float2(-d.S, -d.S);
  return d;
}

// Quotients of a packed pair (signed; -0 inputs give +0, callers take signs from vraw).
__device__ __forceinline__ float2 div2(const Divider& d, float2 a) {
  const float2 q0 = __fmul2_rn(a, d.R2);
  const float2 r = __ffma2_rn(q0, d.nS2, a);
  return __ffma2_rn(r, d.R2, q0);
}

// ------------------------------------------------------------------ grids

// RN(7/6) and RN(6/7) in binary32 (1.16666663, 0.857142866): the IF4 INT4 candidate's scaling
// and dequantization factors.
constexpr float kR76 = 0x1.2aaaaap+0f;
constexpr float kR67 = 0x1.b6db6ep-1f;

template <int G> struct GridInfo;
template <> struct GridInfo<kE2M1> { static constexpr float qmax = 6.0f; };
template <> struct GridInfo<kE1M2> { static constexpr float qmax = 3.5f; };
template <> struct GridInfo<kINT4> { static constexpr float qmax = 7.0f; };
template <> struct GridInfo<kIF4> { static constexpr float qmax = 6.0f; };
template <> struct GridInfo<kE2M1Max4> { static constexpr float qmax = 4.0f; };
template <> struct GridInfo<kE2M1Max3> { static constexpr float qmax = 3.0f; };
template <> struct GridInfo<kE2M1Max2> { static constexpr float qmax = 2.0f; };

// E2M1 codes of two values, hardware round-to-nearest-even with saturation to +-6; the sign of
// each input (including -0) is kept. Result: a in bits 4..7, b in bits 0..3.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float a, float b) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
      : "=r"(r) : "f"(a), "f"(b));
  return r;
}

// Signed value of two E2M1 codes packed in a byte (exact decode): low nibble -> .x.
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte) {
  uint32_t h2;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(h2) : "r"(byte));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

// E2M3 (FP6) codes of two values, round to nearest even, satfinite; each code in the low six
// bits of a byte: sign << 5 | exponent << 3 | mantissa. Result: a in bits 8..13, b in 0..5.
// Below 1 in magnitude E2M3 is subnormal with a uniform step of 1/8, so for |x| <= 7/8 the code
// is sign << 5 | RNE(8 |x|) (ties to the even integer, the sign of zero kept).
__device__ __forceinline__ uint32_t cvt_e2m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(a), "f"(b));
  return r;
}

// E4M3 (satfinite, round to nearest even) of a non-negative float -> byte.
__device__ __forceinline__ uint32_t cvt_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0xFFu;
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
  uint32_t h2;
  const uint16_t b = static_cast<uint16_t>(byte & 0x7Fu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __low2float(h);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ------------------------------------------------------------------ programmatic dependent launch
//
// Quantize kernels are launched with programmatic stream serialization: the next kernel in the
// stream may become resident while this one drains. Each kernel first lets its dependents
// launch, then waits for its own prerequisite grid to complete (and its memory to be visible)
// before touching global memory, so stream order is preserved for inputs and outputs alike.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.launch_dependents;" :::);
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------ bulk copies and barriers
//
// Tile copies into shared memory complete on an mbarrier with a transaction count. Every wait is
// bounded by the global timer: a wait that gives up returns false (the caller records it in the
// library's device status word), so no kernel can hang.

constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0u && global_ns() - t0 > limit_ns) return false;
  }
}

// ------------------------------------------------------------------ stochastic rounding source

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the finalizer of a state, and the output for
// state x + gamma (the generator's next output from state x).
__device__ __forceinline__ uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) { return splitmix64_mix(x + kGamma); }

// The SplitMix64 outputs that hold the draws of the sixteen consecutive elements whose first has
// logical index 4 * quad0 (a multiple of 4), as eight 32-bit words: element 4j + l takes bits
// 16l .. 16l+15 of output quad0 + j of the stream seeded with seedx = seed ^ (stream << 63), whose
// state for output k is seedx + (k + 1) * gamma -- i.e. element e's draw is the low (e even) or
// high (e odd) half of word e >> 1.
__device__ __forceinline__ void sr_words16(uint64_t seedx, uint64_t quad0, uint32_t* d) {
  uint64_t state = seedx + (quad0 + 1u) * kGamma;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint64_t h = splitmix64_mix(state);
    state += kGamma;
    d[2 * j] = (uint32_t)h;
    d[2 * j + 1] = (uint32_t)(h >> 32);
  }
}

// The same draws as sixteen 16-bit values u[e].
__device__ __forceinline__ void sr_draws16(uint64_t seedx, uint64_t quad0, uint32_t* u) {
  uint32_t d[8];
  sr_words16(seedx, quad0, d);
#pragma unroll
  for (int e = 0; e < 16; ++e) u[e] = (e & 1) ? (d[e >> 1] >> 16) : (d[e >> 1] & 0xFFFFu);
}

// 1 + u * 2^-23 for element e's draw u (the draw in the low mantissa bits). The 16-bit field is
// extracted with the integer multiplier (x * 2^16 to drop the high half, the high word of
// x * 2^16 to shift it down) rather than a byte permute: the pass that uses it is bound by the
// integer ALU pipe, and the multiplies issue on the FMA pipe.
__device__ __forceinline__ float sr_one_plus(const uint32_t* d, int e) {
  const uint32_t w = d[e >> 1];
  const uint32_t x = (e & 1) ? w : w * 65536u;
  return __uint_as_float(__umulhi(x, 65536u) + 0x3F800000u);
}

// Round-up decision r < frac with r = u * 2^-16, taken exactly as u < frac * 2^16 (both sides
// exact in FP32).
__device__ __forceinline__ bool sr_up(uint32_t u, float frac) {
  return __uint2float_rn(u) < __fmul_rn(frac, 65536.0f);
}

}  // namespace fp4q

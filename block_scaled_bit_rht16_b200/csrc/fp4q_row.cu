// fp4q_row.cu -- row-orientation kernels of the fused RHT16 + block-scaled 4-bit quantizer.
//
// One thread owns one scale block (16 elements; 32 for UE8M0) end to end: one 256-bit load per
// 16 elements when rows are 32-byte aligned (else two 128-bit loads), sign flips on the bf16 bits, the 16-point butterfly in registers (packed
// f32x2), block absmax, the scale, exact quotients, rounding, nibble packing, one 8-byte
// (16-byte) code store and the scale store. Consecutive threads own consecutive blocks, so a
// warp reads 1 KiB and writes 256 B of codes contiguously. The grid is persistent (SM count x
// resident CTAs) and each thread keeps two blocks in flight.
//
// Sources: "蚂蚁集团揭秘…" (techwalker.com), section 六 Q5 (16-point rotation fused with the
// 16-element quantization block); "当你的 GPU 学不会算账" (zhichai.net/topic/178208020),
// section "UFP4：换一把尺子" (recipe table: 1x16 blocks, FP32 scale, SR on dY);
// "低精度量化技术：IF4…" (bxzpzcl.cn/news/2320061), section 3.2 (E4M3 block scale + FP32
// tensor scale); "AMD全新研究揭示…" (cannews.ca/article/21387), MXFP4 section (32-element
// blocks, shared E8M0 exponent).
#include <cuda_fp16.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_encode.cuh"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {

__device__ int32_t g_device_status = 0;

namespace {

__device__ __forceinline__ int64_t unit_offset(const QuantArgs& a, int64_t u, int unit) {
  if (a.contiguous) return u * unit;
  const int64_t r = u / a.units_per_row;
  return r * a.ld + (u - r * a.units_per_row) * unit;
}

__device__ __forceinline__ void rotate_if(const QuantArgs& a, float2* P) {
  if (a.c != 1.0f) fwht16(P);
}

// Fixed-order reduction of the per-thread statistics into this CTA's raw record.
__device__ void stats_finish(const StatsAcc& acc, double* partials) {
  __shared__ double red[5][kThreads];
  red[0][threadIdx.x] = acc.y2;
  red[1][threadIdx.x] = acc.err2;
  red[2][threadIdx.x] = acc.yx;
  red[3][threadIdx.x] = acc.blocks;
  red[4][threadIdx.x] = acc.if4_fp4;
  __syncthreads();
  double* out = partials + (size_t)blockIdx.x * ST_LEN;
  const int t = threadIdx.x;
  if (t < 5) {
    const int dst[5] = {ST_SUM_Y2, ST_SUM_ERR2, ST_SUM_YXHAT, ST_BLOCKS, ST_IF4_FP4};
    double s = 0.0;
    for (int i = 0; i < kThreads; ++i) s += red[t][i];
    out[dst[t]] = s;
  } else if (t >= 32 && t < 40) {
    const int c = t - 32;
    double s = 0.0, n = 0.0;
    for (int i = 0; i < kThreads; ++i) {
      s += acc.cell_err[c * kThreads + i];
      n += (double)acc.cell_n[c * kThreads + i];
    }
    out[ST_CELL_ERR + c] = s;
    out[ST_CELL_N + c] = n;
  } else if (t == 64) {
    double n = 0.0;
    for (int i = 0; i < 8 * kThreads; ++i) n += (double)acc.cell_n[i];
    out[ST_N] = n;
    out[22] = 0.0;
    out[23] = 0.0;
  }
}

// MXFP4 block: 32 elements (two rotated 16-blocks P, Q) scaled by 2^-e (exact multiply by
// `mult` = 2^-e * cinv), E2M1 with saturation.
template <int R, bool STATS>
__device__ __forceinline__ void encode_mx(const EncCtx& ctx, const float2* P, const float2* Q,
                                          uint64_t quad0, uint8_t* codes, uint16_t* deq, float s,
                                          float mult, bool zero, StatsAcc* acc) {
  const float2 m2 = make_float2(mult, mult);
  uint32_t w[4];
  float val[32], vq[32];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const float2* H = half ? Q : P;
    float2 V[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) V[i] = __fmul2_rn(H[i], m2);   // exact scaling, sign kept
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      vq[16 * half + i] = V[i].x;
      vq[16 * half + 8 + i] = V[i].y;
    }
    uint32_t rnd[16];
    if constexpr (R == kSR) sr_draws16(ctx.seedx, quad0 + 4u * half, rnd);
    uint32_t wa = 0u, wb = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float e0 = V[2 * j].x, e1 = V[2 * j + 1].x, f0 = V[2 * j].y, f1 = V[2 * j + 1].y;
      if constexpr (R == kSR) {
        e0 = e2m1_sr_value(e0, e0, rnd[2 * j]);
        e1 = e2m1_sr_value(e1, e1, rnd[2 * j + 1]);
        f0 = e2m1_sr_value(f0, f0, rnd[2 * j + 8]);
        f1 = e2m1_sr_value(f1, f1, rnd[2 * j + 9]);
      }
      wa |= cvt_e2m1x2(e1, e0) << (8 * j);
      wb |= cvt_e2m1x2(f1, f0) << (8 * j);
    }
    if (zero) {
      wa = 0u;
      wb = 0u;
    }
    w[2 * half] = wa;
    w[2 * half + 1] = wb;
  }
  __stcs(reinterpret_cast<uint4*>(codes), make_uint4(w[0], w[1], w[2], w[3]));
  if (deq != nullptr || STATS) {
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 d = e2m1x2_to_f32((w[k] >> (8 * j)) & 0xFFu);
        val[8 * k + 2 * j] = d.x;
        val[8 * k + 2 * j + 1] = d.y;
      }
    float xh[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) xh[e] = __fmul_rn(val[e], s);
    if (deq != nullptr) {
      uint4* d = reinterpret_cast<uint4*>(deq);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        uint4 o;
        o.x = pack_bf16x2(xh[8 * k + 0], xh[8 * k + 1]);
        o.y = pack_bf16x2(xh[8 * k + 2], xh[8 * k + 3]);
        o.z = pack_bf16x2(xh[8 * k + 4], xh[8 * k + 5]);
        o.w = pack_bf16x2(xh[8 * k + 6], xh[8 * k + 7]);
        __stcs(d + k, o);
      }
    }
    if constexpr (STATS) {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float2* H = (e < 16) ? P : Q;
        const float y = __fmul_rn(elem_x(H, e & 15), ctx.cinv);
        const uint32_t mag = (w[e >> 3] >> (4 * (e & 7))) & 7u;
        acc->element(y, xh[e], mag, val[e], zero ? 0.0f : vq[e]);
      }
      acc->blocks += 1.0;
    }
  }
}

template <int G, int S, int R, bool STATS>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const QuantArgs a) {
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr int kUnit = (S == kUE8M0) ? 32 : 16;
  constexpr int kVec = kUnit / 8;   // 16-byte loads per unit
  pdl_enter();

  float alpha = 0.0f, denom = 0.0f;
  if constexpr (S == kE4M3) {
    if (a.ts_in != nullptr) {
      alpha = *a.ts_in;
    } else {
      const float A = __uint_as_float(a.ws->amax_bits);
      alpha = __fdiv_rn(A, __fmul_rn(qmax, 448.0f));
      if (a.ts_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *a.ts_out = alpha;
    }
    denom = __fmul_rn(alpha, qmax);
  }

  StatsAcc acc;
  if constexpr (STATS) {
    __shared__ double s_cell_err[8 * kThreads];
    __shared__ uint32_t s_cell_n[8 * kThreads];
    acc.y2 = acc.err2 = acc.yx = acc.blocks = acc.if4_fp4 = 0.0;
    acc.cell_err = s_cell_err;
    acc.cell_n = s_cell_n;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      s_cell_err[c * kThreads + threadIdx.x] = 0.0;
      s_cell_n[c * kThreads + threadIdx.x] = 0u;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      a.ws->magic = kWsMagic;
      a.ws->n_partials = gridDim.x;
    }
  }
  const EncCtx ctx{a.cinv, a.seedx};

  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.nunits; u += 2 * stride) {
    uint4 buf[2][kVec];
    const int64_t uu[2] = {u, u + stride};
    const bool has2 = uu[1] < a.nunits;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (k == 1 && !has2) break;
      const uint16_t* src = a.x + unit_offset(a, uu[k], kUnit);
#pragma unroll
      for (int v = 0; v < kVec; v += 2) load16(src + 8 * v, a.vec32 != 0, buf[k][v], buf[k][v + 1]);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (k == 1 && !has2) break;
      const int64_t un = uu[k];
      uint16_t* deq = a.deq ? a.deq + un * kUnit : nullptr;
      if constexpr (S != kUE8M0) {
        float2 P[8];
        unpack16(buf[k][0], buf[k][1], a.flip_lo, a.flip_hi, P);
        rotate_if(a, P);
        const float amax_y = __fmul_rn(absmax16(P), a.cinv);
        float s;
        uint32_t sbyte = 0u;
        if constexpr (S == kFP32) {
          s = div_qmax<G>(amax_y);
        } else {
          const float delta = denom > 0.0f ? __fdiv_rn(amax_y, denom) : 0.0f;
          sbyte = cvt_e4m3(delta);
          s = __fmul_rn(e4m3_to_f32(sbyte), alpha);
        }
        const Divider dv = make_divider(s, a.c);
        const uint32_t flag = encode16<G, R, STATS>(ctx, P, (uint64_t)un * 4u, a.codes + un * 8,
                                                    deq, s, dv, STATS ? &acc : nullptr);
        if constexpr (S == kFP32) {
          __stcs(reinterpret_cast<float*>(a.scales) + un, s);
        } else {
          reinterpret_cast<uint8_t*>(a.scales)[scale_slot(un, a.units_per_row, a.mma_scales)] =
              (uint8_t)(sbyte | flag);
        }
      } else {
        float2 P[8], Q[8];
        unpack16(buf[k][0], buf[k][1], a.flip_lo, a.flip_hi, P);
        unpack16(buf[k][2], buf[k][3], a.flip_lo, a.flip_hi, Q);
        rotate_if(a, P);
        rotate_if(a, Q);
        const float amax_y = __fmul_rn(fmaxf(absmax16(P), absmax16(Q)), a.cinv);
        int e = -127;
        if (amax_y != 0.0f) {
          const int E = (int)(__float_as_uint(amax_y) >> 23);   // biased exponent
          e = (E == 0) ? -127 : max(-127, min(127, E - 127 - 2));
        }
        const float s = (e >= -126) ? __uint_as_float((uint32_t)(127 + e) << 23) : 0x1p-127f;
        const float mult = __fmul_rn(__uint_as_float((uint32_t)(127 - e) << 23), a.cinv);
        encode_mx<R, STATS>(ctx, P, Q, (uint64_t)un * 8u, a.codes + un * 16, deq, s, mult,
                            amax_y == 0.0f, STATS ? &acc : nullptr);
        reinterpret_cast<uint8_t*>(a.scales)[scale_slot(un, a.units_per_row, a.mma_scales)] =
            (uint8_t)(e + 127);
      }
    }
  }
  if constexpr (STATS) stats_finish(acc, a.partials);
}

// The hot path: FP32 1x16 scale, round to nearest even, codes and scales only. FLAT: the
// tensor is contiguous and 32-byte aligned, so unit u is the 32 bytes at 32u (one 256-bit load).
// Each thread encodes one block per iteration while the load of its next block is in flight.
template <int G, bool RHT, bool FLAT>
__device__ __forceinline__ void lean_load(const QuantArgs& a, int64_t u, uint4& lo, uint4& hi) {
  if constexpr (FLAT) load16(a.x + u * 16, true, lo, hi);
  else load16(a.x + unit_offset(a, u, 16), a.vec32 != 0, lo, hi);
}

template <bool FLAT> struct UnitIdx { using T = int64_t; };
template <> struct UnitIdx<true> { using T = uint32_t; };

// FLAT launches index blocks with 32-bit counters and elements as u * 16 in 32 bits, so they
// take tensors of at most 2^28 blocks (2^32 elements); larger ones take the 64-bit path.
constexpr int64_t kFlatMaxUnits = int64_t(1) << 28;
static_assert(kFlatMaxUnits * 16 <= (int64_t(1) << 32), "flat element offsets fit in 32 bits");
static_assert(kFlatMaxUnits + (int64_t(1) << 24) < (int64_t(1) << 32),
              "flat block counters plus one grid stride fit in 32 bits");

__host__ __device__ inline bool flat_launch(const QuantArgs& a) {
  return a.contiguous && a.vec32 && a.nunits <= kFlatMaxUnits;
}

// The two-block kernel stores a pair's codes as one 16-byte word and its scales as one 8-byte word.
inline bool pair_aligned(const QuantArgs& a) {
  return reinterpret_cast<uintptr_t>(a.codes) % 16 == 0 && reinterpret_cast<uintptr_t>(a.scales) % 8 == 0;
}

template <int G, bool RHT, bool FLAT, int R>
__global__ void __launch_bounds__(kThreads) lean_kernel(const QuantArgs a) {
  constexpr float kCinv = RHT ? 0.25f : 1.0f;
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  pdl_enter();
  using Idx = typename UnitIdx<FLAT>::T;
  const Idx n = (Idx)a.nunits;
  const Idx stride = (Idx)gridDim.x * kThreads;
  Idx u = (Idx)blockIdx.x * kThreads + threadIdx.x;
  if (u >= n) return;
  uint4 lo, hi;
  lean_load<G, RHT, FLAT>(a, u, lo, hi);
  for (; u < n; u += stride) {
    uint4 nlo = lo, nhi = hi;
    if (u + stride < n) lean_load<G, RHT, FLAT>(a, u + stride, nlo, nhi);
    float2 P[8];
    unpack16(lo, hi, RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, P);
    if constexpr (RHT) fwht16(P);
    const float s = div_qmax<G>(__fmul_rn(absmax16(P), kCinv));
    uint2 w;
    if constexpr (R == kSR) w = encode_sr<G>(P, s, RHT ? 4.0f : 1.0f, a.seedx, (uint64_t)u * 4u);
    else w = encode_lean<G, RHT>(P, s);
    __stcs(reinterpret_cast<uint2*>(a.codes) + u, w);
    __stcs(reinterpret_cast<float*>(a.scales) + u, s);
    lo = nlo;
    hi = nhi;
  }
}

// The hot path for a flat tensor with round to nearest: two adjacent blocks per thread per
// iteration (64 contiguous bytes: two 256-bit loads, one 16-byte code store, one 8-byte scale
// store), held as A[i] = (element i of the first block, element i of the second) so that every
// butterfly stage and every quotient step runs as packed f32x2 operations for both blocks -- the
// same IEEE operations, in the same order, as the one-block kernel. The next pair's loads are in
// flight while the current pair encodes.
// Codes of block u of a flat tensor with FP32 scale s, recomputed from the input (the same loads
// and operations as the pair kernel's) for a scale outside the correction step's exact range.
// Not inlined, and handed only the arguments' address (a grid constant) and scalars, so that the
// rare path takes neither registers nor a stack frame from the common one: the common path then
// fits 64 registers, four CTAs per SM.
template <int G, bool RHT>
__device__ __noinline__ uint2 lean_block_slow(const QuantArgs* a, uint32_t u, float s) {
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  uint4 lo, hi;
  load16(a->x + (size_t)u * 16, true, lo, hi);
  float2 P[8];
  unpack16(lo, hi, RHT ? a->flip_lo : zero_flip, RHT ? a->flip_hi : zero_flip, P);
  if constexpr (RHT) fwht16(P);
  return encode_lean<G, RHT>(P, s);
}

template <int G, bool RHT>
__global__ void __launch_bounds__(kThreads, 4) lean_pair_kernel(const __grid_constant__ QuantArgs a) {
  constexpr float kCinv = RHT ? 0.25f : 1.0f;
  constexpr float kF = lean_divisor_factor<G, RHT>();
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  pdl_enter();
  const uint32_t npairs = (uint32_t)(a.nunits >> 1);
  const uint32_t stride = gridDim.x * kThreads;
  uint32_t p = blockIdx.x * kThreads + threadIdx.x;
  uint4 v[4];
  if (p < npairs) {
    load16(a.x + (size_t)p * 32, true, v[0], v[1]);
    load16(a.x + (size_t)p * 32 + 16, true, v[2], v[3]);
  }
  for (; p < npairs; p += stride) {
    uint4 nv[4] = {v[0], v[1], v[2], v[3]};
    if (p + stride < npairs) {
      load16(a.x + (size_t)(p + stride) * 32, true, nv[0], nv[1]);
      load16(a.x + (size_t)(p + stride) * 32 + 16, true, nv[2], nv[3]);
    }
    float2 A[16];
    unpack16_pair(v[0], v[1], v[2], v[3], RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, A);
    if constexpr (RHT) fwht16_pair(A);
    const float2 am = absmax16_pair(A);
    const float s0 = div_qmax<G>(__fmul_rn(am.x, kCinv)), s1 = div_qmax<G>(__fmul_rn(am.y, kCinv));
    // a zero block's lane divides by 1 (its codes are zeros whatever its quotients)
    const Divider d0 = make_divider(s0 == 0.0f ? 1.0f : s0, kF), d1 = make_divider(s1 == 0.0f ? 1.0f : s1, kF);
    uint2 w0, w1;
    if (d0.fast && d1.fast) {
      const float2 R2 = make_float2(d0.R, d1.R), nS2 = make_float2(-d0.S, -d1.S);
      float q0[16], q1[16], r0[16], r1[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 qa = __fmul2_rn(A[e], R2);
        const float2 q = __ffma2_rn(__ffma2_rn(qa, nS2, A[e]), R2, qa);
        q0[e] = q.x;
        q1[e] = q.y;
        r0[e] = A[e].x;
        r1[e] = A[e].y;
      }
      w0 = s0 == 0.0f ? make_uint2(0u, 0u) : lean_codes<G, RHT>(q0, r0);
      w1 = s1 == 0.0f ? make_uint2(0u, 0u) : lean_codes<G, RHT>(q1, r1);
    } else {
      w0 = lean_block_slow<G, RHT>(&a, 2 * p, s0);
      w1 = lean_block_slow<G, RHT>(&a, 2 * p + 1, s1);
    }
    __stcs(reinterpret_cast<uint4*>(a.codes) + p, make_uint4(w0.x, w0.y, w1.x, w1.y));
    __stcs(reinterpret_cast<float2*>(a.scales) + p, make_float2(s0, s1));
    v[0] = nv[0];
    v[1] = nv[1];
    v[2] = nv[2];
    v[3] = nv[3];
  }
  // an odd last block
  if ((a.nunits & 1) && blockIdx.x == 0 && threadIdx.x == 0) {
    const uint32_t u = (uint32_t)a.nunits - 1u;
    uint4 lo, hi;
    load16(a.x + (size_t)u * 16, true, lo, hi);
    float2 P[8];
    unpack16(lo, hi, RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, P);
    if constexpr (RHT) fwht16(P);
    const float s = div_qmax<G>(__fmul_rn(absmax16(P), kCinv));
    __stcs(reinterpret_cast<uint2*>(a.codes) + u, encode_lean<G, RHT>(P, s));
    __stcs(reinterpret_cast<float*>(a.scales) + u, s);
  }
}

// Self-test of the bounded wait: one thread waits on a barrier nothing arrives on.
__global__ void wait_timeout_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0u, limit_ns)) atomicOr(&g_device_status, kStatusSelfTest);
  mbar_arrive(&bar);   // complete the phase so the barrier is left consistent
}

// Group of row r: the last g in [0, n) with off[g] <= r (offsets nondecreasing; empty groups
// are skipped). The result is always a valid index, whatever the offsets hold.
__device__ __forceinline__ int group_of(const int64_t* off, int n, int64_t r) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(off + mid) <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// The Divider stored in a scale table entry (scale, S, R, fast).
__device__ __forceinline__ Divider table_divider(const float4& e) {
  Divider dv;
  dv.S = e.y;
  dv.R = e.z;
  dv.fast = e.w != 0.0f;
  dv.R2 = make_float2(dv.R, dv.R);
  dv.nS2 = make_float2(-dv.S, -dv.S);
  return dv;
}

// E4M3 block scale + FP32 tensor scale, round to nearest even, codes and scale bytes only.
// G = kIF4: the per-block FP4 / INT4 choice, flagged in bit 7 of the scale byte.
// GROUPED: the tensor scale is that of the block's row group (group_ts), looked up again only
// when a thread's block leaves the rows of the group it last used.
// Five resident CTAs per SM (48 registers, no spills) measured faster than four; IF4's two
// candidates are held to three CTAs per SM (no spills), the grouped variant's scale cache keeps
// its registers.
template <int G, bool RHT, bool FLAT, bool GROUPED = false>
__global__ void __launch_bounds__(kThreads, G == kIF4 ? 3 : (GROUPED ? 1 : 5)) lean_nv_kernel(const QuantArgs a) {
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr float kCinv = RHT ? 0.25f : 1.0f;
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  pdl_enter();
  float alpha = 0.0f;
  if constexpr (!GROUPED) {
    if (a.ts_in != nullptr) {
      alpha = *a.ts_in;
    } else {
      alpha = __fdiv_rn(__uint_as_float(a.ws->amax_bits), __fmul_rn(qmax, 448.0f));
      if (a.ts_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *a.ts_out = alpha;
    }
  }
  float denom = __fmul_rn(alpha, qmax);
  // RN(amax / denom) for every block through the correction step on one reciprocal (exact for
  // quotients in [2^-20, 2^64); the E4M3 conversion sends anything below 2^-11 to 0 either way)
  Divider dd = make_divider(denom, 1.0f);
  // One tensor scale for the launch: a block scale is RN(decode(d8) * alpha) for one of the 127
  // E4M3 codes d8, so each code's scale and the Divider of its element quotients are formed
  // once per CTA (the same operations as per block) and looked up by code.
  constexpr float kFactor = G == kIF4 ? (RHT ? 4.0f : 1.0f) : lean_divisor_factor<G, RHT>();
  __shared__ float4 s_tab[128];
  if constexpr (!GROUPED) {
    if (threadIdx.x < 128) {
      const float sd = __fmul_rn(e4m3_to_f32(threadIdx.x), alpha);
      const Divider dv = make_divider(sd, kFactor);
      s_tab[threadIdx.x] = make_float4(sd, dv.S, dv.R, dv.fast ? 1.0f : 0.0f);
    }
    __syncthreads();
  }
  int64_t g_lo = 0, g_hi = 0;   // blocks of the group whose scale is loaded (none yet)
  using Idx = typename UnitIdx<FLAT>::T;
  const Idx n = (Idx)a.nunits;
  const Idx stride = (Idx)gridDim.x * kThreads;
  Idx u = (Idx)blockIdx.x * kThreads + threadIdx.x;
  if (u >= n) return;
  uint4 lo, hi;
  lean_load<G, RHT, FLAT>(a, u, lo, hi);
  for (; u < n; u += stride) {
    uint4 nlo = lo, nhi = hi;
    if (u + stride < n) lean_load<G, RHT, FLAT>(a, u + stride, nlo, nhi);
    float2 P[8];
    unpack16(lo, hi, RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, P);
    if constexpr (RHT) fwht16(P);
    const float amax_raw = absmax16(P);
    const float amax_y = __fmul_rn(amax_raw, kCinv);
    if constexpr (GROUPED) {
      if ((int64_t)u < g_lo || (int64_t)u >= g_hi) {
        const int g = group_of(a.group_off, a.n_groups, (int64_t)u / a.units_per_row);
        g_lo = __ldg(a.group_off + g) * a.units_per_row;
        g_hi = __ldg(a.group_off + g + 1) * a.units_per_row;
        alpha = a.group_ts[g];
        denom = __fmul_rn(alpha, qmax);
        dd = make_divider(denom, 1.0f);
      }
    }
    float delta = 0.0f;
    if (dd.fast) delta = div2(dd, make_float2(amax_y, 0.0f)).x;
    // outside the fast range, and for quotients too large for the correction step (a given
    // tensor scale may be tiny), the IEEE division
    if ((!dd.fast || !(delta < 0x1p+64f)) && denom > 0.0f) delta = __fdiv_rn(amax_y, denom);
    const uint32_t sbyte = cvt_e4m3(delta);
    float s;
    Divider dv;
    if constexpr (GROUPED) {
      s = __fmul_rn(e4m3_to_f32(sbyte), alpha);
      dv = make_divider(s, kFactor);
    } else {
      const float4 e = s_tab[sbyte];
      s = e.x;
      dv = table_divider(e);
    }
    uint2 w;
    uint32_t flag = 0u;
    if constexpr (G == kIF4) w = encode_if4<RHT>(P, s, dv, flag);
    else w = encode_lean_dv<G, RHT, true>(P, s, dv, amax_raw);
    __stcs(reinterpret_cast<uint2*>(a.codes) + u, w);
    reinterpret_cast<uint8_t*>(a.scales)[scale_slot((int64_t)u, a.units_per_row, a.mma_scales)] =
        (uint8_t)(sbyte | flag);
    lo = nlo;
    hi = nhi;
  }
}

// Codes of rotated block u of a flat tensor from its scale table entry e, recomputed from the
// input (the same loads and operations as the pair kernel's): encode_lean_dv with the clamp, for
// scales outside the correction step's exact range. Not inlined, and handed only the arguments'
// address (a grid constant) and scalars, so that the rare path takes neither registers nor a
// stack frame from the common one.
template <int G>
__device__ __noinline__ uint2 nv_block_slow(const QuantArgs* a, uint32_t u, float4 e) {
  uint4 lo, hi;
  load16(a->x + (size_t)u * 16, true, lo, hi);
  float2 P[8];
  unpack16(lo, hi, a->flip_lo, a->flip_hi, P);
  fwht16(P);
  return encode_lean_dv<G, true, true>(P, e.x, table_divider(e), absmax16(P));
}

// lean_nv_kernel for a rotated flat tensor with one tensor scale (E2M1, E1M2, INT4): two
// adjacent blocks per thread per iteration, as lean_pair_kernel does for the FP32 scale. The
// block-scale quotients of the pair come from one packed correction step and one paired E4M3
// conversion; the element quotients from packed steps on the two blocks' dividers (looked up by
// scale code in the CTA's table); the same IEEE operations in the same order as the one-block
// kernel. The pair's two scale bytes are adjacent in either scale layout (the MMA layout has a
// multiple of four blocks per row), so they leave as one 16-bit store.
template <int G, int TH>
__global__ void __launch_bounds__(TH) lean_nv_pair_kernel(const __grid_constant__ QuantArgs a) {
  constexpr float qmax = GridInfo<G>::qmax;
  constexpr float kF = lean_divisor_factor<G, true>();
  constexpr float kVScale = (G == kE1M2) ? 4.0f : 1.0f;
  pdl_enter();
  float alpha;
  if (a.ts_in != nullptr) {
    alpha = *a.ts_in;
  } else {
    alpha = __fdiv_rn(__uint_as_float(a.ws->amax_bits), __fmul_rn(qmax, 448.0f));
    if (a.ts_out != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *a.ts_out = alpha;
  }
  const float denom = __fmul_rn(alpha, qmax);
  const Divider dd = make_divider(denom, 1.0f);
  __shared__ float4 s_tab[128];
  static_assert(TH >= 128, "one table entry per thread");
  if (threadIdx.x < 128) {
    const float sd = __fmul_rn(e4m3_to_f32(threadIdx.x), alpha);
    const Divider dv = make_divider(sd, kF);
    s_tab[threadIdx.x] = make_float4(sd, dv.S, dv.R, dv.fast ? 1.0f : 0.0f);
  }
  __syncthreads();
  const uint32_t npairs = (uint32_t)(a.nunits >> 1);
  const uint32_t stride = gridDim.x * TH;
  uint32_t p = blockIdx.x * TH + threadIdx.x;
  uint4 v[4];
  if (p < npairs) {
    load16(a.x + (size_t)p * 32, true, v[0], v[1]);
    load16(a.x + (size_t)p * 32 + 16, true, v[2], v[3]);
  }
  for (; p < npairs; p += stride) {
    uint4 nv[4] = {v[0], v[1], v[2], v[3]};
    if (p + stride < npairs) {
      load16(a.x + (size_t)(p + stride) * 32, true, nv[0], nv[1]);
      load16(a.x + (size_t)(p + stride) * 32 + 16, true, nv[2], nv[3]);
    }
    float2 A[16];
    unpack16_pair(v[0], v[1], v[2], v[3], a.flip_lo, a.flip_hi, A);
    fwht16_pair(A);
    const float2 am = absmax16_pair(A);   // amax of the raw butterfly outputs
    const float2 ay = __fmul2_rn(am, make_float2(0.25f, 0.25f));
    float2 delta = dd.fast ? div2(dd, ay) : make_float2(0.0f, 0.0f);
    // outside the fast range, and for quotients too large for the correction step, the IEEE
    // division (as in the one-block kernel)
    if ((!dd.fast || !(delta.x < 0x1p+64f)) && denom > 0.0f) delta.x = __fdiv_rn(ay.x, denom);
    if ((!dd.fast || !(delta.y < 0x1p+64f)) && denom > 0.0f) delta.y = __fdiv_rn(ay.y, denom);
    uint16_t sb2;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sb2) : "f"(delta.y), "f"(delta.x));
    // the quotients are non-negative, so both codes are in 0..126
    const float4 e0 = s_tab[sb2 & 0x7Fu], e1 = s_tab[(sb2 >> 8) & 0x7Fu];
    uint2 w0, w1;
    if ((e0.w != 0.0f || e0.x == 0.0f) && (e1.w != 0.0f || e1.x == 0.0f)) {
      // a zero-scale lane divides by 1 (its codes are zeros whatever its quotients)
      const float2 R2 = make_float2(e0.x == 0.0f ? 1.0f : e0.z, e1.x == 0.0f ? 1.0f : e1.z);
      const float2 nS2 = make_float2(e0.x == 0.0f ? -1.0f : -e0.y, e1.x == 0.0f ? -1.0f : -e1.y);
      float q0[16], q1[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float2 qa = __fmul2_rn(A[e], R2);
        const float2 q = __ffma2_rn(__ffma2_rn(qa, nS2, A[e]), R2, qa);
        q0[e] = q.x;
        q1[e] = q.y;
      }
      if constexpr (!kIsE2M1<G>) {   // the E2M1 conversion saturates by itself
        constexpr float lim = qmax / kVScale;
        constexpr float half_above = (G == kE1M2 ? 3.75f : 7.5f) / kVScale;   // qmax + step / 2
        const float2 qa = __fmul2_rn(am, R2);
        const float2 qm = __ffma2_rn(__ffma2_rn(qa, nS2, am), R2, qa);
        if (!(qm.x < half_above)) {
#pragma unroll
          for (int e = 0; e < 16; ++e) q0[e] = fminf(fmaxf(q0[e], -lim), lim);
        }
        if (!(qm.y < half_above)) {
#pragma unroll
          for (int e = 0; e < 16; ++e) q1[e] = fminf(fmaxf(q1[e], -lim), lim);
        }
      }
      w0 = e0.x == 0.0f ? make_uint2(0u, 0u) : lean_codes<G, true>(q0, q0);
      w1 = e1.x == 0.0f ? make_uint2(0u, 0u) : lean_codes<G, true>(q1, q1);
    } else {
      // a scale outside the correction step's exact range (tiny or huge data)
      w0 = nv_block_slow<G>(&a, 2 * p, e0);
      w1 = nv_block_slow<G>(&a, 2 * p + 1, e1);
    }
    __stcs(reinterpret_cast<uint4*>(a.codes) + p, make_uint4(w0.x, w0.y, w1.x, w1.y));
    const int64_t slot = scale_slot((int64_t)p * 2, a.units_per_row, a.mma_scales);
    *reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(a.scales) + slot) = sb2;
    v[0] = nv[0];
    v[1] = nv[1];
    v[2] = nv[2];
    v[3] = nv[3];
  }
  // an odd last block (row-major scales only: the MMA layout has an even count)
  if ((a.nunits & 1) && blockIdx.x == 0 && threadIdx.x == 0) {
    const uint32_t u = (uint32_t)a.nunits - 1u;
    uint4 lo, hi;
    load16(a.x + (size_t)u * 16, true, lo, hi);
    float2 P[8];
    unpack16(lo, hi, a.flip_lo, a.flip_hi, P);
    fwht16(P);
    const float amax_raw = absmax16(P);
    const float amax_y = __fmul_rn(amax_raw, 0.25f);
    float delta = 0.0f;
    if (dd.fast) delta = div2(dd, make_float2(amax_y, 0.0f)).x;
    if ((!dd.fast || !(delta < 0x1p+64f)) && denom > 0.0f) delta = __fdiv_rn(amax_y, denom);
    const uint32_t sbyte = cvt_e4m3(delta);
    const float4 e = s_tab[sbyte];
    __stcs(reinterpret_cast<uint2*>(a.codes) + u, encode_lean_dv<G, true, true>(P, e.x, table_divider(e), amax_raw));
    reinterpret_cast<uint8_t*>(a.scales)[scale_slot((int64_t)u, a.units_per_row, a.mma_scales)] = (uint8_t)sbyte;
  }
}

// Amax of the rotated tensor: per-warp maximum of the bit patterns (non-negative floats order
// like unsigned integers), one atomicMax per warp into the workspace header. Like the lean
// kernels: rotation and layout fixed at compile time, the next block's load in flight.
template <bool RHT, bool FLAT>
__global__ void __launch_bounds__(kThreads) amax_kernel(const QuantArgs a) {
  constexpr float kCinv = RHT ? 0.25f : 1.0f;
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  pdl_enter();
  uint32_t m = 0u;
  using Idx = typename UnitIdx<FLAT>::T;
  const Idx n = (Idx)a.nunits;
  const Idx stride = (Idx)gridDim.x * kThreads;
  Idx u = (Idx)blockIdx.x * kThreads + threadIdx.x;
  if (u < n) {
    uint4 lo, hi;
    lean_load<0, RHT, FLAT>(a, u, lo, hi);
    for (; u < n; u += stride) {
      uint4 nlo = lo, nhi = hi;
      if (u + stride < n) lean_load<0, RHT, FLAT>(a, u + stride, nlo, nhi);
      float2 P[8];
      unpack16(lo, hi, RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, P);
      if constexpr (RHT) fwht16(P);
      m = max(m, __float_as_uint(__fmul_rn(absmax16(P), kCinv)));
      lo = nlo;
      hi = nhi;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m != 0u) atomicMax(&a.ws->amax_bits, m);
}

// Per-group amax of the rotated tensor: one warp per row (a row lies in one group), the
// row's blocks strided over the lanes, a warp maximum, one atomicMax per row into the group's
// slot.
template <bool RHT>
__global__ void __launch_bounds__(kThreads) grouped_amax_kernel(const QuantArgs a) {
  constexpr float kCinv = RHT ? 0.25f : 1.0f;
  const uint32_t zero_flip[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < a.rows; r += warps) {
    uint32_t m = 0u;
    for (int64_t b = lane; b < a.units_per_row; b += 32) {
      uint4 lo, hi;
      load16(a.x + r * a.ld + b * 16, a.vec32 != 0, lo, hi);
      float2 P[8];
      unpack16(lo, hi, RHT ? a.flip_lo : zero_flip, RHT ? a.flip_hi : zero_flip, P);
      if constexpr (RHT) fwht16(P);
      m = max(m, __float_as_uint(__fmul_rn(absmax16(P), kCinv)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0 && m != 0u) atomicMax(a.group_amax + group_of(a.group_off, a.n_groups, r), m);
  }
}

// alpha_g = RN(amax_g / RN(qmax * 448)) for every group (0 for an empty or all-zero group).
__global__ void grouped_alpha_kernel(const uint32_t* amax, int n, float qmax, float* ts) {
  for (int g = blockIdx.x * blockDim.x + threadIdx.x; g < n; g += gridDim.x * blockDim.x)
    ts[g] = __fdiv_rn(__uint_as_float(amax[g]), __fmul_rn(qmax, 448.0f));
}

// The rotation alone: y = 1/4 H16 D x, stored bf16 (RNE) or FP32.
__global__ void __launch_bounds__(kThreads) rht16_kernel(const QuantArgs a, int out_fp32, void* out) {
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.nunits; u += stride) {
    uint4 lo, hi;
    load16(a.x + unit_offset(a, u, 16), a.vec32 != 0, lo, hi);
    float2 P[8];
    unpack16(lo, hi, a.flip_lo, a.flip_hi, P);
    fwht16(P);
    float y[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) y[e] = __fmul_rn(elem_x(P, e), 0.25f);
    if (out_fp32) {
      float4* d = reinterpret_cast<float4*>(out) + u * 4;
#pragma unroll
      for (int k = 0; k < 4; ++k) __stcs(d + k, make_float4(y[4 * k], y[4 * k + 1], y[4 * k + 2], y[4 * k + 3]));
    } else {
      uint4 o0, o1;
      o0.x = pack_bf16x2(y[0], y[1]);   o0.y = pack_bf16x2(y[2], y[3]);
      o0.z = pack_bf16x2(y[4], y[5]);   o0.w = pack_bf16x2(y[6], y[7]);
      o1.x = pack_bf16x2(y[8], y[9]);   o1.y = pack_bf16x2(y[10], y[11]);
      o1.z = pack_bf16x2(y[12], y[13]); o1.w = pack_bf16x2(y[14], y[15]);
      uint4* d = reinterpret_cast<uint4*>(out) + u * 2;
      __stcs(d, o0);
      __stcs(d + 1, o1);
    }
  }
}

// Codes back to bf16 (optionally through the inverse rotation x = D 1/4 H16 xhat).
struct DeqArgs {
  const uint8_t* codes;
  const void* scales;
  const float* ts;
  uint16_t* out;
  int64_t nunits;    // 16-element blocks
  int64_t scale_cols;  // scale columns per row (cols/16, MX cols/32)
  uint32_t sw[8];
  int inverse;
  int mma_scales;    // E4M3 / UE8M0 scales in the block-scaled MMA tile layout
};

template <int G, int S>
__global__ void __launch_bounds__(kThreads) dequant_kernel(const DeqArgs a) {
  const float alpha = (S == kE4M3) ? *a.ts : 0.0f;
  const float r67 = kR67;
  const int64_t stride = (int64_t)gridDim.x * kThreads;
  for (int64_t u = (int64_t)blockIdx.x * kThreads + threadIdx.x; u < a.nunits; u += stride) {
    const uint2 cw = __ldcs(reinterpret_cast<const uint2*>(a.codes) + u);
    float s;
    bool int_block = false;
    if constexpr (S == kFP32) {
      s = reinterpret_cast<const float*>(a.scales)[u];
    } else if constexpr (S == kE4M3) {
      const uint32_t b = reinterpret_cast<const uint8_t*>(a.scales)[scale_slot(u, a.scale_cols, a.mma_scales)];
      int_block = (G == kIF4) && (b & 0x80u);
      s = __fmul_rn(e4m3_to_f32(b & 0x7Fu), alpha);
    } else {
      const int e =
          (int)reinterpret_cast<const uint8_t*>(a.scales)[scale_slot(u >> 1, a.scale_cols, a.mma_scales)] - 127;
      s = (e >= -126) ? __uint_as_float((uint32_t)(127 + e) << 23) : 0x1p-127f;
    }
    float v[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const uint32_t nib = ((e < 8 ? cw.x : cw.y) >> (4 * (e & 7))) & 0xFu;
      float q;
      if (G == kINT4 || int_block) {
        const uint32_t m = (nib & 8u) ? 16u - nib : nib;
        const float k = small_int_f32(m);
        q = (nib & 8u) ? -k : k;
        if (int_block) q = __fmul_rn(q, r67);
      } else if (G == kE1M2) {
        const float g = __fmul_rn(small_int_f32(nib & 7u), 0.5f);
        q = __uint_as_float(__float_as_uint(g) | ((nib & 8u) << 28));
      } else {
        const float2 d = e2m1x2_to_f32(nib);
        q = d.x;
      }
      v[e] = __fmul_rn(q, s);
    }
    if (a.inverse) {
      float2 P[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) P[i] = make_float2(v[i], v[i + 8]);
      fwht16(P);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float t = __fmul_rn(elem_x(P, e), 0.25f);
        // element e's sign flip: word e >> 1 of sw, bit 15 (even e) or bit 31 (odd e)
        const uint32_t flip = (a.sw[e >> 1] >> ((e & 1) ? 31 : 15)) & 1u;
        v[e] = __uint_as_float(__float_as_uint(t) ^ (flip << 31));
      }
    }
    uint4 o0, o1;
    o0.x = pack_bf16x2(v[0], v[1]);   o0.y = pack_bf16x2(v[2], v[3]);
    o0.z = pack_bf16x2(v[4], v[5]);   o0.w = pack_bf16x2(v[6], v[7]);
    o1.x = pack_bf16x2(v[8], v[9]);   o1.y = pack_bf16x2(v[10], v[11]);
    o1.z = pack_bf16x2(v[12], v[13]); o1.w = pack_bf16x2(v[14], v[15]);
    uint4* d = reinterpret_cast<uint4*>(a.out) + u * 2;
    __stcs(d, o0);
    __stcs(d + 1, o1);
  }
}

// Fixed-order FP64 reduction of the per-CTA records into the header (one thread per field).
__global__ void stats_reduce_kernel(WsHeader* ws, const double* partials) {
  const int f = threadIdx.x;
  if (f >= ST_LEN) return;
  double s = 0.0;
  const uint32_t n = (ws->magic == kWsMagic) ? min(ws->n_partials, (uint32_t)kStatsCtas) : 0u;
  for (uint32_t i = 0; i < n; ++i) s += partials[(size_t)i * ST_LEN + f];
  ws->reduced[f] = s;
}

// Self-check of the exact-quotient step: pseudo-random pairs (s, y) with s in [2^-60, 2^90)
// and y / s in [2^-20, 8), with and without the folded 1/4, compared with IEEE division.
__global__ void __launch_bounds__(kThreads) division_check_kernel(uint64_t seed, uint64_t n,
                                                                  unsigned long long* bad) {
  unsigned long long local = 0;
  const uint64_t stride = (uint64_t)gridDim.x * kThreads;
  // every mantissa of a in [1, 4) for the six compile-time divisors (the scale quotient
  // a / qmax); by scale invariance this covers all a in [2^-100, 2^100]
  for (uint64_t i = (uint64_t)blockIdx.x * kThreads + threadIdx.x; i < (6ull << 24); i += stride) {
    const uint32_t m = (uint32_t)(i & 0xFFFFFFu);
    const float a = __uint_as_float(((127u + (m >> 23)) << 23) | (m & 0x7FFFFFu));
    const int g = (int)(i >> 24);
    float got, want;
    if (g == 0) { got = div_qmax<kE2M1>(a); want = __fdiv_rn(a, 6.0f); }
    else if (g == 1) { got = div_qmax<kE1M2>(a); want = __fdiv_rn(a, 3.5f); }
    else if (g == 2) { got = div_qmax<kINT4>(a); want = __fdiv_rn(a, 7.0f); }
    else if (g == 3) { got = div_qmax<kE2M1Max4>(a); want = __fdiv_rn(a, 4.0f); }
    else if (g == 4) { got = div_qmax<kE2M1Max3>(a); want = __fdiv_rn(a, 3.0f); }
    else { got = div_qmax<kE2M1Max2>(a); want = __fdiv_rn(a, 2.0f); }
    if (__float_as_uint(got) != __float_as_uint(want)) ++local;
  }
  // the block reciprocal: every float S in [2^-60, 2^91) (151 binades x 2^23 mantissas)
  for (uint64_t i = (uint64_t)blockIdx.x * kThreads + threadIdx.x; i < (151ull << 23); i += stride) {
    const float S = __uint_as_float(((uint32_t)(67 + (i >> 23)) << 23) | (uint32_t)(i & 0x7FFFFFu));
    if (__float_as_uint(rcp_rn_fast(S)) != __float_as_uint(__frcp_rn(S))) ++local;
  }
  for (uint64_t i = (uint64_t)blockIdx.x * kThreads + threadIdx.x; i < n; i += stride) {
    const uint64_t h = splitmix64(seed ^ (i * 0x9E3779B97F4A7C15ull));
    const uint64_t g = splitmix64(h);
    const int es = (int)(h % 151u) - 60;                        // 2^-60 .. 2^90
    const float s = __uint_as_float(((uint32_t)(127 + es) << 23) | (uint32_t)(h >> 41));
    const int et = (int)((h >> 8) % 24u) - 21;                  // 2^-21 .. 2^2 (times [1,2))
    const float t = __uint_as_float(((uint32_t)(127 + et) << 23) | (uint32_t)(g & 0x7FFFFFu));
    float y = __fmul_rn(s, t);
    if (g >> 63) y = -y;
    for (int rot = 0; rot < 2; ++rot) {
      const float c = rot ? 4.0f : 1.0f;
      const Divider dv = make_divider(s, c);
      if (!dv.fast) continue;
      const float vraw = __fmul_rn(y, c);
      const float2 q = div2(dv, make_float2(vraw, -vraw));
      const float want = __fdiv_rn(y, s);
      if (fabsf(want) < 0x1p-20f) continue;
      if (__float_as_uint(fabsf(q.x)) != __float_as_uint(fabsf(want)) ||
          __float_as_uint(fabsf(q.y)) != __float_as_uint(fabsf(want)))
        ++local;
    }
  }
  if (local) atomicAdd(bad, local);
}

// Self-check of the hardware conversions the encoders rely on, each against a rule written here
// from the format's definition (exponent field, step, round half to even through the integer
// conversion, saturation), over every FP32 input in the range the kernels feed it:
//   bad[0]  E2M1 encode (cvt.rn.satfinite.e2m1x2), every non-NaN float
//   bad[1]  E1M2 encode through the FP6 E2M3 conversion (e1m2_word), every float |e| < 15/16
//   bad[2]  E4M3 encode of a block-scale quotient (cvt.rn.satfinite.e4m3x2), every float >= 0
//   bad[3]  the E2M1 (all 256 byte values) and E4M3 (codes 0..0x7E) decoders, and the IF4
//           factors RN(7/6), RN(6/7) against the IEEE quotients
//   bad[4]  bf16 packing of the dequantized values (cvt.rn.bf16x2.f32), every non-NaN float
__device__ __forceinline__ uint32_t e2m1_rule(float x) {
  const uint32_t sgn = __float_as_uint(x) >> 31;
  const float a = fabsf(x);
  uint32_t m;
  if (a < 2.0f) {
    m = (uint32_t)__float2int_rn(a * 2.0f);              // step 1/2: codes 0..4 are k / 2
  } else if (a < 4.0f) {
    m = (uint32_t)__float2int_rn(a) + 2u;                // step 1: 2, 3, 4 -> codes 4, 5, 6
  } else {
    const int k = a >= 16.0f ? 3 : __float2int_rn(a * 0.5f);   // step 2: 4, 6 -> codes 6, 7
    m = (uint32_t)min(k, 3) + 4u;                        // saturation at 6
  }
  return (sgn << 3) | m;
}

__device__ __forceinline__ uint32_t e4m3_rule(float x) {   // x >= 0, not NaN
  if (x >= 448.0f) return 0x7Eu;                           // satfinite: 448 and above -> 448
  if (x < 0x1p-6f) return (uint32_t)__float2int_rn(x * 512.0f);   // subnormal step 2^-9
  const int E = (int)(__float_as_uint(x) >> 23) - 127;        // 2^E <= x < 2^(E+1), E in [-6, 8]
  const float up = __uint_as_float((uint32_t)(127 + 3 - E) << 23);   // 2^(3-E), exact scaling
  const int m = __float2int_rn(x * up);                       // 8 .. 16
  const uint32_t code = (uint32_t)(((E + 7) << 3) + m - 8);   // 16 carries into the exponent
  return min(code, 0x7Eu);
}

__global__ void __launch_bounds__(kThreads) conversion_check_kernel(unsigned long long* bad) {
  unsigned long long nb[5] = {0, 0, 0, 0, 0};
  const uint64_t stride = (uint64_t)gridDim.x * kThreads;
  for (uint64_t i = (uint64_t)blockIdx.x * kThreads + threadIdx.x; i < (1ull << 32); i += stride) {
    const uint32_t u = (uint32_t)i;
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x7FFFFFu)) continue;   // NaN
    const float x = __uint_as_float(u);
    const uint32_t e2 = cvt_e2m1x2(x, x), want2 = e2m1_rule(x);
    if ((e2 & 0xFu) != want2 || (e2 >> 4) != want2) ++nb[0];
    const uint32_t bf = pack_bf16x2(x, x), wantb = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
    if ((bf & 0xFFFFu) != wantb || (bf >> 16) != wantb) ++nb[4];
    if ((u & 0x7FFFFFFFu) < 0x3F700000u) {                 // |x| < 15/16
      const float e[8] = {x, x, x, x, x, x, x, x};
      const uint32_t want = ((u >> 31) << 3) | (uint32_t)__float2int_rn(fabsf(x) * 8.0f);
      if (e1m2_word(e) != want * 0x11111111u) ++nb[1];
    }
    if ((u >> 31) == 0u && cvt_e4m3(x) != e4m3_rule(x)) ++nb[2];
    if (i < 256) {   // the E2M1 decoder on byte i (low nibble -> .x)
      const float2 d = e2m1x2_to_f32((uint32_t)i);
      const float tab[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
      const uint32_t lo = (uint32_t)i & 0xFu, hi = (uint32_t)i >> 4;
      const float wl = (lo & 8u) ? -tab[lo & 7u] : tab[lo & 7u];
      const float wh = (hi & 8u) ? -tab[hi & 7u] : tab[hi & 7u];
      if (__float_as_uint(d.x) != __float_as_uint(wl) || __float_as_uint(d.y) != __float_as_uint(wh)) ++nb[3];
    }
    if (i == 0 && (__float_as_uint(__fdiv_rn(7.0f, 6.0f)) != __float_as_uint(kR76) ||
                   __float_as_uint(__fdiv_rn(6.0f, 7.0f)) != __float_as_uint(kR67)))
      ++nb[3];   // the IF4 factors are the IEEE quotients
    if (i < 0x7F) {   // the E4M3 decoder on code i: m 2^-9 (e = 0) or (8 + m) 2^(e - 10)
      const int e = (int)(i >> 3), m = (int)(i & 7);
      const float want = e == 0 ? (float)m * 0x1p-9f
                                : (float)(8 + m) * __uint_as_float((uint32_t)(127 + e - 10) << 23);
      if (__float_as_uint(e4m3_to_f32((uint32_t)i)) != __float_as_uint(want)) ++nb[3];
    }
  }
#pragma unroll
  for (int k = 0; k < 5; ++k)
    if (nb[k]) atomicAdd(bad + k, nb[k]);
}

// ------------------------------------------------------------------ launch helpers

// Resident CTAs of `kernel` on the current device (SM count x occupancy), queried once per
// (kernel, device) and cached, so that launches inside a stream capture do no queries.
template <class K>
int resident_ctas(K kernel, int threads = kThreads) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev * 4096 + threads);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int sms = 148, per_sm = 1;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
  const int n = sms * std::max(per_sm, 1);
  cache.emplace(key, n);
  return n;
}

// Launch with programmatic stream serialization (the kernels call pdl_enter() first).
template <class... Args>
cudaError_t launch_pdl_n(void (*kernel)(Args...), int grid, int threads, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <class... Args>
cudaError_t launch_pdl(void (*kernel)(Args...), int grid, cudaStream_t st, Args... args) {
  return launch_pdl_n(kernel, grid, kThreads, st, args...);
}

// Grid of a grid-stride kernel: enough CTAs for work_threads threads, at most `waves` times the
// CTAs that fit on the device at once (one wave: a persistent grid).
template <class K>
int persistent_grid(K kernel, int64_t work_threads, int threads = kThreads, int waves = 1) {
  const int64_t need = (work_threads + threads - 1) / threads;
  return (int)std::max<int64_t>(1, std::min<int64_t>(need, (int64_t)waves * resident_ctas(kernel, threads)));
}

// Waves for the one-block and E4M3 quantizers (E4M3 scales, IF4, stochastic rounding, unrotated
// FP32 scales): with four, a CTA that finishes its share early is replaced by a fresh one and the
// SMs keep more warps resident through the launch. Measured on a 16384 x 5120 tensor: NVFP4 with
// the tensor scale given 37.9 against 40.0 us, IF4 71.0 against 73.4 us; E1M2 with stochastic
// rounding on an 8192 x 8192 dY 61.0 against 63.0 us; unrotated E2M1 on a 32768 x 8192 tensor
// 115.9 against 118.5 us. The rotated two-block kernel for FP32 scales (17.05 against 18.07 us on
// stacked 16384 x 2048 operands) and the generic kernel (MXFP4: 35.9 against 37.0 us) stay
// persistent.
constexpr int kIssueBoundWaves = 4;

template <int G, int S, int R, bool STATS>
cudaError_t launch_q(const QuantArgs& a, cudaStream_t st) {
  auto k = quantize_kernel<G, S, R, STATS>;
  int grid;
  if (STATS) {
    grid = kStatsCtas;
  } else {
    // two units per thread per iteration
    grid = persistent_grid(k, (a.nunits + 1) / 2);
  }
  const cudaError_t e = launch_pdl(k, grid, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G, int S, int R>
cudaError_t launch_q_stats(bool stats, const QuantArgs& a, cudaStream_t st) {
  return stats ? launch_q<G, S, R, true>(a, st) : launch_q<G, S, R, false>(a, st);
}

template <int G, int S>
cudaError_t launch_q_round(int round, bool stats, const QuantArgs& a, cudaStream_t st) {
  return round == kSR ? launch_q_stats<G, S, kSR>(stats, a, st)
                      : launch_q_stats<G, S, kRTNE>(stats, a, st);
}

}  // namespace

template <int G, bool RHT, bool FLAT, int R>
cudaError_t launch_lean3(const QuantArgs& a, cudaStream_t st) {
  auto k = lean_kernel<G, RHT, FLAT, R>;
  const cudaError_t e = launch_pdl(k, persistent_grid(k, a.nunits, kThreads, kIssueBoundWaves), st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G, bool RHT, bool FLAT, bool GROUPED>
cudaError_t launch_lean_nv4(const QuantArgs& a, cudaStream_t st) {
  auto k = lean_nv_kernel<G, RHT, FLAT, GROUPED>;
  // the grouped kernel keeps one wave: each thread's first block looks its group up
  const int waves = GROUPED ? 1 : kIssueBoundWaves;
  const cudaError_t e = launch_pdl(k, persistent_grid(k, a.nunits, kThreads, waves), st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G>
cudaError_t launch_lean_nv_pair(const QuantArgs& a, cudaStream_t st) {
  // E2M1 takes 72 registers a thread, at which 128-thread CTAs let 28 warps reside per SM against
  // 24 in three 256-thread CTAs (measured 40.0 against 41.0 us on a 16384 x 5120 tensor); E1M2
  // and INT4 take 80, where smaller CTAs gain no warps (43.3 against 42.3 us for INT4)
  constexpr int kTh = G == kE2M1 ? 128 : 256;
  auto k = lean_nv_pair_kernel<G, kTh>;
  const cudaError_t e = launch_pdl_n(k, persistent_grid(k, (a.nunits + 1) / 2, kTh, kIssueBoundWaves), kTh, st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G, bool GROUPED = false>
cudaError_t launch_lean_nv(const QuantArgs& a, cudaStream_t st) {
  const bool rht = a.c != 1.0f, flat = flat_launch(a);
  // one tensor scale, rotated, flat: two blocks per thread (IF4's two candidates stay on one)
  if constexpr (!GROUPED && G != kIF4) {
    if (rht && flat && reinterpret_cast<uintptr_t>(a.codes) % 16 == 0 && reinterpret_cast<uintptr_t>(a.scales) % 2 == 0)
      return launch_lean_nv_pair<G>(a, st);
  }
  if (rht) return flat ? launch_lean_nv4<G, true, true, GROUPED>(a, st) : launch_lean_nv4<G, true, false, GROUPED>(a, st);
  return flat ? launch_lean_nv4<G, false, true, GROUPED>(a, st) : launch_lean_nv4<G, false, false, GROUPED>(a, st);
}

template <int G, bool RHT>
cudaError_t launch_lean_pair(const QuantArgs& a, cudaStream_t st) {
  auto k = lean_pair_kernel<G, RHT>;
  const cudaError_t e = launch_pdl(k, persistent_grid(k, (a.nunits + 1) / 2), st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G, int R>
cudaError_t launch_lean(const QuantArgs& a, cudaStream_t st) {
  const bool rht = a.c != 1.0f, flat = flat_launch(a);
  // rotated, flat and round to nearest: two blocks per thread when the pair stores are aligned.
  // Unrotated tensors stay on one block per thread: their sign copies take the pair kernel past
  // 64 registers, and a version that copied the signs inside the quotient loop (64 registers,
  // E2M1 spilling 12 bytes) gained 6% on a 33.5 M-element E2M1 tensor but lost 1-5% on the
  // 268 M and 940 M-element ones.
  if (R == kRTNE && rht && flat && pair_aligned(a)) return launch_lean_pair<G, true>(a, st);
  if (rht) return flat ? launch_lean3<G, true, true, R>(a, st) : launch_lean3<G, true, false, R>(a, st);
  return flat ? launch_lean3<G, false, true, R>(a, st) : launch_lean3<G, false, false, R>(a, st);
}

// Range-restricted E2M1 (FP32 scale only): the lean kernel for codes only, else the generic one.
template <int G>
cudaError_t launch_restricted(int round, bool stats, const QuantArgs& a, cudaStream_t st) {
  if (!stats && a.deq == nullptr)
    return round == kSR ? launch_lean<G, kSR>(a, st) : launch_lean<G, kRTNE>(a, st);
  return launch_q_round<G, kFP32>(round, stats, a, st);
}

cudaError_t launch_quantize(int grid, int scale, int round, bool stats, const QuantArgs& a,
                            cudaStream_t st) {
  if (grid >= kE2M1Max4) {
    if (scale != kFP32) return cudaErrorInvalidValue;
    if (grid == kE2M1Max4) return launch_restricted<kE2M1Max4>(round, stats, a, st);
    if (grid == kE2M1Max3) return launch_restricted<kE2M1Max3>(round, stats, a, st);
    if (grid == kE2M1Max2) return launch_restricted<kE2M1Max2>(round, stats, a, st);
    return cudaErrorInvalidValue;
  }
  if (scale == kFP32 && !stats && a.deq == nullptr) {
    if (round == kSR) {
      if (grid == kE2M1) return launch_lean<kE2M1, kSR>(a, st);
      if (grid == kE1M2) return launch_lean<kE1M2, kSR>(a, st);
      if (grid == kINT4) return launch_lean<kINT4, kSR>(a, st);
    } else {
      if (grid == kE2M1) return launch_lean<kE2M1, kRTNE>(a, st);
      if (grid == kE1M2) return launch_lean<kE1M2, kRTNE>(a, st);
      if (grid == kINT4) return launch_lean<kINT4, kRTNE>(a, st);
    }
  }
  if (scale == kE4M3 && round == kRTNE && !stats && a.deq == nullptr) {
    if (grid == kE2M1) return launch_lean_nv<kE2M1>(a, st);
    if (grid == kE1M2) return launch_lean_nv<kE1M2>(a, st);
    if (grid == kINT4) return launch_lean_nv<kINT4>(a, st);
    if (grid == kIF4) return launch_lean_nv<kIF4>(a, st);
  }
  if (scale == kFP32) {
    if (grid == kE2M1) return launch_q_round<kE2M1, kFP32>(round, stats, a, st);
    if (grid == kE1M2) return launch_q_round<kE1M2, kFP32>(round, stats, a, st);
    if (grid == kINT4) return launch_q_round<kINT4, kFP32>(round, stats, a, st);
  } else if (scale == kE4M3) {
    if (grid == kE2M1) return launch_q_round<kE2M1, kE4M3>(round, stats, a, st);
    if (grid == kE1M2) return launch_q_round<kE1M2, kE4M3>(round, stats, a, st);
    if (grid == kINT4) return launch_q_round<kINT4, kE4M3>(round, stats, a, st);
    if (grid == kIF4) return launch_q_stats<kIF4, kE4M3, kRTNE>(stats, a, st);
  } else if (scale == kUE8M0) {
    if (grid == kE2M1) return launch_q_round<kE2M1, kUE8M0>(round, stats, a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_grouped(int grid, const QuantArgs& a, cudaStream_t st) {
  if (grid == kE2M1) return launch_lean_nv<kE2M1, true>(a, st);
  if (grid == kE1M2) return launch_lean_nv<kE1M2, true>(a, st);
  if (grid == kINT4) return launch_lean_nv<kINT4, true>(a, st);
  if (grid == kIF4) return launch_lean_nv<kIF4, true>(a, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_grouped_amax(const QuantArgs& a, cudaStream_t st) {
  auto k = a.c != 1.0f ? grouped_amax_kernel<true> : grouped_amax_kernel<false>;
  const cudaError_t e = launch_pdl(k, persistent_grid(k, a.rows * 32), st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_grouped_alpha(const QuantArgs& a, float qmax, cudaStream_t st) {
  grouped_alpha_kernel<<<(a.n_groups + 255) / 256, 256, 0, st>>>(a.group_amax, a.n_groups, qmax, a.group_ts);
  return cudaGetLastError();
}

template <bool RHT, bool FLAT>
cudaError_t launch_amax2(const QuantArgs& a, cudaStream_t st) {
  auto k = amax_kernel<RHT, FLAT>;
  const cudaError_t e = launch_pdl(k, persistent_grid(k, a.nunits), st, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_amax(const QuantArgs& a, cudaStream_t st) {
  const bool rht = a.c != 1.0f, flat = flat_launch(a);
  if (rht) return flat ? launch_amax2<true, true>(a, st) : launch_amax2<true, false>(a, st);
  return flat ? launch_amax2<false, true>(a, st) : launch_amax2<false, false>(a, st);
}

__global__ void alpha_kernel(const WsHeader* ws, float qmax, float* tensor_scale) {
  *tensor_scale = __fdiv_rn(__uint_as_float(ws->amax_bits), __fmul_rn(qmax, 448.0f));
}

cudaError_t launch_alpha(WsHeader* ws, float qmax, float* tensor_scale, cudaStream_t st) {
  alpha_kernel<<<1, 1, 0, st>>>(ws, qmax, tensor_scale);
  return cudaGetLastError();
}

cudaError_t launch_rht16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                         const uint32_t* sw, void* out, bool out_fp32, cudaStream_t st) {
  QuantArgs a{};
  a.x = x;
  a.rows = rows;
  a.cols = cols;
  a.ld = ld;
  a.units_per_row = cols / 16;
  a.nunits = rows * a.units_per_row;
  a.contiguous = (ld == cols);
  for (int k = 0; k < 8; ++k) a.sw[k] = sw[k];
  sign_flips(a.sw, a.flip_lo, a.flip_hi);
  a.c = 4.0f;
  a.cinv = 0.25f;
  a.vec32 = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (rows == 1 || ld % 16 == 0);
  if (a.nunits == 0) return cudaSuccess;
  rht16_kernel<<<persistent_grid(rht16_kernel, a.nunits), kThreads, 0, st>>>(a, out_fp32 ? 1 : 0, out);
  return cudaGetLastError();
}

template <int G, int S>
cudaError_t launch_dq(const DeqArgs& a, cudaStream_t st) {
  auto k = dequant_kernel<G, S>;
  k<<<persistent_grid(k, a.nunits), kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequant(int grid, int scale, const uint8_t* codes, const void* scales,
                           const float* ts, int64_t rows, int64_t cols, const uint32_t* sw,
                           bool inverse, bool mma_scales, uint16_t* out, cudaStream_t st) {
  DeqArgs a{};
  a.codes = codes;
  a.scales = scales;
  a.ts = ts;
  a.out = out;
  a.nunits = rows * (cols / 16);
  a.scale_cols = scale == kUE8M0 ? cols / 32 : cols / 16;
  a.mma_scales = mma_scales ? 1 : 0;
  for (int k = 0; k < 8; ++k) a.sw[k] = sw[k];
  a.inverse = inverse ? 1 : 0;
  if (a.nunits == 0) return cudaSuccess;
  if (scale == kFP32) {
    if (grid == kE2M1) return launch_dq<kE2M1, kFP32>(a, st);
    if (grid == kE1M2) return launch_dq<kE1M2, kFP32>(a, st);
    if (grid == kINT4) return launch_dq<kINT4, kFP32>(a, st);
  } else if (scale == kE4M3) {
    if (grid == kE2M1) return launch_dq<kE2M1, kE4M3>(a, st);
    if (grid == kE1M2) return launch_dq<kE1M2, kE4M3>(a, st);
    if (grid == kINT4) return launch_dq<kINT4, kE4M3>(a, st);
    if (grid == kIF4) return launch_dq<kIF4, kE4M3>(a, st);
  } else if (scale == kUE8M0) {
    if (grid == kE2M1) return launch_dq<kE2M1, kUE8M0>(a, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_division_check(uint64_t seed, uint64_t n, unsigned long long* bad,
                                  cudaStream_t st) {
  division_check_kernel<<<persistent_grid(division_check_kernel, (int64_t)std::min<uint64_t>(n, 1ull << 40)),
                          kThreads, 0, st>>>(seed, n, bad);
  return cudaGetLastError();
}

cudaError_t launch_conversion_check(unsigned long long* bad, cudaStream_t st) {
  conversion_check_kernel<<<resident_ctas(conversion_check_kernel), kThreads, 0, st>>>(bad);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_check(unsigned long long limit_ns, cudaStream_t st) {
  wait_timeout_kernel<<<1, 1, 0, st>>>(limit_ns);
  return cudaGetLastError();
}

// Device address of the status word on the current device (looked up once per device; kernels
// of other translation units receive it as an argument).
cudaError_t device_status_word(int32_t** out) {
  static std::mutex mu;
  static std::map<int, int32_t*> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) return e;
    it = cache.emplace(dev, static_cast<int32_t*>(p)).first;
  }
  *out = it->second;
  return cudaSuccess;
}

cudaError_t read_device_status(int32_t* out, bool clear, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_device_status, sizeof(int32_t), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  if (clear) {
    static const int32_t zero = 0;
    e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int32_t), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return e;
  }
  return cudaStreamSynchronize(st);
}

cudaError_t launch_stats_reduce(WsHeader* ws, const double* partials, cudaStream_t st) {
  stats_reduce_kernel<<<1, 32, 0, st>>>(ws, partials);
  return cudaGetLastError();
}

}  // namespace fp4q

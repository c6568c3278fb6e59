// fp4q_dual.cu -- dY quantized in both orientations from one read of HBM.
//
// bwd_dx reduces dY over N, so it needs dY blocked along rows; bwd_dw reduces over M, so it
// needs dY^T blocked along rows of dY^T (columns of dY). The UFP4 recipe applies the rotation
// and stochastic rounding to dY on both paths ("当你的 GPU 学不会算账", zhichai.net/topic/
// 178208020, recipe table of section "UFP4：换一把尺子"; "蚂蚁集团揭秘…", techwalker.com,
// section 三 on bwd_dx / bwd_dw).
//
// One CTA per 128 x 64 tile of dY (a 1-D grid over the tiles, columns fastest). Each of its 256
// threads loads two row blocks (16 consecutive bf16 of one row, 32 bytes), encodes them from
// registers and parks them in a padded shared tile; after one barrier, warp g encodes the column
// blocks of rows 16g .. 16g+15, each lane the two adjacent columns 2l, 2l+1 whose elements share
// one 32-bit shared-memory word per row. The column results are staged in shared memory and
// leave as 16-byte stores, each column's 64 bytes of codes and 32 bytes of scales contiguous.
//
// The pass is bound by instruction issue (stochastic rounding's SplitMix64 draws alone are about
// a fifth of its instructions), so the layout favours occupancy: 64 registers and 26 KB of shared
// memory give four resident CTAs (32 warps) per SM. A persistent variant fed by 2-D TMA copies
// through a shared-memory ring was measured slower (three CTAs per SM at its register count).
#include <cuda_fp16.h>

#include "fp4q_device.cuh"
#include "fp4q_encode.cuh"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

constexpr int kTileM = 128, kTileN = 64;
constexpr int kPitch = kTileN + 8;   // elements; 144-byte rows (conflict-free 16-byte stores)
constexpr int kGroups = kTileM / 16;  // column blocks per column of a tile
constexpr int kCodePitch = 10;        // uint2 per staged column (8 used; 16-byte aligned rows)
constexpr int kScalePitch = 12;       // floats per staged column (8 used)

// ROT: both orientations rotated (c = 4 at compile time); otherwise per-orientation flags.
template <int G, int RR, int RC, bool ROT>
__global__ void __launch_bounds__(kThreads, 4) dual_kernel(const DualArgs a) {
  __shared__ __align__(16) uint16_t tile[kTileM * kPitch];
  __shared__ __align__(16) uint2 stage_codes[kTileN * kCodePitch];
  __shared__ __align__(16) float stage_scales[kTileN * kScalePitch];
  const uint32_t tiles_n = (uint32_t)((a.N + kTileN - 1) / kTileN);
  const int64_t m0 = (int64_t)(blockIdx.x / tiles_n) * kTileM;
  const int64_t n0 = (int64_t)(blockIdx.x % tiles_n) * kTileN;
  const int t = threadIdx.x;
  const bool rot_row = ROT || a.c_row != 1.0f;
  const bool rot_col = ROT || a.c_col != 1.0f;
  const float c_row = ROT ? 4.0f : a.c_row, c_col = ROT ? 4.0f : a.c_col;
  const float cinv_row = ROT ? 0.25f : a.cinv_row, cinv_col = ROT ? 0.25f : a.cinv_col;
  pdl_enter();

  // row blocks rb = t, t + 256: row rb / 4, columns 16 * (rb % 4) .. +15 (zeros outside)
  uint4 v[2][2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int rb = t + k * kThreads, r = rb >> 2, b = rb & 3;
    v[k][0] = v[k][1] = make_uint4(0u, 0u, 0u, 0u);
    if (m0 + r < a.M && n0 + 16 * b < a.N)
      load16(a.dy + (m0 + r) * a.ld + n0 + 16 * b, a.vec32 != 0, v[k][0], v[k][1]);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int rb = t + k * kThreads, r = rb >> 2, b = rb & 3;
    uint4* dst = reinterpret_cast<uint4*>(&tile[r * kPitch + 16 * b]);
    dst[0] = v[k][0];
    dst[1] = v[k][1];
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int rb = t + k * kThreads, r = rb >> 2, b = rb & 3;
    const int64_t m = m0 + r, n = n0 + 16 * b;
    if (m >= a.M || n >= a.N) continue;
    float2 P[8];
    unpack16(v[k][0], v[k][1], a.flip_lo_row, a.flip_hi_row, P);
    if (rot_row) fwht16(P);
    const float s = div_qmax<G>(__fmul_rn(absmax16(P), cinv_row));
    const int64_t u = (m * a.N + n) >> 4;   // 16-block index in [M, N/16]
    uint2 w;
    if constexpr (RR == kSR) w = encode_sr<G>(P, s, c_row, a.seedx_row, (uint64_t)u * 4u);
    else w = ROT ? encode_lean<G, true>(P, s) : encode_rtne_rt<G>(P, s, rot_row);
    __stcs(reinterpret_cast<uint2*>(a.codes_row) + u, w);
    __stcs(a.scales_row + u, s);
  }
  __syncthreads();

  // column blocks: rows 16g .. 16g+15, columns 2 * lane + h (N % 16 == 0, M % 16 == 0: a
  // column pair and a group of 16 rows are in range or out of range as a whole)
  const int g = t >> 5, lane = t & 31;
  const int64_t m = m0 + 16 * g, nA = n0 + 2 * lane;
  if (m < a.M && nA < a.N) {
    uint32_t wd[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      wd[i] = *reinterpret_cast<const uint32_t*>(&tile[(16 * g + i) * kPitch + 2 * lane]);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float2 P[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        P[i] = h ? make_float2(bf_hi_flip(wd[i], a.flip_col[i]), bf_hi_flip(wd[i + 8], a.flip_col[i + 8]))
                 : make_float2(bf_lo_flip(wd[i], a.flip_col[i]), bf_lo_flip(wd[i + 8], a.flip_col[i + 8]));
      if (rot_col) fwht16(P);
      const float s = div_qmax<G>(__fmul_rn(absmax16(P), cinv_col));
      const int64_t u = ((nA + h) * a.M + m) >> 4;   // 16-block index in [N, M/16]
      uint2 w;
      if constexpr (RC == kSR) w = encode_sr<G>(P, s, c_col, a.seedx_col, (uint64_t)u * 4u);
      else w = ROT ? encode_lean<G, true>(P, s) : encode_rtne_rt<G>(P, s, rot_col);
      const int c = 2 * lane + h;
      stage_codes[c * kCodePitch + g] = w;
      stage_scales[c * kScalePitch + g] = s;
    }
  }
  __syncthreads();

  // column c's blocks for rows m0 .. m0+127 are kGroups consecutive entries of codes_col /
  // scales_col starting at block (n0 + c) * M/16 + m0/16
  const int64_t rows_left = (a.M - m0) >> 4, cols_left = a.N - n0;
  const int ng = rows_left < kGroups ? (int)rows_left : kGroups;
  const int nc = cols_left < kTileN ? (int)cols_left : kTileN;
  if (a.col16 && ng == kGroups) {
    // 16-byte stores: codes as 4 chunks of 2 blocks, scales as 2 chunks of 4 blocks per column
    {
      const int c = t >> 2, q = t & 3;
      if (c < nc) {
        const uint2 lo = stage_codes[c * kCodePitch + 2 * q], hi = stage_codes[c * kCodePitch + 2 * q + 1];
        uint2* dst = reinterpret_cast<uint2*>(a.codes_col) + (((n0 + c) * a.M + m0) >> 4) + 2 * q;
        __stcs(reinterpret_cast<uint4*>(dst), make_uint4(lo.x, lo.y, hi.x, hi.y));
      }
    }
    if (t < 2 * kTileN) {
      const int c = t >> 1, q = t & 1;
      if (c < nc) {
        const float4 v4 = *reinterpret_cast<const float4*>(&stage_scales[c * kScalePitch + 4 * q]);
        float* dst = a.scales_col + (((n0 + c) * a.M + m0) >> 4) + 4 * q;
        __stcs(reinterpret_cast<float4*>(dst), v4);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = t + k * kThreads, c = e >> 3, gg = e & 7;
      if (c < nc && gg < ng) {
        const int64_t u = (((n0 + c) * a.M + m0) >> 4) + gg;
        __stcs(reinterpret_cast<uint2*>(a.codes_col) + u, stage_codes[c * kCodePitch + gg]);
        __stcs(a.scales_col + u, stage_scales[c * kScalePitch + gg]);
      }
    }
  }
}

template <int G, int RR, int RC>
cudaError_t launch_d(const DualArgs& a, cudaStream_t st) {
  const int64_t tiles = ((a.N + kTileN - 1) / kTileN) * ((a.M + kTileM - 1) / kTileM);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)tiles);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = (a.c_row != 1.0f && a.c_col != 1.0f)
                            ? cudaLaunchKernelEx(&cfg, dual_kernel<G, RR, RC, true>, a)
                            : cudaLaunchKernelEx(&cfg, dual_kernel<G, RR, RC, false>, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G>
cudaError_t launch_d_rounds(const DualArgs& a, cudaStream_t st) {
  if (a.round_row == kSR)
    return a.round_col == kSR ? launch_d<G, kSR, kSR>(a, st) : launch_d<G, kSR, kRTNE>(a, st);
  return a.round_col == kSR ? launch_d<G, kRTNE, kSR>(a, st) : launch_d<G, kRTNE, kRTNE>(a, st);
}

}  // namespace

cudaError_t launch_dual(const DualArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  if (a.grid_row != a.grid_col) return cudaErrorInvalidValue;
  if (a.grid_row == kE2M1) return launch_d_rounds<kE2M1>(a, st);
  if (a.grid_row == kE1M2) return launch_d_rounds<kE1M2>(a, st);
  if (a.grid_row == kINT4) return launch_d_rounds<kINT4>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace fp4q

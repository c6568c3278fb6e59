// fp4q_dual.cu -- dY quantized in both orientations from one read of HBM.
//
// bwd_dx reduces dY over N, so it needs dY blocked along rows; bwd_dw reduces over M, so it
// needs dY^T blocked along rows of dY^T (columns of dY). The UFP4 recipe applies the rotation
// and stochastic rounding to dY on both paths ("当你的 GPU 学不会算账", zhichai.net/topic/
// 178208020, recipe table of section "UFP4：换一把尺子"; "蚂蚁集团揭秘…", techwalker.com,
// section 三 on bwd_dx / bwd_dw).
//
// A CTA stages a 128 x 64 bf16 tile in shared memory (padded pitch: conflict-free 16-byte row
// reads and 2-byte column reads), then each of its 256 threads encodes two row blocks and two
// column blocks with the same per-block encoder as the row kernel. A column's codes for the
// tile are 64 contiguous bytes of codes_col and its scales 32 contiguous bytes of scales_col,
// so every 32-byte sector of both outputs is written whole by one CTA.
#include <cuda_fp16.h>

#include "fp4q_device.cuh"
#include "fp4q_encode.cuh"
#include "fp4q_kernels.cuh"

namespace fp4q {
namespace {

constexpr int kTileM = 128, kTileN = 64;
constexpr int kPitch = kTileN + 8;   // elements; 144-byte rows

template <int G, int RR, int RC>
__global__ void __launch_bounds__(kThreads) dual_kernel(const DualArgs a) {
  __shared__ __align__(16) uint16_t tile[kTileM * kPitch];
  const int64_t m0 = (int64_t)blockIdx.y * kTileM;
  const int64_t n0 = (int64_t)blockIdx.x * kTileN;
  const int t = threadIdx.x;

  // stage: 1024 chunks of 16 bytes (8 per tile row), four per thread, zero outside the tensor
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = t + k * kThreads;
    const int r = c >> 3, cc = c & 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (m0 + r < a.M && n0 + 8 * cc < a.N)
      v = __ldcs(reinterpret_cast<const uint4*>(a.dy + (m0 + r) * a.ld + n0 + 8 * cc));
    *reinterpret_cast<uint4*>(&tile[r * kPitch + 8 * cc]) = v;
  }
  __syncthreads();

  // row blocks: rows t/4 and t/4 + 64, block t%4 (16 columns)
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int r = (t >> 2) + 64 * k, b = t & 3;
    const int64_t m = m0 + r, n = n0 + 16 * b;
    if (m >= a.M || n >= a.N) continue;
    const uint4* src = reinterpret_cast<const uint4*>(&tile[r * kPitch + 16 * b]);
    float2 P[8];
    unpack16(src[0], src[1], a.sw_row, P);
    if (a.c_row != 1.0f) fwht16(P);
    const float s = div_qmax<G>(__fmul_rn(absmax16(P), a.cinv_row));
    const int64_t u = (m * a.N + n) >> 4;   // 16-block index in [M, N/16]
    const uint2 w = (RR == kSR) ? encode_sr<G>(P, s, a.c_row, a.seedx_row, (uint64_t)u * 8u)
                                : encode_rtne_rt<G>(P, s, a.c_row != 1.0f);
    __stcs(reinterpret_cast<uint2*>(a.codes_row) + u, w);
    __stcs(a.scales_row + u, s);
  }

  // column blocks: column (w & 1) * 32 + lane, row groups (w >> 1) and (w >> 1) + 4
  const int w = t >> 5, lane = t & 31;
  const int c = (w & 1) * 32 + lane;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int g = (w >> 1) + 4 * k;
    const int64_t n = n0 + c, m = m0 + 16 * g;
    if (n >= a.N || m >= a.M) continue;
    uint32_t wd[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t lo = tile[(16 * g + 2 * j) * kPitch + c];
      const uint32_t hi = tile[(16 * g + 2 * j + 1) * kPitch + c];
      wd[j] = lo | (hi << 16);
    }
    float2 P[8];
    unpack16(make_uint4(wd[0], wd[1], wd[2], wd[3]), make_uint4(wd[4], wd[5], wd[6], wd[7]),
             a.sw_col, P);
    if (a.c_col != 1.0f) fwht16(P);
    const float s = div_qmax<G>(__fmul_rn(absmax16(P), a.cinv_col));
    const int64_t u = (n * a.M + m) >> 4;   // 16-block index in [N, M/16]
    const uint2 w = (RC == kSR) ? encode_sr<G>(P, s, a.c_col, a.seedx_col, (uint64_t)u * 8u)
                                : encode_rtne_rt<G>(P, s, a.c_col != 1.0f);
    __stcs(reinterpret_cast<uint2*>(a.codes_col) + u, w);
    __stcs(a.scales_col + u, s);
  }
}

template <int G, int RR, int RC>
cudaError_t launch_d(const DualArgs& a, cudaStream_t st) {
  const dim3 grid((unsigned)((a.N + kTileN - 1) / kTileN), (unsigned)((a.M + kTileM - 1) / kTileM));
  dual_kernel<G, RR, RC><<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
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

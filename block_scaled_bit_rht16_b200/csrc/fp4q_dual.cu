// fp4q_dual.cu -- dY quantized in both orientations from one read of HBM.
//
// bwd_dx reduces dY over N, so it needs dY blocked along rows; bwd_dw reduces over M, so it
// needs dY^T blocked along rows of dY^T (columns of dY). The UFP4 recipe applies the rotation
// and stochastic rounding to dY on both paths ("当你的 GPU 学不会算账", zhichai.net/topic/
// 178208020, recipe table of section "UFP4：换一把尺子"; "蚂蚁集团揭秘…", techwalker.com,
// section 三 on bwd_dx / bwd_dw).
//
// Persistent kernel over 128 x 64 tiles of dY (tile t: rows 128 (t / tiles_n), columns
// 64 (t % tiles_n)). Each CTA takes every gridDim.x-th tile, starting at tile blockIdx.x. The tiles reach shared memory through
// a ring of kStages buffers filled by 2-D bulk tensor copies (TMA, this GPU's memory only, no
// multicast) that complete on one mbarrier per buffer, so a CTA's next tiles are in flight
// while it encodes the current one; out-of-range rows and columns of edge tiles arrive as zeros.
// The copies use the 128-byte swizzle: 16-byte chunk j of tile row r sits at chunk j ^ (r % 8),
// which makes both the row reads (two 16-byte chunks of one row per block) and the column reads
// (one 32-bit word, two adjacent columns, per row) free of bank conflicts.
// Per tile and thread: two row blocks (16 consecutive elements of a row), encoded and stored to
// codes_row / scales_row directly, and two column blocks (16 consecutive rows of one column),
// staged in shared memory and stored as 16-byte pieces, each column's 64 bytes of codes and 32
// bytes of scales contiguous. One barrier per tile: after it every thread has finished reading
// the ring buffer (which is then refilled) and writing the staged column results.
// Every wait on a barrier is bounded; a wait that gives up sets bit 0 of the device status word,
// waits (bounded again) for the copies still in flight, and ends the CTA.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_encode.cuh"
#include "fp4q_kernels.cuh"

namespace fp4q {

namespace {

constexpr int kTileM = 128, kTileN = 64;
constexpr int kStages = 3;
constexpr uint32_t kTileBytes = kTileM * kTileN * 2;   // bf16
constexpr int kGroups = kTileM / 16;   // column blocks per column of a tile
constexpr int kCodePitch = 10;         // uint2 per staged column (8 used; 16-byte aligned rows)
constexpr int kScalePitch = 12;        // floats per staged column (8 used)

struct DualSmem {
  uint16_t tile[kStages][kTileM * kTileN];       // 1024-byte aligned (the swizzle's period)
  uint2 stage_codes[2][kTileN * kCodePitch];
  float stage_scales[2][kTileN * kScalePitch];
  uint64_t full[kStages];
};
constexpr size_t kDualSmemBytes = sizeof(DualSmem) + 1024;   // + alignment slack

__device__ __forceinline__ void tma_load_tile(void* dst, const CUtensorMap* map, int x, int y,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
        "r"(smem_u32(bar))
      : "memory");
}

// Byte offset of the 16-byte chunk j of tile row r under the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(int r, int j) { return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4)); }

template <int G, int RR, int RC, bool ROT>
__global__ void __launch_bounds__(kThreads, 3)
    dual_kernel(const __grid_constant__ CUtensorMap tmap, const DualArgs a) {
  extern __shared__ uint8_t smem_raw[];
  DualSmem& sm = *reinterpret_cast<DualSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int t = threadIdx.x, lane = t & 31, wp = t >> 5;
  const bool rot_row = ROT || a.c_row != 1.0f;
  const bool rot_col = ROT || a.c_col != 1.0f;
  const float c_row = ROT ? 4.0f : a.c_row, c_col = ROT ? 4.0f : a.c_col;
  const float cinv_row = ROT ? 0.25f : a.cinv_row, cinv_col = ROT ? 0.25f : a.cinv_col;
  const int64_t tiles_n = (a.N + kTileN - 1) / kTileN;
  const int64_t tiles = tiles_n * ((a.M + kTileM - 1) / kTileM);

  if (t == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&sm.full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  pdl_enter();

  // Tile t is (t / tiles_n, t % tiles_n); walking t by gridDim.x moves that pair by
  // (step_m, step_n) with one carry, so no division is left in the loop.
  const int64_t step_m = gridDim.x / tiles_n, step_n = gridDim.x % tiles_n;
  auto advance = [&](int64_t& tm, int64_t& tn) {
    tm += step_m;
    tn += step_n;
    if (tn >= tiles_n) {
      tn -= tiles_n;
      ++tm;
    }
  };
  const int64_t tm0 = blockIdx.x / tiles_n, tn0 = blockIdx.x % tiles_n;
  auto issue = [&](int64_t tm, int64_t tn, int s) {
    mbar_arrive_expect_tx(&sm.full[s], kTileBytes);
    tma_load_tile(sm.tile[s], &tmap, (int)(tn * kTileN), (int)(tm * kTileM), &sm.full[s]);
  };
  // the tile kStages ahead of the current one (the copy that refills its buffer)
  int64_t am = tm0, an = tn0;
  if (t == 0) {
    for (int s = 0; s < kStages; ++s) {
      if (am * tiles_n + an < tiles) issue(am, an, s);
      advance(am, an);
    }
  }

  int64_t it = 0, tm = tm0, tn = tn0;
  for (;; ++it, advance(tm, tn)) {
    const int64_t tile = tm * tiles_n + tn;
    if (tile >= tiles) break;
    const int s = (int)(it % kStages);
    const uint32_t parity = (uint32_t)((it / kStages) & 1);
    const int fail = mbar_wait(&sm.full[s], parity) ? 0 : 1;
    const int64_t m0 = tm * kTileM, n0 = tn * kTileN;
    const uint8_t* T = reinterpret_cast<const uint8_t*>(sm.tile[s]);

    // row blocks: rows 8 (2 wp + k) + lane % 8, block lane / 8 (columns 16 (lane / 8) ..)
    if constexpr (RR == kSR) {
      // both of the thread's row blocks at once (rows r and r + 8: the 16-row group 16 wp is in
      // range or out of range as a whole, M % 16 == 0)
      const int r = 16 * wp + (lane & 7), b = lane >> 3;
      const int64_t m = m0 + r, n = n0 + 16 * b;
      if (m < a.M && n < a.N) {
        float2 A[16];
        unpack16_pair(*reinterpret_cast<const uint4*>(T + swz(r, 2 * b)),
                      *reinterpret_cast<const uint4*>(T + swz(r, 2 * b + 1)),
                      *reinterpret_cast<const uint4*>(T + swz(r + 8, 2 * b)),
                      *reinterpret_cast<const uint4*>(T + swz(r + 8, 2 * b + 1)), a.flip_lo_row,
                      a.flip_hi_row, A);
        if (rot_row) fwht16_pair(A);
        const float2 am = absmax16_pair(A);
        const float2 sc = make_float2(div_qmax<G>(__fmul_rn(am.x, cinv_row)), div_qmax<G>(__fmul_rn(am.y, cinv_row)));
        const int64_t u0 = (m * a.N + n) >> 4, u1 = ((m + 8) * a.N + n) >> 4;
        uint2 w0, w1;
        encode_sr_pair<G>(A, sc, c_row, a.seedx_row, (uint64_t)u0 * 4u, (uint64_t)u1 * 4u, w0, w1);
        __stcs(reinterpret_cast<uint2*>(a.codes_row) + u0, w0);
        __stcs(a.scales_row + u0, sc.x);
        __stcs(reinterpret_cast<uint2*>(a.codes_row) + u1, w1);
        __stcs(a.scales_row + u1, sc.y);
      }
    } else {
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = 8 * (2 * wp + k) + (lane & 7), b = lane >> 3;
      const int64_t m = m0 + r, n = n0 + 16 * b;
      if (m >= a.M || n >= a.N) continue;
      const uint4 lo = *reinterpret_cast<const uint4*>(T + swz(r, 2 * b));
      const uint4 hi = *reinterpret_cast<const uint4*>(T + swz(r, 2 * b + 1));
      float2 P[8];
      unpack16(lo, hi, a.flip_lo_row, a.flip_hi_row, P);
      if (rot_row) fwht16(P);
      const float sc = div_qmax<G>(__fmul_rn(absmax16(P), cinv_row));
      const int64_t u = (m * a.N + n) >> 4;   // 16-block index in [M, N/16]
      uint2 w;
      if constexpr (RR == kSR) w = encode_sr<G>(P, sc, c_row, a.seedx_row, (uint64_t)u * 4u);
      else w = ROT ? encode_lean<G, true>(P, sc) : encode_rtne_rt<G>(P, sc, rot_row);
      __stcs(reinterpret_cast<uint2*>(a.codes_row) + u, w);
      __stcs(a.scales_row + u, sc);
    }
    }

    // column blocks: rows 16 wp .. 16 wp + 15, columns 2 lane + h (N % 16 == 0, M % 16 == 0: a
    // column pair and a group of 16 rows are in range or out of range as a whole)
    const int buf = (int)(it & 1);
    {
      const int64_t m = m0 + 16 * wp, nA = n0 + 2 * lane;
      if (m < a.M && nA < a.N) {
        uint32_t wd[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = 16 * wp + i;
          wd[i] = *reinterpret_cast<const uint32_t*>(T + swz(r, lane >> 2) + 4 * (lane & 3));
        }
        if constexpr (RC == kSR) {
          // both columns at once: A[i] = (column 2 lane, column 2 lane + 1) of row 16 wp + i
          float2 A[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            A[i] = make_float2(bf_lo_flip(wd[i], a.flip_col[i]), bf_hi_flip(wd[i], a.flip_col[i]));
          if (rot_col) fwht16_pair(A);
          const float2 am = absmax16_pair(A);
          const float2 sc = make_float2(div_qmax<G>(__fmul_rn(am.x, cinv_col)), div_qmax<G>(__fmul_rn(am.y, cinv_col)));
          const int64_t u0 = (nA * a.M + m) >> 4, u1 = ((nA + 1) * a.M + m) >> 4;
          uint2 w0, w1;
          encode_sr_pair<G>(A, sc, c_col, a.seedx_col, (uint64_t)u0 * 4u, (uint64_t)u1 * 4u, w0, w1);
          sm.stage_codes[buf][(2 * lane) * kCodePitch + wp] = w0;
          sm.stage_scales[buf][(2 * lane) * kScalePitch + wp] = sc.x;
          sm.stage_codes[buf][(2 * lane + 1) * kCodePitch + wp] = w1;
          sm.stage_scales[buf][(2 * lane + 1) * kScalePitch + wp] = sc.y;
        } else {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float2 P[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            P[i] = h ? make_float2(bf_hi_flip(wd[i], a.flip_col[i]), bf_hi_flip(wd[i + 8], a.flip_col[i + 8]))
                     : make_float2(bf_lo_flip(wd[i], a.flip_col[i]), bf_lo_flip(wd[i + 8], a.flip_col[i + 8]));
          if (rot_col) fwht16(P);
          const float sc = div_qmax<G>(__fmul_rn(absmax16(P), cinv_col));
          const int64_t u = ((nA + h) * a.M + m) >> 4;   // 16-block index in [N, M/16]
          uint2 w;
          if constexpr (RC == kSR) w = encode_sr<G>(P, sc, c_col, a.seedx_col, (uint64_t)u * 4u);
          else w = ROT ? encode_lean<G, true>(P, sc) : encode_rtne_rt<G>(P, sc, rot_col);
          const int c = 2 * lane + h;
          sm.stage_codes[buf][c * kCodePitch + wp] = w;
          sm.stage_scales[buf][c * kScalePitch + wp] = sc;
        }
        }
      }
    }
    // the tile's barrier; it also tells every thread whether any wait gave up
    if (__syncthreads_or(fail)) break;
    // every thread is done with ring buffer s: refill it with the tile kStages ahead
    if (t == 0) {
      if (am * tiles_n + an < tiles) issue(am, an, s);
      advance(am, an);
    }

    // column c's blocks for rows m0 .. m0+127 are kGroups consecutive entries of codes_col /
    // scales_col starting at block (n0 + c) * M/16 + m0/16
    const int64_t rows_left = (a.M - m0) >> 4, cols_left = a.N - n0;
    const int ng = rows_left < kGroups ? (int)rows_left : kGroups;
    const int nc = cols_left < kTileN ? (int)cols_left : kTileN;
    const uint2* sc_codes = sm.stage_codes[buf];
    const float* sc_scales = sm.stage_scales[buf];
    if (a.col16 && ng == kGroups) {
      // 16-byte stores: codes as 4 chunks of 2 blocks, scales as 2 chunks of 4 blocks per column
      {
        const int c = t >> 2, q = t & 3;
        if (c < nc) {
          const uint2 lo = sc_codes[c * kCodePitch + 2 * q], hi = sc_codes[c * kCodePitch + 2 * q + 1];
          uint2* dst = reinterpret_cast<uint2*>(a.codes_col) + (((n0 + c) * a.M + m0) >> 4) + 2 * q;
          __stcs(reinterpret_cast<uint4*>(dst), make_uint4(lo.x, lo.y, hi.x, hi.y));
        }
      }
      if (t < 2 * kTileN) {
        const int c = t >> 1, q = t & 1;
        if (c < nc) {
          const float4 v4 = *reinterpret_cast<const float4*>(&sc_scales[c * kScalePitch + 4 * q]);
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
          __stcs(reinterpret_cast<uint2*>(a.codes_col) + u, sc_codes[c * kCodePitch + gg]);
          __stcs(a.scales_col + u, sc_scales[c * kScalePitch + gg]);
        }
      }
    }
  }

  if (tm * tiles_n + tn < tiles && t == 0) {
    // a wait gave up: record it, then wait (bounded) for every copy this CTA still has in flight
    // so that none lands in shared memory after the CTA has ended
    atomicOr(a.status, kStatusWaitTimeout);
    for (int64_t j = it; j < it + kStages; ++j, advance(tm, tn)) {
      if (tm * tiles_n + tn >= tiles) break;
      mbar_wait(&sm.full[j % kStages], (uint32_t)((j / kStages) & 1));
    }
  }
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link-time
// dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map of dY (bf16 [M, ld], N columns used) with 64 x 128 boxes and the 128-byte swizzle.
cudaError_t make_dy_map(const DualArgs& a, CUtensorMap* map) {
  auto enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)a.N, (cuuint64_t)a.M};
  const cuuint64_t strides[1] = {(cuuint64_t)a.ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kTileN, (cuuint32_t)kTileM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.dy), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Persistent grid of a dual kernel: SM count x resident CTAs with its dynamic shared memory,
// queried once per (kernel, device) -- after raising the kernel's shared-memory limit on that
// device -- and cached, so that launches inside a stream capture do no queries.
template <class K>
cudaError_t dual_grid(K kernel, int64_t tiles, int* grid) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it == cache.end()) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDualSmemBytes);
    if (e != cudaSuccess) return e;
    int sms = 148, per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, kDualSmemBytes);
    if (e != cudaSuccess) return e;
    it = cache.emplace(key, sms * (per_sm > 0 ? per_sm : 1)).first;
  }
  *grid = (int)(tiles < it->second ? tiles : it->second);
  return cudaSuccess;
}

template <int G, int RR, int RC, bool ROT>
cudaError_t launch_d4(const DualArgs& a, const CUtensorMap& map, cudaStream_t st) {
  auto k = dual_kernel<G, RR, RC, ROT>;
  const int64_t tiles = ((a.N + kTileN - 1) / kTileN) * ((a.M + kTileM - 1) / kTileM);
  int grid = 1;
  const cudaError_t ge = dual_grid(k, tiles, &grid);
  if (ge != cudaSuccess) return ge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kDualSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, map, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int G, int RR, int RC>
cudaError_t launch_d(const DualArgs& a, const CUtensorMap& map, cudaStream_t st) {
  if (a.c_row != 1.0f && a.c_col != 1.0f) return launch_d4<G, RR, RC, true>(a, map, st);
  return launch_d4<G, RR, RC, false>(a, map, st);
}

template <int G>
cudaError_t launch_d_rounds(const DualArgs& a, const CUtensorMap& map, cudaStream_t st) {
  if (a.round_row == kSR)
    return a.round_col == kSR ? launch_d<G, kSR, kSR>(a, map, st) : launch_d<G, kSR, kRTNE>(a, map, st);
  return a.round_col == kSR ? launch_d<G, kRTNE, kSR>(a, map, st) : launch_d<G, kRTNE, kRTNE>(a, map, st);
}

}  // namespace

cudaError_t launch_dual(const DualArgs& a, cudaStream_t st) {
  if (a.M == 0 || a.N == 0) return cudaSuccess;
  if (a.grid_row != a.grid_col) return cudaErrorInvalidValue;
  alignas(64) CUtensorMap map;
  cudaError_t e = make_dy_map(a, &map);
  if (e != cudaSuccess) return e;
  DualArgs b = a;
  e = device_status_word(&b.status);
  if (e != cudaSuccess) return e;
  if (b.grid_row == kE2M1) return launch_d_rounds<kE2M1>(b, map, st);
  if (b.grid_row == kE1M2) return launch_d_rounds<kE1M2>(b, map, st);
  if (b.grid_row == kINT4) return launch_d_rounds<kINT4>(b, map, st);
  return cudaErrorInvalidValue;
}

}  // namespace fp4q

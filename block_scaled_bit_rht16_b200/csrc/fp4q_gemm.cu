// fp4q_gemm.cu -- NVFP4 and MXFP4 GEMMs on the 5th-generation tensor cores (tcgen05, sm_100a)
// consuming the quantizer's outputs unchanged: E2M1 codes (two per byte, element 2j in the low
// nibble) and block scales in the block-scaled MMA layout (FP4Q_OUT_SCALES_MMA): E4M3 per 16
// elements plus each operand's FP32 tensor scale (NVFP4), or UE8M0 per 32 elements (MXFP4).
// D[m, n] = alpha_A alpha_B sum_k A[m, k] B[n, k] (alpha = 1 for MXFP4), A and B both K-major
// (rows of the quantized tensors), accumulated in FP32 in tensor memory, stored as bf16.
//
// The NVFP4 recipe is the hardware path of "低精度量化技术：IF4自适应数据类型的原理与应用"
// (bxzpzcl.cn/news/2320061), section 3.2 (E4M3 block scale per 16 elements + FP32 tensor
// scale); MXFP4 is the 32-element power-of-two block of "AMD全新研究揭示：FP4训练不稳定性源于结构误差
// 而非随机性不足" (cannews.ca/article/21387); "FP4 训练 vs FP4 推理" (reports.10n1j.top) notes that
// Blackwell's FP4 tensor-core path is E2M1-only.
//
// A persistent kernel: one CTA per SM (up to 217 KB of shared memory, 256 or 512 tensor-memory
// columns) walks the 128 x BN tiles of D (BN = 256 when N allows, else 128), tile i of a CTA
// being blockIdx.x + i * gridDim.x with m fastest; when the last round's tiles fit the grid twice
// over, each of them is split into two 128 x 128 halves on two CTAs (GemmItem). The K dimension streams in 256-element steps
// through a ring of shared-memory buffers that runs on across tiles. Ten warps, four roles:
//   thread 0 (producer): per step the A and B code tiles (128 / BN rows x 128 bytes) and the
//     step's 512-byte MMA-layout scale tiles (per 128 rows: four for NVFP4, two for MXFP4) by
//     2-D TMA copies (codes with the 128-byte swizzle), all completing on the buffer's `full`
//     mbarrier; a buffer is refilled once its `empty` barrier says the MMAs that read it have
//     completed, so the next tile's operands load while the current tile drains;
//   warps 6-9 (scales): per step, warp w writes row l of each scale tile into tensor-memory
//     lane 32 (w % 4) + l of the stage's scale columns (tcgen05.st), so that the four warps
//     together fill the four lane quarters with the same 32 rows, the layout the block-scaled
//     MMA reads, and arrive on the buffer's `sf_full` barrier;
//   thread 32 (MMA issuer): per tile, once `acc_empty` says the epilogue has read the previous
//     accumulator, per step waits for `full` and `sf_full`, issues four MMAs of K = 64
//     (tcgen05.mma kind::mxf4nvf4, block16 with E4M3 or block32 with UE8M0 scales, M = 128,
//     N = BN) and commits them to the buffer's `empty` barrier; the tile's last commit goes to
//     `acc_full`;
//   warps 2-5 (epilogue): warp w reads tensor-memory lanes 32 (w % 4) .. +31 (tcgen05.ld, 32
//     columns at a time), scales by alpha_A alpha_B, stores bf16 rows, and arrives on `acc_empty`.
// Every mbarrier wait is bounded by the global timer; a wait that gives up sets bit 0 of the
// library's device status word and the CTA stops (its outputs are then incomplete), draining its
// copies in flight and releasing its tensor memory.
// No copy uses cluster multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

constexpr int kBM = 128, kBKBytes = 128;   // 256 FP4 values per row per step
constexpr int kGThreads = 320;   // warp 0 producer, warp 1 MMA issuer, warps 2-5 epilogue, 6-9 scales
constexpr uint32_t kTileA = kBM * kBKBytes;   // 16 KB
// Per tile width BN (128 or 256) and scale kind (MX: UE8M0 per 32 elements, else E4M3 per 16):
// stages, shared memory, tensor memory. A 512-byte MMA-layout scale tile covers 128 rows and
// 4 scale columns: K = 64 (NVFP4) or 128 (MXFP4), so a 256-deep step takes 4 or 2 of them per 128
// rows.
constexpr uint32_t kSfTile = 512;
template <int BN, bool MX>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr uint32_t kTileB = BN * kBKBytes;
  static constexpr int kSfTiles = MX ? 2 : 4;                     // per 128 rows per step
  static constexpr uint32_t kSfA = kSfTiles * kSfTile;
  static constexpr uint32_t kSfB = (BN / 128) * kSfA;
  static constexpr uint32_t kStageTx = kTileA + kTileB + kSfA + kSfB;
  static constexpr uint32_t kStageTxHalf = kTileA + kTileB / 2 + kSfA + kSfB / 2;   // a half tile (BN = 256)
  static constexpr uint32_t kSfCols = 4 * kSfTiles * (1 + BN / 128);   // A then B, 4 columns a tile
  static constexpr uint32_t kTmemCols = (BN + kStages * kSfCols) <= 256 ? 256 : 512;
  // kind::mxf4nvf4: E2M1 A and B (format 1), K-major, N / 8 in bits 17-22, scale type in bit 23
  // (0 UE4M3, 1 UE8M0), M / 16 in bits 24-28, K = 64; the scale-factor ids (which byte pair of a
  // 32-bit scale column a 32-element-block MMA reads: 0 or 2) in bits 4-5 (B) and 29-30 (A)
  static constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                     ((MX ? 1u : 0u) << 23) | ((uint32_t)(kBM >> 4) << 24);
  // the same with N = BN / 2 (a half tile)
  static constexpr uint32_t kIdescHalf = (kIdesc & ~(0x3Fu << 17)) | ((uint32_t)(BN >> 4) << 17);
};

template <int BN, bool MX>
struct GemmSmem {
  using C = GemmCfg<BN, MX>;
  uint8_t sfa[C::kStages][C::kSfA];   // first: every copy descriptor's reach stays inside the struct
  uint8_t sfb[C::kStages][C::kSfB];
  uint8_t a[C::kStages][kTileA];      // 1024-byte aligned (swizzle period)
  uint8_t b[C::kStages][C::kTileB];
  uint64_t full[C::kStages];
  uint64_t empty[C::kStages];
  uint64_t sf_full[C::kStages];   // the step's scales are in tensor memory (one arrival per scale warp)
  uint64_t acc_full;    // the MMAs of a tile have completed (tcgen05.commit)
  uint64_t acc_empty;   // the epilogue warps have read the accumulator (one arrival per warp)
  uint64_t done;        // every MMA and scale copy issued has completed
  uint32_t tmem_base;
};
template <int BN, bool MX>
constexpr size_t gemm_smem_bytes() { return sizeof(GemmSmem<BN, MX>) + 1024; }
// The code tiles start on the 128-byte swizzle's 1024-byte period (the scale buffers before them
// fill whole periods), shared memory fits one CTA (227 KB) and the accumulator plus every stage's
// scale columns fit the tensor memory allocated.
template <int BN, bool MX>
constexpr bool gemm_layout_ok() {
  using C = GemmCfg<BN, MX>;
  return (C::kStages * (C::kSfA + C::kSfB)) % 1024 == 0 && gemm_smem_bytes<BN, MX>() <= 232448 &&
         BN + C::kStages * C::kSfCols <= C::kTmemCols && C::kTmemCols <= 512;
}
static_assert(gemm_layout_ok<256, false>() && gemm_layout_ok<256, true>() && gemm_layout_ok<128, false>() &&
              gemm_layout_ok<128, true>(), "GEMM shared- or tensor-memory layout");

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits 0-13, leading byte
// offset >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45, version 1 in bits 46-47,
// layout type in bits 61-63 (0 none, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// N consecutive 32-bit tensor-memory columns of the warp's 32 lanes from r[0..N) (tcgen05.st
// 32x32b: thread l writes lane quarter base + l); the caller waits with tcgen05.wait::st.
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t* r);
template <>
__device__ __forceinline__ void tmem_st<8>(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<16>(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                 "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_st<32>(uint32_t taddr, const uint32_t* r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
               "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
               ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
                 "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
                 "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
                 "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
               : "memory");
}

// The 16 bytes of row `lane` of each of n 512-byte scale tiles (tile i at src + i * stride) into
// r[4 i .. 4 i + 3].
__device__ __forceinline__ void load_sf_rows(const uint8_t* src, uint32_t stride, int n, int lane, uint32_t* r) {
#pragma unroll
  for (int i = 0; i < n; ++i) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + i * stride + 16 * lane);
    r[4 * i] = v.x;
    r[4 * i + 1] = v.y;
    r[4 * i + 2] = v.z;
    r[4 * i + 3] = v.w;
  }
}

// Work item i of a launch over ntiles tiles on `grid` CTAs: tile i (m fastest), except that when
// BN = 256 and the last round's rem = ntiles % grid tiles fit the grid twice over, each of those
// tiles becomes two items of half its width (BN / 2 columns at n0 and n0 + BN / 2), so that the
// last round takes about half as long. Every role walks the same items.
struct GemmItem {
  int64_t m0, n0;
  int half;   // 1: a half tile
};
template <int BN>
__device__ __forceinline__ int gemm_split_tiles(int ntiles, int grid) {
  const int rem = ntiles % grid;
  return (BN == 256 && ntiles > grid && 2 * rem <= grid) ? rem : 0;
}
template <int BN>
__device__ __forceinline__ GemmItem gemm_item(int i, int tiles_m, int ntiles, int split) {
  GemmItem w;
  const int nfull = ntiles - split;
  const int tile = i < nfull ? i : nfull + ((i - nfull) >> 1);
  w.half = i < nfull ? 0 : 1;
  w.m0 = (int64_t)(tile % tiles_m) * kBM;
  w.n0 = (int64_t)(tile / tiles_m) * BN + (w.half ? (int64_t)((i - nfull) & 1) * (BN / 2) : 0);
  return w;
}

template <int BN, bool MX>
__global__ void __launch_bounds__(kGThreads, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmBh,
                      const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                      const float* __restrict__ ts_a, const float* __restrict__ ts_b,
                      __nv_bfloat16* __restrict__ out, int64_t ldo, int64_t M, int64_t N, int64_t K,
                      int32_t* status) {
  using C = GemmCfg<BN, MX>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem<BN, MX>& sm = *reinterpret_cast<GemmSmem<BN, MX>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int tiles_m = (int)(M / kBM);
  const int ntiles = tiles_m * (int)(N / BN);
  const int split = gemm_split_tiles<BN>(ntiles, (int)gridDim.x);
  const int nitems = ntiles + split;
  const int ksteps = (int)(K / 256);
  const int row_tiles = (int)(K / (MX ? 128 : 64));   // 512-byte scale tiles per 128-row tile row

  if (t == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      mbar_init(&sm.sf_full[s], 4);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 4);
    mbar_init(&sm.done, 1);
    fence_mbar_init();
  }
  if (warp == 1) {   // tensor memory for the accumulator and the staged scales
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_base)), "r"(C::kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  pdl_enter();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_acc = tmem;                 // lanes 0..127, columns 0..BN-1
  const uint32_t tmem_sf = tmem + BN;             // then S x (A: 16, B: BN/8) columns

  // Items are visited in the same order by every role: item i of this CTA is
  // blockIdx.x + i * gridDim.x (tiles m fastest: CTAs in flight share B tiles in L2).
  int fail = 0;
  int issued = 0;   // producer: steps whose copies have been issued
  if (t == 0) {
    // producer: refills a buffer once the MMAs that read it have completed
    for (int i = blockIdx.x; i < nitems && !fail; i += gridDim.x) {
      const GemmItem w = gemm_item<BN>(i, tiles_m, ntiles, split);
      const int groups = w.half ? BN / 256 : BN / 128;   // 128-row groups of B in the item
      for (int kt = 0; kt < ksteps; ++kt, ++issued) {
        const int s = issued % S;
        if (issued >= S && !mbar_wait(&sm.empty[s], (uint32_t)(((issued / S) - 1) & 1))) { fail = 1; break; }
        mbar_arrive_expect_tx(&sm.full[s], w.half ? C::kStageTxHalf : C::kStageTx);
        tma_load_2d(sm.a[s], &tmA, kt * kBKBytes, (int)w.m0, &sm.full[s]);
        tma_load_2d(sm.b[s], w.half ? &tmBh : &tmB, kt * kBKBytes, (int)w.n0, &sm.full[s]);
        // the step's kSfTiles scale tiles of A and of each 128-row group of B
        tma_load_2d(sm.sfa[s], &tmSA, 0, (int)(w.m0 / 128) * row_tiles + kt * C::kSfTiles, &sm.full[s]);
        for (int j = 0; j < groups; ++j)
          tma_load_2d(sm.sfb[s] + j * C::kSfA, &tmSB, 0, (int)(w.n0 / 128 + j) * row_tiles + kt * C::kSfTiles,
                      &sm.full[s]);
      }
    }
  } else if (t == 32) {
    // MMA issuer: per tile, once the epilogue has read the previous accumulator, scales into
    // tensor memory and four MMAs of K = 64 per step; the tile's last commit goes to acc_full
    int it = 0;
    int j = 0;
    for (int i = blockIdx.x; i < nitems && !fail; i += gridDim.x, ++j) {
      const bool half = i >= ntiles - split;
      // a half tile: N = BN / 2, B's scales in the one-group layout (tile t at sb + 4t)
      const uint32_t idesc_base = half ? C::kIdescHalf : C::kIdesc;
      const uint32_t sfb_stride = half ? 4u : 4u * (uint32_t)(BN / 128);
      if (j > 0 && !mbar_wait(&sm.acc_empty, (uint32_t)((j - 1) & 1))) { fail = 1; break; }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      for (int kt = 0; kt < ksteps; ++kt, ++it) {
        const int s = it % S;
        if (!mbar_wait(&sm.full[s], (uint32_t)((it / S) & 1))) { fail = 1; break; }
        if (!mbar_wait(&sm.sf_full[s], (uint32_t)((it / S) & 1))) { fail = 1; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        // scale tile t of A at columns sa + 4t; tile t of B's 128-row group j at sb + 4 (BN/128) t + 4j
        const uint32_t sa = tmem_sf + (uint32_t)s * C::kSfCols, sb = sa + 4u * C::kSfTiles;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; K-block kb starts 32 bytes in
          const uint64_t adesc = smem_desc(smem_u32(sm.a[s]) + 32u * kb, 16u, 1024u, 2u);
          const uint64_t bdesc = smem_desc(smem_u32(sm.b[s]) + 32u * kb, 16u, 1024u, 2u);
          const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
          // NVFP4: tile kb, all four bytes of each scale column; MXFP4: tile kb / 2, bytes
          // 2 (kb % 2) and 2 (kb % 2) + 1 (the scale-factor ids)
          const int tt = MX ? kb >> 1 : kb;
          const uint32_t id = MX ? 2u * (uint32_t)(kb & 1) : 0u;
          const uint32_t idesc = idesc_base | (id << 4) | (id << 29);
          const uint32_t sfa_col = sa + 4u * tt, sfb_col = sb + sfb_stride * tt;
          if constexpr (MX)
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                ::"r"(tmem_acc), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa_col), "r"(sfb_col)
                : "memory");
          else
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
                ::"r"(tmem_acc), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc), "r"(sfa_col), "r"(sfb_col)
                : "memory");
        }
        umma_commit(&sm.empty[s]);   // the buffer is free again once these MMAs have read it
      }
      if (fail) break;
      umma_commit(&sm.acc_full);     // the tile's accumulator is complete once these have run
    }
    // arrives when every MMA and scale copy issued above has completed
    umma_commit(&sm.done);
  } else if (warp >= 6) {
    // scale warps: warp w writes tensor-memory lanes 32 (w % 4) .. +31. Per step, once the
    // buffer's copies have landed (and so the MMAs that last read the stage's scale columns have
    // completed: the buffer was refilled only after them), row l of each of the step's 512-byte
    // scale tiles goes to lane l of the tile's four columns; the four warps together fill all four
    // lane quarters with the same rows, the layout the MMAs read.
    const uint32_t quarter_base = (uint32_t)(32 * (warp & 3)) << 16;
    int it = 0;
    for (int i = blockIdx.x; i < nitems && !fail; i += gridDim.x) {
      const bool half = i >= ntiles - split;
      for (int kt = 0; kt < ksteps; ++kt, ++it) {
        const int s = it % S;
        // warp-uniform: every lane takes the same branch before the collective stores
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.full[s], (uint32_t)((it / S) & 1)))) { fail = 1; break; }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t sa = tmem_sf + quarter_base + (uint32_t)s * C::kSfCols, sb = sa + 4u * C::kSfTiles;
        {
          uint32_t r[4 * C::kSfTiles];   // A: tile t at columns sa + 4t
          load_sf_rows(sm.sfa[s], kSfTile, C::kSfTiles, lane, r);
          tmem_st<4 * C::kSfTiles>(sa, r);
        }
        if (BN == 256 && half) {
          // a half tile's one 128-row group of B: tile t at columns sb + 4t
          uint32_t r[4 * C::kSfTiles];
          load_sf_rows(sm.sfb[s], kSfTile, C::kSfTiles, lane, r);
          tmem_st<4 * C::kSfTiles>(sb, r);
        } else {
          // B: tile t of 128-row group j at columns sb + 4 (BN / 128) t + 4 j
          constexpr int kG = BN / 128;
          uint32_t r[4 * C::kSfTiles * kG];
#pragma unroll
          for (int j = 0; j < kG; ++j) {
            uint32_t g[4 * C::kSfTiles];
            load_sf_rows(sm.sfb[s] + j * C::kSfA, kSfTile, C::kSfTiles, lane, g);
#pragma unroll
            for (int tt = 0; tt < C::kSfTiles; ++tt)
#pragma unroll
              for (int q = 0; q < 4; ++q) r[4 * (kG * tt + j) + q] = g[4 * tt + q];
          }
          tmem_st<4 * C::kSfTiles * kG>(sb, r);
        }
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.sf_full[s]);
      }
    }
  } else if (warp >= 2) {
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. +31 (rows of the tile) 32 columns
    // at a time, stores them as bf16 x alpha, and releases the accumulator to the next tile's
    // MMAs (the producer has kept loading the next tile's operands meanwhile)
    const float alpha = MX ? 1.0f : __fmul_rn(*ts_a, *ts_b);   // MXFP4 has no tensor scale
    const int quarter = warp & 3;
    int j = 0;
    for (int i = blockIdx.x; i < nitems; i += gridDim.x, ++j) {
      const GemmItem w = gemm_item<BN>(i, tiles_m, ntiles, split);
      const int64_t m0 = w.m0, n0 = w.n0;
      const int cols = w.half ? BN / 2 : BN;
      // warp-uniform: every lane takes the same branch before the collective loads
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sm.acc_full, (uint32_t)(j & 1)))) { fail = 1; break; }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      uint4* dst = reinterpret_cast<uint4*>(out + (m0 + 32 * quarter + lane) * ldo + n0);
#pragma unroll 1
      for (int c0 = 0; c0 < cols; c0 += 32) {
        uint32_t v[32];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
            "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
              "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
              "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
            : "r"(tmem_acc + ((uint32_t)(32 * quarter) << 16) + (uint32_t)c0));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t o[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            o[i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * q + 2 * i]), alpha),
                               __fmul_rn(__uint_as_float(v[8 * q + 2 * i + 1]), alpha));
          dst[c0 / 8 + q] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      // the stores need nothing more from tensor memory: release the accumulator
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
    }
  }
  // a failed wait of any role reaches every thread through the barrier
  fail = __syncthreads_or(fail);
  if (fail && t == 0) {
    // drain: wait (bounded) for the last fill issued into each buffer, steps issued - S ..
    // issued - 1 (a fill the MMA issuer has consumed has completed, and its wait returns at once)
    for (int i = issued > S ? issued - S : 0; i < issued; ++i) mbar_wait(&sm.full[i % S], (uint32_t)((i / S) & 1));
  }
  if (!mbar_wait(&sm.done, 0u)) fail = 1;   // the MMA issuer commits `done` on every path
  fail = __syncthreads_or(fail);
  if (fail && t == 0) atomicOr(status, kStatusWaitTimeout);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (warp == 1)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols) : "memory");
}

PFN_cuTensorMapEncodeTiled_v12000 gemm_tensor_map_encoder() {
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

// 2-D map of a code matrix (uint8 [rows, K/2]) with 128-byte x box_rows boxes, 128-byte swizzle.
cudaError_t make_codes_map(const uint8_t* codes, int64_t rows, int64_t K, int box_rows, CUtensorMap* map) {
  auto enc = gemm_tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kBKBytes, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 2-D map of MMA-layout scales (uint8 [rows / 128 * row_tiles] tiles of 512 bytes) as 32-bit words:
// 128 words of a tile, the tiles; a box of `tiles` consecutive tiles lands contiguously.
cudaError_t make_scales_map(const uint8_t* scales, int64_t total_tiles, int tiles, CUtensorMap* map) {
  auto enc = gemm_tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {128, (cuuint64_t)total_tiles};
  const cuuint64_t strides[1] = {512};
  const cuuint32_t box[2] = {128, (cuuint32_t)tiles};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(scales), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Raises the kernel's shared-memory limit once per (kernel, device).
template <int BN, bool MX>
cudaError_t gemm_prepare() {
  static std::mutex mu;
  static std::map<int, cudaError_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find(dev);
  if (it == done.end())
    it = done.emplace(dev, cudaFuncSetAttribute(fp4_gemm_kernel<BN, MX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)gemm_smem_bytes<BN, MX>())).first;
  return it->second;
}

template <int BN, bool MX>
cudaError_t launch_gemm_bn(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts,
                           const uint8_t* b_codes, const uint8_t* b_scales, const float* b_ts,
                           int64_t M, int64_t N, int64_t K, uint16_t* out, int64_t ldo, cudaStream_t st) {
  using C = GemmCfg<BN, MX>;
  alignas(64) CUtensorMap ma, mb, mbh, msa, msb;
  cudaError_t e = make_codes_map(a_codes, M, K, kBM, &ma);
  if (e != cudaSuccess) return e;
  e = make_codes_map(b_codes, N, K, BN, &mb);
  if (e != cudaSuccess) return e;
  e = make_codes_map(b_codes, N, K, BN / 2, &mbh);   // half tiles' B (used only when BN = 256)
  if (e != cudaSuccess) return e;
  const int64_t row_tiles = K / (MX ? 128 : 64);
  e = make_scales_map(a_scales, M / 128 * row_tiles, C::kSfTiles, &msa);
  if (e != cudaSuccess) return e;
  e = make_scales_map(b_scales, N / 128 * row_tiles, C::kSfTiles, &msb);
  if (e != cudaSuccess) return e;
  e = gemm_prepare<BN, MX>();
  if (e != cudaSuccess) return e;
  int32_t* status = nullptr;
  e = device_status_word(&status);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t tiles = (M / kBM) * (N / BN);
  cfg.gridDim = dim3((unsigned)std::min<int64_t>(tiles, sms));   // one persistent CTA per SM
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = gemm_smem_bytes<BN, MX>();
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, fp4_gemm_kernel<BN, MX>, ma, mb, mbh, msa, msb, a_ts, b_ts,
                         reinterpret_cast<__nv_bfloat16*>(out), ldo, M, N, K, status);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts,
                              const uint8_t* b_codes, const uint8_t* b_scales, const float* b_ts,
                              int64_t M, int64_t N, int64_t K, uint16_t* out, int64_t ldo,
                              cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (N % 256 == 0)
    return launch_gemm_bn<256, false>(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, M, N, K, out, ldo, st);
  return launch_gemm_bn<128, false>(a_codes, a_scales, a_ts, b_codes, b_scales, b_ts, M, N, K, out, ldo, st);
}

cudaError_t launch_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                              const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, uint16_t* out,
                              int64_t ldo, cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (N % 256 == 0)
    return launch_gemm_bn<256, true>(a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, M, N, K, out, ldo, st);
  return launch_gemm_bn<128, true>(a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, M, N, K, out, ldo, st);
}

}  // namespace fp4q

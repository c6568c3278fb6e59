// fp4q_gemm.cu -- NVFP4 GEMM on the 5th-generation tensor cores (tcgen05, sm_100a) consuming the
// quantizer's outputs unchanged: E2M1 codes (two per byte, element 2j in the low nibble) and
// E4M3 block scales in the block-scaled MMA layout (FP4Q_OUT_SCALES_MMA), plus each operand's
// FP32 tensor scale. D[m, n] = alpha_A alpha_B sum_k A[m, k] B[n, k], A and B both K-major
// (rows of the quantized tensors), accumulated in FP32 in tensor memory, stored as bf16.
//
// The NVFP4 recipe is the hardware path of "低精度量化技术：IF4自适应数据类型的原理与应用"
// (bxzpzcl.cn/news/2320061), section 3.2 (E4M3 block scale per 16 elements + FP32 tensor
// scale); "FP4 训练 vs FP4 推理" (reports.10n1j.top) notes that Blackwell's FP4 tensor-core path
// is E2M1-only.
//
// One CTA computes a 128 x 128 tile of D with 128 threads. Thread 0 streams the K dimension in
// 256-element steps through a ring of kStages shared-memory buffers: per step the A and B code
// tiles (128 rows x 128 bytes each) arrive by 2-D TMA copies with the 128-byte swizzle, and the
// two 2 KB scale blocks (four 512-byte MMA-layout tiles each) by 1-D bulk copies, all completing
// on the buffer's mbarrier. It then copies the scales into tensor memory (tcgen05.cp, 32 lanes x
// 128 bits, replicated to the four lane quarters) and issues four MMAs of K = 64
// (tcgen05.mma kind::mxf4nvf4, block16 scaling, M = 128, N = 128), and tcgen05.commit arrives
// on the buffer's release barrier when they have read it. The accumulator is 128 lanes x 128
// FP32 columns of tensor memory; after the last step every warp reads its 32 lanes back
// (tcgen05.ld), scales by alpha_A alpha_B and stores bf16. Every mbarrier wait is bounded by the
// global timer; a wait that gives up sets bit 0 of the library's device status word and the CTA
// skips the rest of its work (its outputs are then incomplete), releasing its tensor memory.
// No copy uses cluster multicast.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <map>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"

namespace fp4q {
namespace {

constexpr int kBM = 128, kBN = 128, kBKBytes = 128;   // 256 FP4 values per row per step
constexpr int kGStages = 4;
constexpr int kGThreads = 128;
constexpr uint32_t kTileA = kBM * kBKBytes, kTileB = kBN * kBKBytes;   // 16 KB each
constexpr uint32_t kSfBytes = 4 * 512;                                 // 4 K-blocks of 64
constexpr uint32_t kStageTx = kTileA + kTileB + 2 * kSfBytes;
constexpr uint32_t kTmemCols = 256;   // 128 accumulator + kGStages x 2 x 16 scale columns

struct GemmSmem {
  uint8_t a[kGStages][kTileA];      // 1024-byte aligned (swizzle period)
  uint8_t b[kGStages][kTileB];
  uint8_t sfa[kGStages][kSfBytes];
  uint8_t sfb[kGStages][kSfBytes];
  uint64_t full[kGStages];
  uint64_t empty[kGStages];
  uint64_t done;
  uint32_t tmem_base;
};
constexpr size_t kGemmSmemBytes = sizeof(GemmSmem) + 1024;

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address >> 4 in bits 0-13, leading byte
// offset >> 4 in bits 16-29, stride byte offset >> 4 in bits 32-45, version 1 in bits 46-47,
// layout type in bits 61-63 (0 none, 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of kind::mxf4nvf4 with E2M1 A and B (format 1), K-major A and B, N / 8
// in bits 17-22, UE4M3 scales (bit 23 = 0), M / 16 in bits 24-28, scale-factor ids 0, K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

__global__ void __launch_bounds__(kGThreads, 1)
    nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb,
                      const float* __restrict__ ts_a, const float* __restrict__ ts_b,
                      __nv_bfloat16* __restrict__ out, int64_t ldo, int64_t K, int32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int64_t m0 = (int64_t)blockIdx.y * kBM, n0 = (int64_t)blockIdx.x * kBN;
  const int ksteps = (int)(K / 256);
  const int64_t kb64 = K / 64;   // scale tiles (of 4 K-blocks of 16) per 128-row tile row

  if (t == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.done, 1);
    fence_mbar_init();
  }
  if (warp == 0) {   // tensor memory for the accumulator and the staged scales
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&sm.tmem_base)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  pdl_enter();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t tmem_acc = tmem;                 // lanes 0..127, columns 0..127
  const uint32_t tmem_sf = tmem + kBN;            // then kGStages x (A: 16, B: 16) columns

  int fail = 0;
  if (t == 0) {
    const uint8_t* sfa_row = sfa + (m0 / 128) * kb64 * 512;
    const uint8_t* sfb_row = sfb + (n0 / 128) * kb64 * 512;
    auto issue = [&](int kt, int s) {
      mbar_arrive_expect_tx(&sm.full[s], kStageTx);
      tma_load_2d(sm.a[s], &tmA, kt * kBKBytes, (int)m0, &sm.full[s]);
      tma_load_2d(sm.b[s], &tmB, kt * kBKBytes, (int)n0, &sm.full[s]);
      bulk_load_1d(sm.sfa[s], sfa_row + (int64_t)kt * kSfBytes, kSfBytes, &sm.full[s]);
      bulk_load_1d(sm.sfb[s], sfb_row + (int64_t)kt * kSfBytes, kSfBytes, &sm.full[s]);
    };
    int issued = 0;   // steps whose copies have been issued
    for (; issued < kGStages && issued < ksteps; ++issued) issue(issued, issued);
    int kt = 0;
    for (; kt < ksteps; ++kt) {
      const int s = kt % kGStages;
      const uint32_t ph = (uint32_t)((kt / kGStages) & 1);
      if (!mbar_wait(&sm.full[s], ph)) { fail = 1; break; }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t sa = tmem_sf + (uint32_t)s * 32u, sb = sa + 16u;
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        // 512 bytes = 32 rows of 16 bytes, 8-row groups 128 bytes apart
        const uint64_t da = smem_desc(smem_u32(sm.sfa[s] + kb * 512), 16u, 128u, 0u);
        const uint64_t db = smem_desc(smem_u32(sm.sfb[s] + kb * 512), 16u, 128u, 0u);
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sa + 4u * kb), "l"(da) : "memory");
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(sb + 4u * kb), "l"(db) : "memory");
      }
#pragma unroll
      for (int kb = 0; kb < 4; ++kb) {
        // K-major, 128-byte swizzle: 8-row groups 1024 bytes apart; K-block kb starts 32 bytes in
        const uint64_t adesc = smem_desc(smem_u32(sm.a[s]) + 32u * kb, 16u, 1024u, 2u);
        const uint64_t bdesc = smem_desc(smem_u32(sm.b[s]) + 32u * kb, 16u, 1024u, 2u);
        const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
            ::"r"(tmem_acc), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(acc), "r"(sa + 4u * kb), "r"(sb + 4u * kb)
            : "memory");
      }
      // the buffer is free again once these MMAs have read it
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                   ::"r"(smem_u32(&sm.empty[s])) : "memory");
      if (issued < ksteps) {
        if (!mbar_wait(&sm.empty[s], ph)) { fail = 1; break; }
        issue(issued, s);
        ++issued;
      }
    }
    if (fail) {
      // drain: the copies still in flight (steps kt + 1 .. issued - 1, and kt's own if its wait
      // gave up), each wait bounded again
      for (int j = kt; j < issued; ++j) mbar_wait(&sm.full[j % kGStages], (uint32_t)((j / kGStages) & 1));
    }
    // arrives when every MMA and scale copy issued above has completed
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(&sm.done)) : "memory");
  }
  // the other threads wait at the barrier (not spinning beside thread 0) until every step is
  // issued; then all wait for the last MMAs (bounded), and a failed wait anywhere reaches every
  // thread through the second barrier (then nothing reads tensor memory)
  fail = __syncthreads_or(fail);
  if (!mbar_wait(&sm.done, 0u)) fail = 1;   // thread 0 commits `done` on every path
  fail = __syncthreads_or(fail);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (fail) {
    if (t == 0) atomicOr(status, kStatusWaitTimeout);
  } else {
    const float alpha = __fmul_rn(*ts_a, *ts_b);
    const int64_t row = m0 + 32 * warp + lane;
#pragma unroll
    for (int c0 = 0; c0 < kBN; c0 += 32) {
      uint32_t v[32];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
          "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
            "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
            "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
          : "r"(tmem_acc + ((uint32_t)(32 * warp) << 16) + (uint32_t)c0));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      uint4* dst = reinterpret_cast<uint4*>(out + row * ldo + n0 + c0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 o;
        o.x = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * q + 0]), alpha), __fmul_rn(__uint_as_float(v[8 * q + 1]), alpha));
        o.y = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * q + 2]), alpha), __fmul_rn(__uint_as_float(v[8 * q + 3]), alpha));
        o.z = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * q + 4]), alpha), __fmul_rn(__uint_as_float(v[8 * q + 5]), alpha));
        o.w = pack_bf16x2(__fmul_rn(__uint_as_float(v[8 * q + 6]), alpha), __fmul_rn(__uint_as_float(v[8 * q + 7]), alpha));
        dst[q] = o;
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
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

// 2-D map of a code matrix (uint8 [rows, K/2]) with 128-byte x 128-row boxes, 128-byte swizzle.
cudaError_t make_codes_map(const uint8_t* codes, int64_t rows, int64_t K, CUtensorMap* map) {
  auto enc = gemm_tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  const cuuint32_t box[2] = {(cuuint32_t)kBKBytes, (cuuint32_t)kBM};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                         box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t gemm_prepare(int* ok) {
  static std::mutex mu;
  static std::map<int, cudaError_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find(dev);
  if (it == done.end())
    it = done.emplace(dev, cudaFuncSetAttribute(nvfp4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)kGemmSmemBytes)).first;
  *ok = it->second == cudaSuccess;
  return it->second;
}

}  // namespace

cudaError_t launch_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts,
                              const uint8_t* b_codes, const uint8_t* b_scales, const float* b_ts,
                              int64_t M, int64_t N, int64_t K, uint16_t* out, int64_t ldo,
                              cudaStream_t st) {
  if (M == 0 || N == 0) return cudaSuccess;
  alignas(64) CUtensorMap ma, mb;
  cudaError_t e = make_codes_map(a_codes, M, K, &ma);
  if (e != cudaSuccess) return e;
  e = make_codes_map(b_codes, N, K, &mb);
  if (e != cudaSuccess) return e;
  int ok = 0;
  e = gemm_prepare(&ok);
  if (e != cudaSuccess) return e;
  int32_t* status = nullptr;
  e = device_status_word(&status);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(N / kBN), (unsigned)(M / kBM));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGemmSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, nvfp4_gemm_kernel, ma, mb, a_scales, b_scales, a_ts, b_ts,
                         reinterpret_cast<__nv_bfloat16*>(out), ldo, K, status);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fp4q

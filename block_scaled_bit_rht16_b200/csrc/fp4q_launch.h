// fp4q_launch.h -- host-side launchers of the library's kernels (each defined with its kernels
// in the .cu file that holds them; the C ABI in fp4q_api.cu calls them). Kept apart from the
// device-side argument structs so that a launcher added or changed touches no kernel's sources.
#pragma once
#include "fp4q_kernels.cuh"

namespace fp4q {

// Host-side launchers (fp4q_row.cu / fp4q_dual.cu). Return the CUDA error of the launch.
cudaError_t launch_quantize(int grid, int scale, int round, bool stats, const QuantArgs& a,
                            cudaStream_t st);
cudaError_t launch_amax(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_grouped_amax(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_grouped_alpha(const QuantArgs& a, float qmax, cudaStream_t st);
cudaError_t launch_quantize_grouped(int grid, const QuantArgs& a, cudaStream_t st);
cudaError_t launch_alpha(WsHeader* ws, float qmax, float* tensor_scale, cudaStream_t st);
cudaError_t launch_rht16(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                         const uint32_t* sw, void* out, bool out_fp32, cudaStream_t st);
cudaError_t launch_dequant(int grid, int scale, const uint8_t* codes, const void* scales,
                           const float* ts, int64_t rows, int64_t cols, const uint32_t* sw,
                           bool inverse, bool mma_scales, uint16_t* out, cudaStream_t st);
cudaError_t launch_stats_reduce(WsHeader* ws, const double* partials, cudaStream_t st);
cudaError_t launch_dual(const DualArgs& a, cudaStream_t st);
cudaError_t launch_division_check(uint64_t seed, uint64_t n, unsigned long long* bad,
                                  cudaStream_t st);
cudaError_t launch_wait_timeout_check(unsigned long long limit_ns, cudaStream_t st);
cudaError_t launch_conversion_check(unsigned long long* bad, cudaStream_t st);
cudaError_t read_device_status(int32_t* out, bool clear, cudaStream_t st);
cudaError_t device_status_word(int32_t** out);
cudaError_t launch_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_ts,
                              const uint8_t* b_codes, const uint8_t* b_scales, const float* b_ts,
                              int64_t M, int64_t N, int64_t K, uint16_t* out, int64_t ldo,
                              cudaStream_t st);
cudaError_t launch_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                              const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, uint16_t* out,
                              int64_t ldo, cudaStream_t st);

cudaError_t launch_ws_clear(void* p, size_t bytes, cudaStream_t st);   // fp4q_workspace.cu; bytes % 16 == 0

}  // namespace fp4q

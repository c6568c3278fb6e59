// fp4q_workspace.cu -- clearing workspace before a call that accumulates into it (the header's
// rotated-tensor amax for a computed E4M3 tensor scale and its statistics record counts; the
// grouped call's per-group amax slots).
//
// A kernel rather than a memset: launched with programmatic stream serialization like
// the quantize kernels, it keeps a chain of back-to-back calls (quantize, clear, amax, quantize,
// ...) free of the copy-engine node a memset would put between them. It waits for the preceding
// kernel on the stream (which may still be reading the header) before it clears it.
#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

// Zeroes n16 16-byte words at p, grid-stride.
__global__ void __launch_bounds__(kThreads) ws_clear_kernel(uint4* p, size_t n16) {
  pdl_enter();
  const size_t stride = (size_t)gridDim.x * kThreads;
  for (size_t i = (size_t)blockIdx.x * kThreads + threadIdx.x; i < n16; i += stride) p[i] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

cudaError_t launch_ws_clear(void* p, size_t bytes, cudaStream_t st) {
  if (bytes == 0) return cudaSuccess;
  if (bytes % 16 != 0 || reinterpret_cast<uintptr_t>(p) % 16 != 0) return cudaErrorInvalidValue;
  const size_t n16 = bytes / 16;
  const size_t blocks = (n16 + kThreads - 1) / kThreads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(blocks < 592 ? blocks : 592));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, ws_clear_kernel, reinterpret_cast<uint4*>(p), n16);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fp4q

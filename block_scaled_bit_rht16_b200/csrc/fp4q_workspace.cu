// fp4q_workspace.cu -- clearing the workspace header before a call that accumulates into it (the
// rotated tensor's amax for a computed E4M3 tensor scale, the statistics record counts).
//
// A one-CTA kernel rather than a memset: launched with programmatic stream serialization like
// the quantize kernels, it keeps a chain of back-to-back calls (quantize, clear, amax, quantize,
// ...) free of the copy-engine node a memset would put between them. It waits for the preceding
// kernel on the stream (which may still be reading the header) before it clears it.
#include "fp4q_device.cuh"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace fp4q {
namespace {

__global__ void __launch_bounds__(kThreads) ws_reset_kernel(WsHeader* ws) {
  pdl_enter();
  constexpr int kWords = (int)(sizeof(WsHeader) / sizeof(uint32_t));
  static_assert(kWords <= kThreads, "one word per thread");
  if (threadIdx.x < kWords) reinterpret_cast<uint32_t*>(ws)[threadIdx.x] = 0u;
}

}  // namespace

cudaError_t launch_ws_reset(WsHeader* ws, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, ws_reset_kernel, ws);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fp4q

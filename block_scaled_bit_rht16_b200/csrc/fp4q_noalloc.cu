// fp4q_noalloc.cu -- the quantizer for callers that cannot allocate device memory.
//
// fp4q_rht_quantize takes its scratch memory (a 256-byte header holding the rotated tensor's
// amax while it computes an E4M3 tensor scale) from the caller. Some callers cannot provide it:
// a plugin boundary of an inference or training runtime that hands a library only its input and
// output buffers, code whose device memory is budgeted and owned entirely by a host framework,
// or work enqueued where cudaMalloc is off limits (it may synchronize the device, and it cannot
// be captured into a CUDA graph). For them this file keeps that scratch in a fixed array in
// device memory that the library itself carries, and calls the same kernels with it.
#include <map>
#include <mutex>

#include "../../include/fp4q.h"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

namespace {

// The built-in scratch: one workspace header. Every GPU that loads the library holds these
// 256 bytes until the process exits.
constexpr size_t kNoAllocScratchBytes = 256;
static_assert(sizeof(fp4q::WsHeader) <= kNoAllocScratchBytes, "header fits the static scratch");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch on the current device. In host code the array's name is only a
// host-side stand-in, so the address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, and cached.
fp4q_status scratch_address(void** out) {
  static std::mutex mu;
  static std::map<int, void*> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FP4Q_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FP4Q_ERR_CUDA;
    it = cache.emplace(dev, p).first;
  }
  *out = it->second;
  return FP4Q_OK;
}

}  // namespace

extern "C" fp4q_status fp4q_rht_quantize_noalloc(const fp4q_config* cfg, const void* x,
                                                 int64_t rows, int64_t cols, int64_t ld,
                                                 uint8_t* codes, void* scales, float* tensor_scale,
                                                 int32_t tensor_scale_given, void* dequant,
                                                 fp4q_stream_t stream) {
  if (cfg == nullptr) return FP4Q_ERR_INVALID_ARG;
  // Only configurations whose scratch fits the built-in array are accepted: everything except
  // statistics, whose per-CTA records need fp4q_workspace_size() bytes from the caller.
  const size_t need = fp4q_workspace_size(cfg, rows, cols);
  if (need > kNoAllocScratchBytes) return FP4Q_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const fp4q_status st = scratch_address(&scratch);
    if (st != FP4Q_OK) return st;
  }
  // fp4q_rht_quantize zeroes the header on the stream before its kernels read it.
  return fp4q_rht_quantize(cfg, x, rows, cols, ld, codes, scales, tensor_scale, tensor_scale_given,
                           dequant, scratch, need > 0 ? kNoAllocScratchBytes : 0, stream);
}

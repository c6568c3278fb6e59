// fp4q_api.cu -- the C ABI declared in include/fp4q.h: host-side validation, workspace layout
// and kernel dispatch. Every argument is checked before anything is enqueued; a rejected call
// launches nothing.
#include <climits>
#include <cmath>
#include <cstring>

#include "../../include/fp4q.h"
#include "fp4q_kernels.cuh"
#include "fp4q_launch.h"

using namespace fp4q;

namespace {

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

uint64_t host_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Per bf16 pair k: bit 15 flips element 2k, bit 31 flips element 2k+1.
void sign_words(uint32_t mask, bool rht, uint32_t* sw) {
  for (int k = 0; k < 8; ++k) {
    sw[k] = 0u;
    if (!rht) continue;
    if ((mask >> (2 * k)) & 1u) sw[k] |= 0x00008000u;
    if ((mask >> (2 * k + 1)) & 1u) sw[k] |= 0x80000000u;
  }
}

fp4q_status check_cfg(const fp4q_config* cfg) {
  if (cfg == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (cfg->grid < FP4Q_GRID_E2M1 || cfg->grid > FP4Q_GRID_IF4) return FP4Q_ERR_INVALID_ARG;
  if (cfg->scale < FP4Q_SCALE_FP32_1x16 || cfg->scale > FP4Q_SCALE_UE8M0_1x32) return FP4Q_ERR_INVALID_ARG;
  if (cfg->round != FP4Q_ROUND_RTNE && cfg->round != FP4Q_ROUND_SR) return FP4Q_ERR_INVALID_ARG;
  if (cfg->rht != 0 && cfg->rht != 1) return FP4Q_ERR_INVALID_ARG;
  if (cfg->sign_mask > 0xFFFFu) return FP4Q_ERR_INVALID_ARG;
  if (cfg->outputs & ~(uint32_t)(FP4Q_OUT_CODES | FP4Q_OUT_DEQUANT | FP4Q_OUT_STATS | FP4Q_OUT_SCALES_MMA))
    return FP4Q_ERR_INVALID_ARG;
  if ((cfg->outputs & FP4Q_OUT_SCALES_MMA) &&
      (cfg->scale == FP4Q_SCALE_FP32_1x16 || cfg->grid == FP4Q_GRID_IF4))
    return FP4Q_ERR_UNSUPPORTED;
  if (cfg->e2m1_max != 0u && cfg->e2m1_max != 4u && cfg->e2m1_max != 3u && cfg->e2m1_max != 2u)
    return FP4Q_ERR_INVALID_ARG;
  if (cfg->e2m1_max != 0u &&
      (cfg->grid != FP4Q_GRID_E2M1 || cfg->scale != FP4Q_SCALE_FP32_1x16))
    return FP4Q_ERR_UNSUPPORTED;
  if (cfg->grid == FP4Q_GRID_IF4 &&
      (cfg->scale != FP4Q_SCALE_E4M3_1x16_TENSOR || cfg->round != FP4Q_ROUND_RTNE))
    return FP4Q_ERR_UNSUPPORTED;
  if (cfg->scale == FP4Q_SCALE_UE8M0_1x32 && cfg->grid != FP4Q_GRID_E2M1) return FP4Q_ERR_UNSUPPORTED;
  return FP4Q_OK;
}

// Kernel grid id: the ABI grid, or the range-restricted E2M1 table selected by e2m1_max.
int kernel_grid(const fp4q_config* cfg) {
  if (cfg->e2m1_max == 4u) return kE2M1Max4;
  if (cfg->e2m1_max == 3u) return kE2M1Max3;
  if (cfg->e2m1_max == 2u) return kE2M1Max2;
  return cfg->grid;
}

// The block-scaled MMA scale layout tiles 128 rows x 4 scale columns.
fp4q_status check_mma_shape(const fp4q_config* cfg, int64_t rows, int64_t cols) {
  if (!(cfg->outputs & FP4Q_OUT_SCALES_MMA) || rows == 0 || cols == 0) return FP4Q_OK;
  const int64_t scale_cols = cols / (cfg->scale == FP4Q_SCALE_UE8M0_1x32 ? 32 : 16);
  return (rows % 128 == 0 && scale_cols % 4 == 0) ? FP4Q_OK : FP4Q_ERR_SHAPE;
}

int block_elems(const fp4q_config* cfg) { return cfg->scale == FP4Q_SCALE_UE8M0_1x32 ? 32 : 16; }

size_t stats_bytes() { return (size_t)kStatsCtas * ST_LEN * sizeof(double); }

// Largest M and N of fp4q_quantize_dual (and its 128 x 64 tiles must number below 2^31: one CTA
// each on the grid's x axis).
constexpr int64_t kDualMaxDim = (int64_t(1) << 31) - 128;

fp4q_status check_shape(int64_t rows, int64_t cols, int64_t ld, int unit) {
  if (rows < 0 || cols < 0) return FP4Q_ERR_SHAPE;
  if (cols % unit != 0) return FP4Q_ERR_SHAPE;
  if (rows == 0 || cols == 0) return FP4Q_OK;            // empty: nothing is read
  if (ld < cols) return FP4Q_ERR_SHAPE;
  if (rows > 1 && ld % 8 != 0) return FP4Q_ERR_ALIGN;   // every row starts 16-byte aligned
  return FP4Q_OK;
}

fp4q_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA; }

// Kernel arguments common to the row quantizers (a valid configuration and shape).
QuantArgs base_args(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols, int64_t ld,
                    uint8_t* codes, void* scales) {
  QuantArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.rows = rows;
  a.cols = cols;
  a.ld = ld;
  a.units_per_row = cols / block_elems(cfg);
  a.nunits = rows * a.units_per_row;
  a.codes = codes;
  a.scales = scales;
  sign_words(cfg->sign_mask, cfg->rht != 0, a.sw);
  sign_flips(a.sw, a.flip_lo, a.flip_hi);
  a.c = cfg->rht ? 4.0f : 1.0f;
  a.cinv = cfg->rht ? 0.25f : 1.0f;
  a.seedx = cfg->sr_seed ^ ((uint64_t)(cfg->sr_stream & 1u) << 63);
  a.contiguous = (ld == cols) ? 1 : 0;
  a.vec32 = (reinterpret_cast<uintptr_t>(x) % 32 == 0 && (rows == 1 || ld % 16 == 0)) ? 1 : 0;
  a.mma_scales = (cfg->outputs & FP4Q_OUT_SCALES_MMA) ? 1 : 0;
  return a;
}
}  // namespace

extern "C" {

const char* fp4q_status_string(fp4q_status s) {
  switch (s) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_INVALID_ARG: return "invalid argument";
    case FP4Q_ERR_SHAPE: return "invalid shape";
    case FP4Q_ERR_ALIGN: return "misaligned pointer or row pitch";
    case FP4Q_ERR_UNSUPPORTED: return "unsupported configuration";
    case FP4Q_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4Q_ERR_CUDA: return "CUDA error";
    case FP4Q_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

uint32_t fp4q_sign_mask_from_seed(uint64_t seed) { return (uint32_t)(host_splitmix64(seed) & 0xFFFFu); }

size_t fp4q_workspace_size(const fp4q_config* cfg, int64_t rows, int64_t cols) {
  if (check_cfg(cfg) != FP4Q_OK || rows < 0 || cols < 0) return 0;
  const bool stats = (cfg->outputs & FP4Q_OUT_STATS) != 0;
  const bool nv = cfg->scale == FP4Q_SCALE_E4M3_1x16_TENSOR;
  if (!stats && !nv) return 0;
  return sizeof(WsHeader) + (stats ? stats_bytes() : 0);
}


fp4q_status fp4q_rht_quantize(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                              int64_t ld, uint8_t* codes, void* scales, float* tensor_scale,
                              int32_t tensor_scale_given, void* dequant, void* workspace,
                              size_t workspace_bytes, fp4q_stream_t stream) {
  fp4q_status st = check_cfg(cfg);
  if (st != FP4Q_OK) return st;
  const int unit = block_elems(cfg);
  st = check_shape(rows, cols, ld, unit);
  if (st != FP4Q_OK) return st;
  st = check_mma_shape(cfg, rows, cols);
  if (st != FP4Q_OK) return st;
  const bool want_deq = (cfg->outputs & FP4Q_OUT_DEQUANT) != 0;
  const bool want_stats = (cfg->outputs & FP4Q_OUT_STATS) != 0;
  const bool nv = cfg->scale == FP4Q_SCALE_E4M3_1x16_TENSOR;
  const bool compute_alpha = nv && !tensor_scale_given;
  const bool empty = rows == 0 || cols == 0;
  if (!empty && (x == nullptr || codes == nullptr || scales == nullptr)) return FP4Q_ERR_INVALID_ARG;
  if (want_deq && !empty && dequant == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (nv && tensor_scale == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, unit == 32 ? 16 : 8) || !aligned(scales, 4) ||
      !aligned(dequant, 16) || !aligned(tensor_scale, 4) || !aligned(workspace, 256))
    return FP4Q_ERR_ALIGN;
  const size_t need = fp4q_workspace_size(cfg, rows, cols);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return FP4Q_ERR_WORKSPACE;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* ws = reinterpret_cast<WsHeader*>(workspace);
  // the header is read only for a computed tensor scale (its amax) and for statistics; with a
  // given scale the quantize kernel is the call's only work (no memset between back-to-back
  // launches, which would also cut their programmatic overlap)
  const bool use_ws = compute_alpha || want_stats;
  if (use_ws) {
    if (launch_ws_clear(ws, sizeof(WsHeader), s) != cudaSuccess) return FP4Q_ERR_CUDA;
  }
  if (empty) {
    if (compute_alpha && cudaMemsetAsync(tensor_scale, 0, sizeof(float), s) != cudaSuccess)
      return FP4Q_ERR_CUDA;
    return FP4Q_OK;
  }

  QuantArgs a = base_args(cfg, x, rows, cols, ld, codes, scales);
  a.deq = want_deq ? static_cast<uint16_t*>(dequant) : nullptr;
  a.ts_in = (nv && tensor_scale_given) ? tensor_scale : nullptr;
  a.ts_out = compute_alpha ? tensor_scale : nullptr;
  a.ws = use_ws ? ws : nullptr;
  a.partials = want_stats ? reinterpret_cast<double*>(static_cast<char*>(workspace) + sizeof(WsHeader)) : nullptr;

  if (compute_alpha) {
    QuantArgs am = a;
    if (cfg->scale == FP4Q_SCALE_E4M3_1x16_TENSOR) {
      am.units_per_row = cols / 16;
      am.nunits = rows * am.units_per_row;
    }
    if (launch_amax(am, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  }
  return cuda_status(launch_quantize(kernel_grid(cfg), cfg->scale, cfg->round, want_stats, a, s));
}

size_t fp4q_grouped_workspace_size(const fp4q_config* cfg, int32_t n_groups) {
  if (cfg == nullptr || n_groups < 1 || n_groups > (1 << 24)) return 0;
  if (cfg->scale != FP4Q_SCALE_E4M3_1x16_TENSOR) return 0;
  return ((size_t)n_groups * sizeof(uint32_t) + 255) / 256 * 256;
}

fp4q_status fp4q_rht_quantize_grouped(const fp4q_config* cfg, const void* x, int64_t rows,
                                      int64_t cols, int64_t ld, const int64_t* group_offsets,
                                      int32_t n_groups, uint8_t* codes, void* scales,
                                      float* tensor_scales, int32_t tensor_scales_given,
                                      void* workspace, size_t workspace_bytes,
                                      fp4q_stream_t stream) {
  fp4q_status st = check_cfg(cfg);
  if (st != FP4Q_OK) return st;
  if (cfg->outputs & (FP4Q_OUT_DEQUANT | FP4Q_OUT_STATS)) return FP4Q_ERR_UNSUPPORTED;
  if (cfg->scale == FP4Q_SCALE_E4M3_1x16_TENSOR && cfg->round != FP4Q_ROUND_RTNE)
    return FP4Q_ERR_UNSUPPORTED;   // the grouped E4M3 kernel rounds to nearest
  if (n_groups < 1 || n_groups > (1 << 24)) return FP4Q_ERR_INVALID_ARG;
  if (tensor_scales_given != 0 && tensor_scales_given != 1) return FP4Q_ERR_INVALID_ARG;
  if (cfg->scale != FP4Q_SCALE_E4M3_1x16_TENSOR)   // no per-group state
    return fp4q_rht_quantize(cfg, x, rows, cols, ld, codes, scales, nullptr, 0, nullptr, nullptr,
                             0, stream);
  st = check_shape(rows, cols, ld, 16);
  if (st != FP4Q_OK) return st;
  st = check_mma_shape(cfg, rows, cols);
  if (st != FP4Q_OK) return st;
  const bool empty = rows == 0 || cols == 0;
  if (group_offsets == nullptr || tensor_scales == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!empty && (x == nullptr || codes == nullptr || scales == nullptr)) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(codes, 8) || !aligned(scales, 4) || !aligned(group_offsets, 8) ||
      !aligned(tensor_scales, 4) || !aligned(workspace, 256))
    return FP4Q_ERR_ALIGN;
  const bool given = tensor_scales_given != 0;
  const size_t need = given ? 0 : fp4q_grouped_workspace_size(cfg, n_groups);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need)) return FP4Q_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!given && launch_ws_clear(workspace, need, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  QuantArgs a = base_args(cfg, x, rows, cols, ld, codes, scales);
  a.group_off = group_offsets;
  a.n_groups = n_groups;
  a.group_ts = tensor_scales;
  a.group_amax = static_cast<uint32_t*>(workspace);
  if (!given) {
    // every group's alpha, 0 for the empty ones (all of them when the tensor is empty)
    if (!empty && launch_grouped_amax(a, s) != cudaSuccess) return FP4Q_ERR_CUDA;
    const float qmax = cfg->grid == FP4Q_GRID_INT4 ? 7.0f : (cfg->grid == FP4Q_GRID_E1M2 ? 3.5f : 6.0f);
    if (launch_grouped_alpha(a, qmax, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  }
  if (empty) return FP4Q_OK;
  return cuda_status(launch_quantize_grouped(cfg->grid, a, s));
}

fp4q_status fp4q_tensor_scale(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                              int64_t ld, float* tensor_scale, void* workspace,
                              size_t workspace_bytes, fp4q_stream_t stream) {
  fp4q_status st = check_cfg(cfg);
  if (st != FP4Q_OK) return st;
  if (cfg->scale != FP4Q_SCALE_E4M3_1x16_TENSOR) return FP4Q_ERR_UNSUPPORTED;
  st = check_shape(rows, cols, ld, 16);
  if (st != FP4Q_OK) return st;
  const bool empty = rows == 0 || cols == 0;
  if (tensor_scale == nullptr || (!empty && x == nullptr)) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(tensor_scale, 4) || !aligned(workspace, 256)) return FP4Q_ERR_ALIGN;
  if (workspace == nullptr || workspace_bytes < sizeof(WsHeader)) return FP4Q_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* ws = reinterpret_cast<WsHeader*>(workspace);
  if (launch_ws_clear(ws, sizeof(WsHeader), s) != cudaSuccess) return FP4Q_ERR_CUDA;
  if (!empty) {
    QuantArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.rows = rows;
    a.cols = cols;
    a.ld = ld;
    a.units_per_row = cols / 16;
    a.nunits = rows * a.units_per_row;
    a.ws = ws;
    sign_words(cfg->sign_mask, cfg->rht != 0, a.sw);
    sign_flips(a.sw, a.flip_lo, a.flip_hi);
  sign_flips(a.sw, a.flip_lo, a.flip_hi);
    a.c = cfg->rht ? 4.0f : 1.0f;
    a.cinv = cfg->rht ? 0.25f : 1.0f;
    a.contiguous = (ld == cols) ? 1 : 0;
    a.vec32 = (reinterpret_cast<uintptr_t>(x) % 32 == 0 && (rows == 1 || ld % 16 == 0)) ? 1 : 0;
    if (launch_amax(a, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  }
  const float qmax = cfg->grid == FP4Q_GRID_INT4 ? 7.0f : (cfg->grid == FP4Q_GRID_E1M2 ? 3.5f : 6.0f);
  return cuda_status(launch_alpha(ws, qmax, tensor_scale, s));
}

fp4q_status fp4q_if4_select(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* codes, uint8_t* scales_flagged,
                            float* tensor_scale, int32_t tensor_scale_given, void* dequant,
                            void* workspace, size_t workspace_bytes, fp4q_stream_t stream) {
  if (cfg == nullptr) return FP4Q_ERR_INVALID_ARG;
  fp4q_config c = *cfg;
  c.grid = FP4Q_GRID_IF4;
  c.scale = FP4Q_SCALE_E4M3_1x16_TENSOR;
  return fp4q_rht_quantize(&c, x, rows, cols, ld, codes, scales_flagged, tensor_scale,
                           tensor_scale_given, dequant, workspace, workspace_bytes, stream);
}

fp4q_status fp4q_quantize_dual(const fp4q_config* row_cfg, const fp4q_config* col_cfg,
                               const void* dy, int64_t M, int64_t N, int64_t ld,
                               uint8_t* codes_row, void* scales_row, uint8_t* codes_col,
                               void* scales_col, void* workspace, size_t workspace_bytes,
                               fp4q_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  fp4q_status st = check_cfg(row_cfg);
  if (st != FP4Q_OK) return st;
  st = check_cfg(col_cfg);
  if (st != FP4Q_OK) return st;
  for (const fp4q_config* c : {row_cfg, col_cfg}) {
    if (c->scale != FP4Q_SCALE_FP32_1x16 || c->grid == FP4Q_GRID_IF4) return FP4Q_ERR_UNSUPPORTED;
    if (c->outputs & (FP4Q_OUT_DEQUANT | FP4Q_OUT_STATS)) return FP4Q_ERR_UNSUPPORTED;
  }
  if (row_cfg->grid != col_cfg->grid) return FP4Q_ERR_UNSUPPORTED;
  if (row_cfg->e2m1_max != 0u || col_cfg->e2m1_max != 0u) return FP4Q_ERR_UNSUPPORTED;
  if (M < 0 || N < 0 || M % 16 != 0 || N % 16 != 0) return FP4Q_ERR_SHAPE;
  if (M > kDualMaxDim || N > kDualMaxDim) return FP4Q_ERR_SHAPE;
  if (((M + 127) / 128) * ((N + 63) / 64) > INT32_MAX) return FP4Q_ERR_SHAPE;   // one CTA per tile
  if (M > 0 && N > 0 && ld < N) return FP4Q_ERR_SHAPE;
  if (M > 1 && N > 0 && ld % 8 != 0) return FP4Q_ERR_ALIGN;
  const bool empty = M == 0 || N == 0;
  if (!empty && (dy == nullptr || codes_row == nullptr || scales_row == nullptr ||
                 codes_col == nullptr || scales_col == nullptr))
    return FP4Q_ERR_INVALID_ARG;
  if (!aligned(dy, 16) || !aligned(codes_row, 8) || !aligned(codes_col, 8) ||
      !aligned(scales_row, 4) || !aligned(scales_col, 4))
    return FP4Q_ERR_ALIGN;
  if (empty) return FP4Q_OK;
  DualArgs a{};
  a.dy = static_cast<const uint16_t*>(dy);
  a.M = M;
  a.N = N;
  a.ld = ld;
  a.codes_row = codes_row;
  a.scales_row = static_cast<float*>(scales_row);
  a.codes_col = codes_col;
  a.scales_col = static_cast<float*>(scales_col);
  uint32_t sw_row[8];
  sign_words(row_cfg->sign_mask, row_cfg->rht != 0, sw_row);
  sign_flips(sw_row, a.flip_lo_row, a.flip_hi_row);
  for (int i = 0; i < 16; ++i)
    a.flip_col[i] = (col_cfg->rht != 0 && ((col_cfg->sign_mask >> i) & 1u)) ? 0x80000000u : 0u;
  a.vec32 = ((reinterpret_cast<uintptr_t>(dy) & 31u) == 0 && ld % 16 == 0) ? 1 : 0;
  a.col16 = (M % 64 == 0 && aligned(codes_col, 16) && aligned(scales_col, 16)) ? 1 : 0;
  a.c_row = row_cfg->rht ? 4.0f : 1.0f;
  a.cinv_row = row_cfg->rht ? 0.25f : 1.0f;
  a.c_col = col_cfg->rht ? 4.0f : 1.0f;
  a.cinv_col = col_cfg->rht ? 0.25f : 1.0f;
  a.seedx_row = row_cfg->sr_seed ^ ((uint64_t)(row_cfg->sr_stream & 1u) << 63);
  a.seedx_col = col_cfg->sr_seed ^ ((uint64_t)(col_cfg->sr_stream & 1u) << 63);
  a.round_row = row_cfg->round;
  a.round_col = col_cfg->round;
  a.grid_row = row_cfg->grid;
  a.grid_col = col_cfg->grid;
  return cuda_status(launch_dual(a, reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_dequantize(const fp4q_config* cfg, const uint8_t* codes, const void* scales,
                            const float* tensor_scale, int64_t rows, int64_t cols,
                            int32_t inverse_rht, void* out, fp4q_stream_t stream) {
  fp4q_status st = check_cfg(cfg);
  if (st != FP4Q_OK) return st;
  if (inverse_rht != 0 && inverse_rht != 1) return FP4Q_ERR_INVALID_ARG;
  st = check_shape(rows, cols, cols, block_elems(cfg));
  if (st != FP4Q_OK) return st;
  st = check_mma_shape(cfg, rows, cols);
  if (st != FP4Q_OK) return st;
  const bool empty = rows == 0 || cols == 0;
  const bool nv = cfg->scale == FP4Q_SCALE_E4M3_1x16_TENSOR;
  if (!empty && (codes == nullptr || scales == nullptr || out == nullptr)) return FP4Q_ERR_INVALID_ARG;
  if (!empty && nv && tensor_scale == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(codes, 8) || !aligned(out, 16) || !aligned(scales, 4) || !aligned(tensor_scale, 4))
    return FP4Q_ERR_ALIGN;
  if (empty) return FP4Q_OK;
  uint32_t sw[8];
  sign_words(cfg->sign_mask, true, sw);
  return cuda_status(launch_dequant(cfg->grid, cfg->scale, codes, scales, tensor_scale, rows, cols,
                                    sw, inverse_rht != 0, (cfg->outputs & FP4Q_OUT_SCALES_MMA) != 0,
                                    static_cast<uint16_t*>(out),
                                    reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_rht16(const void* x, int64_t rows, int64_t cols, int64_t ld, uint32_t sign_mask,
                       void* out, int32_t out_fp32, fp4q_stream_t stream) {
  if (sign_mask > 0xFFFFu || (out_fp32 != 0 && out_fp32 != 1)) return FP4Q_ERR_INVALID_ARG;
  fp4q_status st = check_shape(rows, cols, ld, 16);
  if (st != FP4Q_OK) return st;
  const bool empty = rows == 0 || cols == 0;
  if (!empty && (x == nullptr || out == nullptr)) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(out, 16)) return FP4Q_ERR_ALIGN;
  if (empty) return FP4Q_OK;
  uint32_t sw[8];
  sign_words(sign_mask, true, sw);
  return cuda_status(launch_rht16(static_cast<const uint16_t*>(x), rows, cols, ld, sw, out,
                                  out_fp32 != 0, reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_stats(const void* workspace, size_t workspace_bytes, fp4q_stats_t* host_out,
                       fp4q_stream_t stream) {
  if (workspace == nullptr || host_out == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return FP4Q_ERR_ALIGN;
  if (workspace_bytes < sizeof(WsHeader) + stats_bytes()) return FP4Q_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* ws = reinterpret_cast<WsHeader*>(const_cast<void*>(workspace));
  const double* partials = reinterpret_cast<const double*>(static_cast<const char*>(workspace) + sizeof(WsHeader));
  if (launch_stats_reduce(ws, partials, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  WsHeader h;
  if (cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, s) != cudaSuccess) return FP4Q_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP4Q_ERR_CUDA;

  std::memset(host_out, 0, sizeof *host_out);
  const double* r = h.reduced;
  host_out->sum_y2 = r[ST_SUM_Y2];
  host_out->sum_err2 = r[ST_SUM_ERR2];
  host_out->sum_y_xhat = r[ST_SUM_YXHAT];
  host_out->n = r[ST_N];
  for (int c = 0; c < 8; ++c) {
    host_out->cell_count[c] = r[ST_CELL_N + c];
    host_out->cell_err[c] = r[ST_CELL_ERR + c];
    host_out->cell_mean_err[c] = r[ST_CELL_N + c] > 0 ? r[ST_CELL_ERR + c] / r[ST_CELL_N + c] : NAN;
  }
  host_out->if4_fp4_blocks = r[ST_IF4_FP4];
  host_out->blocks = r[ST_BLOCKS];
  const double y2 = host_out->sum_y2, e2 = host_out->sum_err2;
  host_out->sqnr_db = e2 == 0.0 ? INFINITY : (y2 > 0.0 ? 10.0 * std::log10(y2 / e2) : -INFINITY);
  host_out->alpha = y2 > 0.0 ? host_out->sum_y_xhat / y2 : 1.0;
  host_out->mse = host_out->n > 0 ? e2 / host_out->n : 0.0;
  host_out->nmse = y2 > 0.0 ? e2 / y2 : 0.0;
  host_out->if4_fp4_fraction = host_out->blocks > 0 ? host_out->if4_fp4_blocks / host_out->blocks : 0.0;
  host_out->status = h.status == 0 ? FP4Q_OK : FP4Q_ERR_TIMEOUT;
  return host_out->status == FP4Q_OK ? FP4Q_OK : FP4Q_ERR_TIMEOUT;
}

fp4q_status fp4q_check_division(uint64_t seed, uint64_t n, unsigned long long* mismatches,
                                fp4q_stream_t stream) {
  if (mismatches == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(mismatches, 8)) return FP4Q_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(mismatches, 0, sizeof(unsigned long long), s) != cudaSuccess) return FP4Q_ERR_CUDA;
  return cuda_status(launch_division_check(seed, n, mismatches, s));
}

fp4q_status fp4q_device_status(int32_t* status_bits, int32_t clear, fp4q_stream_t stream) {
  if (status_bits == nullptr || (clear != 0 && clear != 1)) return FP4Q_ERR_INVALID_ARG;
  return cuda_status(read_device_status(status_bits, clear != 0, reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_tensor_scale,
                            const uint8_t* b_codes, const uint8_t* b_scales, const float* b_tensor_scale,
                            int64_t M, int64_t N, int64_t K, void* out, int64_t ldo,
                            fp4q_stream_t stream) {
  if (M < 0 || N < 0 || K < 256 || M % 128 != 0 || N % 128 != 0 || K % 256 != 0) return FP4Q_ERR_SHAPE;
  if (M / 128 > 65535 || K > (int64_t(1) << 31) || (M / 128) * (N / 128) > (int64_t(1) << 30)) return FP4Q_ERR_SHAPE;
  if ((M / 128) * (K / 64) > INT32_MAX || (N / 128) * (K / 64) > INT32_MAX) return FP4Q_ERR_SHAPE;   // scale tiles
  if (M > 0 && N > 0 && ldo < N) return FP4Q_ERR_SHAPE;
  if (M == 0 || N == 0) return FP4Q_OK;
  if (a_codes == nullptr || a_scales == nullptr || a_tensor_scale == nullptr || b_codes == nullptr ||
      b_scales == nullptr || b_tensor_scale == nullptr || out == nullptr)
    return FP4Q_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) || !aligned(b_scales, 16) ||
      !aligned(out, 16) || ldo % 8 != 0 || !aligned(a_tensor_scale, 4) || !aligned(b_tensor_scale, 4))
    return FP4Q_ERR_ALIGN;
  return cuda_status(launch_gemm_nvfp4(a_codes, a_scales, a_tensor_scale, b_codes, b_scales, b_tensor_scale,
                                       M, N, K, static_cast<uint16_t*>(out), ldo,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                            const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, void* out, int64_t ldo,
                            fp4q_stream_t stream) {
  if (M < 0 || N < 0 || K < 256 || M % 128 != 0 || N % 128 != 0 || K % 256 != 0) return FP4Q_ERR_SHAPE;
  if (M / 128 > 65535 || K > (int64_t(1) << 31) || (M / 128) * (N / 128) > (int64_t(1) << 30)) return FP4Q_ERR_SHAPE;
  if ((M / 128) * (K / 64) > INT32_MAX || (N / 128) * (K / 64) > INT32_MAX) return FP4Q_ERR_SHAPE;   // scale tiles
  if (M > 0 && N > 0 && ldo < N) return FP4Q_ERR_SHAPE;
  if (M == 0 || N == 0) return FP4Q_OK;
  if (a_codes == nullptr || a_scales == nullptr || b_codes == nullptr || b_scales == nullptr || out == nullptr)
    return FP4Q_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) || !aligned(b_scales, 16) ||
      !aligned(out, 16) || ldo % 8 != 0)
    return FP4Q_ERR_ALIGN;
  return cuda_status(launch_gemm_mxfp4(a_codes, a_scales, b_codes, b_scales, M, N, K, static_cast<uint16_t*>(out),
                                       ldo, reinterpret_cast<cudaStream_t>(stream)));
}

fp4q_status fp4q_check_conversions(unsigned long long* mismatches, fp4q_stream_t stream) {
  if (mismatches == nullptr) return FP4Q_ERR_INVALID_ARG;
  if (!aligned(mismatches, 8)) return FP4Q_ERR_ALIGN;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(mismatches, 0, 5 * sizeof(unsigned long long), s) != cudaSuccess) return FP4Q_ERR_CUDA;
  return cuda_status(launch_conversion_check(mismatches, s));
}

fp4q_status fp4q_check_wait_timeout(uint64_t limit_ns, fp4q_stream_t stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return FP4Q_ERR_INVALID_ARG;
  return cuda_status(launch_wait_timeout_check(limit_ns, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

/*
 * fp4q.h -- C ABI of libfp4q: fused 16-point random Hadamard rotation (RHT16) + block-scaled
 * 4-bit quantization on NVIDIA B200 (sm_100a).
 *
 * What it computes (the method is described on these web pages; cited by title and section):
 *   [UFP4-A] "当你的 GPU 学不会算账：FP4 训练里那个被忽视了 30 年的几何陷阱"
 *            (zhichai.net/topic/178208020): E2M1/E1M2 grids, UFP4 recipe table (1x16 blocks,
 *            FP32 single-level scale, RHT on fwd_y/bwd_dx/bwd_dw, stochastic rounding on dY).
 *   [UFP4-B] "蚂蚁集团揭秘：为什么给AI"降精度省电"会悄悄让它越来越笨？"
 *            (techwalker.com/2026/0624/3191429.shtml), section 六 Q5: the rotation block equals
 *            the 16-element quantization block, so rotation and quantization fuse in one pass.
 *   [MXFP4]  "AMD全新研究揭示：FP4训练不稳定性源于结构误差而非随机性不足"
 *            (cannews.ca/article/21387): MXFP4 = 32-element blocks with a shared E8M0 exponent.
 *   [IF4]    "低精度量化技术：IF4自适应数据类型的原理与应用" (bxzpzcl.cn/news/2320061):
 *            NVFP4/NVINT4 two-level scales (section 3.2), IF4 per-block FP4-or-INT4 choice
 *            flagged in the scale's sign bit (sections 3.1, 3.2).
 *
 * Per 16-element block along the reduction axis (the contiguous axis of a row):
 *   y = 1/4 * H16 * D * x            H16 Sylvester-ordered Hadamard, D = diag(+-1) from sign_mask,
 *                                    butterfly stages h = 1, 2, 4, 8, each (a+b, a-b), in FP32
 *   s = block scale (see fp4q_scale)
 *   v = y / s                         IEEE FP32 division (MX: exact power-of-two multiply)
 *   q = round(v) onto the grid        RTNE (ties to the even code) or stochastic rounding
 *   codes: element 2j in the low nibble of byte j; dequant xhat = q * s (FP32), stored bf16.
 * Results are bit-identical to the CPU oracle in oracle/ for every configuration.
 *
 * Conventions for every entry point:
 *  - Pointers named x / dy / codes / scales / dequant / workspace / tensor_scale are DEVICE
 *    pointers owned by the caller; the library allocates nothing and keeps no state between
 *    calls. Tensors are row-major; `ld` is the row pitch in elements.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream), except fp4q_stats, which
 *    synchronizes the stream. Calls on different streams with disjoint outputs may overlap.
 *  - Arguments are validated on the host before anything is launched; the first failure is
 *    returned and nothing runs. A launch failure returns FP4Q_ERR_CUDA.
 *  - Inputs must be finite bfloat16. Results for NaN/Inf inputs are unspecified.
 *  - Required alignment: x / dy 16 bytes (and ld a multiple of 8 elements), codes 8 bytes,
 *    FP32 scales 4 bytes, dequant 16 bytes, workspace 256 bytes.
 */
#ifndef FP4Q_H
#define FP4Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; this header does not need the CUDA headers. */
typedef struct CUstream_st* fp4q_stream_t;

typedef enum {
  FP4Q_OK = 0,
  FP4Q_ERR_INVALID_ARG = 1, /* null pointer for a requested output, bad enum, bad flag */
  FP4Q_ERR_SHAPE = 2,       /* cols not a multiple of the block, ld < cols, negative size */
  FP4Q_ERR_ALIGN = 3,       /* a pointer or ld breaks the alignment rules above */
  FP4Q_ERR_UNSUPPORTED = 4, /* valid enums in a combination the library does not implement */
  FP4Q_ERR_WORKSPACE = 5,   /* workspace missing or smaller than fp4q_workspace_size() */
  FP4Q_ERR_CUDA = 6,        /* a CUDA call or kernel launch failed */
  FP4Q_ERR_TIMEOUT = 7      /* a bounded device-side wait gave up (reported by fp4q_stats) */
} fp4q_status;

/* Element grid [UFP4-A "E2M1：一块刻度不均的尺子", "UFP4：换一把尺子"; IF4 sections 2.2, 3.1].
 *   E2M1: {0,.5,1,1.5,2,3,4,6}, sign-magnitude code S EE M; a negative value that rounds to
 *         zero is -0 (code 0x8). qmax 6.
 *   E1M2: {0,.5,...,3.5} (exponent bias 0), sign-magnitude code S E MM, -0 as for E2M1. qmax 3.5.
 *   INT4: integers -7..7, two's complement code (0x8 unused). qmax 7.
 *   IF4:  per block E2M1 or INT4 scaled by 6/7, whichever has the smaller squared error;
 *         only with FP4Q_SCALE_E4M3_1x16_TENSOR and RTNE. */
typedef enum { FP4Q_GRID_E2M1 = 0, FP4Q_GRID_E1M2 = 1, FP4Q_GRID_INT4 = 2, FP4Q_GRID_IF4 = 3 } fp4q_grid;

/* Block scale.
 *   FP32_1x16: s = amax(y) / qmax per 16 elements, stored as float [rows, cols/16]
 *              [UFP4-A recipe table: "FP32 单层"].
 *   E4M3_1x16_TENSOR: alpha = A / RN(qmax*448) with A the amax of the whole rotated tensor;
 *              per block d8 = E4M3_rne_satfinite(amax / RN(alpha*qmax)), s = decode(d8)*alpha;
 *              stored as uint8 [rows, cols/16] (IF4: bit 7 = 1 marks an INT4 block) plus one
 *              float alpha [IF4 section 3.2].
 *   UE8M0_1x32: s = 2^e, e = floor(log2 amax(y)) - 2 clamped to [-127, 127], stored as uint8
 *              e + 127 per 32 elements, [rows, cols/32]; E2M1 grid only [MXFP4]. */
typedef enum {
  FP4Q_SCALE_FP32_1x16 = 0,
  FP4Q_SCALE_E4M3_1x16_TENSOR = 1,
  FP4Q_SCALE_UE8M0_1x32 = 2
} fp4q_scale;

/* Rounding [UFP4-B section 二 (RTNE); IF4 section 6.1 (stochastic rounding); UFP4-A recipe
 * table (SR on dY only)]. SR rounds |v| up between adjacent grid points lo <= |v| < hi iff
 * r < (|v|-lo)/(hi-lo), r = u * 2^-16, u = bits 16l .. 16l+15 (l = idx & 3) of output idx>>2
 * of the SplitMix64 stream seeded with sr_seed ^ (sr_stream << 63), i.e. of the finalizer of
 * state seed + ((idx>>2) + 1) * 0x9E3779B97F4A7C15; idx = row * cols + col in the output
 * orientation. The expected code differs from |v| by at most 2^-16 of the cell width. */
typedef enum { FP4Q_ROUND_RTNE = 0, FP4Q_ROUND_SR = 1 } fp4q_round;

/* Output bits of fp4q_config.outputs. Codes and scales are always written.
 * FP4Q_OUT_SCALES_MMA: E4M3 / UE8M0 block scales in the scale-factor layout that sm_100
 *   block-scaled tensor-core MMA (NVFP4, MXFP4) consumes, instead of row-major: the [rows, C]
 *   scale matrix (C = cols/16, MX cols/32) as 512-byte tiles of 128 rows x 4 columns, row-major
 *   over tiles, with row r, column c of a tile at byte (r % 32) * 16 + (r / 32 % 4) * 4 + c % 4.
 *   The buffer size is unchanged. Needs rows % 128 == 0 and C % 4 == 0 (else FP4Q_ERR_SHAPE);
 *   FP32 scales and IF4 (flagged scale bytes): FP4Q_ERR_UNSUPPORTED. fp4q_dequantize reads the
 *   scales in the layout the same bit names. The pages give no interface; this serves the
 *   hardware FP4 GEMM path the NVFP4 recipe targets ("低精度量化技术：IF4…", section 3.2). */
enum { FP4Q_OUT_CODES = 1u, FP4Q_OUT_DEQUANT = 2u, FP4Q_OUT_STATS = 4u, FP4Q_OUT_SCALES_MMA = 8u };

typedef struct {
  int32_t grid;        /* fp4q_grid */
  int32_t scale;       /* fp4q_scale */
  int32_t round;       /* fp4q_round */
  int32_t rht;         /* 0: y = x (no rotation). 1: y = 1/4 * H16 * D * x */
  uint32_t sign_mask;  /* bit j (0..15) set <=> D_jj = -1; 0 gives the deterministic H16 */
  uint32_t sr_stream;  /* SR counter stream: 0 row orientation, 1 column orientation */
  uint64_t sr_seed;    /* SR counter seed */
  uint32_t outputs;    /* FP4Q_OUT_* bits */
  uint32_t e2m1_max;   /* 0: the grid as named. 4, 3 or 2: range-restricted E2M1, the E2M1 table
                          up to that largest value ("当你的 GPU 学不会算账", section "124B MoE 上的
                          验证"; "蚂蚁集团揭秘…", section 六) -- grid E2M1 with the FP32 1x16
                          scale only, s = amax / e2m1_max, RTNE or SR onto the restricted table,
                          E2M1 codes (dequantize as E2M1). Other values: FP4Q_ERR_INVALID_ARG;
                          with another grid or scale, or in fp4q_quantize_dual:
                          FP4Q_ERR_UNSUPPORTED. */
} fp4q_config;

/* Statistics of one quantizer call, in the rotated domain (y vs the FP32 xhat). */
typedef struct {
  double sum_y2;            /* sum y^2 */
  double sum_err2;          /* sum (y - xhat)^2 */
  double sum_y_xhat;        /* sum y * xhat */
  double n;                 /* elements */
  double cell_count[8];     /* elements per magnitude code (FP grids: code & 7; INT4: |k|; IF4:
                               the chosen representation's, so FP4 and INT4 blocks share cells) */
  double cell_err[8];       /* sum (|q| - |v|) per magnitude code, in scaled (v) units */
  double if4_fp4_blocks;    /* IF4 blocks that kept FP4 */
  double blocks;            /* scale blocks */
  /* derived */
  double sqnr_db;           /* 10 log10(sum_y2 / sum_err2); +inf when sum_err2 == 0 */
  double alpha;             /* sum_y_xhat / sum_y2 (signal attenuation) */
  double mse;               /* sum_err2 / n */
  double nmse;              /* sum_err2 / sum_y2 */
  double cell_mean_err[8];  /* cell_err / cell_count (NaN for an empty cell): shrinkage bias */
  double if4_fp4_fraction;  /* if4_fp4_blocks / blocks */
  int32_t status;           /* FP4Q_OK, or FP4Q_ERR_TIMEOUT if a device wait gave up (the
                               statistics-producing kernels do not wait: FP4Q_OK) */
  int32_t reserved;
} fp4q_stats_t;

/* Human-readable name of a status. Never NULL. */
const char* fp4q_status_string(fp4q_status status);

/* The sign mask for a seed: low 16 bits of SplitMix64(seed) (Steele, Lea & Flood 2014).
 * [UFP4-A "治病药反而喂养了病菌": the rotation is random]. Pure host function. */
uint32_t fp4q_sign_mask_from_seed(uint64_t seed);

/* Bytes of device workspace a call with this configuration and shape needs: 0 when neither
 * statistics nor a computed E4M3 tensor scale are requested. Returns 0 for invalid arguments. */
size_t fp4q_workspace_size(const fp4q_config* cfg, int64_t rows, int64_t cols);

/* Fused RHT16 + quantize along rows [UFP4-B section 六 Q5 (fused kernel); UFP4-A recipe table].
 *  x            bf16 [rows, ld], quantized along the row (cols contiguous).
 *  codes        uint8 [rows, cols/2].
 *  scales       float [rows, cols/16] | uint8 [rows, cols/16] | uint8 [rows, cols/32] per cfg->scale.
 *  tensor_scale E4M3 scale only, one device float alpha. tensor_scale_given != 0: read alpha
 *               from it (delayed scaling); == 0: compute A over the rotated tensor (an extra
 *               read of x) and write alpha there. Ignored (may be NULL) for other scales.
 *  dequant      bf16 [rows, cols] (xhat in the rotated domain) if FP4Q_OUT_DEQUANT, else NULL.
 *  workspace    device scratch of fp4q_workspace_size() bytes (NULL if that is 0). With
 *               FP4Q_OUT_STATS the statistics stay in it for fp4q_stats().
 * cfg->grid may be FP4Q_GRID_IF4 here too (then scales carry the INT4 flag in bit 7). */
fp4q_status fp4q_rht_quantize(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                              int64_t ld, uint8_t* codes, void* scales, float* tensor_scale,
                              int32_t tensor_scale_given, void* dequant, void* workspace,
                              size_t workspace_bytes, fp4q_stream_t stream);

/* dY in both orientations from one read [UFP4-A recipe table (SR on dY, RHT on bwd_dx and
 * bwd_dw); UFP4-B section 三 (bwd_dx reduces over N, bwd_dw over M)].
 *  dy         bf16 [M, ld], ld >= N.
 *  codes_row  uint8 [M, N/2], scales_row float [M, N/16]: blocks along N (row_cfg).
 *  codes_col  uint8 [N, M/2], scales_col float [N, M/16]: blocks along M, i.e. dy^T
 *             quantized along its rows (col_cfg; SR index n * M + m).
 * Both configs must use FP4Q_SCALE_FP32_1x16 and no dequant/stats outputs; M and N must be
 * multiples of 16, at most 2^31 - 128, and (M/128) * (N/64) (rounded up) below 2^31 (else
 * FP4Q_ERR_SHAPE). workspace may be NULL. */
fp4q_status fp4q_quantize_dual(const fp4q_config* row_cfg, const fp4q_config* col_cfg,
                               const void* dy, int64_t M, int64_t N, int64_t ld,
                               uint8_t* codes_row, void* scales_row, uint8_t* codes_col,
                               void* scales_col, void* workspace, size_t workspace_bytes,
                               fp4q_stream_t stream);

/* Codes back to bf16: xhat = q * s in FP32 (IF4 INT4 blocks: RN(k * RN(6/7)) * s), then, if
 * inverse_rht, x = D * 1/4 * H16 * xhat per 16 elements in FP32; stored bf16 (RNE).
 *  codes uint8 [rows, cols/2]; scales as fp4q_rht_quantize; tensor_scale device float alpha
 *  (E4M3 scales only); out bf16 [rows, cols]. cfg->grid/scale/sign_mask describe the codes. */
fp4q_status fp4q_dequantize(const fp4q_config* cfg, const uint8_t* codes, const void* scales,
                            const float* tensor_scale, int64_t rows, int64_t cols,
                            int32_t inverse_rht, void* out, fp4q_stream_t stream);

/* IF4 [IF4 sections 3.1, 3.2]: NVFP4 scales; per block both the E2M1 candidate and
 * round(v * RN(7/6)) on INT4 are formed, their squared errors in scaled units summed in a
 * fixed pairwise order, and INT4 kept iff strictly smaller (bit 7 of the scale byte).
 * Same arguments as fp4q_rht_quantize with cfg->grid forced to IF4, cfg->scale to E4M3. */
fp4q_status fp4q_if4_select(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                            int64_t ld, uint8_t* codes, uint8_t* scales_flagged,
                            float* tensor_scale, int32_t tensor_scale_given, void* dequant,
                            void* workspace, size_t workspace_bytes, fp4q_stream_t stream);

/* The FP32 tensor scale alone (the first pass of the E4M3 two-level scale [IF4 section 3.2]):
 * alpha = A / RN(qmax * 448), A the amax of the rotated x (cfg->grid, rht, sign_mask apply).
 * Writes alpha to the device float *tensor_scale. For a tensor split by rows over ranks, the
 * global alpha is the maximum of the ranks' alphas (rounding is monotonic), which is then passed
 * to fp4q_rht_quantize with tensor_scale_given = 1. workspace: fp4q_workspace_size() of an
 * E4M3 configuration (256 bytes). */
fp4q_status fp4q_tensor_scale(const fp4q_config* cfg, const void* x, int64_t rows, int64_t cols,
                              int64_t ld, float* tensor_scale, void* workspace,
                              size_t workspace_bytes, fp4q_stream_t stream);

/* fp4q_rht_quantize for callers that cannot allocate device memory (a runtime's plugin
 * boundary that hands over only input and output buffers, a host framework that owns all
 * device memory, or work where cudaMalloc is off limits). The pages have no counterpart: this
 * is a calling convention of the library, not part of the method.
 * Same arguments and results as fp4q_rht_quantize without the workspace: the scratch an E4M3
 * tensor scale computed on the device needs (256 bytes) lives in a static array inside the
 * library, which every GPU that loads the library keeps until the process exits. A
 * configuration that needs more scratch than that -- statistics (FP4Q_OUT_STATS) -- is rejected
 * with FP4Q_ERR_WORKSPACE before anything runs.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call outside any stream capture. All calls share the
 * one array, which each call clears on its stream before use: calls that can overlap on the GPU
 * (different streams, or different host threads, on the same device) race on it and must be
 * ordered by the caller. No allocation happens in this call. */
fp4q_status fp4q_rht_quantize_noalloc(const fp4q_config* cfg, const void* x, int64_t rows,
                                      int64_t cols, int64_t ld, uint8_t* codes, void* scales,
                                      float* tensor_scale, int32_t tensor_scale_given,
                                      void* dequant, fp4q_stream_t stream);

/* Grouped quantization of the rows of x as n_groups consecutive tensors, e.g. the experts of an
 * MoE layer with variable token counts ("当你的 GPU 学不会算账", section "124B MoE 上的验证"
 * and the MoE rows of the scale table): group g is rows [group_offsets[g], group_offsets[g+1]).
 * With the E4M3 scale (NVFP4, NVINT4, IF4) every group has its own FP32 tensor scale
 * alpha_g = RN(A_g / RN(qmax * 448)), A_g the amax of the group's rotated rows: tensor_scales
 * (device float[n_groups]) receives the alpha_g, or supplies them when tensor_scales_given; an
 * empty or all-zero group gets alpha 0. Codes and scales are laid out as for one
 * fp4q_rht_quantize call over all rows (FP4Q_OUT_SCALES_MMA included); SR indices are global.
 * With the FP32 or UE8M0 scale no state is per group, and the call is fp4q_rht_quantize over all
 * rows (group_offsets and tensor_scales are not read).
 *   group_offsets: device int64[n_groups + 1], nondecreasing, [0] = 0, [n_groups] = rows. Other
 *   values give an unspecified grouping but never an out-of-bounds access.
 *   workspace: fp4q_grouped_workspace_size(cfg, n_groups) bytes, 256-byte aligned (per-group
 *   amax slots; zeroed by the call on its stream).
 * Errors as fp4q_rht_quantize; n_groups < 1 or > 2^24, or a null group_offsets / tensor_scales
 * that is needed: FP4Q_ERR_INVALID_ARG; FP4Q_OUT_DEQUANT / FP4Q_OUT_STATS, or stochastic
 * rounding with the E4M3 scale: FP4Q_ERR_UNSUPPORTED. */
size_t fp4q_grouped_workspace_size(const fp4q_config* cfg, int32_t n_groups);
fp4q_status fp4q_rht_quantize_grouped(const fp4q_config* cfg, const void* x, int64_t rows,
                                      int64_t cols, int64_t ld, const int64_t* group_offsets,
                                      int32_t n_groups, uint8_t* codes, void* scales,
                                      float* tensor_scales, int32_t tensor_scales_given,
                                      void* workspace, size_t workspace_bytes,
                                      fp4q_stream_t stream);

/* NVFP4 GEMM on the tensor cores (tcgen05 block-scaled MMA, sm_100a), consuming the quantizer's
 * outputs unchanged: out[m, n] = alpha_a * alpha_b * sum_k A[m, k] B[n, k] (bf16, RNE), where A and B
 * are the E2M1 codes of two NVFP4 quantizations along K (fp4q_rht_quantize with grid E2M1,
 * FP4Q_SCALE_E4M3_1x16_TENSOR and FP4Q_OUT_SCALES_MMA) times their E4M3 block scales, and alpha_a,
 * alpha_b their FP32 tensor scales ("低精度量化技术：IF4…", section 3.2: the two-level NVFP4 scale
 * of the hardware path; both operands rotated with the same sign mask keep A B^T, since the
 * 16-point rotation is orthogonal). Products accumulate in FP32.
 *  a_codes uint8 [M, K/2], a_scales uint8 [M, K/16] in the MMA layout, a_tensor_scale one device
 *  float; b_* the same with N rows; out bf16 [M, ldo], ldo >= N, ldo % 8 == 0.
 *  M and N multiples of 128 (M at most 65535 * 128, at most 2^30 tiles of 128 x 128, and
 *  M / 128 * K / 64 and N / 128 * K / 64 at most 2^31 - 1), K a multiple of 256 up to 2^31 (else
 *  FP4Q_ERR_SHAPE);
 *  every pointer 16-byte aligned (tensor scales 4) (else FP4Q_ERR_ALIGN); a null pointer:
 *  FP4Q_ERR_INVALID_ARG. The first call on a device looks up cached launch parameters; make it
 *  outside any stream capture. A tile whose bounded waits (2 s) give up is left incomplete and
 *  sets bit 0 of the device status word (fp4q_device_status). */
fp4q_status fp4q_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                            const float* a_tensor_scale, const uint8_t* b_codes,
                            const uint8_t* b_scales, const float* b_tensor_scale, int64_t M,
                            int64_t N, int64_t K, void* out, int64_t ldo, fp4q_stream_t stream);

/* MXFP4 GEMM on the tensor cores (tcgen05 block-scaled MMA with 32-element blocks, sm_100a),
 * consuming the quantizer's outputs unchanged: out[m, n] = sum_k A[m, k] B[n, k] (bf16, RNE), where
 * A and B are the E2M1 codes of two MXFP4 quantizations along K (fp4q_rht_quantize with grid E2M1,
 * FP4Q_SCALE_UE8M0_1x32 and FP4Q_OUT_SCALES_MMA) times their UE8M0 block scales
 * ("AMD全新研究揭示：FP4训练不稳定性源于结构误差而非随机性不足", cannews.ca/article/21387: MXFP4 = 32-element
 * blocks sharing one power-of-two scale; no tensor scale). Products accumulate in FP32.
 *  a_codes uint8 [M, K/2], a_scales uint8 [M, K/32] in the MMA layout; b_* the same with N rows;
 *  out bf16 [M, ldo], ldo >= N, ldo % 8 == 0.
 *  Shapes, alignment, errors, the first call and the bounded waits as fp4q_gemm_nvfp4. */
fp4q_status fp4q_gemm_mxfp4(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                            const uint8_t* b_scales, int64_t M, int64_t N, int64_t K, void* out, int64_t ldo,
                            fp4q_stream_t stream);

/* Reduce the statistics a previous fp4q_rht_quantize / fp4q_if4_select call with
 * FP4Q_OUT_STATS left in `workspace` (in a fixed order, FP64), copy them to *host_out and
 * derive SQNR, alpha, MSE and the per-cell mean error [UFP4-A "E2M1", "复利效应的反向版本",
 * "治病药反而喂养了病菌"; IF4 section 6.2]. Synchronizes `stream`. */
fp4q_status fp4q_stats(const void* workspace, size_t workspace_bytes, fp4q_stats_t* host_out,
                       fp4q_stream_t stream);

/* The rotation alone (first pass of the unfused pipeline the fused kernel is compared with
 * [UFP4-B section 六 Q5]): y = 1/4 * H16 * D * x per 16 elements, written as bf16 (RNE) or
 * FP32 [rows, cols]. out_fp32 != 0 selects FP32. */
fp4q_status fp4q_rht16(const void* x, int64_t rows, int64_t cols, int64_t ld, uint32_t sign_mask,
                       void* out, int32_t out_fp32, fp4q_stream_t stream);

/* Diagnostic: checks the kernels' exact-quotient steps (one correctly rounded reciprocal plus
 * an FMA correction, after P. Markstein, IBM J. Res. Dev. 34(1), 1990) against IEEE division:
 * the scale quotient a / qmax for every mantissa of a in [1, 4) and qmax in {6, 3.5, 7}; the
 * block reciprocal (hardware approximation + one Newton-Raphson step) for every float in
 * [2^-60, 2^91); and the element quotient y / s on `n` pseudo-random pairs from `seed` with s in
 * [2^-60, 2^90) and |y/s| in [2^-20, 8), with and without the folded rotation normalisation.
 * Writes the number of results that differ in any bit to the device counter *mismatches
 * (zeroed first). */
fp4q_status fp4q_check_division(uint64_t seed, uint64_t n, unsigned long long* mismatches,
                                fp4q_stream_t stream);

/* Diagnostic: checks the hardware conversions the encoders use, each against a rule written from
 * the format's definition (exponent field, grid step, round half to even, saturation), over every
 * FP32 input in the range the kernels feed it, and writes the number of inputs whose result
 * differs in any bit to the device counters mismatches[0..4] (zeroed first; 8-byte aligned):
 *  [0] E2M1 encode (round to nearest even, saturating at 6, sign of zero kept), every non-NaN
 *      float ["当你的 GPU 学不会算账", section "E2M1：一块刻度不均的尺子"]
 *  [1] E1M2 encode as the kernels form it (quarters of the scaled value through the FP6 E2M3
 *      conversion), every float of magnitude below 15/16 ["UFP4：换一把尺子"]
 *  [2] E4M3 encode of a block-scale quotient (round to nearest even, 448 and above -> 448), every
 *      float >= 0 including +inf ["低精度量化技术：IF4…", section 3.2]
 *  [3] the E2M1 decoder on all 256 bytes, the E4M3 decoder on codes 0..0x7E, and IF4's
 *      factors RN(7/6), RN(6/7) against the IEEE quotients
 *  [4] bf16 rounding of dequantized values (round to nearest even), every non-NaN float */
fp4q_status fp4q_check_conversions(unsigned long long* mismatches, fp4q_stream_t stream);

/* Device status word of the library on the current device: bit 0 is set when a bounded wait
 * inside a quantize kernel gives up (fp4q_quantize_dual waits on the tile copies it has issued,
 * at most 2 s each; that launch's outputs are then incomplete); the row quantizers read their
 * inputs with plain loads and never wait. Bit 1 is set by fp4q_check_wait_timeout. Copies the
 * word to *status_bits (host), clears it when `clear` is 1, and synchronizes `stream`. */
fp4q_status fp4q_device_status(int32_t* status_bits, int32_t clear, fp4q_stream_t stream);

/* Diagnostic: launches one thread that waits, with a limit of limit_ns (1 ns .. 1 s), on a
 * barrier nothing arrives on; when the limit runs out it sets bit 1 of the status word and
 * returns. Exercises the timeout path of the kernels' bounded waits without any fault. */
fp4q_status fp4q_check_wait_timeout(uint64_t limit_ns, fp4q_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* FP4Q_H */

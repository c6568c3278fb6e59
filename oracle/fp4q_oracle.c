/*
 * fp4q_oracle.c -- CPU oracle for the fused RHT16 + block-scaled 4-bit quantizer.
 *
 * TEST INFRASTRUCTURE. This is the plain, slow, obviously-correct restatement of what the
 * quantizer computes. Only the test suite, the package smoke check and the benchmark's
 * CPU-baseline leg load it; the CUDA library never does, and the two share no source.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC (oracle/build.py).
 * On x86-64 every float operation below is one IEEE-754 binary32 operation, rounded to
 * nearest-even, in the written order, with no fused multiply-add.
 *
 * Sources (web pages on FP4 training formats; cited by title and section):
 *   [UFP4-A]  "当你的 GPU 学不会算账：FP4 训练里那个被忽视了 30 年的几何陷阱"
 *             (zhichai.net/topic/178208020) -- UFP4 explainer.
 *   [UFP4-B]  "蚂蚁集团揭秘：为什么给AI"降精度省电"会悄悄让它越来越笨？"
 *             (techwalker.com/2026/0624/3191429.shtml) -- second UFP4 explainer, sections 一..七.
 *   [MXFP4]   "AMD全新研究揭示：FP4训练不稳定性源于结构误差而非随机性不足"
 *             (cannews.ca/article/21387) -- MXFP4 pretraining on MI355X.
 *   [IF4]     "低精度量化技术：IF4自适应数据类型的原理与应用"
 *             (bxzpzcl.cn/news/2320061) -- IF4 adaptive data type, sections 1..6.
 *
 * Where the pages leave a step open, the reading taken is stated at the step (R1..R16 below
 * name the readings; the repository's design notes list them with their reasons).
 *
 * Parity status: every function here is pinned by a CPU test (tests/test_oracle_*.py)
 * except the stats of real-data experiments, which the pages print without their data.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------------ */
/* Configuration (the oracle's own encoding; the test layer maps the library's onto it). */

enum { ORC_GRID_E2M1 = 0, ORC_GRID_E1M2 = 1, ORC_GRID_INT4 = 2, ORC_GRID_IF4 = 3,
       /* E2M1 with the largest magnitude restricted to 4, 3 or 2 (codes above it unused) */
       ORC_GRID_E2M1_MAX4 = 4, ORC_GRID_E2M1_MAX3 = 5, ORC_GRID_E2M1_MAX2 = 6 };
enum { ORC_SCALE_FP32_1x16 = 0, ORC_SCALE_E4M3_1x16 = 1, ORC_SCALE_UE8M0_1x32 = 2 };
enum { ORC_ROUND_RTNE = 0, ORC_ROUND_SR = 1 };

typedef struct {
  int32_t grid;
  int32_t scale;
  int32_t round;
  int32_t rht;          /* 0: no rotation, y = x. 1: y = 1/4 * H16 * D * x per 16-block. */
  uint32_t sign_mask;   /* bit j set <=> D_jj = -1 (R1) */
  uint32_t sr_stream;   /* 0 row orientation, 1 column orientation (R12) */
  uint64_t sr_seed;
} orc_cfg;

/* Layout of the raw statistics record (doubles), accumulated with += so that callers can
 * chain calls over row chunks. */
enum {
  ORC_ST_SUM_Y2 = 0,      /* sum y^2 over elements (rotated domain, R15) */
  ORC_ST_SUM_ERR2 = 1,    /* sum (y - xhat)^2, xhat the FP32 dequant value */
  ORC_ST_SUM_YXHAT = 2,   /* sum y * xhat */
  ORC_ST_N = 3,           /* element count */
  ORC_ST_CELL_N = 4,      /* [8] element count per magnitude code */
  ORC_ST_CELL_ERR = 12,   /* [8] sum (|q| - |v|) per magnitude code, in scaled units */
  ORC_ST_IF4_FP4 = 20,    /* IF4 blocks that kept FP4 */
  ORC_ST_BLOCKS = 21,     /* scale blocks */
  ORC_ST_LEN = 24
};

/* ------------------------------------------------------------------------------------ */
/* Scalar helpers. */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* Nearest bfloat16 to a finite float, ties to the even bfloat16 (the two candidates are the
 * truncation and the next value away from zero; their distances are exact in double). */
static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u = bits_from_f32(f);
  uint32_t lo = u & 0xFFFF0000u;
  if (lo == u) return (uint16_t)(u >> 16);
  uint32_t hi = lo + 0x10000u;
  double dlo = fabs((double)f - (double)f32_from_bits(lo));
  double dhi = fabs((double)f - (double)f32_from_bits(hi));
  if (dlo < dhi) return (uint16_t)(lo >> 16);
  if (dhi < dlo) return (uint16_t)(hi >> 16);
  return ((lo >> 16) & 1u) ? (uint16_t)(hi >> 16) : (uint16_t)(lo >> 16);
}

uint16_t orc_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }

/* ------------------------------------------------------------------------------------ */
/* Number formats [UFP4-A "E2M1：一块刻度不均的尺子", "UFP4：换一把尺子"; IF4 section 2.2 table].
 * Magnitudes are enumerated from the bit fields of each format, not typed in.
 *
 * E2M1: 2 exponent bits (bias 1), 1 mantissa bit.   -> {0, .5, 1, 1.5, 2, 3, 4, 6}
 * E1M2: 1 exponent bit, 2 mantissa bits. The pages print only the value set
 *       {0, .5, ..., 3.5}; bias 0 is the one bias under which this bit layout gives that set.
 * INT4: two's complement, magnitudes 0..7 (IF4 section 2.2: max 7 with an E4M3 scale).   */

static double minifloat_magnitude(int mbits, int bias, int e, int m) {
  double frac = (double)m / (double)(1 << mbits);
  if (e == 0) return ldexp(frac, 1 - bias);    /* subnormal */
  return ldexp(1.0 + frac, e - bias);          /* normal */
}

/* Fills g[0..7] with the non-negative magnitudes of `grid`, indexed by magnitude code, and
 * returns how many codes the grid rounds to (8; 0 for an unknown grid). IF4 uses the E2M1
 * table for its FP4 blocks.
 * Range-restricted E2M1 ["当你的 GPU 学不会算账", section "124B MoE 上的验证": E2M1 limited
 * to a largest value of 2, i.e. {0, .5, 1, 1.5, 2}; "蚂蚁集团揭秘…", section 六: largest
 * value 6 lowered to 4, 3 or 2]: the E2M1 table, of which only the codes up to the new largest
 * magnitude are used (7, 6 or 5 codes); the rest keep their E2M1 values for decoding. */
int orc_grid_magnitudes(int grid, double* g) {
  if (grid == ORC_GRID_E2M1 || grid == ORC_GRID_IF4 || grid == ORC_GRID_E2M1_MAX4 ||
      grid == ORC_GRID_E2M1_MAX3 || grid == ORC_GRID_E2M1_MAX2) {
    for (int c = 0; c < 8; ++c) g[c] = minifloat_magnitude(1, 1, c >> 1, c & 1);
    if (grid == ORC_GRID_E2M1_MAX4) return 7;   /* ... 3, 4 */
    if (grid == ORC_GRID_E2M1_MAX3) return 6;   /* ... 2, 3 */
    if (grid == ORC_GRID_E2M1_MAX2) return 5;   /* ... 1.5, 2 */
    return 8;
  }
  if (grid == ORC_GRID_E1M2) {
    for (int c = 0; c < 8; ++c) g[c] = minifloat_magnitude(2, 0, c >> 2, c & 3);
    return 8;
  }
  if (grid == ORC_GRID_INT4) {
    for (int c = 0; c < 8; ++c) g[c] = (double)c;
    return 8;
  }
  return 0;
}

/* 4-bit code of a signed grid point given its magnitude code. E2M1/E1M2 are
 * sign-magnitude: a negative value that rounds to zero keeps its sign (-0 is 0x8; R6).
 * INT4 is two's complement, so there is no -0. */
static uint8_t encode_nibble(int grid, int negative, int mag) {
  if (grid == ORC_GRID_INT4) {
    int k = negative ? -mag : mag;
    return (uint8_t)(k & 0xF);
  }
  return (uint8_t)((negative ? 8 : 0) | mag);
}

/* Signed value of a 4-bit code on `grid` (IF4's FP4 blocks decode as E2M1). */
double orc_decode_nibble(int grid, uint8_t nib) {
  double g[8];
  orc_grid_magnitudes(grid, g);
  nib &= 0xF;
  if (grid == ORC_GRID_INT4) {
    int k = (nib & 8) ? (int)nib - 16 : (int)nib;
    return (double)k;
  }
  double m = g[nib & 7];
  return (nib & 8) ? -m : m;
}

/* ------------------------------------------------------------------------------------ */
/* Rounding.
 *
 * RTNE [UFP4-B section 二]: the nearest grid point; on a tie the even code (R5). Values at or
 * beyond the largest magnitude map to it (saturation). Below it, distances are exact in double
 * (a float under 8 minus a grid point of few bits); far above it they would not be, which is
 * why saturation is decided first. */

static int nearest_magnitude_code(const double* g, int n, double a) {
  if (a >= g[n - 1]) return n - 1;
  int best = 0;
  double bd = fabs(a - g[0]);
  for (int c = 1; c < n; ++c) {
    double d = fabs(a - g[c]);
    if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
  }
  return best;
}

uint8_t orc_round_rtne(int grid, float v) {
  double g[8];
  int n = orc_grid_magnitudes(grid, g);
  int neg = signbit(v) ? 1 : 0;
  return encode_nibble(grid, neg, nearest_magnitude_code(g, n, fabs((double)v)));
}

/* Stochastic rounding [IF4 section 6.1 pseudo-code: floor(x) + (random() < frac)], applied on
 * the non-uniform grids by its meaning: between the adjacent grid points lo <= |v| <= hi,
 * round away from zero iff r < (|v| - lo) / (hi - lo), with r = u * 2^-16 for the element's
 * 16-bit draw u from the counter hash (R12). |v| is first clamped to the largest magnitude
 * (R4, R13). */
static int sr_magnitude_code(const double* g, int n, double a, uint32_t u) {
  if (a >= g[n - 1]) return n - 1;
  int c = 0;
  while (g[c + 1] <= a) ++c;
  double frac = (a - g[c]) / (g[c + 1] - g[c]);
  double r = (double)(u & 0xFFFFu) * 0x1p-16;
  return (r < frac) ? c + 1 : c;
}

uint8_t orc_round_sr(int grid, float v, uint32_t u) {
  double g[8];
  int n = orc_grid_magnitudes(grid, g);
  int neg = signbit(v) ? 1 : 0;
  return encode_nibble(grid, neg, sr_magnitude_code(g, n, fabs((double)v), u));
}

/* ------------------------------------------------------------------------------------ */
/* Counter-based random source for stochastic rounding (R12).
 * SplitMix64 finalizer (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014): the output for state increment x. */

uint64_t orc_splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* The 16-bit draw u of element `idx` (linear index in its output orientation). The draws are
 * the output stream of the SplitMix64 generator seeded with seed ^ (stream << 63): output k is
 * the finalizer of state seed' + (k + 1) * gamma, i.e. orc_splitmix64(seed' + k * gamma).
 * Elements 4k .. 4k+3 share output k: element 4k + l takes bits 16l .. 16l+15 of it. */
uint32_t orc_sr_bits(uint64_t seed, uint32_t stream, uint64_t idx) {
  uint64_t seed_s = seed ^ ((uint64_t)(stream & 1u) << 63);
  uint64_t h = orc_splitmix64(seed_s + (idx >> 2) * 0x9E3779B97F4A7C15ull);
  return (uint32_t)((h >> (16u * (unsigned)(idx & 3u))) & 0xFFFFu);
}

/* Sign diagonal from a seed (R1): low 16 bits of SplitMix64(seed). */
uint32_t orc_sign_mask_from_seed(uint64_t seed) { return (uint32_t)(orc_splitmix64(seed) & 0xFFFFu); }

/* ------------------------------------------------------------------------------------ */
/* The 16-point Hadamard rotation [UFP4-A "治病药反而喂养了病菌"; UFP4-B sections 四, 六 Q5:
 * block size 16, equal to the quantization block].
 *
 * Sylvester construction H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]; used by the tests only,
 * to pin the butterfly below. */
void orc_sylvester_h16(int32_t* h) {
  int32_t m[16][16];
  m[0][0] = 1;
  for (int n = 1; n < 16; n <<= 1)
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) {
        m[i][j + n] = m[i][j];
        m[i + n][j] = m[i][j];
        m[i + n][j + n] = -m[i][j];
      }
  for (int i = 0; i < 16; ++i)
    for (int j = 0; j < 16; ++j) h[i * 16 + j] = m[i][j];
}

/* Butterfly in fixed order (R3): stages h = 1, 2, 4, 8; each pair (i, i+h) with i & h == 0
 * becomes (a + b, a - b). Output is in natural (Sylvester) order, i.e. v <- H16 v. */
static void butterfly16(float* v) {
  for (int h = 1; h < 16; h <<= 1)
    for (int i = 0; i < 16; ++i)
      if ((i & h) == 0) {
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

/* y = 1/4 * H16 * D * x (R2: signs first). */
void orc_rht16(const float* x, uint32_t mask, float* y) {
  float v[16];
  for (int j = 0; j < 16; ++j) v[j] = ((mask >> j) & 1u) ? -x[j] : x[j];
  butterfly16(v);
  for (int j = 0; j < 16; ++j) y[j] = 0.25f * v[j];
}

/* x = D * 1/4 * H16 * y, the inverse of orc_rht16 (H16 H16 = 16 I and D D = I). */
void orc_inverse_rht16(const float* y, uint32_t mask, float* x) {
  float v[16];
  for (int j = 0; j < 16; ++j) v[j] = y[j];
  butterfly16(v);
  for (int j = 0; j < 16; ++j) {
    float t = 0.25f * v[j];
    x[j] = ((mask >> j) & 1u) ? -t : t;
  }
}

/* ------------------------------------------------------------------------------------ */
/* E4M3 (FP8) block-scale encoding [IF4 section 2.2 table: E4M3 scale, max 448; section 3.2].
 * 4 exponent bits (bias 7), 3 mantissa bits, no infinities, 0x7F is NaN. */

float orc_e4m3_decode(uint8_t b) {
  int e = (b >> 3) & 0xF, m = b & 7;
  double mag = (e == 0) ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return (float)((b & 0x80) ? -mag : mag);
}

/* Nearest non-negative finite E4M3 value, ties to the even code, saturating at 448
 * (R8: "E4M3 by RNE, saturating to 448"). Input is a non-negative float. */
uint8_t orc_e4m3_encode(float x) {
  if (!(x < 448.0f)) return 0x7E;   /* 448 and above (and +inf) saturate */
  int best = 0;
  double bd = fabs((double)x - (double)orc_e4m3_decode(0));
  for (int c = 1; c <= 0x7E; ++c) {
    double d = fabs((double)x - (double)orc_e4m3_decode((uint8_t)c));
    if (d < bd || (d == bd && (c & 1) == 0)) { best = c; bd = d; }
  }
  return (uint8_t)best;
}

/* UE8M0 shared exponent of an MX block (R10, the OCP MX rule): e = floor(log2 amax) - 2,
 * clamped to [-127, 127]; stored as e + 127. floor(log2 amax) comes from frexp. */
int orc_mx_exponent(float amax) {
  if (amax == 0.0f) return -127;
  int ex;
  frexp((double)amax, &ex);        /* amax = f * 2^ex with f in [0.5, 1) */
  int e = (ex - 1) - 2;
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* ------------------------------------------------------------------------------------ */
/* Rotated block loader: y[0..n-1] for n = 16 or 32 elements of one row. */

static void load_rotated(const orc_cfg* cfg, const uint16_t* src, int n, float* y) {
  for (int b = 0; b < n; b += 16) {
    float x[16];
    for (int j = 0; j < 16; ++j) x[j] = bf16_to_f32(src[b + j]);
    if (cfg->rht) orc_rht16(x, cfg->sign_mask, y + b);
    else for (int j = 0; j < 16; ++j) y[b + j] = x[j];
  }
}

/* Amax of the rotated tensor (the NV-family tensor amax A, R8). */
float orc_tensor_amax(const orc_cfg* cfg, const uint16_t* x, int64_t rows, int64_t cols, int64_t ld) {
  float a = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; c += 16) {
      float y[16];
      load_rotated(cfg, x + r * ld + c, 16, y);
      for (int j = 0; j < 16; ++j) if (fabsf(y[j]) > a) a = fabsf(y[j]);
    }
  return a;
}

/* Balanced pairwise sum of 16 floats (R14): ((e0+e1)+(e2+e3)) ... in FP32. */
static float tree_sum16(const float* e) {
  float t[16];
  for (int j = 0; j < 16; ++j) t[j] = e[j];
  for (int h = 1; h < 16; h <<= 1)
    for (int i = 0; i < 16; i += 2 * h) t[i] = t[i] + t[i + h];
  return t[0];
}

static void stats_add_element(double* st, float y, float xhat, int mag, double cell_err) {
  if (!st) return;
  st[ORC_ST_SUM_Y2] += (double)y * (double)y;
  double d = (double)y - (double)xhat;
  st[ORC_ST_SUM_ERR2] += d * d;
  st[ORC_ST_SUM_YXHAT] += (double)y * (double)xhat;
  st[ORC_ST_N] += 1.0;
  st[ORC_ST_CELL_N + mag] += 1.0;
  st[ORC_ST_CELL_ERR + mag] += cell_err;
}

/* ------------------------------------------------------------------------------------ */
/* The quantizer.
 *
 * For every row and every block along the row (the reduction axis):
 *   1. y = rotated block (or x itself when cfg->rht == 0)
 *   2. scale, by format:
 *      FP32 1x16 [UFP4-A recipe table "FP32 单层"; UFP4-B section 五] (R4):
 *          s = amax / qmax   (qmax 6 E2M1, 3.5 E1M2, 7 INT4)
 *      E4M3 1x16 + FP32 tensor scale [IF4 section 3.2] (R8, R9):
 *          alpha = A / (qmax * 448), denom = alpha * qmax, delta = amax / denom,
 *          d8 = E4M3(delta), s = decode(d8) * alpha
 *      UE8M0 1x32 [MXFP4 "MXFP4：一种基于微缩放的低精度数据格式"] (R10):
 *          s = 2^e, e = floor(log2 amax) - 2
 *   3. v = y / s (IEEE division; MX: v = y * 2^-e), then RTNE or SR to the grid
 *   4. IF4 [IF4 sections 3.1, 3.1.1, 3.2] (R11): both the E2M1 candidate and the INT4 candidate
 *      round(v * 7/6) are formed; the one with the smaller squared error in scaled units wins,
 *      ties to FP4; the choice is bit 7 of the E4M3 scale byte; INT4 dequantizes times 6/7.
 *   5. pack: element 2j in the low nibble of byte j (R7); dequant xhat = q * s in FP32, stored
 *      as bfloat16 (R16); statistics (R15).
 * A block whose scale is zero (all of its y are zero) encodes as all-zero codes.
 *
 * codes: [rows, cols/2] bytes. scales: FP32 [rows, cols/16] | u8 [rows, cols/16] |
 * u8 [rows, cols/32]. tensor_scale: alpha (read when tensor_scale_given, else written).
 * row0: logical index of the first row (for the stochastic-rounding counter).
 * deq (optional): bfloat16 [rows, cols]. st (optional): raw statistics, accumulated.
 * Returns 0, or -1 for an invalid configuration or shape. */
int orc_quantize(const orc_cfg* cfg, const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                 int64_t row0, uint8_t* codes, void* scales, float* tensor_scale,
                 int32_t tensor_scale_given, uint16_t* deq, double* st) {
  const int grid = cfg->grid, scale = cfg->scale;
  const int bs = (scale == ORC_SCALE_UE8M0_1x32) ? 32 : 16;
  if (rows < 0 || cols < 0 || cols % bs != 0 || ld < cols) return -1;
  if (grid < 0 || grid > 6 || scale < 0 || scale > 2 || cfg->round < 0 || cfg->round > 1) return -1;
  if (grid == ORC_GRID_IF4 && (scale != ORC_SCALE_E4M3_1x16 || cfg->round != ORC_ROUND_RTNE)) return -1;
  if (scale == ORC_SCALE_UE8M0_1x32 && grid != ORC_GRID_E2M1) return -1;
  if (grid >= ORC_GRID_E2M1_MAX4 && scale != ORC_SCALE_FP32_1x16) return -1;

  double g[8];
  const int ncodes = orc_grid_magnitudes(grid, g);
  const float qmax = (float)g[ncodes - 1];
  const int elem_grid = (grid == ORC_GRID_IF4) ? ORC_GRID_E2M1 : grid;

  float alpha = 0.0f;
  if (scale == ORC_SCALE_E4M3_1x16) {
    if (tensor_scale_given) {
      alpha = *tensor_scale;
    } else {
      float A = orc_tensor_amax(cfg, x, rows, cols, ld);
      float qmax448 = qmax * 448.0f;
      alpha = A / qmax448;
      *tensor_scale = alpha;
    }
  }
  const float r76 = 7.0f / 6.0f;   /* RN(7/6) */
  const float r67 = 6.0f / 7.0f;   /* RN(6/7) */

  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c0 = 0; c0 < cols; c0 += bs) {
      const int64_t bidx = (r * cols + c0) / bs;   /* block index in the scale array */
      float y[32];
      load_rotated(cfg, x + r * ld + c0, bs, y);
      float amax = 0.0f;
      for (int j = 0; j < bs; ++j) if (fabsf(y[j]) > amax) amax = fabsf(y[j]);

      /* -- scale -- */
      float s = 0.0f;       /* dequant multiplier */
      float inv_pow2 = 0.0f; /* MX only: 2^-e */
      uint8_t sbyte = 0;
      if (scale == ORC_SCALE_FP32_1x16) {
        s = amax / qmax;
        ((float*)scales)[bidx] = s;
      } else if (scale == ORC_SCALE_E4M3_1x16) {
        float denom = alpha * qmax;
        float delta = (denom > 0.0f) ? amax / denom : 0.0f;
        sbyte = orc_e4m3_encode(delta);
        s = orc_e4m3_decode(sbyte) * alpha;
      } else {
        int e = orc_mx_exponent(amax);
        sbyte = (uint8_t)(e + 127);
        s = ldexpf(1.0f, e);
        inv_pow2 = ldexpf(1.0f, -e);
        ((uint8_t*)scales)[bidx] = sbyte;
      }
      const int zero_block = (scale == ORC_SCALE_UE8M0_1x32) ? (amax == 0.0f) : (s == 0.0f);

      /* -- scaled values -- */
      float v[32];
      for (int j = 0; j < bs; ++j) {
        if (zero_block) v[j] = 0.0f;
        else if (scale == ORC_SCALE_UE8M0_1x32) v[j] = y[j] * inv_pow2;
        else v[j] = y[j] / s;
      }

      /* -- round -- */
      uint8_t nib[32];
      float val[32];   /* dequant value in scaled units (the grid point, or INT4 * 6/7) */
      int mag[32];
      int use_int = 0;
      for (int j = 0; j < bs; ++j) {
        if (zero_block) { nib[j] = 0; val[j] = 0.0f; mag[j] = 0; continue; }
        if (cfg->round == ORC_ROUND_SR) {
          uint64_t idx = (uint64_t)((row0 + r) * cols + c0 + j);
          nib[j] = orc_round_sr(elem_grid, v[j], orc_sr_bits(cfg->sr_seed, cfg->sr_stream, idx));
        } else {
          nib[j] = orc_round_rtne(elem_grid, v[j]);
        }
        val[j] = (float)orc_decode_nibble(elem_grid, nib[j]);
        mag[j] = (elem_grid == ORC_GRID_INT4) ? (int)fabs((double)val[j]) : (nib[j] & 7);
      }
      if (grid == ORC_GRID_IF4 && !zero_block) {
        uint8_t nib_i[16];
        float val_i[16], e_fp[16], e_int[16];
        for (int j = 0; j < 16; ++j) {
          float w = v[j] * r76;
          nib_i[j] = orc_round_rtne(ORC_GRID_INT4, w);
          float k = (float)orc_decode_nibble(ORC_GRID_INT4, nib_i[j]);
          val_i[j] = k * r67;
          float dfp = val[j] - v[j], dint = val_i[j] - v[j];
          e_fp[j] = dfp * dfp;
          e_int[j] = dint * dint;
        }
        float sse_fp = tree_sum16(e_fp), sse_int = tree_sum16(e_int);
        use_int = sse_int < sse_fp;
        if (use_int)
          for (int j = 0; j < 16; ++j) {
            nib[j] = nib_i[j];
            val[j] = val_i[j];
            mag[j] = (int)fabs((double)orc_decode_nibble(ORC_GRID_INT4, nib_i[j]));
          }
      }
      if (scale == ORC_SCALE_E4M3_1x16)
        ((uint8_t*)scales)[bidx] = (uint8_t)(sbyte | (use_int ? 0x80 : 0));

      /* -- pack, dequant, stats -- */
      for (int j = 0; j < bs; ++j) {
        int64_t e = r * cols + c0 + j;
        if ((j & 1) == 0) codes[e >> 1] = nib[j];
        else codes[e >> 1] |= (uint8_t)(nib[j] << 4);
        float xhat = zero_block ? 0.0f : val[j] * s;
        if (deq) deq[e] = f32_to_bf16_rne(xhat);
        if (st) {
          double cell_err = zero_block ? 0.0 : fabs((double)val[j]) - fabs((double)v[j]);
          stats_add_element(st, y[j], xhat, mag[j], cell_err);
        }
      }
      if (st) {
        st[ORC_ST_BLOCKS] += 1.0;
        if (grid == ORC_GRID_IF4 && !use_int) st[ORC_ST_IF4_FP4] += 1.0;
      }
    }
  }
  return 0;
}

/* Dequantize codes back to bfloat16: xhat = q * s in FP32 (IF4 INT4 blocks: (k * 6/7) * s),
 * optionally followed by the inverse rotation x = D * 1/4 * H16 * xhat per 16-block in FP32.
 * Returns 0, or -1 for an invalid configuration. */
int orc_dequantize(const orc_cfg* cfg, const uint8_t* codes, const void* scales,
                   float tensor_scale, int64_t rows, int64_t cols, int32_t inverse_rht,
                   uint16_t* out) {
  const int grid = cfg->grid, scale = cfg->scale;
  const int bs = (scale == ORC_SCALE_UE8M0_1x32) ? 32 : 16;
  if (rows < 0 || cols < 0 || cols % bs != 0) return -1;
  if (grid == ORC_GRID_IF4 && scale != ORC_SCALE_E4M3_1x16) return -1;
  if (scale == ORC_SCALE_UE8M0_1x32 && grid != ORC_GRID_E2M1) return -1;
  const float r67 = 6.0f / 7.0f;
  const int elem_grid = (grid == ORC_GRID_IF4) ? ORC_GRID_E2M1 : grid;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c0 = 0; c0 < cols; c0 += 16) {
      float xh[16];
      int64_t bidx = (r * cols + c0) / bs;
      float s;
      int int_block = 0;
      if (scale == ORC_SCALE_FP32_1x16) {
        s = ((const float*)scales)[bidx];
      } else if (scale == ORC_SCALE_E4M3_1x16) {
        uint8_t b = ((const uint8_t*)scales)[bidx];
        int_block = (grid == ORC_GRID_IF4) && (b & 0x80);
        s = orc_e4m3_decode((uint8_t)(b & 0x7F)) * tensor_scale;
      } else {
        s = ldexpf(1.0f, (int)((const uint8_t*)scales)[bidx] - 127);
      }
      for (int j = 0; j < 16; ++j) {
        int64_t e = r * cols + c0 + j;
        uint8_t nib = (uint8_t)((codes[e >> 1] >> ((e & 1) ? 4 : 0)) & 0xF);
        float val;
        if (int_block) val = (float)orc_decode_nibble(ORC_GRID_INT4, nib) * r67;
        else val = (float)orc_decode_nibble(elem_grid, nib);
        xh[j] = val * s;
      }
      if (inverse_rht) {
        float xr[16];
        orc_inverse_rht16(xh, cfg->sign_mask, xr);
        for (int j = 0; j < 16; ++j) out[r * cols + c0 + j] = f32_to_bf16_rne(xr[j]);
      } else {
        for (int j = 0; j < 16; ++j) out[r * cols + c0 + j] = f32_to_bf16_rne(xh[j]);
      }
    }
  }
  return 0;
}

/* The rotation alone, as the first pass of the unfused pipeline: y = 1/4 H16 D x per 16-block,
 * written as FP32 (exact) and as bfloat16 (RNE of the FP32 value); either output may be NULL. */
int orc_rht16_rows(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t mask,
                   float* y_f32, uint16_t* y_bf16) {
  if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return -1;
  orc_cfg cfg;
  memset(&cfg, 0, sizeof cfg);
  cfg.rht = 1;
  cfg.sign_mask = mask;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c0 = 0; c0 < cols; c0 += 16) {
      float y[16];
      load_rotated(&cfg, x + r * ld + c0, 16, y);
      for (int j = 0; j < 16; ++j) {
        if (y_f32) y_f32[r * cols + c0 + j] = y[j];
        if (y_bf16) y_bf16[r * cols + c0 + j] = f32_to_bf16_rne(y[j]);
      }
    }
  return 0;
}

/* ------------------------------------------------------------------------------------ */
/* Array forms of the scalar rules, for exhaustive tests. */

void orc_round_rtne_n(int grid, const float* v, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_round_rtne(grid, v[i]);
}

void orc_round_sr_n(int grid, const float* v, const uint32_t* u, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_round_sr(grid, v[i], u[i]);
}

void orc_e4m3_encode_n(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}

void orc_f32_to_bf16_n(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(x[i]);
}

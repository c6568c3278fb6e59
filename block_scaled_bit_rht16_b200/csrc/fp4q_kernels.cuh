// fp4q_kernels.cuh -- kernel argument blocks and launch entry points shared by the host layer.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace fp4q {

// kE2M1Max4/3/2: E2M1 with the largest magnitude lowered to 4, 3 or 2 (internal ids; the C
// ABI selects them with fp4q_config.e2m1_max). Codes and decoding are E2M1's.
enum Grid { kE2M1 = 0, kE1M2 = 1, kINT4 = 2, kIF4 = 3, kE2M1Max4 = 4, kE2M1Max3 = 5, kE2M1Max2 = 6 };

// Grids encoded by the E2M1 converter (the full table or a range-restricted one).
template <int G> constexpr bool kIsE2M1 = (G == kE2M1 || G == kE2M1Max4 || G == kE2M1Max3 || G == kE2M1Max2);
enum Scale { kFP32 = 0, kE4M3 = 1, kUE8M0 = 2 };
enum Round { kRTNE = 0, kSR = 1 };

// Raw statistics record (doubles), one per CTA in the workspace and once reduced.
enum {
  ST_SUM_Y2 = 0, ST_SUM_ERR2 = 1, ST_SUM_YXHAT = 2, ST_N = 3, ST_CELL_N = 4, ST_CELL_ERR = 12,
  ST_IF4_FP4 = 20, ST_BLOCKS = 21, ST_LEN = 24
};

// Workspace layout: a 256-byte header, then (with statistics) kStatsCtas raw records.
struct WsHeader {
  uint32_t magic;       // kWsMagic once a statistics-producing call has been enqueued
  uint32_t n_partials;  // raw records that follow
  uint32_t amax_bits;   // rotated-tensor amax (bit pattern of a non-negative float)
  int32_t status;       // device status word (0 ok)
  double reduced[ST_LEN];  // fp4q_stats writes the fixed-order reduction here
  uint8_t pad[256 - 16 - 8 * ST_LEN];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");
constexpr uint32_t kWsMagic = 0x51345046u;   // "FP4Q"
constexpr int kStatsCtas = 512;               // fixed grid of statistics-producing launches
constexpr int kThreads = 256;

struct QuantArgs {
  const uint16_t* x;
  int64_t rows, cols, ld;
  int64_t nunits;          // blocks of 16 (32 for UE8M0) in the tensor
  int64_t units_per_row;
  uint8_t* codes;
  void* scales;
  uint16_t* deq;           // optional
  const float* ts_in;      // E4M3: alpha supplied by the caller
  float* ts_out;           // E4M3: where the computed alpha goes
  WsHeader* ws;            // header (amax, status) or null
  double* partials;        // statistics records or null
  uint32_t sw[8];          // sign flips per bf16 pair (all 0 without rotation)
  uint32_t flip_lo[8], flip_hi[8];   // the same flips at bit 31: element 2k / 2k+1 of a block
  float c, cinv;           // 4, 1/4 with rotation; 1, 1 without
  uint64_t seedx;          // SR: seed ^ (stream << 63)
  int contiguous;          // ld == cols
  int vec32;               // every unit starts 32-byte aligned: one 256-bit load per 16 elements
  int mma_scales;          // E4M3 / UE8M0 scales in the block-scaled MMA tile layout
  // grouped (E4M3): rows [group_off[g], group_off[g+1]) form group g, with tensor scale
  // group_ts[g]; group_amax: per-group rotated amax bits (workspace) for the computed scales
  const int64_t* group_off;
  int32_t n_groups;
  float* group_ts;
  uint32_t* group_amax;
};

// Byte position of scale (r, c) of a [rows, C] scale matrix in the scale-factor layout that
// sm_100 block-scaled MMA (NVFP4 / MXFP4) consumes: 512-byte tiles of 128 rows x 4 columns,
// row-major over tiles (C / 4 tiles per tile row); inside a tile, row r and column c sit at
// (r % 32) * 16 + (r / 32 % 4) * 4 + c % 4. Needs rows % 128 == 0 and C % 4 == 0.
__host__ __device__ inline int64_t mma_scale_slot(int64_t r, int64_t c, int64_t C) {
  return ((r >> 7) * (C >> 2) + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// Slot of block u (row-major block index, C scale columns per row) in either layout.
__host__ __device__ inline int64_t scale_slot(int64_t u, int64_t C, int mma) {
  if (!mma) return u;
  const int64_t r = u / C;
  return mma_scale_slot(r, u - r * C, C);
}

struct DualArgs {
  const uint16_t* dy;
  int64_t M, N, ld;
  uint8_t* codes_row; float* scales_row;
  uint8_t* codes_col; float* scales_col;
  uint32_t flip_lo_row[8], flip_hi_row[8];   // row blocks: bit 31 flips elements 2k / 2k+1
  uint32_t flip_col[16];    // column blocks: bit 31 flips element i (both columns of a word)
  int vec32;                // dy 32-byte aligned and ld % 16 == 0: 256-bit row-block loads
  int col16;                // M % 64 == 0 and codes_col, scales_col 16-byte aligned
  float c_row, cinv_row, c_col, cinv_col;
  uint64_t seedx_row, seedx_col;
  int round_row, round_col;   // per orientation
  int grid_row, grid_col;
};

// Host: the per-element flips at bit 31 from sign words sw (bit 15: element 2k, bit 31:
// element 2k+1), the form unpack16 adds to the unpacked bf16 halves.
inline void sign_flips(const uint32_t* sw, uint32_t* flip_lo, uint32_t* flip_hi) {
  for (int k = 0; k < 8; ++k) {
    flip_lo[k] = (sw[k] & 0x8000u) << 16;
    flip_hi[k] = sw[k] & 0x80000000u;
  }
}

// Bits of the device status word (defined in fp4q_row.cu): bit 0 a bounded wait in a kernel gave
// up (the GEMM's waits on its tile copies and MMAs), bit 1 the timeout self-test fired. Sticky
// until read with clear.
constexpr int32_t kStatusWaitTimeout = 1;
constexpr int32_t kStatusSelfTest = 2;

}  // namespace fp4q

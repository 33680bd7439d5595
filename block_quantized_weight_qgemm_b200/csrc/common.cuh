// common.cuh -- definitions shared by the host layer and the kernels of libqgemm.
#pragma once
#include <cuda.h>
#include <cstdint>

namespace qg {

enum Fmt : int { FMT_Q8_0 = 0, FMT_NVFP4 = 1, FMT_MXFP4 = 2 };

// ---- tile geometry (tcgen05, swap-AB: weight rows are the MMA M dimension) -------------
constexpr int kTileRows = 128;                    // weight rows per subtile (MMA M)
constexpr int kWRowBytes = 128;                   // code bytes per row in one weight stage
constexpr int kWCodeBytes = kTileRows * kWRowBytes;        // 16 KB, 128-byte swizzled
constexpr int kScaleRowBytes = 16;                // scale bytes per row in one weight stage
constexpr int kWStageBytes = kWCodeBytes + kTileRows * kScaleRowBytes;  // 18 KB
constexpr int kSubK = 64;                         // K per x stage (one 128-byte swizzle atom)
constexpr int kAStageK = 128;                     // K per A stage (TMEM)
constexpr int kMaxAStages = 4;                    // A ring depth limit
constexpr int kAColsPerStage = kAStageK / 2;      // 16-bit elements, 2 per TMEM column
constexpr int kDequantWarps = 8;                  // 2 per TMEM lane quarter
constexpr int kThreads = (2 + kDequantWarps) * 32;
constexpr int kMaxNB = 256;                       // MMA N limit
constexpr int kSmemLimit = 227 * 1024;

// K covered by one weight stage (128 code bytes per row).
__host__ __device__ constexpr int chunk_k(int fmt) { return fmt == FMT_Q8_0 ? 128 : 256; }
__host__ __device__ constexpr int block_k(int fmt) { return fmt == FMT_NVFP4 ? 16 : 32; }
__host__ __device__ constexpr int64_t roundup16(int64_t v) { return (v + 15) / 16 * 16; }
__host__ __device__ constexpr int64_t code_pitch(int fmt, int64_t K) {
  return fmt == FMT_Q8_0 ? roundup16(K) : roundup16(K / 2);
}
__host__ __device__ constexpr int64_t scale_pitch(int fmt, int64_t K) {
  return fmt == FMT_Q8_0 ? roundup16(K / 16) : fmt == FMT_NVFP4 ? roundup16(K / 16) : roundup16(K / 32);
}

// Everything the GEMM kernel needs besides its tensor maps.
struct GemmParams {
  int N, K, B;
  int NB;        // batch columns per tile (MMA N), multiple of 16, <= 256
  int R;         // weight subtiles (of 128 rows) sharing each x stage
  int NMAT;      // 1: plain GEMM; 2: fused gate/up (subtile r reads matrix r % 2)
  int S;         // K splits (fixed by fmt, N, K for B <= 256)
  int n_groups;  // ceil(row tiles / (R / NMAT))
  int b_tiles;   // ceil(B / NB)
  int chunks;    // ceil(K / chunk_k)
  int XS, WS;    // x ring and weight ring depths
  int AS;        // A ring depth (TMEM stages of kAStageK)
  int tmem_cols; // allocated TMEM columns
  uint32_t smem_x, smem_w, smem_bar;  // byte offsets in the 1024-aligned dynamic smem
  const int* x_exp;          // f16 operands: x row b was scaled by 2^-x_exp[b]
  const float* ts[2];        // NVFP4 tensor scales (device), else nullptr
  const uint8_t* scales[2];  // packed scales (MXFP4 exponent pre-pass)
  int64_t spitch;            // scale row pitch
  float* ws;                 // split-K partials [S][NMAT][B][N]
  int* counters;             // [n_groups * b_tiles], zero on entry, left zero
  void* out;                 // y [B][N] (fp32 or bf16), or h [B][N] bf16 for NMAT == 2
  int out_bf16;
  int* dev_err;
};

// Per-row power-of-two scaling of x before the bf16 -> f16 conversion.
struct PrepParams {
  const uint16_t* x;  // bf16 [B][K]
  uint16_t* xh;       // f16 [B][K]
  int* x_exp;         // [B]
  int B, K;
  int* counters;      // zeroed here (split-K arrival counters of the following GEMM)
  int n_counters;
};

// Device error codes written to the library's error word.
constexpr int kErrTimeout = 1;

}  // namespace qg

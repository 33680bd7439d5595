// common.cuh -- definitions shared by the host layer and the kernels of libqgemm.
#pragma once
#include <cuda.h>
#include <cstdint>

namespace qg {

enum Fmt : int { FMT_Q8_0 = 0, FMT_NVFP4 = 1, FMT_MXFP4 = 2, FMT_FP8 = 3 };

// ---- tile geometry (tcgen05, swap-AB: weight rows are the MMA M dimension) -------------
constexpr int kTileRows = 128;                    // weight rows per subtile (MMA M)
constexpr int kWRowBytes = 128;                   // code bytes per row in one weight stage
constexpr int kWCodeBytes = kTileRows * kWRowBytes;        // 16 KB, 128-byte swizzled
constexpr int kSubK = 64;                         // K per x stage (one 128-byte swizzle atom)
constexpr int kMaxWStages = 8;                    // weight ring depth limit
// CTA-pair kernel: warp 0 producer, warp 1 TMEM owner / pair MMA issuer, then dequant warps
constexpr int kPairDequantWarps = 8;              // 2 per TMEM lane quarter
constexpr int kPairFirstDequantWarp = 2;
constexpr int kPairIssuer2Warp = kPairFirstDequantWarp + kPairDequantWarps;  // second MMA issuer
constexpr int kPairXWarp = kPairIssuer2Warp + 1;  // x producer
constexpr int kPairThreads = (kPairXWarp + 1) * 32;
constexpr int kPairSMs = 74;                      // CTA pairs resident at once (148 SMs)
constexpr int kPairAK = 256;                      // K per weight stage / x group of the pair kernel
constexpr int kPairSlotK = 128;                   // K per A slot (one half of a stage)
constexpr int kPairACols = kPairSlotK / 2;        // its TMEM columns (f16 pairs)
constexpr int kMaxNB = 256;                       // MMA N limit
constexpr int kSmemLimit = 227 * 1024;

// one byte per element (Q8_0, FP8) or two (NVFP4, MXFP4)
__host__ __device__ constexpr bool byte_codes(int fmt) { return fmt == FMT_Q8_0 || fmt == FMT_FP8; }
// K covered by one weight stage (128 code bytes per row).
__host__ __device__ constexpr int chunk_k(int fmt) { return byte_codes(fmt) ? 128 : 256; }
// K granularity: the scale block (FP8 has none; 16 keeps every x row 32-byte aligned)
__host__ __device__ constexpr int block_k(int fmt) {
  return (fmt == FMT_NVFP4 || fmt == FMT_FP8) ? 16 : 32;
}
// scale bytes per row per chunk: Q8_0 4 x fp16, NVFP4 16 x E4M3, MXFP4 8 x E8M0, FP8 none
__host__ __device__ constexpr int scale_row_bytes(int fmt) {
  return fmt == FMT_NVFP4 ? 16 : fmt == FMT_FP8 ? 0 : 8;
}
// formats with an fp32 tensor scale applied in the epilogue
__host__ __device__ constexpr bool has_tensor_scale(int fmt) {
  return fmt == FMT_NVFP4 || fmt == FMT_FP8;
}
__host__ __device__ constexpr int64_t row_tiles(int64_t N) { return (N + kTileRows - 1) / kTileRows; }
__host__ __device__ constexpr int64_t k_chunks(int fmt, int64_t K) {
  return (K + chunk_k(fmt) - 1) / chunk_k(fmt);
}
// Weight stage of the pair kernel: one A slot of one subtile, i.e. kPairAK / chunk_k chunks
// of a 128-row tile (contiguous in the tile-major layout): their codes, then their scales.
__host__ __device__ constexpr int pair_wstage_bytes(int fmt) {
  return (kPairAK / chunk_k(fmt)) * (kWCodeBytes + kTileRows * scale_row_bytes(fmt));
}
// Row-major interchange layout (qgemm_repack_rowmajor input): codes [N][code pitch],
// scales [N][scale pitch], rows 16-byte aligned.
__host__ __device__ constexpr int64_t roundup16(int64_t v) { return (v + 15) / 16 * 16; }
__host__ __device__ constexpr int64_t rm_code_bytes_per_row(int fmt, int64_t K) {
  return byte_codes(fmt) ? K : K / 2;
}
__host__ __device__ constexpr int64_t rm_scale_bytes_per_row(int fmt, int64_t K) {
  return fmt == FMT_Q8_0 ? 2 * (K / 32) : fmt == FMT_NVFP4 ? K / 16 : fmt == FMT_FP8 ? 0 : K / 32;
}
__host__ __device__ constexpr int64_t rm_code_pitch(int fmt, int64_t K) {
  return roundup16(rm_code_bytes_per_row(fmt, K));
}
__host__ __device__ constexpr int64_t rm_scale_pitch(int fmt, int64_t K) {
  return roundup16(rm_scale_bytes_per_row(fmt, K));
}
// Tile-major packed layout: for row tile t and chunk c, one contiguous block of
// 128 rows x 128 code bytes (16-byte groups of row r stored at group ^ (r & 7)) and one
// contiguous block of 128 rows x scale_row_bytes.
__host__ __device__ constexpr int64_t packed_code_bytes(int fmt, int64_t N, int64_t K) {
  return row_tiles(N) * k_chunks(fmt, K) * kWCodeBytes;
}
__host__ __device__ constexpr int64_t packed_scale_bytes(int fmt, int64_t N, int64_t K) {
  return row_tiles(N) * k_chunks(fmt, K) * kTileRows * scale_row_bytes(fmt);
}
// byte offset of code byte `b` (0..127) of row n, chunk c
__host__ __device__ constexpr int64_t code_offset(int64_t C, int64_t n, int64_t c, int b) {
  return (((n / kTileRows) * C + c) * kTileRows + (n % kTileRows)) * kWRowBytes +
         ((((b >> 4) ^ (int)(n & 7)) << 4) | (b & 15));
}
// byte offset of the scale bytes of row n, chunk c
__host__ __device__ constexpr int64_t scale_offset(int fmt, int64_t C, int64_t n, int64_t c) {
  return (((n / kTileRows) * C + c) * kTileRows + (n % kTileRows)) * scale_row_bytes(fmt);
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
  int units;     // work units of the call; the persistent grid's CTA pairs share them out
  int chunks;    // ceil(K / chunk_k)
  int XS, WS;    // x ring and weight ring depths
  int AS;        // A ring depth (TMEM slots of kPairSlotK; even: each stage half owns AS/2)
  int tmem_cols; // allocated TMEM columns
  int x3d;       // pair kernel: x map is 3-D {64, B, K/64} (one TMA load per x stage)
  int NACC;      // pair kernel: accumulators per subtile (1, or 2 for the f16 path)
  uint32_t smem_x, smem_w, smem_bar;  // byte offsets in the 1024-aligned dynamic smem
  const int* x_exp;          // f16 operands: x row b was scaled by 2^-x_exp[b]
  const float* ts[2];        // NVFP4 / FP8 tensor scales (device), else nullptr
  const uint8_t* codes[2];   // tile-major packed codes of each matrix
  const uint8_t* scales[2];  // tile-major packed scales of each matrix
  float* ws;                 // split-K partials [S][NMAT][B][N], fully scaled
  void* out;                 // y [B][N] (fp32 or bf16), or h [B][N] bf16 for NMAT == 2
  int out_bf16;
  int* dev_err;
  // Grouped experts (routed mixture-of-experts): when moe_off is set, x's B rows are grouped
  // by expert (rows moe_off[e] .. moe_off[e+1]-1 belong to expert e, offsets clamped to
  // [0, B]); a work unit is (expert, row-tile pair group, batch tile) with S = 1, and expert
  // e's weights come from the device pointer tables below instead of codes/scales/ts.
  const int* moe_off;
  const uint8_t* const* moe_codes[2];
  const uint8_t* const* moe_scales[2];
  const float* const* moe_ts[2];
};

// Fixed-order sum of the split-K partials and the output epilogue.  The partials carry every
// scale already (the GEMM epilogue applies the tensor scale and the powers of two).
struct ReduceParams {
  const float* ws;     // partials [S][NMAT][B][N]
  int S, NMAT, B, N;
  void* out;           // y [B][N] fp32 / bf16, or h [B][N] bf16 for NMAT == 2
  int out_bf16;
};

// Conversion of the row-major packed layout into the tile-major one.
struct RepackParams {
  const uint8_t* codes_rm;
  const uint8_t* scales_rm;
  int64_t code_pitch, scale_pitch;  // row pitches of the row-major arrays (bytes)
  uint8_t* codes;
  uint8_t* scales;
  int64_t N, K;
  int fmt;
};

// Per-row power-of-two scaling of x before the bf16 -> f16 conversion.
struct PrepParams {
  const uint16_t* x;  // bf16 [B][K]
  uint16_t* xh;       // f16 [B][Kp], columns K..Kp-1 zero
  int* x_exp;         // [B]
  int B, K, Kp;       // Kp: row pitch of xh in elements (K rounded up to 64)
};

// Device error codes written to the library's error word.
constexpr int kErrTimeout = 1;
constexpr int kErrArg = 2;  // an argument found in device memory is invalid (an expert table entry)

}  // namespace qg

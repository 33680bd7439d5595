// bs.cu -- the block-scaled tensor-core path (sm_100a).
//
// y[m][n] = sum_k x[m][k] * dequant(W)[n][k] with W in MXFP4 (E2M1 codes, one E8M0 scale per
// 32 elements; OCP Microscaling format as the Atlas issue's "Fix: F16 operands with an exact
// dequant" section describes it), NVFP4 (E2M1, one UE4M3 scale per 16, a tensor scale) or FP8
// (E4M3 with a tensor scale), and x in bf16, on tcgen05.mma.kind::mxf4nvf4 (FP4) or
// kind::mxf8f6f4 (FP8) with block scales on both operands, so that the packed weights reach
// the tensor cores as they are, without a dequantisation pass.
//
// x is not an MMA type here.  The split kernel writes each row as the sum of terms in the
// weights' element kind with their own power-of-two scale per block: per block, r_0 = x *
// 2^-x_exp (x_exp = the row's floor(log2 max|x|) less a per-format shift, an exact power of
// two that the epilogue restores), e_j = floor(log2 max|r_j|) - top, q_j = CODE(r_j / 2^e_j)
// (round to nearest even, saturating), r_{j+1} = r_j - q_j 2^e_j.  Three E2M1 terms (top 2)
// leave a residual below 2^-6 of each block's maximum before rounding; two E4M3 terms (top 7)
// one below 2^-8.  Measured against the exact product the normalised error is below 1e-4 at
// the 27B shapes.  A term whose scale would fall below the scale type's range is dropped.
//
// Layout of the split x (device, written by qgemm_bs_split_x, read by the GEMM), with CK = 256
// (FP4) or 128 (FP8) elements per chunk and T = 3 (FP4) or 2 (FP8) terms:
//   codes : [Mt][C][T][128 rows][128 bytes]   Mt = ceil(M/128) token tiles, C = ceil(K/CK)
//           chunks; row r of a (tile, chunk, term) block holds elements CK c .. CK c + CK-1 of
//           token 128 t + r (E2M1: two per byte, even element in the low nibble; E4M3: one per
//           byte), its 16-byte groups stored at group ^ (r & 7) (the 128-byte swizzle of the
//           MMA operand, as the tile-major weights).  Tokens past M and elements past K are 0.
//   scales: [Mt][C][T][128 rows][sbr]   one scale byte per block (sbr 8 MXFP4, 16 NVFP4, 4 FP8).
//   x_exp : [Mt * 128] int32.
//
// Prefill GEMM (more than 128 rows): one CTA per SM (persistent).  A tile is 128 tokens (MMA M,
// the x terms as operand A) x 256 weight rows (MMA N, two tile-major weight tiles as operand B)
// over all of K.  Per chunk the producer brings the x-term blocks and the two weight blocks
// with their scales into one of the shared-memory stages (1-D bulk copies); four staging warps
// place the stage's scale factors in tensor memory with tcgen05.st in the layout the
// block-scaled MMA reads (per MMA K-block: scale j of row r = r0 + 32 r1 at lane r0 of every
// lane quarter, column r1, byte j); one thread issues 4 K-blocks x T terms of M128 N256 MMAs
// into one fp32 accumulator; four epilogue warps read it out, restore 2^x_exp (and the tensor
// scale) and store y.  Decode widths use the second kernel below, with the operands' roles
// swapped.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "common.cuh"
#include "ptx.cuh"

namespace qg {

constexpr int kBsM = 128;                     // tokens per tile
constexpr int kBsWT = 2;                      // weight tiles (of 128 rows) per tile
constexpr int kBsN = 128 * kBsWT;             // weight rows per tile (MMA N)
// (one weight tile per tile with three stages measured faster only at M = 2048 of the
// 5120 x 17408 MXFP4 shape and slower at M = 8192: x is then re-read for every 128 weight rows)
constexpr int kBsBlock = kBsM * 128;          // one 128-row x 128-byte code block: 16 KB
constexpr int kBsBCodes = kBsWT * kBsBlock;
constexpr int kBsKB = 4;                      // MMA K-blocks per chunk (32 bytes of codes each)
constexpr int kBsTmemCols = 512;
constexpr int kBsEpiWarp0 = 6;    // warps 6..9 run the epilogue
constexpr int kBsThreads = 10 * 32;

// Weight formats of the path: 0 MXFP4, 1 NVFP4 (both kind::mxf4nvf4, E2M1 operands),
// 2 FP8 E4M3 with a per-tensor scale (kind::mxf8f6f4, E4M3 operands).
constexpr int kBsMx = 0, kBsNv = 1, kBsF8 = 2;

struct BsSplitParams {
  const uint16_t* x;  // bf16 [M][K]
  int M, K, C, Mt;
  int f;              // weight format (kBsMx, kBsNv, kBsF8)
  uint8_t* codes;     // [Mt][C][terms][128][128]
  uint8_t* scales;    // [Mt][C][terms][128][sbr]
  int* x_exp;
};

// Parameters of the split per weight format: terms, K per chunk (one weight chunk of the
// tile-major layout), block size, prescale shift (the row maximum lands in
// [2^xshift, 2^(xshift+1))), smallest block-scale exponent, top (the block maximum / 2^e lands
// in [2^top, 2^(top+1))), x-term and weight scale bytes per row and chunk.  MXFP4: three E2M1
// terms, E8M0 scales per 32 elements, whose range covers every bf16 row after a prescale to
// [1, 2).  NVFP4: three E2M1 terms, UE4M3 scales per 16, restricted to the powers of two it
// holds exactly (2^-9 .. 2^8, so that every step stays exact); the prescale to [2^10, 2^11)
// keeps every block scale <= 2^8 and gives blocks 2^17 of range below the row maximum.  FP8:
// two E4M3 terms with E8M0 scales per 32 (the weights carry only a per-tensor scale; their
// block scales are 1).
__host__ __device__ constexpr int bs_terms(int f) { return f == kBsF8 ? 2 : 3; }
__host__ __device__ constexpr int bs_chunk(int f) { return f == kBsF8 ? 128 : 256; }
__host__ __device__ constexpr int bs_blk(int f) { return f == kBsNv ? 16 : 32; }
__host__ __device__ constexpr int bs_xshift(int f) { return f == kBsNv ? 10 : 0; }
__host__ __device__ constexpr int bs_emin(int f) { return f == kBsNv ? -9 : -127; }
__host__ __device__ constexpr int bs_top(int f) { return f == kBsF8 ? 7 : 2; }
__host__ __device__ constexpr int bs_sbr(int f) { return f == kBsNv ? 16 : (f == kBsF8 ? 4 : 8); }
__host__ __device__ constexpr int bs_wsbr(int f) { return f == kBsNv ? 16 : (f == kBsF8 ? 0 : 8); }
// The scale byte of 2^e: E8M0 e + 127; UE4M3 (bias 7, three mantissa bits) (e + 7) << 3 for a
// normal value, 2^(e + 9) as the subnormal mantissa below 2^-6.
__host__ __device__ constexpr int bs_scale_byte(int f, int e) {
  return f == kBsNv ? (e >= -6 ? (e + 7) << 3 : 1 << (e + 9)) : e + 127;
}

// Instruction descriptor of the block-scaled MMA with M = 128 and N = n, both operands
// K-major, scale factor ids 0.  kind::mxf4nvf4: A and B E2M1 (format 1), K = 64 per
// instruction, scale type UE4M3 (NVFP4) or E8M0 (MXFP4).  kind::mxf8f6f4: A and B E4M3
// (format 0), K = 32 per instruction, scale type E8M0.
__host__ __device__ constexpr uint32_t bs_idesc(int f, int n) {
  return (f == kBsF8 ? 0u : ((1u << 7) | (1u << 10))) | ((uint32_t)(n >> 3) << 17) |
         ((f == kBsNv ? 0u : 1u) << 23) | ((uint32_t)(kBsM >> 4) << 24);
}

// Prefill-kernel stage layout per weight format: [x-term codes terms x 16 KB][weight codes
// 32 KB][x-term scales terms x 128 x sbr][weight scales 2 x 128 x wsbr] (85 KB MXFP4, 90 KB
// NVFP4, 65 KB FP8).  Tensor memory: the accumulator in columns [0, 256), then per stage SfCols
// columns of scale factors: x term t, K-block kb at (t * 4 + kb) * 4 (4 columns: row groups
// r1 = 0..3), the weights' K-block kb at ASf + kb * 8 (8 columns: r1 = 0..7).
template <int F>
struct BsLay {
  static constexpr int Terms = bs_terms(F);
  static constexpr int ACodes = Terms * kBsBlock;
  static constexpr int SB = kBsM * bs_sbr(F);    // x-term scales of one 128-row block
  static constexpr int WSB = kBsM * bs_wsbr(F);  // weight scales of one 128-row block
  static constexpr int AScales = Terms * SB;
  static constexpr int BScales = kBsWT * WSB;
  static constexpr int Stage = ACodes + kBsBCodes + AScales + BScales;
  static constexpr int Stages = F == kBsF8 ? 3 : 2;  // FP8 chunks hold half the K
  static constexpr int ASf = Terms * kBsKB * 4;
  static constexpr int SfCols = ASf + kBsKB * 4 * kBsWT;
  static constexpr int Smem = 1024 + Stages * Stage + 256;
  static constexpr uint32_t Idesc = bs_idesc(F, kBsN);
  static_assert(Stage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(Smem <= 227 * 1024, "shared memory");
  static_assert(kBsN + Stages * SfCols <= kBsTmemCols, "TMEM budget");
  static_assert(SfCols % 16 == 0, "scale factors are stored 16 columns at a time");
};

struct BsParams {
  int M, N, K, C, Mt, Nt, units;
  const uint8_t* xcodes;
  const uint8_t* xscales;
  const int* x_exp;
  const uint8_t* wcodes;   // tile-major MXFP4 / NVFP4 codes
  const uint8_t* wscales;  // tile-major scales
  const float* ts;         // NVFP4 / FP8 tensor scale (device), else nullptr
  void* out;               // y [M][N] fp32 or bf16
  int out_bf16;
  int* dev_err;
};

// ---------------------------------------------------------------------------------------
// Split: one CTA of 256 threads per token row of the padded tile range (rows past M write
// zeros).  Phase 1: the row maximum and x_exp.  Phase 2: each 256-element span is one warp's,
// lane l holding elements 8l .. 8l+7 of it (one E2M1 chunk, or two E4M3 chunks of 128), so
// four lanes share a 32-element block (two a 16-element one).
// Every step is exact in fp32: bf16 values times powers of two, a code times a power of two,
// and r - q 2^e, whose significand fits 24 bits because |r - q 2^e| is at most half a code
// step at |r|'s magnitude (or, for E2M1, the saturation error 2^(e+1) where |r| >= 2^(e+2)).
// ---------------------------------------------------------------------------------------
constexpr int kBsSplitThreads = 256;
constexpr int kBsSplitRegs = 3;  // 8-element words per thread kept from phase 1 (rows to 6144)

__device__ __forceinline__ float bs_pow2(int e) {  // 2^e for -149 <= e <= 127, exact
  return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << (e + 149));
}
// floor(log2 v) for a finite v > 0, from the bits (normal: biased exponent - 127; subnormal:
// the leading mantissa bit's position - 149)
__device__ __forceinline__ int bs_flog2(float v) {
  const uint32_t b = __float_as_uint(v);
  return (b >> 23) != 0u ? (int)(b >> 23) - 127 : -118 - __clz((int)b);
}
__device__ __forceinline__ float bs_amax8(float m, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
  return m;
}

// Two elements as one code pair (element 2i first: the low nibble or byte), rounded to
// nearest even and saturated by the hardware conversion, and their values back (exact in f16).
template <int F>
__device__ __forceinline__ uint32_t bs_enc2(float a, float b, float& qa, float& qb) {
  if (F == kBsF8) {
    const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(c2, __NV_E4M3);
    qa = __half2float(__half(__half_raw{h.x}));
    qb = __half2float(__half(__half_raw{h.y}));
    return (uint32_t)c2;
  }
  const __nv_fp4x2_storage_t c2 = __nv_cvt_float2_to_fp4x2(make_float2(a, b), __NV_E2M1, cudaRoundNearest);
  const __half2_raw h = __nv_cvt_fp4x2_to_halfraw2(c2, __NV_E2M1);
  qa = __half2float(__half(__half_raw{h.x}));
  qb = __half2float(__half(__half_raw{h.y}));
  return (uint32_t)c2;
}

// The terms of one lane's 8 elements (a quarter of a 32-element block or half of a 16-element
// one), written to the split layout when `store` (lanes past the padded K only take part in
// the block reductions).  All lanes of the block take the same decisions (the block maximum is
// reduced over them first).  The prescale 2^-x_exp is f1 (TWO: f1 * f2, for exponents past
// the normal range).
template <int F, bool TWO>
__device__ __forceinline__ void bs_split8(const BsSplitParams& p, const uint4& v, bool in, bool store,
                                          float f1, float f2, int t, int r, int k, int lane) {
  constexpr int kTerms = bs_terms(F), kChunk = bs_chunk(F), kBlk = bs_blk(F), kSbr = bs_sbr(F);
  constexpr int kLpb = kBlk / 8;  // lanes per block
  float rv[8];
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16) * f1, hi = __uint_as_float(w[i] & 0xFFFF0000u) * f1;
    rv[2 * i] = in ? (TWO ? lo * f2 : lo) : 0.f;
    rv[2 * i + 1] = in ? (TWO ? hi * f2 : hi) : 0.f;
  }
  const int c = k / kChunk, o = k % kChunk;  // chunk, element offset in it
  const int j = o / kBlk;                    // block of the chunk
  // byte offset of the 8 elements' codes in the row: 16-byte group ob / 16, stored at group
  // (ob / 16) ^ (r & 7)
  const int ob = F == kBsF8 ? o : o / 2;
  const int pos = ((((ob >> 4) ^ r) & 7) << 4) + (ob & 15);
  bool done = false;
#pragma unroll
  for (int term = 0; term < kTerms; ++term) {
    float bmax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) bmax = fmaxf(bmax, fabsf(rv[i]));
    bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
    const float b2 = __shfl_xor_sync(0xffffffffu, bmax, 2);
    if (kLpb == 4) bmax = fmaxf(bmax, b2);
    int sb = 0;  // scale byte
    uint32_t packed[2] = {0u, 0u};
    if (!done && bmax > 0.f) {
      const int e = bs_flog2(bmax) - bs_top(F);  // block maximum / 2^e in [2^top, 2^(top+1))
      if (e >= bs_emin(F)) {
        sb = bs_scale_byte(F, e);
        // 2^-e is a normal float: e runs from emin >= -127 to at most 8 (the largest prescaled
        // block maximum is below 2^11)
        const float inv = __int_as_float((127 - e) << 23), sc = bs_pow2(e);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float qa, qb;
          const uint32_t c2 = bs_enc2<F>(rv[2 * i] * inv, rv[2 * i + 1] * inv, qa, qb);
          if (term + 1 < kTerms) {  // the last term's residual is not needed
            rv[2 * i] = fmaf(-qa, sc, rv[2 * i]);
            rv[2 * i + 1] = fmaf(-qb, sc, rv[2 * i + 1]);
          }
          if (F == kBsF8) packed[i >> 1] |= c2 << (16 * (i & 1));
          else packed[0] |= c2 << (8 * i);
        }
      } else {
        done = true;  // below the scale range: this and the later terms are dropped
      }
    } else {
      done = true;
    }
    if (store) {
      const size_t bidx = ((size_t)t * p.C + c) * kTerms + term;
      uint8_t* crow = p.codes + bidx * kBsBlock + (size_t)r * 128;
      if (F == kBsF8) *reinterpret_cast<uint2*>(crow + pos) = make_uint2(packed[0], packed[1]);
      else *reinterpret_cast<uint32_t*>(crow + pos) = packed[0];
      if (lane % kLpb == 0) p.scales[bidx * (size_t)(kBsM * kSbr) + (size_t)r * kSbr + j] = (uint8_t)(done ? 0 : sb);
    }
  }
}

template <int F>
__global__ void __launch_bounds__(kBsSplitThreads) qgemm_bs_split_kernel(const BsSplitParams p) {
  // x may come from the preceding grid.  Only once that grid has completed may the GEMM
  // launch: it reads the weights before it waits for this grid, and the grid before may have
  // written them.
  griddep_wait();
  griddep_launch_dependents();
  const int m = blockIdx.x;
  const bool live = m < p.M;
  const uint16_t* xr = p.x + (size_t)(live ? m : 0) * p.K;
  __shared__ float red[kBsSplitThreads / 32];
  // Phase 1: the row maximum.  Thread i reads the 8-element words k = 8 (i + 256 n); the same
  // thread converts them in phase 2 (word n is lane i % 32 of the warp span starting at
  // 256 (8 n + i / 32)), so the first kBsSplitRegs words stay in registers.
  const int Kp = p.C * bs_chunk(F);
  uint4 v[kBsSplitRegs];
  float amax = 0.f;
#pragma unroll
  for (int n = 0; n < kBsSplitRegs; ++n) {
    const int k = (threadIdx.x + n * kBsSplitThreads) * 8;
    v[n] = (live && k < p.K) ? *reinterpret_cast<const uint4*>(xr + k) : make_uint4(0u, 0u, 0u, 0u);
    amax = bs_amax8(amax, v[n]);
  }
  if (live)
    for (int k = (threadIdx.x + kBsSplitRegs * kBsSplitThreads) * 8; k < p.K; k += kBsSplitThreads * 8)
      amax = bs_amax8(amax, *reinterpret_cast<const uint4*>(xr + k));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < kBsSplitThreads / 32; ++i) amax = fmaxf(amax, red[i]);
  int xe = 0;
  if (amax > 0.f && amax <= 3.4e38f)
    xe = bs_flog2(amax) - bs_xshift(F);  // row maximum * 2^-xe in [2^xshift, 2^(xshift+1))
  if (threadIdx.x == 0) p.x_exp[m] = live ? xe : 0;
  // 2^-xe as two exact factors (xe runs from -143 to 127)
  const int a1 = max(min(-xe, 126), -126);
  const float f1 = bs_pow2(a1), f2 = bs_pow2(-xe - a1);
  const int t = m / kBsM, r = m % kBsM;
  const int lane = threadIdx.x & 31;
  // Phase 2, over the warp spans that start inside the padded K (warp-uniform conditions:
  // every lane of a span takes part in its block reductions)
  auto phase2 = [&](auto two) {
    constexpr bool kTwo = decltype(two)::value;
#pragma unroll
    for (int n = 0; n < kBsSplitRegs; ++n) {
      const int k = (threadIdx.x + n * kBsSplitThreads) * 8;
      if (k - 8 * lane < Kp) bs_split8<F, kTwo>(p, v[n], live && k < p.K, k < Kp, f1, f2, t, r, k, lane);
    }
    for (int k = (threadIdx.x + kBsSplitRegs * kBsSplitThreads) * 8; k - 8 * lane < Kp; k += kBsSplitThreads * 8) {
      const bool in = live && k < p.K;
      const uint4 w = in ? *reinterpret_cast<const uint4*>(xr + k) : make_uint4(0u, 0u, 0u, 0u);
      bs_split8<F, kTwo>(p, w, in, k < Kp, f1, f2, t, r, k, lane);
    }
  };
  if (f2 == 1.0f) phase2(std::false_type{});  // the row's 2^-xe is one normal float (uniform)
  else phase2(std::true_type{});
}

// ---------------------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void bs_tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void bs_tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void bs_tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A * B^T with block scales: A, B K-major in shared memory, the scale factors in
// tensor memory at sfa / sfb.  E2M1 with 16-element UE4M3 blocks (NVFP4) or 32-element E8M0
// (MXFP4); E4M3 with 32-element E8M0 blocks (FP8).
template <int F>
__device__ __forceinline__ void bs_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  if (F == kBsF8)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  else if (F == kBsNv)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// The 4-byte scale word of one row for MMA K-block kb: NVFP4 keeps 4 scales per 64 K (16 bytes
// per row and chunk), MXFP4 2 (8 bytes), FP8 x terms 1 per 32 K (4 bytes); the upper bytes of
// the word are unused.
template <int F>
__device__ __forceinline__ uint32_t bs_sf_word(const uint8_t* row, int kb) {
  if (F == kBsNv) return reinterpret_cast<const uint32_t*>(row)[kb];
  if (F == kBsF8) return (uint32_t)row[kb];
  return (uint32_t)reinterpret_cast<const uint16_t*>(row)[kb];
}
// The FP8 weights' block scales: 2^0 in E8M0 (their tensor scale is applied in the epilogue)
constexpr uint32_t kBsUnitSf = 0x7F7F7F7Fu;
__device__ __forceinline__ void bs_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// Each lane writes 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void bs_tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
// Each lane reads 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void bs_tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// Each lane reads 16 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void bs_tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}


__device__ __forceinline__ float bs_scale_pow2(float v, int e) {
  return (e >= -126 && e <= 127) ? v * __int_as_float((e + 127) << 23) : ldexpf(v, e);
}

template <int F>
__global__ void __launch_bounds__(kBsThreads, 1) qgemm_bs_kernel(const __grid_constant__ BsParams p) {
  using L = BsLay<F>;
  constexpr int kTerms = L::Terms;
  constexpr int kBsStages = L::Stages;
  constexpr int kBsStage = L::Stage;
  constexpr int kBsACodes = L::ACodes;
  constexpr int kBsAScales = L::AScales;
  constexpr int kBsSBlock = L::SB;
  constexpr int kBsWSBlock = L::WSB;
  constexpr int kBsSfCols = L::SfCols;
  constexpr int kSbr = bs_sbr(F);
  constexpr int kWSbr = bs_wsbr(F);
  constexpr bool kTs = F != kBsMx;  // a per-tensor scale (NVFP4, FP8)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBsStages * kBsStage);
  const uint32_t bar_full = smem_u32(bars);                  // [2] stage data landed
  const uint32_t bar_empty = bar_full + 8 * kBsStages;       // [2] the stage's MMAs are done
  const uint32_t bar_sf = bar_empty + 8 * kBsStages;         // [2] its scale factors are in TMEM
  const uint32_t bar_acc = bar_sf + 8 * kBsStages;           // a tile's accumulator is complete
  const uint32_t bar_acc_free = bar_acc + 8;                 // the epilogue has read it
  const uint32_t bar_drain = bar_acc_free + 8;               // the issuer's MMAs are done
  int* ctl = reinterpret_cast<int*>(bars + 3 * kBsStages + 3);
  volatile int* abort_flag = ctl + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kBsStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_sf + 8 * s, 4);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_acc_free, 4);
    mbar_init(bar_drain, 1);
    ctl[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    bs_tmem_alloc(smem_u32(ctl), kBsTmemCols);
    bs_tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(ctl[0]);
  const int64_t n_row_tiles = row_tiles(p.N);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_last();
      const uint64_t pol_x = policy_evict_last();
      RingPos sp;
      int issued = 0;
      bool ok = true;
      bool waited = false;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        const int mt = u % p.Mt, nt = u / p.Mt;
        for (int c = 0; c < p.C; ++c) {
          if (issued >= kBsStages &&
              !mbar_wait(bar_empty + 8 * sp.slot, sp.phase ^ 1u, abort_flag, p.dev_err, kErrTimeout)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * sp.slot;
          const uint32_t st = sbase + (uint32_t)(sp.slot * kBsStage);
          uint32_t bytes = kBsACodes + kBsAScales;
          for (int j = 0; j < kBsWT; ++j)
            if (kBsWT * nt + j < n_row_tiles) bytes += kBsBlock + kBsWSBlock;
          mbar_arrive_expect_tx(fb, bytes);
          for (int j = 0; j < kBsWT; ++j) {
            const int64_t t = kBsWT * (int64_t)nt + j;
            if (t >= n_row_tiles) continue;
            const int64_t blk = t * p.C + c;
            bulk_load(st + kBsACodes + j * kBsBlock, p.wcodes + blk * kBsBlock, kBsBlock, fb, pol_w);
            if (kBsWSBlock > 0)
              bulk_load(st + kBsACodes + kBsBCodes + kBsAScales + j * kBsWSBlock,
                        p.wscales + blk * kBsWSBlock, kBsWSBlock, fb, pol_w);
          }
          // the split x comes from the preceding grid
          if (!waited) {
            griddep_wait();
            waited = true;
          }
          const int64_t xb = ((int64_t)mt * p.C + c) * kTerms;
          bulk_load(st, p.xcodes + xb * kBsBlock, kBsACodes, fb, pol_x);
          bulk_load(st + kBsACodes + kBsBCodes, p.xscales + xb * kBsSBlock, kBsAScales, fb, pol_x);
          sp.next(kBsStages);
          ++issued;
        }
      }
      if (!ok) {
        // let the copies in flight land before the CTA leaves
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      RingPos sp;
      bool ok = true;
      int ti = 0;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++ti) {
        if (ti > 0) {
          if (!mbar_wait_spin(bar_acc_free, (uint32_t)(ti - 1) & 1u, false, abort_flag, p.dev_err,
                              kErrTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int c = 0; c < p.C; ++c) {
          if (!mbar_wait_spin(bar_full + 8 * sp.slot, sp.phase, false, abort_flag, p.dev_err, kErrTimeout) ||
              !mbar_wait_spin(bar_sf + 8 * sp.slot, sp.phase, false, abort_flag, p.dev_err, kErrTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + (uint32_t)(sp.slot * kBsStage);
          const uint64_t bdesc0 = smem_desc_sw128(st + kBsACodes);
          const uint32_t sf0 = tmem + (uint32_t)(kBsN + sp.slot * kBsSfCols);
#pragma unroll
          for (int kb = 0; kb < kBsKB; ++kb) {
#pragma unroll
            for (int t = 0; t < kTerms; ++t) {
              const uint64_t adesc = smem_desc_sw128(st + (uint32_t)(t * kBsBlock)) + (uint64_t)(kb * 2);
              bs_mma<F>(tmem, adesc, bdesc0 + (uint64_t)(kb * 2), L::Idesc,
                        sf0 + (uint32_t)((t * 4 + kb) * 4), sf0 + (uint32_t)(L::ASf + kb * 4 * kBsWT),
                        (c | kb | t) != 0 ? 1u : 0u);
            }
          }
          bs_commit(bar_empty + 8 * sp.slot);
          sp.next(kBsStages);
        }
        if (!ok) break;
        bs_commit(bar_acc);
      }
      bs_commit(bar_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_drain, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else if (warp < kBsEpiWarp0) {
    // ------------------------------------------------------------ scale-factor staging
    // Every warp writes the same values into its own lane quarter (the MMA reads the scale
    // factors of row r0 + 32 r1 from lane r0 of each quarter).
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    RingPos sp;
    int used = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      for (int c = 0; c < p.C; ++c) {
        if (used >= kBsStages) {
          ok = mbar_wait(bar_empty + 8 * sp.slot, sp.phase ^ 1u, abort_flag, p.dev_err, kErrTimeout);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        ok = mbar_wait(bar_full + 8 * sp.slot, sp.phase, abort_flag, p.dev_err, kErrTimeout);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* st = smem + sp.slot * kBsStage;
        const uint8_t* sa = st + kBsACodes + kBsBCodes;  // x-term scales [terms][128][sbr]
        const uint8_t* sb = sa + kBsAScales;              // weight scales [kBsWT][128][wsbr]
        uint32_t v[kBsSfCols];
#pragma unroll
        for (int t = 0; t < kTerms; ++t)
#pragma unroll
          for (int r1 = 0; r1 < 4; ++r1) {
            const uint8_t* row = sa + t * kBsSBlock + (r1 * 32 + lane) * kSbr;
#pragma unroll
            for (int kb = 0; kb < kBsKB; ++kb) v[(t * 4 + kb) * 4 + r1] = bs_sf_word<F>(row, kb);
          }
#pragma unroll
        for (int r1 = 0; r1 < 4 * kBsWT; ++r1) {
          const uint8_t* row = sb + (r1 >> 2) * kBsWSBlock + ((r1 & 3) * 32 + lane) * kWSbr;
#pragma unroll
          for (int kb = 0; kb < kBsKB; ++kb)
            v[L::ASf + kb * 4 * kBsWT + r1] = kWSbr == 0 ? kBsUnitSf : bs_sf_word<F>(row, kb);
        }
        const uint32_t ta = tmem + lane_base + (uint32_t)(kBsN + sp.slot * kBsSfCols);
#pragma unroll
        for (int i = 0; i < kBsSfCols / 16; ++i)
          bs_tmem_st16(ta + (uint32_t)(16 * i), *reinterpret_cast<const uint32_t(*)[16]>(&v[16 * i]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sf + 8 * sp.slot);
        sp.next(kBsStages);
        ++used;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    griddep_wait();  // x_exp comes from the split kernel
    int ti = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++ti) {
      const int mt = u % p.Mt, nt = u / p.Mt;
      const int m = mt * kBsM + q * 32 + lane;
      const int xe = (m < p.M) ? p.x_exp[m] : 0;
      const float tsv = kTs ? __ldg(p.ts) : 1.0f;  // tensor scale, applied before 2^xe
      // y = (acc * ts) * 2^xe: the tensor scale rounds once, the power of two is exact.  When
      // every row of the warp has a normal 2^xe (the common case) it is one multiply by a
      // factor taken once per unit; otherwise the warp takes bs_scale_pow2 per element.
      const bool fast = xe >= -126 && xe <= 127;
      const float sc = __int_as_float(((fast ? xe : 0) + 127) << 23);
      const bool all_fast = __all_sync(0xffffffffu, fast);
      bool ok = mbar_wait(bar_acc, (uint32_t)ti & 1u, abort_flag, p.dev_err, kErrTimeout);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      // one 32-column block: scale and store (FAST: the one-multiply scale)
      auto store_block = [&](const uint32_t (&v)[32], int cb, auto fastc) {
        constexpr bool FAST = decltype(fastc)::value;
        auto yv = [&](uint32_t w) {
          const float a = kTs ? __uint_as_float(w) * tsv : __uint_as_float(w);
          return FAST ? a * sc : bs_scale_pow2(a, xe);
        };
        const int n0 = nt * kBsN + cb;
        if (m < p.M && n0 < p.N) {
          if (p.out_bf16) {
            __nv_bfloat16* yr = reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)m * p.N + n0;
            if (n0 + 32 <= p.N && (p.N % 8) == 0) {
#pragma unroll
              for (int i = 0; i < 32; i += 8) {
                uint32_t w[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const __nv_bfloat16 lo = __float2bfloat16_rn(yv(v[i + 2 * h]));
                  const __nv_bfloat16 hi = __float2bfloat16_rn(yv(v[i + 2 * h + 1]));
                  w[h] = (uint32_t)__bfloat16_as_ushort(lo) | ((uint32_t)__bfloat16_as_ushort(hi) << 16);
                }
                *reinterpret_cast<uint4*>(yr + i) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = __float2bfloat16_rn(yv(v[i]));
            }
          } else {
            float* yr = reinterpret_cast<float*>(p.out) + (size_t)m * p.N + n0;
            if (n0 + 32 <= p.N && (p.N % 4) == 0) {
#pragma unroll
              for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4*>(yr + i) =
                    make_float4(yv(v[i]), yv(v[i + 1]),
                                yv(v[i + 2]), yv(v[i + 3]));
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (n0 + i < p.N) yr[i] = yv(v[i]);
            }
          }
        }
      };
#pragma unroll 1
      for (int cb = 0; cb < kBsN; cb += 32) {
        uint32_t v[32];
        bs_tmem_ld32(tmem + lane_base + (uint32_t)cb, v);
        tmem_ld_wait();
        if (all_fast) store_block(v, cb, std::true_type{});
        else store_block(v, cb, std::false_type{});
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_free);
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    bs_tmem_dealloc(tmem, kBsTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// Decode widths (M <= 128): the roles of the operands swap.  The weights are the MMA M
// operand (one 128-row weight tile per unit, its scales SFA), the split x the N operand
// (N = M rounded up to 16 rows of the first token tile, its scales SFB), and K is split
// over S ranges so that the units fill the SMs; S > 1 writes fp32 partials that the split-K
// reduce kernel sums in the order s = 0..S-1.  Per chunk: 4 K-blocks x terms MMAs of
// M128 N(M) (K64 E2M1 or K32 E4M3).  At these widths the issuing thread bounds the MMA stream,
// so two issuers take alternate chunks of a unit, each into its own accumulator; the epilogue
// adds them in the order even + odd.  Stage: [weight codes 16 KB][terms x N x 128 term codes]
// [weight scales 128 x wsbr][terms x N x sbr term scales], rounded up to 1 KB; an even number
// of stages, so that a stage's previous use belongs to the same issuer.  TMEM: the two
// accumulators (N columns each), then per stage 16 + 16 terms columns of scale factors: the
// weights' K-block kb at 4 kb (4 row groups), term j's K-block kb at 16 + 4 (4 j + kb).
// ---------------------------------------------------------------------------------------
__host__ __device__ constexpr int bd_sf_cols(int f) { return 16 + bs_terms(f) * 16; }
__host__ __device__ constexpr int bd_max_stages(int f) { return f == kBsF8 ? 8 : 6; }
constexpr int kBdIssuer2Warp = 10;
constexpr int kBdThreads = 11 * 32;

struct BsDecParams {
  int M, N, K, C, Nb, S, units, stages, stage_bytes;
  const uint8_t* xcodes;
  const uint8_t* xscales;
  const int* x_exp;
  const uint8_t* wcodes;
  const uint8_t* wscales;
  const float* ts;  // NVFP4 / FP8 tensor scale (device), else nullptr
  float* ws;  // S > 1: partials [S][M][N], fully scaled
  void* out;
  int out_bf16;
  int* dev_err;
};

template <int F>
__global__ void __launch_bounds__(kBdThreads, 1) qgemm_bs_dec_kernel(const __grid_constant__ BsDecParams p) {
  constexpr int kTerms = bs_terms(F);
  constexpr int kSbr = bs_sbr(F), kWSbr = bs_wsbr(F);
  constexpr int kSBlock = kBsM * kSbr;    // one 128-row block of term scales in the split
  constexpr int kWSBlock = kBsM * kWSbr;  // one 128-row block of weight scales
  constexpr int kBdSfCols = bd_sf_cols(F);
  constexpr bool kTs = F != kBsMx;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const int NST = p.stages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NST * p.stage_bytes);
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = bar_full + 8 * NST;
  const uint32_t bar_sf = bar_empty + 8 * NST;
  const uint32_t bar_acc = bar_sf + 8 * NST;
  const uint32_t bar_acc_free = bar_acc + 8;
  const uint32_t bar_drain = bar_acc_free + 8;
  int* ctl = reinterpret_cast<int*>(bars + 3 * NST + 4);
  volatile int* abort_flag = ctl + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Nb = p.Nb;
  const uint32_t xterm = (uint32_t)Nb * 128u;      // one term's codes in a stage
  const uint32_t off_ws = kBsBlock + kTerms * xterm;  // weight scales
  const uint32_t off_xs = off_ws + kWSBlock;           // term scales
  const uint32_t idesc = bs_idesc(F, Nb);
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_sf + 8 * s, 4);
    }
    mbar_init(bar_acc, 2);  // one commit of each issuer per unit
    mbar_init(bar_acc_free, 4);
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 8, 1);
    ctl[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    bs_tmem_alloc(smem_u32(ctl), kBsTmemCols);
    bs_tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(ctl[0]);
  const int64_t n_row_tiles = row_tiles(p.N);
  const uint32_t sf_col0 = (uint32_t)(2 * Nb);  // scale factors after the two accumulators
  auto unit_range = [&](int u, int& t, int& s, int& c0, int& c1) {
    t = u % (int)n_row_tiles;
    s = u / (int)n_row_tiles;
    c0 = (int)((int64_t)s * p.C / p.S);
    c1 = (int)((int64_t)(s + 1) * p.C / p.S);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      RingPos sp;
      int issued = 0;
      bool ok = true, waited = false;
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
        int t, s, c0, c1;
        unit_range(u, t, s, c0, c1);
        for (int c = c0; c < c1; ++c) {
          if (issued >= NST &&
              !mbar_wait(bar_empty + 8 * sp.slot, sp.phase ^ 1u, abort_flag, p.dev_err, kErrTimeout)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * sp.slot;
          const uint32_t st = sbase + (uint32_t)(sp.slot * p.stage_bytes);
          mbar_arrive_expect_tx(fb, kBsBlock + kWSBlock + kTerms * (xterm + (uint32_t)(Nb * kSbr)));
          const int64_t blk = (int64_t)t * p.C + c;
          bulk_load(st, p.wcodes + blk * kBsBlock, kBsBlock, fb, pol_w);
          if (kWSBlock > 0) bulk_load(st + off_ws, p.wscales + blk * kWSBlock, kWSBlock, fb, pol_w);
          if (!waited) {
            griddep_wait();  // the split x comes from the preceding grid
            waited = true;
          }
          for (int j = 0; j < kTerms; ++j) {
            const int64_t xb = (int64_t)c * kTerms + j;  // token tile 0
            bulk_load(st + kBsBlock + (uint32_t)j * xterm, p.xcodes + xb * kBsBlock, xterm, fb, pol_x);
            bulk_load(st + off_xs + (uint32_t)(j * Nb * kSbr), p.xscales + xb * kSBlock, (uint32_t)(Nb * kSbr), fb, pol_x);
          }
          sp.next(NST);
          ++issued;
        }
      }
      if (!ok) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == kBdIssuer2Warp) {
    // ------------------------------------------------------------ MMA issuers
    // issuer e takes the chunks c of each unit with (c - c0) % 2 == e into accumulator e
    const int e = (warp == 1) ? 0 : 1;
    if (lane == 0) {
      RingPos sp;
      bool ok = true;
      int ti = 0;
      const uint32_t d = tmem + (uint32_t)(e * Nb);
      for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x, ++ti) {
        int t, s, c0, c1;
        unit_range(u, t, s, c0, c1);
        if (ti > 0) {
          if (!mbar_wait_spin(bar_acc_free, (uint32_t)(ti - 1) & 1u, false, abort_flag, p.dev_err,
                              kErrTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int c = c0; c < c1; ++c) {
          if (((c - c0) & 1) != e) {  // the other issuer's chunk: keep the ring position
            sp.next(NST);
            continue;
          }
          if (!mbar_wait_spin(bar_full + 8 * sp.slot, sp.phase, false, abort_flag, p.dev_err, kErrTimeout) ||
              !mbar_wait_spin(bar_sf + 8 * sp.slot, sp.phase, false, abort_flag, p.dev_err, kErrTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + (uint32_t)(sp.slot * p.stage_bytes);
          const uint64_t adesc0 = smem_desc_sw128(st);
          const uint32_t sf0 = tmem + sf_col0 + (uint32_t)(sp.slot * kBdSfCols);
#pragma unroll
          for (int kb = 0; kb < kBsKB; ++kb) {
#pragma unroll
            for (int j = 0; j < kTerms; ++j) {
              const uint64_t bdesc = smem_desc_sw128(st + kBsBlock + (uint32_t)j * xterm) + (uint64_t)(kb * 2);
              bs_mma<F>(d, adesc0 + (uint64_t)(kb * 2), bdesc, idesc, sf0 + (uint32_t)(kb * 4),
                     sf0 + (uint32_t)(16 + (j * 4 + kb) * 4), (c - c0 >= 2 || kb || j) ? 1u : 0u);
            }
          }
          bs_commit(bar_empty + 8 * sp.slot);
          sp.next(NST);
        }
        if (!ok) break;
        bs_commit(bar_acc);  // this issuer's part of the unit (nothing pending if it had none)
      }
      bs_commit(bar_drain + 8 * e);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_drain + 8 * e, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else if (warp < kBsEpiWarp0) {
    // ------------------------------------------------------------ scale-factor staging
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    RingPos sp;
    int used = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < p.units && ok; u += gridDim.x) {
      int t, s, c0, c1;
      unit_range(u, t, s, c0, c1);
      for (int c = c0; c < c1; ++c) {
        if (used >= NST) {
          ok = mbar_wait(bar_empty + 8 * sp.slot, sp.phase ^ 1u, abort_flag, p.dev_err, kErrTimeout);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
        }
        ok = mbar_wait(bar_full + 8 * sp.slot, sp.phase, abort_flag, p.dev_err, kErrTimeout);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint8_t* st = smem + sp.slot * p.stage_bytes;
        uint32_t v[kBdSfCols];
#pragma unroll
        for (int r1 = 0; r1 < 4; ++r1) {
          const uint8_t* row = st + off_ws + (r1 * 32 + lane) * kWSbr;
#pragma unroll
          for (int kb = 0; kb < kBsKB; ++kb) v[kb * 4 + r1] = kWSbr == 0 ? kBsUnitSf : bs_sf_word<F>(row, kb);
        }
#pragma unroll
        for (int j = 0; j < kTerms; ++j)
#pragma unroll
          for (int r1 = 0; r1 < 4; ++r1) {
            const int rw = r1 * 32 + lane;
            const uint8_t* row = st + off_xs + j * Nb * kSbr + rw * kSbr;
#pragma unroll
            for (int kb = 0; kb < kBsKB; ++kb)
              v[16 + (j * 4 + kb) * 4 + r1] = rw < Nb ? bs_sf_word<F>(row, kb) : 0u;
          }
        const uint32_t ta = tmem + lane_base + sf_col0 + (uint32_t)(sp.slot * kBdSfCols);
#pragma unroll
        for (int i = 0; i < kBdSfCols / 16; ++i)
          bs_tmem_st16(ta + (uint32_t)(16 * i), *reinterpret_cast<const uint32_t(*)[16]>(&v[16 * i]));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_sf + 8 * sp.slot);
        sp.next(NST);
        ++used;
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // lane = weight row n of the tile; columns = tokens b (scaled by 2^x_exp[b])
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    griddep_wait();  // x_exp comes from the split kernel
    const size_t MN = (size_t)p.M * p.N;
    const float tsv = kTs ? __ldg(p.ts) : 1.0f;  // tensor scale, applied before 2^x_exp
    // 2^x_exp of token column b = lane + 32 j held by lane `lane` as fac[j] (M <= 128); when
    // every column's exponent is in the normal range the restore is one multiply by a factor
    // fetched with a shuffle, otherwise bs_scale_pow2 per element
    float fac[4];
    bool fast = true;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int b = lane + 32 * j;
      const int e = (b < p.M) ? __ldg(p.x_exp + b) : 0;
      const bool f = e >= -126 && e <= 127;
      fast = fast && f;
      fac[j] = __int_as_float(((f ? e : 0) + 127) << 23);
    }
    const bool all_fast = __all_sync(0xffffffffu, fast);
    int ti = 0;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x, ++ti) {
      int t, s, c0, c1;
      unit_range(u, t, s, c0, c1);
      const int64_t n64 = (int64_t)t * kBsM + q * 32 + lane;
      bool ok = mbar_wait(bar_acc, (uint32_t)ti & 1u, abort_flag, p.dev_err, kErrTimeout);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const bool two = (c1 - c0) >= 2;  // the odd chunks' accumulator holds data
#pragma unroll 1
      for (int cb = 0; cb < Nb; cb += 16) {
        uint32_t v[16];
        bs_tmem_ld16(tmem + lane_base + (uint32_t)cb, v);
        tmem_ld_wait();
        if (two) {
          uint32_t w[16];
          bs_tmem_ld16(tmem + lane_base + (uint32_t)(Nb + cb), w);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w[i]));
        }
        // the factors of columns cb .. cb+15 (all lanes take part in the shuffles)
        const int jb = cb >> 5;
        const float fr = jb == 0 ? fac[0] : jb == 1 ? fac[1] : jb == 2 ? fac[2] : fac[3];
        float fv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) fv[i] = __shfl_sync(0xffffffffu, fr, (cb & 16) + i);
        if (n64 < p.N) {
          const int n = (int)n64;
          auto put = [&](int b, float val) {
            if (p.S > 1) p.ws[(size_t)s * MN + (size_t)b * p.N + n] = val;
            else if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)b * p.N + n] = __float2bfloat16_rn(val);
            else reinterpret_cast<float*>(p.out)[(size_t)b * p.N + n] = val;
          };
          if (all_fast) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (cb + i < p.M) put(cb + i, (kTs ? __uint_as_float(v[i]) * tsv : __uint_as_float(v[i])) * fv[i]);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (cb + i < p.M)
                put(cb + i, bs_scale_pow2(kTs ? __uint_as_float(v[i]) * tsv : __uint_as_float(v[i]),
                                          __ldg(p.x_exp + cb + i)));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_free);
    }
    griddep_launch_dependents();  // the split-K reduce may launch
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    bs_tmem_dealloc(tmem, kBsTmemCols);
  }
}

// ---------------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------------
cudaError_t launch_bs_split(int f, const uint16_t* x, int M, int K, uint8_t* codes,
                            uint8_t* scales, int* x_exp, cudaStream_t stream) {
  if (f < kBsMx || f > kBsF8) return cudaErrorInvalidValue;
  BsSplitParams p{};
  p.x = x;
  p.M = M;
  p.K = K;
  p.C = (K + bs_chunk(f) - 1) / bs_chunk(f);
  p.Mt = (M + kBsM - 1) / kBsM;
  p.f = f;
  p.codes = codes;
  p.scales = scales;
  p.x_exp = x_exp;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.Mt * kBsM), 1, 1);
  cfg.blockDim = dim3(kBsSplitThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return f == kBsF8   ? cudaLaunchKernelEx(&cfg, qgemm_bs_split_kernel<kBsF8>, p)
         : f == kBsNv ? cudaLaunchKernelEx(&cfg, qgemm_bs_split_kernel<kBsNv>, p)
                      : cudaLaunchKernelEx(&cfg, qgemm_bs_split_kernel<kBsMx>, p);
}

// SMs of device `dev`, read once per device (devices beyond 64 read it on every launch).
static int bs_sm_count(int dev) {
  static std::atomic<int> cached[64];
  int v = (dev >= 0 && dev < 64) ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) v = 148;
  if (dev >= 0 && dev < 64) cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

// Raises a kernel's dynamic shared-memory limit once per device (devices beyond 64 on every
// launch); one mask per kernel instantiation.
static cudaError_t bs_smem_attr(const void* fn, std::atomic<uint64_t>& mask, int dev, int bytes) {
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit != 0 && (mask.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) mask.fetch_or(bit, std::memory_order_release);
  return e;
}

static cudaError_t bs_launch_pdl(cudaLaunchConfig_t& cfg, cudaStream_t stream, cudaLaunchAttribute* at) {
  cfg.stream = stream;
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaSuccess;
}

template <int F>
static cudaError_t launch_bs_gemm_t(int M, int N, int K, const uint8_t* xcodes,
                                    const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                                    const uint8_t* wscales, const float* ts, void* out,
                                    int out_bf16, int* dev_err, cudaStream_t stream) {
  static std::atomic<uint64_t> set_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = bs_smem_attr((const void*)qgemm_bs_kernel<F>, set_mask, dev, BsLay<F>::Smem);
  if (e != cudaSuccess) return e;
  BsParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.C = (K + bs_chunk(F) - 1) / bs_chunk(F);
  p.Mt = (M + kBsM - 1) / kBsM;
  p.Nt = (N + kBsN - 1) / kBsN;
  p.units = p.Mt * p.Nt;
  p.xcodes = xcodes;
  p.xscales = xscales;
  p.x_exp = x_exp;
  p.wcodes = wcodes;
  p.wscales = wscales;
  p.ts = ts;
  p.out = out;
  p.out_bf16 = out_bf16;
  p.dev_err = dev_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min(p.units, bs_sm_count(dev)), 1, 1);
  cfg.blockDim = dim3(kBsThreads, 1, 1);
  cfg.dynamicSmemBytes = BsLay<F>::Smem;
  cudaLaunchAttribute at[1];
  bs_launch_pdl(cfg, stream, at);
  return cudaLaunchKernelEx(&cfg, qgemm_bs_kernel<F>, p);
}

cudaError_t launch_bs_gemm(int f, int M, int N, int K, const uint8_t* xcodes,
                           const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                           const uint8_t* wscales, const float* ts, void* out, int out_bf16,
                           int* dev_err, cudaStream_t stream) {
  switch (f) {
    case kBsMx:
      return launch_bs_gemm_t<kBsMx>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, out,
                                     out_bf16, dev_err, stream);
    case kBsNv:
      return launch_bs_gemm_t<kBsNv>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, out,
                                     out_bf16, dev_err, stream);
    case kBsF8:
      return launch_bs_gemm_t<kBsF8>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, out,
                                     out_bf16, dev_err, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

// K split of the decode kernel: a function of (format, N, K) only (the unit count is weighed
// against the 148 SMs of a B200), the smallest S of least cost (waves of units x (K per unit +
// a fixed cost of ~768 K) + a small charge per split for the partials), in units of 256 K.
constexpr int kBsSplitSMs = 148;
int bs_dec_split(int f, int64_t N, int64_t K, int sms) {
  const int64_t T = row_tiles(N), C = (K + bs_chunk(f) - 1) / bs_chunk(f);
  const double ck = double(bs_chunk(f)) / 256.0;
  int best = 1;
  double best_cost = 0.0;
  for (int64_t S = 1; S <= std::min<int64_t>(16, C); ++S) {
    const int64_t waves = (T * S + sms - 1) / sms;
    const double cost = double(waves) * (double((C + S - 1) / S) * ck + 3.0) + 0.25 * double(S);
    if (S == 1 || cost < best_cost - 1e-9) {
      best_cost = cost;
      best = (int)S;
    }
  }
  return best;
}

// Workspace of the block-scaled path: split codes, split scales, row exponents and, for
// decode widths with a K split, the fp32 partials.
size_t bs_workspace_bytes(int f, int64_t M, int64_t N, int64_t K, size_t* off_scales,
                          size_t* off_exp, size_t* off_part) {
  const int64_t C = (K + bs_chunk(f) - 1) / bs_chunk(f), Mt = (M + kBsM - 1) / kBsM;
  const size_t codes = (size_t)(Mt * C * bs_terms(f)) * kBsBlock;
  const size_t scales = (size_t)(Mt * C * bs_terms(f)) * (size_t)(kBsM * bs_sbr(f));
  if (off_scales) *off_scales = codes;
  if (off_exp) *off_exp = codes + scales;
  size_t total = codes + scales + (size_t)Mt * kBsM * 4;
  total = (total + 255) / 256 * 256;
  if (off_part) *off_part = total;
  if (M <= kBsM && N > 0) {
    const int S = bs_dec_split(f, N, K, kBsSplitSMs);
    if (S > 1) total += (size_t)S * (size_t)M * (size_t)N * 4;
  }
  return total;
}

cudaError_t launch_reduce(const ReduceParams& rp, cudaStream_t stream);

template <int F>
static cudaError_t launch_bs_dec_t(int M, int N, int K, const uint8_t* xcodes,
                                   const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                                   const uint8_t* wscales, const float* ts, float* part, void* out,
                                   int out_bf16, int* dev_err, cudaStream_t stream) {
  static std::atomic<uint64_t> set_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = bs_smem_attr((const void*)qgemm_bs_dec_kernel<F>, set_mask, dev, kSmemLimit);
  if (e != cudaSuccess) return e;
  constexpr int kTerms = bs_terms(F);
  BsDecParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.C = (K + bs_chunk(F) - 1) / bs_chunk(F);
  p.Nb = (M + 15) / 16 * 16;
  p.S = bs_dec_split(F, N, K, kBsSplitSMs);
  p.units = (int)row_tiles(N) * p.S;
  p.stage_bytes = (kBsBlock + kTerms * p.Nb * 128 + kBsM * bs_wsbr(F) + kTerms * p.Nb * bs_sbr(F) + 1023) /
                  1024 * 1024;
  p.stages = std::min({bd_max_stages(F), (kSmemLimit - 1024 - 256) / p.stage_bytes,
                       (kBsTmemCols - 2 * p.Nb) / bd_sf_cols(F)}) & ~1;  // even
  if (p.stages < 2) return cudaErrorInvalidValue;
  p.xcodes = xcodes;
  p.xscales = xscales;
  p.x_exp = x_exp;
  p.wcodes = wcodes;
  p.wscales = wscales;
  p.ts = ts;
  p.ws = part;
  p.out = out;
  p.out_bf16 = out_bf16;
  p.dev_err = dev_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min(p.units, bs_sm_count(dev)), 1, 1);
  cfg.blockDim = dim3(kBdThreads, 1, 1);
  cfg.dynamicSmemBytes = 1024 + (size_t)p.stages * p.stage_bytes + 256;
  cudaLaunchAttribute at[1];
  bs_launch_pdl(cfg, stream, at);
  e = cudaLaunchKernelEx(&cfg, qgemm_bs_dec_kernel<F>, p);
  if (e != cudaSuccess || p.S == 1) return e;
  ReduceParams rp{};
  rp.ws = part;
  rp.S = p.S;
  rp.NMAT = 1;
  rp.B = M;
  rp.N = N;
  rp.out = out;
  rp.out_bf16 = out_bf16;
  return launch_reduce(rp, stream);
}

// Decode widths: queues the GEMM (and the split-K reduce when S > 1).
cudaError_t launch_bs_dec(int f, int M, int N, int K, const uint8_t* xcodes,
                          const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                          const uint8_t* wscales, const float* ts, float* part, void* out,
                          int out_bf16, int* dev_err, cudaStream_t stream) {
  switch (f) {
    case kBsMx:
      return launch_bs_dec_t<kBsMx>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, part,
                                    out, out_bf16, dev_err, stream);
    case kBsNv:
      return launch_bs_dec_t<kBsNv>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, part,
                                    out, out_bf16, dev_err, stream);
    case kBsF8:
      return launch_bs_dec_t<kBsF8>(M, N, K, xcodes, xscales, x_exp, wcodes, wscales, ts, part,
                                    out, out_bf16, dev_err, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace qg

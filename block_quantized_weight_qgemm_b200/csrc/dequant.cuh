// dequant.cuh -- device helpers shared by the GEMM kernels: bit tricks, the per-format
// dequantisation of 32 packed K elements into 16-bit MMA operands, and output stores.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "ptx.cuh"

namespace qg {

// ---------------------------------------------------------------------------------------
// Small bit helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
__device__ __forceinline__ uint32_t b2u(__nv_bfloat162 h) {
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ __nv_bfloat162 u2b(uint32_t u) {
  return *reinterpret_cast<__nv_bfloat162*>(&u);
}

__device__ __forceinline__ __half2 half2_bcast(uint16_t bits) {
  const uint32_t u = (uint32_t)bits | ((uint32_t)bits << 16);
  return u2h(u);
}

// f16 bit pattern of 2^ex, or 0 below the f16 subnormal range.  ex <= 15.
__device__ __forceinline__ uint16_t f16_pow2_bits(int ex) {
  if (ex >= -14) return (uint16_t)((ex + 15) << 10);
  if (ex >= -24) return (uint16_t)(1u << (ex + 24));
  return 0;
}

// Load a 16-byte chunk `ci` (0..7) of a 128-byte row stored with the 128-byte TMA swizzle.
__device__ __forceinline__ uint4 ld_sw128(const uint8_t* row_base, int row, int ci) {
  return *reinterpret_cast<const uint4*>(row_base + ((ci ^ (row & 7)) << 4));
}

// ---------------------------------------------------------------------------------------
// Dequantisation of 32 consecutive K elements of one weight row into 16 packed words
// (element 2i in the low half of word i), the layout of an A row in TMEM.
//   crow: the row's 128 code bytes in the weight stage (swizzled); srow: its 16 scale bytes.
//   c: chunk index (selects the half of a scale line shared by two chunks);
//   e0: first element within the chunk (multiple of 32).
// ---------------------------------------------------------------------------------------
template <int FMT, bool BF16OP>
struct Dequant;

// Q8_0 -> f16: q + 1152 built as f16 from the byte (0x64XX = 1024 + XX with XX = q ^ 0x80),
// minus 1152 gives q exactly; one rounding in q * d.
template <>
struct Dequant<FMT_Q8_0, false> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int c, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 4);
    const uint4 b = ld_sw128(crow, row, (e0 >> 4) + 1);
    const uint16_t dbits =
        *reinterpret_cast<const uint16_t*>(srow + 2 * (e0 >> 5));
    const __half2 d2 = half2_bcast(dbits);
    const __half2 off = half2_bcast(0x6480);  // 1152.0
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t t = w[i] ^ 0x80808080u;
      const uint32_t lo = prmt(t, 0x64646464u, 0x4140u);
      const uint32_t hi = prmt(t, 0x64646464u, 0x4342u);
      v[2 * i] = h2u(__hmul2(__hsub2(u2h(lo), off), d2));
      v[2 * i + 1] = h2u(__hmul2(__hsub2(u2h(hi), off), d2));
    }
  }
};

// Q8_0 -> bf16: q (sign-extended) + 1.5*2^23 as fp32 bits, fma with d and -1.5*2^23*d gives
// q*d exactly in fp32; one rounding to bf16.
template <>
struct Dequant<FMT_Q8_0, true> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int c, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 4);
    const uint4 b = ld_sw128(crow, row, (e0 >> 4) + 1);
    const uint16_t dbits =
        *reinterpret_cast<const uint16_t*>(srow + 2 * (e0 >> 5));
    const float d = __half2float(__ushort_as_half(dbits));
    const float nd = -12582912.0f * d;
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float f[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        int q;
        asm("bfe.s32 %0, %1, %2, 8;" : "=r"(q) : "r"(w[i]), "r"(8 * j));
        f[j] = __fmaf_rn(__int_as_float(0x4B400000 + q), d, nd);
      }
      v[2 * i] = b2u(__floats2bfloat162_rn(f[0], f[1]));
      v[2 * i + 1] = b2u(__floats2bfloat162_rn(f[2], f[3]));
    }
  }
};

// E2M1 byte pair -> f16x2 (hardware conversion), times a broadcast f16 scale (exact).
__device__ __forceinline__ uint32_t e2m1x2_f16(uint32_t byte, __half2 s) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)byte, __NV_E2M1);
  __half2 h;
  *reinterpret_cast<__half2_raw*>(&h) = r;
  return h2u(__hmul2(h, s));
}

template <>
struct Dequant<FMT_NVFP4, false> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int /*c*/, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 5);
    const uint16_t sb = *reinterpret_cast<const uint16_t*>(srow + (e0 >> 4));
    const __half2_raw sr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)sb, __NV_E4M3);
    const __half2 s0 = half2_bcast(sr.x), s1 = half2_bcast(sr.y);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * i + j] = e2m1x2_f16((w[i] >> (8 * j)) & 0xFFu, i < 2 ? s0 : s1);
    }
  }
};

template <>
struct Dequant<FMT_MXFP4, false> {
  // ex = E - Emax_row, the exponent of this block relative to the row's largest block;
  // the f16 scale is 2^(ex + 13) so the largest block's values stay below 2^16.
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int c, int e0, int emax, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 5);
    const int e = srow[e0 >> 5];
    const __half2 s = half2_bcast(f16_pow2_bits(e - emax + 13));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[4 * i + j] = e2m1x2_f16((w[i] >> (8 * j)) & 0xFFu, s);
    }
  }
};

// FP8 (E4M3) -> f16: the hardware E4M3x2 -> f16x2 conversion (every E4M3 value is exact in
// f16); the tensor scale is applied in the epilogue.
template <>
struct Dequant<FMT_FP8, false> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* /*srow*/,
                                             int /*c*/, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 4);
    const uint4 b = ld_sw128(crow, row, (e0 >> 4) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] & 0xFFFFu), __NV_E4M3);
      const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w[i] >> 16), __NV_E4M3);
      v[2 * i] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
      v[2 * i + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
    }
  }
};

// FP8 (E4M3) -> bf16 through f16 and fp32 (every E4M3 value is exact in each).
template <>
struct Dequant<FMT_FP8, true> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* /*srow*/,
                                             int /*c*/, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 4);
    const uint4 b = ld_sw128(crow, row, (e0 >> 4) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const __half2_raw r =
            __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)((w[i] >> (16 * j)) & 0xFFFFu), __NV_E4M3);
        __half2 h;
        *reinterpret_cast<__half2_raw*>(&h) = r;
        v[2 * i + j] = b2u(__float22bfloat162_rn(__half22float2(h)));
      }
    }
  }
};

// E2M1 -> bf16 for 8 codes in one word (two prmt byte tables for the magnitude, prmt sign
// replication for the sign bits), times a broadcast bf16 scale (exact).
__device__ __forceinline__ void e2m1x8_bf16(uint32_t w, __nv_bfloat162 s, uint32_t* out) {
  // bf16 high / low bytes of the magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} by code 0..7
  constexpr uint32_t HI0 = 0x3F3F3F00u, HI1 = 0x40404040u;
  constexpr uint32_t LO0 = 0xC0800000u, LO1 = 0xC0804000u;
  const uint32_t m = w & 0x77777777u;
  const uint32_t m2 = m >> 16;
  const uint32_t w4 = w << 4;  // byte i's msb = sign of the even code 2i; w's = odd code 2i+1
  const uint32_t H = prmt(HI0, HI1, m), L = prmt(LO0, LO1, m);
  const uint32_t H2 = prmt(HI0, HI1, m2), L2 = prmt(LO0, LO1, m2);
  uint32_t o[4];
  o[0] = prmt(L, H, 0x5140u);
  o[1] = prmt(L, H, 0x7362u);
  o[2] = prmt(L2, H2, 0x5140u);
  o[3] = prmt(L2, H2, 0x7362u);
  const uint32_t sel[4] = {0xC080u, 0xD090u, 0xE0A0u, 0xF0B0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t sg;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(sg) : "r"(w4), "r"(w), "r"(sel[i]));
    const uint32_t val = (o[i] & 0x7FFF7FFFu) | (sg & 0x80008000u);
    out[i] = b2u(__hmul2(u2b(val), s));
  }
}

template <>
struct Dequant<FMT_NVFP4, true> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int /*c*/, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 5);
    const uint16_t sb = *reinterpret_cast<const uint16_t*>(srow + (e0 >> 4));
    const __half2_raw sr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)sb, __NV_E4M3);
    const __nv_bfloat16 b0 = __float2bfloat16_rn(__half2float(__ushort_as_half(sr.x)));
    const __nv_bfloat16 b1 = __float2bfloat16_rn(__half2float(__ushort_as_half(sr.y)));
    const __nv_bfloat162 s0 = __halves2bfloat162(b0, b0), s1 = __halves2bfloat162(b1, b1);
    e2m1x8_bf16(a.x, s0, &v[0]);
    e2m1x8_bf16(a.y, s0, &v[4]);
    e2m1x8_bf16(a.z, s1, &v[8]);
    e2m1x8_bf16(a.w, s1, &v[12]);
  }
};

template <>
struct Dequant<FMT_MXFP4, true> {
  __device__ __forceinline__ static void run(const uint8_t* crow, int row, const uint8_t* srow,
                                             int c, int e0, int /*ex*/, uint32_t (&v)[16]) {
    const uint4 a = ld_sw128(crow, row, e0 >> 5);
    const uint32_t e = srow[e0 >> 5];
    const uint32_t bits = e ? (e << 7) : 0x0040u;  // 2^(e-127) as bf16 (e = 0: subnormal)
    const __nv_bfloat162 s = u2b(bits | (bits << 16));
    e2m1x8_bf16(a.x, s, &v[0]);
    e2m1x8_bf16(a.y, s, &v[4]);
    e2m1x8_bf16(a.z, s, &v[8]);
    e2m1x8_bf16(a.w, s, &v[12]);
  }
};


// ---------------------------------------------------------------------------------------
// Epilogue helpers
// ---------------------------------------------------------------------------------------
// 2^e as a float, exact for -149 <= e <= 127 (subnormal below -126), 0 below -149.
__device__ __forceinline__ float exp2_exact(int e) {
  if (e >= -126) return __int_as_float((min(e, 127) + 127) << 23);
  return e >= -149 ? __int_as_float(1 << (e + 149)) : 0.0f;
}

// Epilogue exponents within +-kFastExp take plain multiplies by exact powers of two.
constexpr int kFastExp = 60;

// v * 2^ex with a single rounding, for any ex (x rows of bf16 subnormals give ex down to
// -147); kept out of line, off the epilogue's fast path.
static __device__ __noinline__ float scale_pow2_exact(float v, int ex) { return ldexpf(v, ex); }

// y[m][n] (m: row of x and y)
__device__ __forceinline__ void store_y(const GemmParams& p, int m, int n, float v) {
  if (p.out_bf16)
    reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(p.out)[(size_t)m * p.N + n] = v;
}

// SiLU(g) * u rounded to bf16.  The fast exponential's relative error (~2^-21) is far
// below the bf16 rounding of h, and it keeps the epilogue from being bound by expf.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return g / (1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ void store_h(const GemmParams& p, int m, int n, float g, float u) {
  reinterpret_cast<__nv_bfloat16*>(p.out)[(size_t)m * p.N + n] = __float2bfloat16_rn(silu_mul(g, u));
}



}  // namespace qg

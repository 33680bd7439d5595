// pack.cu -- weight quantisation into the packed layout of qgemm.h (not performance critical).
//
// Recipes (the pages name the formats but not their quantisers; see qgemm.h):
//   Q8_0 : d = fp16_RNE(amax/127) kept finite; q = clamp(RNE(w/d), -127, 127).
//   NVFP4: ts = fp32_RNE(amax(W)/2688); s = E4M3_RNE_sat(amax_blk/(6 ts));
//          code = E2M1_RNE_sat(w/(e4m3(s) ts)).
//   MXFP4: e = clamp(floor(log2 amax_blk) - 2 + 127, 0, 254); code = E2M1_RNE_sat(w/2^(e-127)).
//   FP8  : ts = fp32_RNE(amax(W)/448); code = E4M3_RNE_sat(w/ts), sign kept at zero.
// Every quotient is formed once in fp64 from exact operands (the divisor products are exact
// in fp64), then rounded once to the target format -- fp16 by the integer routine below,
// E4M3 / E2M1 by NVIDIA's double -> fp8 / fp4 conversions -- so ties are decided on the
// exact value.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace qg {

__device__ __forceinline__ uint32_t e2m1_code(double v) {
  // sign is kept for values whose magnitude rounds to zero
  const uint32_t mag = (uint32_t)__nv_cvt_double_to_fp4(fabs(v), __NV_E2M1, cudaRoundNearest) & 7u;
  return (v < 0.0 ? 8u : 0u) | mag;
}

// binary16 bit pattern nearest to a (0 <= a <= 65504), ties to even, computed from the exact
// fp64 significand with integer arithmetic.
__device__ __forceinline__ uint16_t f16_bits_rne(double a) {
  if (!(a > 0.0)) return 0;
  const uint64_t u = static_cast<uint64_t>(__double_as_longlong(a));
  const int e = (int)((u >> 52) & 0x7FF) - 1023;                  // a = 1.f * 2^e
  const uint64_t m = (u & ((1ull << 52) - 1)) | (1ull << 52);     // 53-bit significand
  int drop = 52 - 10;                                             // keep 11 significant bits
  if (e < -14) drop += -14 - e;                                   // subnormals: quantum 2^-24
  if (drop > 63) return 0;
  uint64_t q = m >> drop;
  const uint64_t rem = m & ((1ull << drop) - 1);
  const uint64_t half = 1ull << (drop - 1);
  if (rem > half || (rem == half && (q & 1))) ++q;
  if (e < -14) return (uint16_t)q;  // q = 1024 is the smallest normal: same bits
  int E = e;
  if (q == 2048) {
    q = 1024;
    ++E;
  }
  return (uint16_t)(((E + 15) << 10) | (q & 1023));
}

// One thread per 32-element block.
__global__ void pack_q8_0_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                 uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int64_t nb = K / 32;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * nb) return;
  const int64_t n = idx / nb, kb = idx % nb;
  const float* w = W + n * K + kb * 32;
  float amax = 0.f;
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(w[i]));
  double dq = (double)amax / 127.0;
  if (dq > 65504.0) dq = 65504.0;
  const uint16_t hb = f16_bits_rne(dq);
  const double d = (double)__half2float(__ushort_as_half(hb));
  const int64_t C = k_chunks(FMT_Q8_0, K);
  const int64_t k0 = kb * 32, c = k0 / 128;
  const int b0 = (int)(k0 % 128);
  uint8_t* sp = scales + scale_offset(FMT_Q8_0, C, n, c) + 2 * (b0 / 32);
  sp[0] = (uint8_t)(hb & 0xFF);
  sp[1] = (uint8_t)(hb >> 8);
  for (int i = 0; i < 32; ++i) {
    double q = 0.0;
    if (d != 0.0) q = fmin(127.0, fmax(-127.0, rint((double)w[i] / d)));
    codes[code_offset(C, n, c, b0 + i)] = (uint8_t)(int8_t)q;
  }
}

// amax over the whole matrix into *amax_bits (non-negative floats order like their bits).
__global__ void amax_kernel(const float* __restrict__ W, int64_t total, unsigned int* amax_bits) {
  float m = 0.f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(W[i]));
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(m));
}

__device__ __forceinline__ float nvfp4_ts_from_amax(float amax) {
  return __double2float_rn((double)amax / (6.0 * 448.0));
}

__device__ __forceinline__ float fp8_ts_from_amax(float amax) {
  return __double2float_rn((double)amax / 448.0);
}

// One thread per 16-element block.  amax_bits holds max|W| (written by amax_kernel).
__global__ void pack_nvfp4_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                  const unsigned int* amax_bits) {
  const int64_t nb = K / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * nb) return;
  const int64_t n = idx / nb, kb = idx % nb;
  const float ts = nvfp4_ts_from_amax(__uint_as_float(*amax_bits));
  const float* w = W + n * K + kb * 16;
  float ab = 0.f;
  for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(w[i]));
  uint32_t s = 0;
  if (ab != 0.f && ts != 0.f)
    s = (uint32_t)__nv_cvt_double_to_fp8((double)ab / (6.0 * (double)ts), __NV_SATFINITE, __NV_E4M3);
  const __half_raw sr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)s, __NV_E4M3);
  const double sv = (double)__half2float(__ushort_as_half(sr.x));
  const int64_t C = k_chunks(FMT_NVFP4, K);
  const int64_t k0 = kb * 16, c = k0 / 256;
  const int e0 = (int)(k0 % 256);
  scales[scale_offset(FMT_NVFP4, C, n, c) + e0 / 16] = (uint8_t)s;
  const double den = sv * (double)ts;
  for (int i = 0; i < 8; ++i) {
    uint32_t lo = 0, hi = 0;
    if (sv != 0.0) {
      lo = e2m1_code((double)w[2 * i] / den);
      hi = e2m1_code((double)w[2 * i + 1] / den);
    }
    codes[code_offset(C, n, c, e0 / 2 + i)] = (uint8_t)(lo | (hi << 4));
  }
}

__global__ void nvfp4_finish_kernel(float* tensor_scale) {
  const unsigned int bits = *reinterpret_cast<unsigned int*>(tensor_scale);
  *tensor_scale = nvfp4_ts_from_amax(__uint_as_float(bits));
}

// One thread per 16 consecutive elements of a row.  amax_bits holds max|W|.
__global__ void pack_fp8_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                uint8_t* __restrict__ codes, const unsigned int* amax_bits) {
  const int64_t nb = K / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * nb) return;
  const int64_t n = idx / nb, kb = idx % nb;
  const float ts = fp8_ts_from_amax(__uint_as_float(*amax_bits));
  const float* w = W + n * K + kb * 16;
  const int64_t C = k_chunks(FMT_FP8, K);
  const int64_t k0 = kb * 16, c = k0 / 128;
  const int b0 = (int)(k0 % 128);
  for (int i = 0; i < 16; ++i) {
    uint32_t code = 0;
    if (ts != 0.f) {
      const double v = (double)w[i] / (double)ts;
      code = ((uint32_t)__nv_cvt_double_to_fp8(fabs(v), __NV_SATFINITE, __NV_E4M3) & 0x7Fu) |
             (v < 0.0 ? 0x80u : 0u);
    }
    codes[code_offset(C, n, c, b0 + i)] = (uint8_t)code;
  }
}

__global__ void fp8_finish_kernel(float* tensor_scale) {
  const unsigned int bits = *reinterpret_cast<unsigned int*>(tensor_scale);
  *tensor_scale = fp8_ts_from_amax(__uint_as_float(bits));
}

// One thread per 32-element block.
__global__ void pack_mxfp4_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int64_t nb = K / 32;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= N * nb) return;
  const int64_t n = idx / nb, kb = idx % nb;
  const float* w = W + n * K + kb * 32;
  float ab = 0.f;
  for (int i = 0; i < 32; ++i) ab = fmaxf(ab, fabsf(w[i]));
  int e = 0;
  if (ab != 0.f) {
    int ex;
    (void)frexp((double)ab, &ex);  // floor(log2 ab) = ex - 1 exactly
    e = min(254, max(0, (ex - 1) - 2 + 127));
  }
  const int64_t C = k_chunks(FMT_MXFP4, K);
  const int64_t k0 = kb * 32, c = k0 / 256;
  const int e0 = (int)(k0 % 256);
  scales[scale_offset(FMT_MXFP4, C, n, c) + e0 / 32] = (uint8_t)e;
  const double sc = ldexp(1.0, e - 127);
  for (int i = 0; i < 16; ++i) {
    uint32_t lo = 0, hi = 0;
    if (ab != 0.f) {
      lo = e2m1_code((double)w[2 * i] / sc);
      hi = e2m1_code((double)w[2 * i + 1] / sc);
    }
    codes[code_offset(C, n, c, e0 / 2 + i)] = (uint8_t)(lo | (hi << 4));
  }
}

// Row-major interchange layout -> tile-major layout.  One thread per (row, chunk); rows and
// chunks past the matrix are written as zeros.
__global__ void repack_kernel(const RepackParams p) {
  const int64_t C = k_chunks(p.fmt, p.K);
  const int64_t T = row_tiles(p.N);
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T * kTileRows * C) return;
  const int64_t n = idx / C, c = idx % C;
  const int64_t row_bytes = rm_code_bytes_per_row(p.fmt, p.K);
  const int64_t srow_bytes = rm_scale_bytes_per_row(p.fmt, p.K);
  const int SBr = scale_row_bytes(p.fmt);
  for (int b = 0; b < kWRowBytes; ++b) {
    const int64_t src = c * kWRowBytes + b;
    const uint8_t v = (n < p.N && src < row_bytes) ? p.codes_rm[n * p.code_pitch + src] : 0;
    p.codes[code_offset(C, n, c, b)] = v;
  }
  for (int b = 0; b < SBr; ++b) {
    const int64_t src = c * SBr + b;
    const uint8_t v = (n < p.N && src < srow_bytes) ? p.scales_rm[n * p.scale_pitch + src] : 0;
    p.scales[scale_offset(p.fmt, C, n, c) + b] = v;
  }
}

cudaError_t launch_repack(const RepackParams& rp, cudaStream_t stream) {
  const int64_t total = row_tiles(rp.N) * kTileRows * k_chunks(rp.fmt, rp.K);
  const int threads = 256;
  repack_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(rp);
  return cudaGetLastError();
}

cudaError_t launch_pack(int fmt, const float* W, int64_t N, int64_t K, void* codes, void* scales,
                        float* tensor_scale, cudaStream_t stream) {
  cudaError_t e = cudaSuccess;
  // padding rows and K past the last block are zero
  e = cudaMemsetAsync(codes, 0, (size_t)packed_code_bytes(fmt, N, K), stream);
  if (e != cudaSuccess) return e;
  if (packed_scale_bytes(fmt, N, K) > 0) {
    e = cudaMemsetAsync(scales, 0, (size_t)packed_scale_bytes(fmt, N, K), stream);
    if (e != cudaSuccess) return e;
  }
  const int threads = 256;
  if (fmt == FMT_Q8_0) {
    const int64_t blocks = (N * (K / 32) + threads - 1) / threads;
    pack_q8_0_kernel<<<(unsigned)blocks, threads, 0, stream>>>(W, N, K, (uint8_t*)codes,
                                                              (uint8_t*)scales);
  } else if (fmt == FMT_NVFP4) {
    e = cudaMemsetAsync(tensor_scale, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    amax_kernel<<<1184, threads, 0, stream>>>(W, N * K, reinterpret_cast<unsigned int*>(tensor_scale));
    const int64_t blocks = (N * (K / 16) + threads - 1) / threads;
    pack_nvfp4_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        W, N, K, (uint8_t*)codes, (uint8_t*)scales, reinterpret_cast<unsigned int*>(tensor_scale));
    nvfp4_finish_kernel<<<1, 1, 0, stream>>>(tensor_scale);
  } else if (fmt == FMT_FP8) {
    e = cudaMemsetAsync(tensor_scale, 0, sizeof(float), stream);
    if (e != cudaSuccess) return e;
    amax_kernel<<<1184, threads, 0, stream>>>(W, N * K, reinterpret_cast<unsigned int*>(tensor_scale));
    const int64_t blocks = (N * (K / 16) + threads - 1) / threads;
    pack_fp8_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
        W, N, K, (uint8_t*)codes, reinterpret_cast<unsigned int*>(tensor_scale));
    fp8_finish_kernel<<<1, 1, 0, stream>>>(tensor_scale);
  } else {
    const int64_t blocks = (N * (K / 32) + threads - 1) / threads;
    pack_mxfp4_kernel<<<(unsigned)blocks, threads, 0, stream>>>(W, N, K, (uint8_t*)codes,
                                                               (uint8_t*)scales);
  }
  return cudaGetLastError();
}

}  // namespace qg

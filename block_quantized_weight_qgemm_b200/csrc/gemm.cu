// gemm.cu -- the kernels around the GEMM of libqgemm (sm_100a): the x preparation for the
// f16-operand path, the fixed-order split-K reduction with the output epilogue, and the
// library's device error word.  The GEMM itself is the CTA-pair kernel in pair.cu.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "dequant.cuh"
#include "ptx.cuh"

namespace qg {

// The library's device error word (bounded waits that ran out write kErrTimeout).
__device__ int g_dev_err = 0;

// ---------------------------------------------------------------------------------------
// x preparation for the f16 path (widths <= 256): per row, e = floor(log2 amax) - 14,
// xh = f16(x * 2^-e) (exact for every bf16 value within 2^-38 of the row maximum), and the
// row's exponent e, which the GEMM epilogue restores.  Rows of xh are padded with zeros to
// a multiple of 64 elements.  e runs from -147 (a row of bf16 subnormals) to 113, so 2^-e
// can exceed the largest fp32 power of two; it is applied as two exact factors, 2^n1 with
// n1 = min(-e, 126) and 2^(-e - n1) (which is 1 unless the row's maximum is below 2^-112).
// ---------------------------------------------------------------------------------------
constexpr int kPrepThreads = 1024;  // one CTA per x row
constexpr int kPrepRegs = 3;        // 16-byte words per thread held in registers (rows to 24576)

__device__ __forceinline__ float amax8(float m, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = fmaxf(m, fabsf(__uint_as_float(w[i] << 16)));
    m = fmaxf(m, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
  }
  return m;
}

// 8 bf16 values times 2^n1 * 2^n2 (both factors normal powers of two: each product is exact
// unless it leaves the f16 range), rounded once to f16
__device__ __forceinline__ uint4 to_f16x8(const uint4& v, float sc1, float sc2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half lo = __float2half_rn(__uint_as_float(w[i] << 16) * sc1 * sc2);
    const __half hi = __float2half_rn(__uint_as_float(w[i] & 0xFFFF0000u) * sc1 * sc2);
    o[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__global__ void __launch_bounds__(kPrepThreads) qgemm_prep_x_kernel(const PrepParams p) {
  // The GEMM that follows may start its set-up and weight streaming now; it waits for this
  // grid before it reads xh or x_exp.  Its weight reads are not ordered after the grid before
  // this one: weights must come from a grid that has completed, or that does not let its
  // dependents launch early (the library's packers do not).
  griddep_launch_dependents();
  // x may come from the grid before this one, which may also still read xh and x_exp
  griddep_wait();
  const int b = blockIdx.x;
  const uint16_t* xr = p.x + (size_t)b * p.K;
  __shared__ float red[kPrepThreads / 32];
  // one pass over the row: the first kPrepRegs words of each thread stay in registers, any
  // longer tail is read again for the conversion
  uint4 v[kPrepRegs];
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < kPrepRegs; ++j) {
    const int k = (threadIdx.x + j * kPrepThreads) * 8;
    v[j] = (k < p.K) ? *reinterpret_cast<const uint4*>(xr + k) : make_uint4(0u, 0u, 0u, 0u);
    amax = amax8(amax, v[j]);
  }
  for (int k = (threadIdx.x + kPrepRegs * kPrepThreads) * 8; k < p.K; k += kPrepThreads * 8)
    amax = amax8(amax, *reinterpret_cast<const uint4*>(xr + k));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  if (threadIdx.x < 32) {
    float m = red[threadIdx.x];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) red[0] = m;
  }
  __syncthreads();
  amax = red[0];
  int e = 0;
  if (amax > 0.f && amax <= 3.4e38f) {
    int ex;
    (void)frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
    e = (ex - 1) - 14;        // amax * 2^-e in [2^14, 2^15)
  }
  const int n1 = min(-e, 126);
  const float sc1 = __int_as_float((n1 + 127) << 23);      // 2^n1, n1 in [-113, 126]
  const float sc2 = __int_as_float((-e - n1 + 127) << 23);  // 2^(-e-n1), exponent in [0, 21]
  uint16_t* xo = p.xh + (size_t)b * p.Kp;
#pragma unroll
  for (int j = 0; j < kPrepRegs; ++j) {
    const int k = (threadIdx.x + j * kPrepThreads) * 8;
    if (k < p.K) *reinterpret_cast<uint4*>(xo + k) = to_f16x8(v[j], sc1, sc2);
  }
  for (int k = (threadIdx.x + kPrepRegs * kPrepThreads) * 8; k < p.K; k += kPrepThreads * 8)
    *reinterpret_cast<uint4*>(xo + k) =
        to_f16x8(*reinterpret_cast<const uint4*>(xr + k), sc1, sc2);
  for (int k = p.K + threadIdx.x * 8; k < p.Kp; k += kPrepThreads * 8)
    *reinterpret_cast<uint4*>(xo + k) = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) p.x_exp[b] = e;
}

// ---------------------------------------------------------------------------------------
// Split-K reduction: out = epilogue(sum_{s=0..S-1} partial_s), in that fixed order, one
// 4-wide column group (b, n..n+3) per thread.  The epilogue is the output conversion, or
// SiLU(g) * u for the fused gate+up.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qgemm_splitk_reduce_kernel(const ReduceParams p) {
  griddep_launch_dependents();  // the next call's preparation may launch and wait
  griddep_wait();  // launched as a programmatic dependent of the GEMM that wrote the partials
  const int64_t nq = (p.N + 3) / 4;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)p.B * nq) return;
  const int b = (int)(idx / nq);
  const int n = (int)(idx % nq) * 4;
  const size_t BN = (size_t)p.B * p.N;
  const size_t off = (size_t)b * p.N + n;
  const int lim = min(4, p.N - n);
  const bool vec = ((p.N & 3) == 0);
  float g[4] = {0.f, 0.f, 0.f, 0.f}, u[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < p.S; ++s) {
    const float* src = p.ws + (size_t)(s * p.NMAT) * BN + off;
    if (vec) {
      const float4 t = __ldcs(reinterpret_cast<const float4*>(src));
      g[0] += t.x; g[1] += t.y; g[2] += t.z; g[3] += t.w;
      if (p.NMAT == 2) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(src + BN));
        u[0] += v.x; u[1] += v.y; u[2] += v.z; u[3] += v.w;
      }
    } else {
      for (int e = 0; e < lim; ++e) {
        g[e] += __ldcs(src + e);
        if (p.NMAT == 2) u[e] += __ldcs(src + BN + e);
      }
    }
  }
  // the partials already carry every scale (tensor scale, x and row exponents)
  for (int e = 0; e < lim; ++e) {
    if (p.NMAT == 1) {
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.out)[off + e] = __float2bfloat16_rn(g[e]);
      else
        reinterpret_cast<float*>(p.out)[off + e] = g[e];
    } else {
      reinterpret_cast<__nv_bfloat16*>(p.out)[off + e] = __float2bfloat16_rn(silu_mul(g[e], u[e]));
    }
  }
}

// ---------------------------------------------------------------------------------------
// Host-side launchers (called by the C-ABI layer)
// ---------------------------------------------------------------------------------------
int* device_error_word() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_dev_err) != cudaSuccess) return nullptr;
  return static_cast<int*>(ptr);
}

// The small kernels around the GEMM ask for the largest shared-memory carveout, the one the
// GEMM runs with, so that the SMs need no L1/shared reconfiguration between the launches.
static void prefer_max_shared(const void* fn) {
  (void)cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
}

cudaError_t launch_reduce(const ReduceParams& rp, cudaStream_t stream) {
  static const bool once = (prefer_max_shared((const void*)qgemm_splitk_reduce_kernel), true);
  (void)once;
  const int64_t total = (int64_t)rp.B * ((rp.N + 3) / 4);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((total + 255) / 256), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qgemm_splitk_reduce_kernel, rp);
}

cudaError_t launch_prep(const PrepParams& pp, cudaStream_t stream) {
  static const bool once = (prefer_max_shared((const void*)qgemm_prep_x_kernel), true);
  (void)once;
  // a programmatic dependent of whatever precedes it: it launches early and waits for that
  // grid (griddepcontrol.wait) before it reads x or writes the workspace
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)pp.B, 1, 1);
  cfg.blockDim = dim3(kPrepThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, qgemm_prep_x_kernel, pp);
}

}  // namespace qg

// gemm.cu -- the block-quantized-weight GEMM kernels of libqgemm (sm_100a).
//
// y[b][n] = sum_k x[b][k] * dequant(W)[n][k]     (hipfire PR "fix(mtp): chunk scalar Q8
// batched GEMM above 64 rows"; Atlas issue "Qwen3.8-27B on Strix Halo: prefill 2.4x gap",
// kernel ranking and exact-F16-dequant sections)
//
// Design (swap-AB on the 5th-generation tensor cores):
//   * Weights are the MMA M operand: one subtile = 128 weight rows, held in tensor memory
//     (TMEM) as 16-bit values that dequant warps write with tcgen05.st.
//   * Activations are the MMA N operand: NB <= 256 batch rows of x, loaded by TMA into
//     128-byte-swizzled shared memory and read by the MMA through a smem descriptor.
//   * Accumulators live in TMEM (fp32), one NB-column block per weight subtile.
//   * Warp roles: warp 0 issues TMA loads, warp 1 allocates TMEM and issues tcgen05.mma,
//     warps 2..9 dequantize packed weights from the smem ring into the TMEM A ring and then
//     run the epilogue.
//   * K is split into S contiguous ranges (S fixed by format, N, K); partials are summed in
//     the fixed order s = 0..S-1 by whichever CTA of a tile arrives last.  Nothing in the
//     arithmetic depends on the batch width, so row b of y is bit-identical for B <= 256.
//   * Widths 1..256 use f16 operands: x rows are rescaled by a power of two chosen from the
//     row's own maximum (exact), then rounded to f16 (exact for every bf16 value within
//     2^-38 of the row maximum), and the power of two is restored in the epilogue.  The
//     dequantized weights are exact in f16 for NVFP4 (E2M1 x E4M3 has <= 6 significant bits,
//     range [2^-10, 2688]) and for MXFP4 (after a per-row power-of-two rebase of the E8M0
//     exponents); Q8_0 products q*d are rounded once.
//   * Widths above 256 (prefill) use bf16 operands straight from the caller's x, no split.
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
// x preparation for the f16 path: per row, e = floor(log2 amax) - 14, xh = f16(x * 2^-e).
// Also clears the split-K arrival counters of the GEMM that follows on the stream.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qgemm_prep_x_kernel(const PrepParams p) {
  const int b = blockIdx.x;
  const uint16_t* xr = p.x + (size_t)b * p.K;
  __shared__ float red[8];
  float amax = 0.f;
  for (int k = threadIdx.x * 8; k < p.K; k += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) amax = fmaxf(amax, red[i]);
  int e = 0;
  if (amax > 0.f && amax <= 3.4e38f) {
    int ex;
    (void)frexpf(amax, &ex);  // amax = f * 2^ex, f in [0.5, 1)
    e = (ex - 1) - 14;        // amax * 2^-e in [2^14, 2^15)
  }
  const float sc = ldexpf(1.0f, -e);
  uint16_t* xo = p.xh + (size_t)b * p.Kp;
  for (int k = p.K + threadIdx.x * 8; k < p.Kp; k += blockDim.x * 8)
    *reinterpret_cast<uint4*>(xo + k) = make_uint4(0u, 0u, 0u, 0u);
  for (int k = threadIdx.x * 8; k < p.K; k += blockDim.x * 8) {
    const uint4 v = *reinterpret_cast<const uint4*>(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half lo = __float2half_rn(__uint_as_float(w[i] << 16) * sc);
      const __half hi = __float2half_rn(__uint_as_float(w[i] & 0xFFFF0000u) * sc);
      o[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
    }
    *reinterpret_cast<uint4*>(xo + k) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (threadIdx.x == 0) p.x_exp[b] = e;
  if (b == 0)
    for (int i = threadIdx.x; i < p.n_counters; i += blockDim.x) p.counters[i] = 0;
}

// ---------------------------------------------------------------------------------------
// The GEMM kernel.  One CTA = one work unit (row group g, batch tile bt, K split s).
// ---------------------------------------------------------------------------------------
template <int FMT, bool BF16OP>
__global__ void __launch_bounds__(kThreads, 1)
    qgemm_tc_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tm_x) {
  constexpr int KW = chunk_k(FMT);
  constexpr int J = KW / kSubK;       // x stages per chunk
  constexpr int JA = KW / kAStageK;   // A stages per chunk
  constexpr int SB = scale_row_bytes(FMT);
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by pointer arithmetic on the shared array so that every access
  // through it stays a shared-memory access (an integer round trip would make them generic)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sx = sbase + p.smem_x;
  const uint32_t sw = sbase + p.smem_w;
  const int XS = p.XS, WS = p.WS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.smem_bar);
  const uint32_t bar_x_full = smem_u32(bars);
  const uint32_t bar_x_empty = bar_x_full + 8 * XS;
  const uint32_t bar_w_full = bar_x_empty + 8 * XS;
  const uint32_t bar_w_empty = bar_w_full + 8 * WS;
  const uint32_t bar_a_full = bar_w_empty + 8 * WS;
  const int AS = p.AS;
  const uint32_t bar_a_empty = bar_a_full + 8 * AS;
  const uint32_t bar_acc = bar_a_empty + 8 * AS;
  int* ctl = reinterpret_cast<int*>(bars + 2 * XS + 2 * WS + 2 * AS + 1);
  volatile int* abort_flag = ctl + 1;
  float* col_fac = reinterpret_cast<float*>(ctl + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int u = blockIdx.x;
  const int g = u % p.n_groups;
  u /= p.n_groups;
  const int bt = u % p.b_tiles;
  const int s = u / p.b_tiles;
  const int c0 = (int)((int64_t)s * p.chunks / p.S);
  const int c1 = (int)((int64_t)(s + 1) * p.chunks / p.S);
  const int tiles_per_group = p.R / p.NMAT;
  const int64_t n_row_tiles = row_tiles(p.N);
  const uint32_t a_col0 = (uint32_t)(p.R * p.NB);

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    for (int i = 0; i < XS; ++i) {
      mbar_init(bar_x_full + 8 * i, 1);
      mbar_init(bar_x_empty + 8 * i, (uint32_t)p.R);  // every MMA issuer releases each x stage
    }
    for (int i = 0; i < WS; ++i) {
      mbar_init(bar_w_full + 8 * i, 1);
      mbar_init(bar_w_empty + 8 * i, kDequantWarps);
    }
    for (int i = 0; i < AS; ++i) {
      mbar_init(bar_a_full + 8 * i, kDequantWarps);
      mbar_init(bar_a_empty + 8 * i, 1);
    }
    mbar_init(bar_acc, (uint32_t)p.R);  // one commit per MMA issuer
    ctl[1] = 0;
    ctl[2] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctl), (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  if (warp >= kFirstDequantWarp) {
    for (int i = threadIdx.x - kFirstDequantWarp * 32; i < p.NB; i += kDequantWarps * 32) {
      const int b = bt * p.NB + i;
      col_fac[i] = (b < p.B) ? (p.x_exp ? ldexpf(1.0f, p.x_exp[b]) : 1.0f) : 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(ctl[0]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Two independent streams, each limited only by its own ring: weight stages in the
    // order (c, r) and x stages in the order (c, j).  Lane 0 polls both without blocking
    // on either, so weight prefetch never waits behind an x slot (and vice versa).
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      const int nchunks = c1 - c0;
      const int w_total = nchunks * p.R, x_total = nchunks * J;
      RingPos xp, wp;
      int x_issued = 0, w_issued = 0;
      int wc = c0, wr = 0;  // next weight stage (chunk, subtile)
      int xc = c0, xj = 0;  // next x stage (chunk, slice)
      bool ok = true;
      uint64_t idle_since = 0;
      while (ok && (w_issued < w_total || x_issued < x_total)) {
        bool progressed = false;
        if (w_issued < w_total &&
            (w_issued < WS || mbar_test_wait(bar_w_empty + 8 * wp.slot, wp.phase ^ 1u))) {
          const uint32_t fb = bar_w_full + 8 * wp.slot;
          const int m = (p.NMAT == 2) ? (wr & 1) : 0;
          const int64_t t = (int64_t)g * tiles_per_group + (p.NMAT == 2 ? (wr >> 1) : wr);
          const uint32_t dst = sw + (uint32_t)(wp.slot * kWStageBytes);
          if (t < n_row_tiles) {
            // one contiguous block of codes and one of scales per (tile, chunk)
            const int64_t blk = t * p.chunks + wc;
            mbar_arrive_expect_tx(fb, (uint32_t)(kWCodeBytes + kTileRows * SB));
            bulk_load(dst, p.codes[m] + blk * kWCodeBytes, kWCodeBytes, fb, pol_w);
            bulk_load(dst + kWCodeBytes, p.scales[m] + blk * (kTileRows * SB),
                      (uint32_t)(kTileRows * SB), fb, pol_w);
          } else {
            mbar_arrive(fb);  // a tile past the matrix: its rows are never stored
          }
          wp.next(WS);
          ++w_issued;
          if (++wr == p.R) {
            wr = 0;
            ++wc;
          }
          progressed = true;
        }
        if (x_issued < x_total &&
            (x_issued < XS || mbar_test_wait(bar_x_empty + 8 * xp.slot, xp.phase ^ 1u))) {
          const uint32_t fb = bar_x_full + 8 * xp.slot;
          mbar_arrive_expect_tx(fb, (uint32_t)p.NB * 128u);
          tma_load_2d(sx + (uint32_t)(xp.slot * p.NB * 128), &tm_x, fb, xc * KW + xj * kSubK,
                      bt * p.NB, pol_x);
          xp.next(XS);
          ++x_issued;
          if (++xj == J) {
            xj = 0;
            ++xc;
          }
          progressed = true;
        }
        if (progressed) {
          idle_since = 0;
        } else {
          const uint64_t now = globaltimer_ns();
          if (idle_since == 0) idle_since = now;
          if (*abort_flag) ok = false;
          if (now - idle_since > kWaitLimitNs) {
            *abort_flag = 1;
            atomicExch(p.dev_err, kErrTimeout);
            ok = false;
          }
          __nanosleep(20);
        }
      }
      if (!ok) {
        // let every load already issued land before the CTA leaves: the last use of each
        // slot is at most one ring depth back
        for (int k = 0; k < XS && k < x_issued; ++k) {
          xp.slot = (xp.slot == 0) ? XS - 1 : xp.slot - 1;
          if (xp.slot == XS - 1) xp.phase ^= 1u;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar_x_full + 8 * xp.slot, xp.phase) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
        for (int k = 0; k < WS && k < w_issued; ++k) {
          wp.slot = (wp.slot == 0) ? WS - 1 : wp.slot - 1;
          if (wp.slot == WS - 1) wp.phase ^= 1u;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(bar_w_full + 8 * wp.slot, wp.phase) &&
                 globaltimer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp < kFirstDequantWarp) {
    // ------------------------------------------------------------ MMA issuers
    // One thread per weight subtile r (warp 1 + r): it owns accumulator r, so the issuers'
    // MMAs never touch the same accumulator and each accumulator still receives its K slices
    // in ascending order.  Several issuers keep the tensor pipe fed while one of them is busy
    // with its waits and commits.
    const int r = warp - 1;
    if (lane == 0 && r < p.R) {
      const uint32_t idesc = idesc_f16(BF16OP, (uint32_t)p.NB);
      const uint32_t xstage_bytes = (uint32_t)p.NB * 128u;
      const uint32_t d = tmem + (uint32_t)(r * p.NB);
      // this issuer's A slots: spr = AS / R of them, used in turn, so each slot's uses
      // alternate phase within one thread (no parity aliasing between issuers)
      const int spr = AS / p.R;
      RingPos xc;  // first x stage of the current chunk
      bool ok = true;
      for (int c = c0; c < c1 && ok; ++c) {
        RingPos xp = xc;
        for (int ja = 0; ja < JA && ok; ++ja) {
          const int li = (c - c0) * JA + ja;  // this subtile's A stage count
          const int aslot = r * spr + li % spr;
          if (!mbar_wait(bar_a_full + 8 * aslot, (uint32_t)(li / spr) & 1u, abort_flag, p.dev_err,
                         kErrTimeout)) {
            ok = false;
            break;
          }
          const uint32_t a = tmem + a_col0 + (uint32_t)(aslot * kAColsPerStage);
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            if (!mbar_wait(bar_x_full + 8 * xp.slot, xp.phase, abort_flag, p.dev_err, kErrTimeout)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t bx = sx + (uint32_t)xp.slot * xstage_bytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = (c > c0 || ja > 0 || jj > 0 || kk > 0) ? 1u : 0u;
              mma_f16_ts(d, a + (uint32_t)(jj * 32 + kk * 8), smem_desc_sw128(bx + kk * 32), idesc,
                         acc);
            }
            mma_commit(bar_x_empty + 8 * xp.slot);
            xp.next(XS);
          }
          mma_commit(bar_a_empty + 8 * aslot);
        }
        for (int j = 0; j < J; ++j) xc.next(XS);
      }
      mma_commit(bar_acc);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    const int dw = warp - kFirstDequantWarp;
    const int q = warp & 3;       // TMEM lane quarter this warp may access
    const int h = dw >> 2;        // which 64-element half of each 128-element A stage
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;

    // MXFP4 on f16 operands: largest block exponent of this row within the split
    int emax[4] = {0, 0, 0, 0};
    if (FMT == FMT_MXFP4 && !BF16OP) {
      // (padding blocks past K are zero and cannot raise the maximum)
      for (int r = 0; r < p.R; ++r) {
        const int64_t n = (int64_t)(g * tiles_per_group + r / p.NMAT) * kTileRows + row;
        uint32_t mx = 0;
        if (n < p.N) {
          const uint8_t* sb = p.scales[r % p.NMAT];
          for (int c = c0; c < c1; ++c) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(sb + scale_offset(FMT, p.chunks, n, c)));
            mx = __vmaxu4(mx, __vmaxu4(v.x, v.y));
          }
        }
        mx = max(max(mx & 0xFFu, (mx >> 8) & 0xFFu), max((mx >> 16) & 0xFFu, mx >> 24));
        emax[r] = (int)mx;
      }
    }

    RingPos wp;
    const int spr = AS / p.R;  // A slots per subtile (see the MMA issuers)
    bool ok = true;
    for (int c = c0; c < c1 && ok; ++c) {
      for (int r = 0; r < p.R && ok; ++r) {
        ok = mbar_wait(bar_w_full + 8 * wp.slot, wp.phase, abort_flag, p.dev_err, kErrTimeout);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint8_t* stage = smem + p.smem_w + wp.slot * kWStageBytes;
        const uint8_t* crow = stage + row * kWRowBytes;
        const uint8_t* srow = stage + kWCodeBytes + row * SB;
        const int ex = emax[r & 3];
        for (int ja = 0; ja < JA; ++ja) {
          const int li = (c - c0) * JA + ja;
          const int aslot = r * spr + li % spr;
          const int use = li / spr;
          if (use > 0) {
            ok = mbar_wait(bar_a_empty + 8 * aslot, (uint32_t)(use - 1) & 1u, abort_flag, p.dev_err,
                           kErrTimeout);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          tc_fence_after();
          // this warp's 64 elements of the 128-element A stage, as two independent halves
          const int e0 = ja * kAStageK + h * 64;
          uint32_t v[32];
          Dequant<FMT, BF16OP>::run(crow, row, srow, c, e0, ex,
                                    *reinterpret_cast<uint32_t(*)[16]>(&v[0]));
          Dequant<FMT, BF16OP>::run(crow, row, srow, c, e0 + 32, ex,
                                    *reinterpret_cast<uint32_t(*)[16]>(&v[16]));
          tmem_st32(tmem + lane_base + a_col0 + (uint32_t)(aslot * kAColsPerStage + h * 32), v);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_a_full + 8 * aslot);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_w_empty + 8 * wp.slot);
        wp.next(WS);
      }
    }

    if (ok) {
      ok = mbar_wait(bar_acc, 0, abort_flag, p.dev_err, kErrTimeout);
      ok = __all_sync(0xffffffffu, ok);
    }
    tc_fence_after();
    const int half_cols = p.NB >> 1;
    const int cb0 = h * half_cols;
    const size_t BN = (size_t)p.B * p.N;
    float ts[2] = {1.0f, 1.0f};
    if (FMT == FMT_NVFP4) {
      ts[0] = __ldg(p.ts[0]);
      if (p.NMAT == 2) ts[1] = __ldg(p.ts[1]);
    }
    float rowfac[4] = {1.0f, 1.0f, 1.0f, 1.0f};
    if (FMT == FMT_MXFP4 && !BF16OP)
      for (int r = 0; r < p.R; ++r) rowfac[r & 3] = ldexpf(1.0f, emax[r & 3] - 140);
    if (ok) {
      // pass 1: scale the accumulators; store finals (S == 1) or partials (S > 1)
      for (int t2 = 0; t2 < tiles_per_group; ++t2) {
        const int n = (g * tiles_per_group + t2) * kTileRows + row;
        const float rf_g = rowfac[(t2 * p.NMAT) & 3];
        const float rf_u = rowfac[(t2 * p.NMAT + 1) & 3];
        for (int cb = cb0; cb < cb0 + half_cols; cb += 32) {
          const int nchunk = min(32, cb0 + half_cols - cb) >> 3;  // groups of 8 columns
          uint32_t va[4][8], vb[4][8];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            if (q8 < nchunk) {
              tmem_ld8(tmem + lane_base + (uint32_t)(t2 * p.NMAT * p.NB + cb + q8 * 8), va[q8]);
              if (p.NMAT == 2)
                tmem_ld8(tmem + lane_base + (uint32_t)((t2 * 2 + 1) * p.NB + cb + q8 * 8), vb[q8]);
            }
          }
          tmem_ld_wait();
          if (n >= p.N) continue;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            if (q8 >= nchunk) break;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int col = cb + q8 * 8 + i;
              const int b = bt * p.NB + col;
              if (b >= p.B) break;
              const float cf = col_fac[col];
              const float ga = __uint_as_float(va[q8][i]) * cf * rf_g;
              if (p.NMAT == 1) {
                if (p.S > 1) p.ws[(size_t)s * BN + (size_t)b * p.N + n] = ga;
                else store_y(p, b, n, ga * ts[0]);
              } else {
                const float ua = __uint_as_float(vb[q8][i]) * cf * rf_u;
                if (p.S > 1) {
                  p.ws[(size_t)(2 * s) * BN + (size_t)b * p.N + n] = ga;
                  p.ws[(size_t)(2 * s + 1) * BN + (size_t)b * p.N + n] = ua;
                } else {
                  store_h(p, b, n, ga * ts[0], ua * ts[1]);
                }
              }
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0 && *abort_flag) {
      // the final commit arrives once every MMA issued by this CTA has completed
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_acc, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, (uint32_t)p.tmem_cols);
  }
}

// ---------------------------------------------------------------------------------------
// Split-K reduction: out = epilogue(sum_{s=0..S-1} partial_s), in that fixed order, one
// 4-wide column group (b, n..n+3) per thread.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qgemm_splitk_reduce_kernel(const ReduceParams p) {
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
  const float ts0 = p.ts[0] ? __ldg(p.ts[0]) : 1.0f;
  const float ts1 = (p.NMAT == 2 && p.ts[1]) ? __ldg(p.ts[1]) : 1.0f;
  for (int e = 0; e < lim; ++e) {
    if (p.NMAT == 1) {
      const float v = g[e] * ts0;
      if (p.out_bf16)
        reinterpret_cast<__nv_bfloat16*>(p.out)[off + e] = __float2bfloat16_rn(v);
      else
        reinterpret_cast<float*>(p.out)[off + e] = v;
    } else {
      const float gv = g[e] * ts0, uv = u[e] * ts1;
      reinterpret_cast<__nv_bfloat16*>(p.out)[off + e] =
          __float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv);
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
  qgemm_splitk_reduce_kernel<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(rp);
  return cudaGetLastError();
}

cudaError_t launch_prep(const PrepParams& pp, cudaStream_t stream) {
  static const bool once = (prefer_max_shared((const void*)qgemm_prep_x_kernel), true);
  (void)once;
  qgemm_prep_x_kernel<<<pp.B, 256, 0, stream>>>(pp);
  return cudaGetLastError();
}

template <int FMT, bool BF16OP>
static cudaError_t launch_tc_impl(const GemmParams& p, size_t smem_bytes, int grid,
                                  const CUtensorMap* maps, cudaStream_t stream) {
  auto kern = qgemm_tc_kernel<FMT, BF16OP>;
  static size_t configured = 0;  // per instantiation: largest dynamic smem granted so far
  if (smem_bytes > configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem_bytes));
    if (e != cudaSuccess) return e;
    configured = smem_bytes;
  }
  kern<<<grid, kThreads, smem_bytes, stream>>>(p, maps[0]);
  return cudaGetLastError();
}

cudaError_t launch_tc(int fmt, bool bf16op, const GemmParams& p, size_t smem_bytes, int grid,
                      const CUtensorMap* maps, cudaStream_t stream) {
  switch (fmt * 2 + (bf16op ? 1 : 0)) {
    case FMT_Q8_0 * 2: return launch_tc_impl<FMT_Q8_0, false>(p, smem_bytes, grid, maps, stream);
    case FMT_Q8_0 * 2 + 1: return launch_tc_impl<FMT_Q8_0, true>(p, smem_bytes, grid, maps, stream);
    case FMT_NVFP4 * 2: return launch_tc_impl<FMT_NVFP4, false>(p, smem_bytes, grid, maps, stream);
    case FMT_NVFP4 * 2 + 1: return launch_tc_impl<FMT_NVFP4, true>(p, smem_bytes, grid, maps, stream);
    case FMT_MXFP4 * 2: return launch_tc_impl<FMT_MXFP4, false>(p, smem_bytes, grid, maps, stream);
    case FMT_MXFP4 * 2 + 1: return launch_tc_impl<FMT_MXFP4, true>(p, smem_bytes, grid, maps, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qg

// pair.cu -- the block-quantized-weight GEMM on CTA pairs (sm_100a).
//
// y[b][n] = sum_k x[b][k] * dequant(W)[n][k]     (hipfire PR "fix(mtp): chunk scalar Q8
// batched GEMM above 64 rows"; Atlas issue "Qwen3.8-27B on Strix Halo: prefill 2.4x gap",
// kernel ranking and exact-F16-dequant sections)
//
// Swap-AB on the 5th-generation tensor cores, two SMs per MMA:
//   * A cluster of two CTAs shares one tcgen05.mma.cta_group::2 stream.  The MMA M operand
//     is 256 weight rows: the even CTA's 128 rows in its tensor memory (TMEM), the odd CTA's
//     128 rows at the same TMEM address of its own SM.  At small widths the issuing thread,
//     not the tensor pipe, bounds the MMA stream (about 58 cycles per instruction), and one
//     M=256 instruction costs it what an M=128 one does, so the pair halves the instruction
//     count per weight byte.
//   * The MMA N operand is NB batch rows of x: rows [0, NB/2) in the even CTA's shared
//     memory, [NB/2, NB) in the odd CTA's, both loaded by TMA in the 128-byte swizzle.
//     Each CTA's TMEM receives the fp32 accumulator of its own 128 rows x all NB columns.
//   * Warp roles per CTA: warp 0 lane 0 streams packed weight stages (1-D bulk copies, the
//     tile-major layout makes each stage contiguous); warp 11 lane 0 streams x stages (tiled
//     TMA whose byte count lands on the even CTA's barrier); warp 1 allocates TMEM and, with
//     warp 10, issues the pair MMAs from the even CTA (two accumulators, alternate A-slot
//     groups); warps 2..9 dequantize weight stages from shared memory into the TMEM A ring
//     (tcgen05.st) and run the epilogue.
//   * The grid is persistent: at most one CTA pair per two SMs, each walking its share of
//     the work units (row-tile pair group x batch tile x K range, or x expert) with its rings
//     running on from unit to unit.  After a unit's last MMA the issuers commit its
//     accumulators; the dequant warps read them out in the epilogue and hand them back
//     before the issuers start the next unit, while the producers already stream its data.
//   * K is split into S contiguous ranges, S fixed by (format, N, K).  Partials are summed
//     in the fixed order s = 0..S-1 by the reduce kernel; nothing in the arithmetic depends
//     on the batch width, so row b of y is bit-identical for every width up to 256.
//   * Operand types: f16 (x rescaled per row by a power of two) for widths up to 256, bf16
//     straight from the caller above that.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <atomic>

#include "common.cuh"
#include "dequant.cuh"
#include "ptx.cuh"

namespace qg {

// a[i] for a runtime i in 0..3 without indexing the array dynamically (which would place
// it in local memory)
template <typename T>
__device__ __forceinline__ T sel4(const T (&a)[4], int i) {
  return i == 0 ? a[0] : i == 1 ? a[1] : i == 2 ? a[2] : a[3];
}

// One work unit of the pair kernel, as every role of a CTA computes it: the row-tile pair
// group g, the batch tile bt, the K range [c0, c1) in chunks and, for grouped experts, the
// expert's rows [rb, rb + nrows) of x and its weight buffers.
struct PairUnit {
  int g, bt, rb, nrows, c0, c1, ngroups;
  int s;  // K split index (partials slot)
  const uint8_t* codes[2];
  const uint8_t* scales[2];
  const float* ts[2];
};

// Unit u of the call (u < p.units).  Returns false for a unit with nothing to do (an expert
// without rows in the tile, or one whose table entries the kernel refuses); every thread
// that asks gets the same answer.
template <int FMT>
__device__ __forceinline__ bool pair_unit(const GemmParams& p, int u, PairUnit& U) {
  U.rb = 0;
  U.nrows = p.B;
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    U.codes[m] = p.codes[m];
    U.scales[m] = p.scales[m];
    U.ts[m] = p.ts[m];
  }
  if (p.moe_off) {
    U.bt = u % p.b_tiles;
    u /= p.b_tiles;
    U.g = u % p.n_groups;
    const int ex = u / p.n_groups;
    U.s = 0;
    const int lo = min(max(__ldg(p.moe_off + ex), 0), p.B);
    const int hi = min(max(__ldg(p.moe_off + ex + 1), lo), p.B);
    U.rb = lo;
    U.nrows = hi - lo;
    if (U.bt * p.NB >= U.nrows) return false;  // no rows of this expert in the tile
    bool bad = false;
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int mm = (m < p.NMAT) ? m : 0;
      U.codes[m] = p.moe_codes[mm][ex];
      U.scales[m] = p.moe_scales[mm] ? p.moe_scales[mm][ex] : nullptr;
      U.ts[m] = p.moe_ts[mm] ? p.moe_ts[mm][ex] : nullptr;
      // the bulk copies need present, 16-byte aligned buffers: refuse the expert otherwise
      bad |= (U.codes[m] == nullptr) || ((reinterpret_cast<uintptr_t>(U.codes[m]) & 15u) != 0);
      if (scale_row_bytes(FMT) > 0)
        bad |= (U.scales[m] == nullptr) || ((reinterpret_cast<uintptr_t>(U.scales[m]) & 15u) != 0);
      if (has_tensor_scale(FMT))
        bad |= (U.ts[m] == nullptr) || ((reinterpret_cast<uintptr_t>(U.ts[m]) & 3u) != 0);
    }
    if (bad) {
      atomicExch(p.dev_err, kErrArg);
      return false;
    }
  } else {
    U.g = u % p.n_groups;
    u /= p.n_groups;
    U.bt = u % p.b_tiles;
    U.s = u / p.b_tiles;
  }
  U.c0 = (int)((int64_t)U.s * p.chunks / p.S);
  U.c1 = (int)((int64_t)(U.s + 1) * p.chunks / p.S);
  constexpr int CPA = kPairAK / chunk_k(FMT);
  U.ngroups = (U.c1 - U.c0 + CPA - 1) / CPA;
  return true;
}

template <int FMT, bool BF16OP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    qgemm_pair_kernel(const __grid_constant__ GemmParams p,
                      const __grid_constant__ CUtensorMap tm_x) {
  constexpr int KW = chunk_k(FMT);
  constexpr int J = KW / kSubK;       // 64-element x slices per chunk
  constexpr int CPA = kPairAK / KW;   // chunks per weight stage (Q8_0/FP8: 2, FP4: 1)
  constexpr int SB = scale_row_bytes(FMT);
  constexpr int WSTAGE = pair_wstage_bytes(FMT);
  constexpr int WSCALES = (kPairAK / chunk_k(FMT)) * kWCodeBytes;  // offset of the scales in a stage
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, by pointer arithmetic on the shared array so that every access
  // through it stays a shared-memory access (an integer round trip would make them generic)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sx = sbase + p.smem_x;
  const uint32_t sw = sbase + p.smem_w;
  const int XS = p.XS, WS = p.WS, AS = p.AS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.smem_bar);
  const uint32_t bar_x_full = smem_u32(bars);
  const uint32_t bar_x_empty = bar_x_full + 8 * XS;
  const uint32_t bar_w_full = bar_x_empty + 8 * XS;
  const uint32_t bar_w_empty = bar_w_full + 8 * WS;
  // A ring: AS TMEM slots of kPairSlotK.  Stage s's half h goes to slot 2 (s % (AS/2)) + h, so
  // each half owns the ring positions of its parity.
  const uint32_t bar_a_full = bar_w_empty + 8 * WS;
  const uint32_t bar_a_empty = bar_a_full + 8 * AS;
  const uint32_t bar_acc = bar_a_empty + 8 * AS;  // a unit's accumulators are complete
  const uint32_t bar_acc_free = bar_acc + 8;      // the epilogue has read them
  const uint32_t bar_drain = bar_acc_free + 8;    // [2]: each issuer's MMAs are done
  int* ctl = reinterpret_cast<int*>(bars + 2 * XS + 2 * WS + 2 * AS + 4);
  volatile int* abort_flag = ctl + 1;
  // per batch column: the x row's power-of-two exponent, and 2^exponent as an exact float
  int* col_exp = ctl + 4;
  float* col_fac = reinterpret_cast<float*>(ctl + 4 + p.NB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: even CTA (issues the MMAs), 1: odd CTA
  // persistent: CTA pair q of Q takes units q, q + Q, q + 2Q, ... (every role walks the same
  // list and skips the same empty units)
  const int pid = (int)(blockIdx.x >> 1);
  const int npairs = (int)(gridDim.x >> 1);
  const int tpg = p.R / p.NMAT;  // tile pairs per group
  const int64_t n_row_tiles = row_tiles(p.N);
  const uint32_t a_col0 = (uint32_t)(p.R * p.NACC * p.NB);  // accumulators, then the A ring
  const int half = p.NB >> 1;  // x rows (MMA N) held by each CTA
  const uint32_t xslice = (uint32_t)half * 128u;  // one 64-element K slice of those rows
  const uint32_t xstage = xslice * (uint32_t)(CPA * J);  // one group's K range
  const bool by_matrix = (p.NMAT == 2);
  const int n_issuers = by_matrix ? 2 : p.NACC;  // issuers that commit per unit

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_x);
    for (int i = 0; i < XS; ++i) {
      mbar_init(bar_x_full + 8 * i, 1);   // the even CTA's producer arrives (expect_tx)
      mbar_init(bar_x_empty + 8 * i, (p.NMAT == 2) ? 2u : 1u);  // each issuer using the group
    }
    for (int i = 0; i < WS; ++i) {
      mbar_init(bar_w_full + 8 * i, 1);
      mbar_init(bar_w_empty + 8 * i, kPairDequantWarps);  // both halves' warps read the stage
    }
    for (int i = 0; i < AS; ++i) {
      mbar_init(bar_a_full + 8 * i, kPairDequantWarps);  // the half's 4 warps in each CTA
      mbar_init(bar_a_empty + 8 * i, 1);
    }
    mbar_init(bar_acc, (uint32_t)n_issuers);            // one commit per active issuer per unit
    mbar_init(bar_acc_free, 2 * kPairDequantWarps);     // every dequant warp of both CTAs
    mbar_init(bar_drain, 1);
    mbar_init(bar_drain + 8, 1);
    ctl[1] = 0;
    ctl[2] = 0;
    ctl[3] = 0;  // set when a column's exponent leaves the epilogue's fast range
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(ctl), (uint32_t)p.tmem_cols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = static_cast<uint32_t>(ctl[0]);

  if (warp == 0) {
    // ------------------------------------------------------------ weight producer
    // This CTA's weight stages, unit after unit, in the order (group, subtile) into its own
    // ring: one bulk copy of the stage's codes and one of its scales, completing on the
    // CTA's own barrier.  The ring runs on across units.
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      RingPos wp;
      int w_issued = 0;
      bool ok = true;
      for (int u = pid; u < p.units && ok; u += npairs) {
        PairUnit U;
        if (!pair_unit<FMT>(p, u, U)) continue;
        for (int wg = 0; wg < U.ngroups && ok; ++wg) {
          for (int wr = 0; wr < p.R; ++wr) {
            if (w_issued >= WS &&
                !mbar_wait(bar_w_empty + 8 * wp.slot, wp.phase ^ 1u, abort_flag, p.dev_err,
                           kErrTimeout)) {
              ok = false;
              break;
            }
            const uint32_t fb = bar_w_full + 8 * wp.slot;
            const int m = (p.NMAT == 2) ? (wr & 1) : 0;
            const int64_t t = 2 * ((int64_t)U.g * tpg + wr / p.NMAT) + rank;
            const int cg = U.c0 + wg * CPA;
            const int n = min(CPA, U.c1 - cg);
            const uint32_t dst = sw + (uint32_t)(wp.slot * WSTAGE);
            if (t < n_row_tiles) {
              const int64_t blk = t * p.chunks + cg;
              const uint32_t cbytes = (uint32_t)n * kWCodeBytes;
              const uint32_t sbytes = (uint32_t)n * (kTileRows * SB);
              mbar_arrive_expect_tx(fb, cbytes + sbytes);
              bulk_load(dst, (m ? U.codes[1] : U.codes[0]) + blk * kWCodeBytes, cbytes, fb, pol_w);
              if (SB > 0)
                bulk_load(dst + WSCALES, (m ? U.scales[1] : U.scales[0]) + blk * (kTileRows * SB), sbytes,
                          fb, pol_w);
            } else {
              mbar_arrive(fb);  // a tile past the matrix: its rows are never stored
            }
            wp.next(WS);
            ++w_issued;
          }
        }
      }
      if (!ok) {
        // let this CTA's weight loads land before it leaves (their barrier is local)
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
  } else if (warp == kPairXWarp) {
    // ------------------------------------------------------------ x producer
    // This CTA's half of x for each group (4 slices of 64 K elements) into the x ring, unit
    // after unit.  The bytes of both CTAs count on the even CTA's x barrier, which the even
    // CTA arms with the pair's total.  x comes from the preceding grid (the preparation
    // kernel), so the first load waits for it.
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();
      const uint32_t xbar0 = mapa_shared(bar_x_full, 0);  // even CTA's x_full[0]
      RingPos xp;
      int x_issued = 0;
      bool ok = true;
      griddep_wait();
      for (int u = pid; u < p.units && ok; u += npairs) {
        PairUnit U;
        if (!pair_unit<FMT>(p, u, U)) continue;
        const int row0 = U.rb + U.bt * p.NB + (int)rank * half;
        for (int gi = 0; gi < U.ngroups; ++gi) {
          if (x_issued >= XS &&
              !mbar_wait(bar_x_empty + 8 * xp.slot, xp.phase ^ 1u, abort_flag, p.dev_err,
                         kErrTimeout)) {
            ok = false;
            break;
          }
          const int cg = U.c0 + gi * CPA;
          const uint32_t dst = sx + (uint32_t)xp.slot * xstage;
          const uint32_t cbar = xbar0 + 8u * (uint32_t)xp.slot;
          if (p.x3d) {
            // one box of 4 slices (slices past K read zeros from the padded rows or the
            // out-of-range fill)
            if (rank == 0) mbar_arrive_expect_tx(bar_x_full + 8 * xp.slot, 2u * xstage);
            tma_load_3d_pair(dst, &tm_x, cbar, 0, row0, cg * KW / kSubK, pol_x);
          } else {
            const int nsl = min(CPA, U.c1 - cg) * J;  // slices in this group
            if (rank == 0)
              mbar_arrive_expect_tx(bar_x_full + 8 * xp.slot, 2u * xslice * (uint32_t)nsl);
            for (int j = 0; j < nsl; ++j)
              tma_load_2d_pair(dst + (uint32_t)j * xslice, &tm_x, cbar, cg * KW + j * kSubK,
                               row0, pol_x);
          }
          xp.next(XS);
          ++x_issued;
        }
      }
      if (!ok) {
        // the x loads complete on the even CTA's barrier: give them a fixed grace period
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000) __nanosleep(1000);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == kPairIssuer2Warp) {
    // ------------------------------------------------------------ pair MMA issuers
    // One tcgen05.mma takes its issuing thread about as long as the tensor pipe needs for
    // an N=128 tile, so at small N the issue rate, not the pipe, bounds the MMA stream.  Two
    // threads of the even CTA therefore issue concurrently, each into its own accumulators:
    //   * plain GEMM, NACC = 2: issuer e takes the groups gi with gi % 2 == e and
    //     accumulates them into D[i][e]; the epilogue adds D[i][0] + D[i][1];
    //   * fused gate+up (NMAT = 2, NACC = 1): issuer e takes matrix e's subtiles (gate or up),
    //     one accumulator each;
    //   * NACC = 1 plain GEMM (widths > 256): issuer 0 alone.
    // A-ring slots hold one half of a stage each (kPairSlotK of K); half h of stage s sits at
    // slot 2 (s % (AS/2)) + h, so the two halves run as independent rings.  An issuer's
    // previous slot of the same half lies at most AS/2 stages back (two issuers alternate
    // groups of one stage, or take alternate matrices), so its wait on a slot's "full"
    // barrier never aliases an older phase.  Within each accumulator the K slices arrive in
    // ascending order.  Per slot: wait for it (a_full counts the half's warps of both CTAs),
    // issue its K=16 MMAs, release it to both CTAs with a multicast commit; per group: wait
    // for the pair's x stage first and release it after the issuer's last slot of the group.
    // Per unit: before the first MMA, wait until the epilogue has read the previous unit's
    // accumulators; after the last, commit the unit's accumulator barrier.
    const int e = (warp == 1) ? 0 : 1;
    if (rank == 0 && lane == 0 && e < n_issuers) {
      const uint32_t idesc = idesc_f16_pair(BF16OP, (uint32_t)p.NB);
      const uint32_t xs16 = xslice >> 4;
      RingPos xc;  // x stage of the current group
      RingPos sp;  // stage position in the A ring (AS/2 per half)
      RingPos au;  // units with work: accumulator hand-over
      int nu = 0;  // units with work issued so far
      const int HS = AS / 2;
      bool ok = true;
      for (int u = pid; u < p.units && ok; u += npairs) {
        PairUnit U;
        if (!pair_unit<FMT>(p, u, U)) continue;
        if (nu > 0) {
          // the epilogue of the previous unit has read the accumulators
          if (!mbar_wait_spin(bar_acc_free, au.phase ^ 1u, false, abort_flag, p.dev_err,
                              kErrTimeout)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int gi = 0; gi < U.ngroups && ok; ++gi) {
          if (!by_matrix && gi % p.NACC != e) {
            // another issuer's group: keep the ring positions in step
            for (int i = 0; i < p.R; ++i) sp.next(HS);
            xc.next(XS);
            continue;
          }
          const int kvalid = min(CPA, U.c1 - (U.c0 + gi * CPA)) * KW;  // K of the group with data
          if (!mbar_wait_spin(bar_x_full + 8 * xc.slot, xc.phase, false, abort_flag, p.dev_err,
                              kErrTimeout)) {
            ok = false;
            break;
          }
          const uint32_t xbase = sx + (uint32_t)xc.slot * xstage;
          const uint64_t bd0 = smem_desc_sw128(xbase);
          for (int i = 0; i < p.R && ok; ++i) {
            if (by_matrix && (i & 1) != e) {  // the other matrix's stage
              sp.next(HS);
              continue;
            }
            const int acc_i = by_matrix ? i : i * p.NACC + e;
            const uint32_t d = tmem + (uint32_t)(acc_i * p.NB);
            const bool first = by_matrix ? (gi == 0) : (gi < p.NACC);  // accumulator's first group
#pragma unroll
            for (int hh = 0; hh < kPairAK / kPairSlotK; ++hh) {
              const int slot = 2 * sp.slot + hh;
              if (!mbar_wait_spin(bar_a_full + 8 * slot, sp.phase, false, abort_flag, p.dev_err,
                                  kErrTimeout)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t a = tmem + a_col0 + (uint32_t)(slot * kPairACols);
              const int ksteps = max(0, min(kPairSlotK, kvalid - hh * kPairSlotK)) / 16;
              // The issuing thread, not the tensor pipe, bounds small-N MMA streams, so a full
              // slot is one straight run of 8 MMAs whose operand addresses are the group's
              // descriptor plus constants (descriptor address units are 16 bytes).
              if (ksteps == kPairSlotK / 16) {
#pragma unroll
                for (int ks = 0; ks < kPairSlotK / 16; ++ks) {
                  const int kk = hh * (kPairSlotK / 16) + ks;  // K=16 step within the group
                  mma_f16_ts_pair(d, a + (uint32_t)(ks * 8),
                                  bd0 + (uint64_t)((kk >> 2) * xs16 + (kk & 3) * 2), idesc,
                                  (first && kk == 0) ? 0u : 1u);
                }
              } else {
                for (int ks = 0; ks < ksteps; ++ks) {
                  const int kk = hh * (kPairSlotK / 16) + ks;
                  mma_f16_ts_pair(d, a + (uint32_t)(ks * 8),
                                  bd0 + (uint64_t)((kk >> 2) * xs16 + (kk & 3) * 2), idesc,
                                  (first && kk == 0) ? 0u : 1u);
                }
              }
              mma_commit_pair(bar_a_empty + 8 * slot);
            }
            sp.next(HS);
          }
          if (!ok) break;
          mma_commit_pair(bar_x_empty + 8 * xc.slot);
          xc.next(XS);
        }
        if (!ok) break;
        mma_commit_pair(bar_acc);  // the unit's accumulators, once its MMAs complete
        au.next(1);
        ++nu;
      }
      // every MMA this thread issued has completed before the CTA may free TMEM
      mma_commit_pair(bar_drain + 8 * e);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(bar_drain + 8 * e, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ dequant + epilogue
    // Warp w may touch TMEM lanes 32*(w%4)..+31 (its lane quarter q); the kWPQ warps of a
    // quarter take the halves of each weight stage (warp h half h), each into its own A slot,
    // so the two halves advance independently within the weight ring.
    constexpr int kWPQ = kPairDequantWarps / 4;
    static_assert(kWPQ * kPairSlotK == kPairAK, "one A slot per warp of a quarter per stage");
    const int dw = warp - kPairFirstDequantWarp;
    const int q = warp & 3;
    const int h = dw >> 2;
    const int row = q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t afull0 = mapa_shared(bar_a_full, 0);      // even CTA's a_full[0]
    const uint32_t afree0 = mapa_shared(bar_acc_free, 0);    // even CTA's acc_free
    const int HS = AS / 2;
    const int ccw = (h * kPairSlotK) / KW;  // chunk of the stage holding this warp's half
    const int eo = (h * kPairSlotK) % KW;   // its first element within the chunk
    RingPos wp;  // weight stage
    RingPos sp;  // this half's A-ring position (AS/2 per half)
    RingPos au;  // units with work: accumulator hand-over
    int ns = 0;  // stages consumed
    bool ok = true;
    for (int u = pid; u < p.units; u += npairs) {
      PairUnit U;
      if (!pair_unit<FMT>(p, u, U)) continue;

      // MXFP4 on f16 operands: largest block exponent of this row within the unit's K range
      int emax[4] = {0, 0, 0, 0};
      if (FMT == FMT_MXFP4 && !BF16OP) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (r >= p.R) break;
          const int64_t t = 2 * ((int64_t)U.g * tpg + r / p.NMAT) + rank;
          const int64_t n = t * kTileRows + row;
          uint32_t mx = 0;
          if (n < p.N) {
            const uint8_t* sb = (r % p.NMAT) ? U.scales[1] : U.scales[0];
            for (int c = U.c0; c < U.c1; ++c) {
              const uint2 v = __ldg(reinterpret_cast<const uint2*>(sb + scale_offset(FMT, p.chunks, n, c)));
              mx = __vmaxu4(mx, __vmaxu4(v.x, v.y));
            }
          }
          mx = max(max(mx & 0xFFu, (mx >> 8) & 0xFFu), max((mx >> 16) & 0xFFu, mx >> 24));
          emax[r] = (int)mx;
        }
      }

      // (a warp whose wait failed skips the stages and meets the others at the barrier below)
      for (int gi = 0; gi < U.ngroups && ok; ++gi) {
        const int cg = U.c0 + gi * CPA;
        const int n = min(CPA, U.c1 - cg);
        for (int r = 0; r < p.R; ++r) {
          const int slot = 2 * sp.slot + h;
          if (ns >= HS) {
            // the pair MMAs of this slot's previous use (this half's stage ns - AS/2) are done
            ok = mbar_wait(bar_a_empty + 8 * slot, sp.phase ^ 1u, abort_flag, p.dev_err,
                           kErrTimeout);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
          }
          ok = mbar_wait(bar_w_full + 8 * wp.slot, wp.phase, abort_flag, p.dev_err, kErrTimeout);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          const uint8_t* stage = smem + p.smem_w + wp.slot * WSTAGE;
          tc_fence_after();
          if (ccw < n) {
            // this warp's half of the stage: kPairSlotK elements of its 32 rows
            const uint8_t* crow = stage + ccw * kWCodeBytes + row * kWRowBytes;
            const uint8_t* srow = stage + WSCALES + ccw * (kTileRows * SB) + row * SB;
            // two 64-element pieces, each stored as soon as it is converted (the stores read
            // their registers at issue), so that only one piece is held in registers
            const int ex = sel4(emax, r);
            const uint32_t ta = tmem + lane_base + a_col0 + (uint32_t)(slot * kPairACols);
#pragma unroll
            for (int pc = 0; pc < kPairSlotK / 64; ++pc) {
              uint32_t v[32];
#pragma unroll
              for (int i = 0; i < 2; ++i)
                Dequant<FMT, BF16OP>::run(crow, row, srow, cg + ccw, eo + 64 * pc + 32 * i, ex,
                                          *reinterpret_cast<uint32_t(*)[16]>(&v[16 * i]));
              if (pc == kPairSlotK / 64 - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_w_empty + 8 * wp.slot);  // registers hold the data
              }
              tmem_st32(ta + (uint32_t)(32 * pc), v);
            }
            tmem_st_wait();
          } else {
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_w_empty + 8 * wp.slot);  // nothing of this stage to read
          }
          tc_fence_before();
          __syncwarp();
          // the stores above are complete (wait::st): the even CTA's warps arrive locally, the
          // odd CTA's with a relaxed remote arrive (a cluster-scope release here would cost
          // about a thousand cycles per slot)
          if (lane == 0) {
            if (rank == 0) mbar_arrive(bar_a_full + 8 * slot);
            else mbar_arrive_cluster_relaxed(afull0 + 8u * (uint32_t)slot);
          }
          wp.next(WS);
          sp.next(HS);
          ++ns;
        }
      }

      // ---- epilogue of the unit
      // Every dequant warp meets here once per unit, failed or not, so that the named
      // barriers below see all of them; they leave together if any wait failed.  The
      // barrier also tells them that the previous unit's epilogue no longer reads the
      // column arrays.
      ok = bar_and(1, kPairDequantWarps * 32, ok);
      if (!ok) break;
      // the output may be read by a dependent grid only after it completes; let it launch
      griddep_launch_dependents();
      // per-column exponents x_exp[b] (f16 path); x_exp comes from the preceding grid.
      // Loaded before the accumulator wait so that their latency hides behind the last MMAs.
      griddep_wait();
      for (int i = threadIdx.x - kPairFirstDequantWarp * 32; i < p.NB; i += kPairDequantWarps * 32) {
        const int b = U.bt * p.NB + i;
        const int ce = (b < U.nrows && p.x_exp) ? p.x_exp[U.rb + b] : 0;
        col_exp[i] = ce;
        col_fac[i] = exp2_exact(ce);
        if (ce < -kFastExp || ce > kFastExp) ctl[3] = 1;
      }
      asm volatile("bar.sync 1, %0;" ::"r"(kPairDequantWarps * 32) : "memory");
      ok = mbar_wait(bar_acc, au.phase, abort_flag, p.dev_err, kErrTimeout);
      ok = __all_sync(0xffffffffu, ok);
      au.next(1);
      if (!ok) continue;  // to the next unit's barrier, which all warps reach
      tc_fence_after();
      const int qcols = p.NB / kWPQ;  // columns per warp of a lane quarter (multiple of 4)
      const int cb0 = h * qcols;
      const size_t BN = (size_t)p.B * p.N;
      float ts[2] = {1.0f, 1.0f};
      if (has_tensor_scale(FMT)) {
        ts[0] = __ldg(U.ts[0]);
        if (p.NMAT == 2) ts[1] = __ldg(U.ts[1]);
      }
      // per-row exponent restored by the epilogue: the MXFP4 f16 rebase (2^(E - Emax + 13) in
      // the operand for a block scale 2^(E - 127))
      constexpr bool kRowExp = (FMT == FMT_MXFP4 && !BF16OP);
      int rowexp[4] = {0, 0, 0, 0};
      if (kRowExp)
#pragma unroll
        for (int r = 0; r < 4; ++r) rowexp[r] = emax[r] - 140;
      // Fast path: with every exponent within +-kFastExp, ((acc * ts) * 2^re) * 2^ce rounds
      // once except at subnormal magnitudes far below the accuracy bound; otherwise (x rows
      // near the ends of the bf16 range) each output is scaled by one exactly rounded ldexpf.
      const bool cols_fast = (ctl[3] == 0);
      const bool two_acc = (p.NACC == 2 && U.ngroups > 1);
      // scale the accumulators; store finals (S == 1) or partials (S > 1)
      for (int lt = 0; lt < tpg; ++lt) {
        const int64_t t = 2 * ((int64_t)U.g * tpg + lt) + rank;
        const int64_t n64 = t * kTileRows + row;
        const int n = (int)n64;
        const int re_g = sel4(rowexp, lt * p.NMAT);
        const int re_u = sel4(rowexp, lt * p.NMAT + 1);
        const float rf_g = exp2_exact(re_g), rf_u = exp2_exact(re_u);
        const bool fast_g = cols_fast && re_g >= -kFastExp && re_g <= kFastExp;
        const bool fast_u = cols_fast && re_u >= -kFastExp && re_u <= kFastExp;
        for (int cb = cb0; cb < cb0 + qcols; cb += 16) {
          const int ngrp = min(16, cb0 + qcols - cb) >> 2;  // groups of 4 columns
          // va: the accumulator of subtile ig (issuer 0); vb: the up matrix's accumulator
          // (fused gate/up), or the odd groups' accumulator of subtile ig (two issuers), which
          // is added to va in the fixed order even + odd.  The two cases never meet (fused
          // gate/up has one accumulator per subtile), so one pair of arrays serves both.
          uint32_t va[4][4], vb[4][4];
          // accumulator of subtile i, issuer e: columns ((i * NACC) + e) * NB
          const int ig = lt * p.NMAT;
          const uint32_t col_a = (uint32_t)(ig * p.NACC * p.NB + cb);
          const uint32_t col_b = (uint32_t)((p.NMAT == 2 ? (ig + 1) * p.NACC : ig * p.NACC + 1) * p.NB + cb);
          const bool second = (p.NMAT == 2) || two_acc;
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            if (g4 < ngrp) {
              tmem_ld4(tmem + lane_base + col_a + (uint32_t)(g4 * 4), va[g4]);
              if (second) tmem_ld4(tmem + lane_base + col_b + (uint32_t)(g4 * 4), vb[g4]);
            }
          }
          tmem_ld_wait();
          if (p.NMAT == 1 && two_acc) {
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4)
#pragma unroll
              for (int j = 0; j < 4; ++j)
                va[g4][j] = __float_as_uint(__uint_as_float(va[g4][j]) + __uint_as_float(vb[g4][j]));
          }
          if (n64 >= p.N) continue;
#pragma unroll
          for (int g4 = 0; g4 < 4; ++g4) {
            if (g4 >= ngrp) break;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int col = cb + g4 * 4 + i;
              const int b = U.bt * p.NB + col;
              if (b >= U.nrows) break;
              // tensor scale first, then the row's and the column's powers of two
              const float cf = col_fac[col];
              const float vg = __uint_as_float(va[g4][i]) * ts[0];
              const float ga = fast_g ? (kRowExp ? vg * rf_g : vg) * cf
                                      : scale_pow2_exact(vg, col_exp[col] + re_g);
              if (p.NMAT == 1) {
                if (p.S > 1) p.ws[(size_t)U.s * BN + (size_t)b * p.N + n] = ga;
                else store_y(p, U.rb + b, n, ga);
              } else {
                const float vu = __uint_as_float(vb[g4][i]) * ts[1];
                const float ua = fast_u ? (kRowExp ? vu * rf_u : vu) * cf
                                        : scale_pow2_exact(vu, col_exp[col] + re_u);
                if (p.S > 1) {
                  p.ws[(size_t)(2 * U.s) * BN + (size_t)b * p.N + n] = ga;
                  p.ws[(size_t)(2 * U.s + 1) * BN + (size_t)b * p.N + n] = ua;
                } else {
                  store_h(p, U.rb + b, n, ga, ua);
                }
              }
            }
          }
        }
      }
      // every accumulator load of this warp has completed (wait::ld above): hand the
      // accumulators back to the issuers (the odd CTA with a relaxed remote arrive, as for
      // the A slots)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0) mbar_arrive(bar_acc_free);
        else mbar_arrive_cluster_relaxed(afree0);
      }
    }
  }

  // ------------------------------------------------------------ teardown
  // the issuers drained their MMAs above; neither CTA leaves (or frees TMEM the pair MMAs
  // write) while its peer may still use it
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, (uint32_t)p.tmem_cols);
  }
}

// CTA pairs resident at once on device `dev` (one CTA per SM): half its SM count, read once
// per device (devices beyond 64 read it on every launch).
static int pair_slots(int dev) {
  static std::atomic<int> cached[64];
  int v = (dev >= 0 && dev < 64) ? cached[dev].load(std::memory_order_relaxed) : 0;
  if (v > 0) return v;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 2)
    sms = 2 * kPairSMs;
  v = sms / 2;
  if (dev >= 0 && dev < 64) cached[dev].store(v, std::memory_order_relaxed);
  return v;
}

// ---------------------------------------------------------------------------------------
// Launcher: a persistent grid of at most one CTA pair per two SMs (clusters of 2 from the
// kernel attribute); the pairs share out the call's work units.
// ---------------------------------------------------------------------------------------
template <int FMT, bool BF16OP>
cudaError_t launch_pair_impl(const GemmParams& p, size_t smem_bytes, int units,
                             const CUtensorMap* maps, bool pdl, cudaStream_t stream) {
  auto kern = qgemm_pair_kernel<FMT, BF16OP>;
  // raise the dynamic shared-memory limit (a per-device function attribute) once per device
  // and instantiation; devices beyond 64 set it on every launch
  static std::atomic<uint64_t> set_mask{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
  if (bit == 0 || !(set_mask.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return e;
    set_mask.fetch_or(bit, std::memory_order_release);
  }
  if (smem_bytes > (size_t)kSmemLimit) return cudaErrorInvalidValue;
  if (units <= 0) return cudaSuccess;
  const int pairs = std::min(units, pair_slots(dev));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(kPairThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, p, maps[0]);
}

cudaError_t launch_pair(int fmt, bool bf16op, const GemmParams& p, size_t smem_bytes, int units,
                        const CUtensorMap* maps, bool pdl, cudaStream_t stream) {
  switch (fmt) {
    case FMT_Q8_0:
      return bf16op ? launch_pair_impl<FMT_Q8_0, true>(p, smem_bytes, units, maps, pdl, stream)
                    : launch_pair_impl<FMT_Q8_0, false>(p, smem_bytes, units, maps, pdl, stream);
    case FMT_NVFP4:
      return bf16op ? launch_pair_impl<FMT_NVFP4, true>(p, smem_bytes, units, maps, pdl, stream)
                    : launch_pair_impl<FMT_NVFP4, false>(p, smem_bytes, units, maps, pdl, stream);
    case FMT_MXFP4:
      return bf16op ? launch_pair_impl<FMT_MXFP4, true>(p, smem_bytes, units, maps, pdl, stream)
                    : launch_pair_impl<FMT_MXFP4, false>(p, smem_bytes, units, maps, pdl, stream);
    default:
      return bf16op ? launch_pair_impl<FMT_FP8, true>(p, smem_bytes, units, maps, pdl, stream)
                    : launch_pair_impl<FMT_FP8, false>(p, smem_bytes, units, maps, pdl, stream);
  }
}

}  // namespace qg

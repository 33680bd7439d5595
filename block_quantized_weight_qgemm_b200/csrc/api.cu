// api.cu -- the C ABI of libqgemm (declared in include/qgemm.h): argument checks, the fixed
// K-split rule, per-call tile configuration, workspace layout, TMA descriptors, launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/qgemm.h"
#include "common.cuh"

namespace qg {
cudaError_t launch_prep(const PrepParams& pp, cudaStream_t stream);
cudaError_t launch_bs_split(int f, const uint16_t* x, int M, int K, uint8_t* codes,
                            uint8_t* scales, int* x_exp, cudaStream_t stream);
cudaError_t launch_bs_gemm(int f, int M, int N, int K, const uint8_t* xcodes,
                           const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                           const uint8_t* wscales, const float* ts, void* out, int out_bf16,
                           int* dev_err, cudaStream_t stream);
size_t bs_workspace_bytes(int f, int64_t M, int64_t N, int64_t K, size_t* off_scales,
                          size_t* off_exp, size_t* off_part);
cudaError_t launch_bs_dec(int f, int M, int N, int K, const uint8_t* xcodes,
                          const uint8_t* xscales, const int* x_exp, const uint8_t* wcodes,
                          const uint8_t* wscales, const float* ts, float* part, void* out,
                          int out_bf16, int* dev_err, cudaStream_t stream);
cudaError_t launch_pair(int fmt, bool bf16op, const GemmParams& p, size_t smem_bytes, int units,
                        const CUtensorMap* maps, bool pdl, cudaStream_t stream);
cudaError_t launch_pack(int fmt, const float* W, int64_t N, int64_t K, void* codes, void* scales,
                        float* tensor_scale, cudaStream_t stream);
cudaError_t launch_repack(const RepackParams& rp, cudaStream_t stream);
cudaError_t launch_reduce(const ReduceParams& rp, cudaStream_t stream);
int* device_error_word();
}  // namespace qg

using namespace qg;

// Scratch of qgemm_run_noalloc: a device global sized QGEMM_NOALLOC_SCRATCH_BYTES, reserved on
// every GPU that loads this library for as long as the process lives.  Host code never reads
// this name as an address: it asks the runtime for the device address of the current GPU's copy.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QGEMM_NOALLOC_SCRATCH_BYTES];

namespace {

thread_local char g_last_cuda_error[256] = "";
thread_local cudaEvent_t g_prof_begin = nullptr;
thread_local cudaEvent_t g_prof_end = nullptr;

int cuda_fail(cudaError_t e, const char* where) {
  snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", where, cudaGetErrorString(e));
  return QGEMM_ERR_CUDA;
}

// ---- driver entry point for TMA descriptor encoding (no link-time libcuda dependency) ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows][inner] array with the given row pitch (bytes).
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* base, uint64_t inner,
              uint64_t rows, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  (void)esize;
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D map {64, rows, slices} over a row-major [rows][pitch] array of 16-bit elements whose
// rows are read in slices of 64: box {64, box_rows, box_slices}.
bool make_map3(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t rows,
               uint64_t pitch_elems, uint32_t box_rows, uint32_t box_slices) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {64, rows, pitch_elems / 64};
  const cuuint64_t strides[2] = {pitch_elems * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, box_slices};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int64_t pad64(int64_t k) { return (k + 63) / 64 * 64; }

// A weight matrix's buffers are present: codes; block scales unless the format has none
// (FP8); the fp32 tensor scale for the formats that have one (NVFP4, FP8).
bool weights_given(int fmt, const void* codes, const void* scales, const float* ts) {
  return codes && (scales || scale_row_bytes(fmt) == 0) && (ts || !has_tensor_scale(fmt));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_fmt_shape(int fmt, int64_t N, int64_t K) {
  if (fmt != FMT_Q8_0 && fmt != FMT_NVFP4 && fmt != FMT_MXFP4 && fmt != FMT_FP8)
    return QGEMM_ERR_FORMAT;
  if (N < 1 || K < 1 || N > 0x7FFFFFFF || K > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (K % block_k(fmt) != 0) return QGEMM_ERR_K_BLOCK;
  return QGEMM_OK;
}

// Per-device facts looked up once: whether the device is an sm_100 part, and the device
// addresses of the library's error word and no-alloc scratch there.  Devices beyond
// kMaxDevices are looked up on every call.
constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_dev_cc[kMaxDevices] = {};          // 0 unknown, 1 sm_100, 2 other
int* g_dev_err_ptr[kMaxDevices] = {};

int current_device(int* dev) {
  const cudaError_t e = cudaGetDevice(dev);
  return e == cudaSuccess ? QGEMM_OK : cuda_fail(e, "cudaGetDevice");
}

int device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_dev_cc[dev] != 0) return g_dev_cc[dev] == 1;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return 0;
  const int v = (major == 10) ? 1 : 2;
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    g_dev_cc[dev] = v;
  }
  return v == 1;
}

// Device address of the library's error word on the current device (nullptr on failure).
int* error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
  if (dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_dev_err_ptr[dev]) return g_dev_err_ptr[dev];
  }
  int* w = device_error_word();
  if (w && dev >= 0 && dev < kMaxDevices) {
    std::lock_guard<std::mutex> lock(g_dev_mu);
    g_dev_err_ptr[dev] = w;
  }
  return w;
}

// The K split of the CTA-pair kernel for widths 1..256: a function of (fmt, N, K) only.  A
// work unit is one pair of 128-row tiles over K/S; kPairSMs units run at once.  A unit costs
// its A slots (kPairAK elements of K each) plus a fixed cost of about kUnitOverheadSlots slots
// (set-up, the first weight latency, the MMA tail and the epilogue, measured); the time of a
// split is (waves of units) x (cost per unit), plus a small charge per split for the
// partials the reduction reads.  The smallest S of least cost wins.
constexpr int kUnitOverheadSlots = 6;

int split_for_pair(int fmt, int64_t N, int64_t K) {
  const int64_t chunks = (K + chunk_k(fmt) - 1) / chunk_k(fmt);
  const int64_t cpa = kPairAK / chunk_k(fmt);  // chunks per A slot
  const int64_t pairs = (row_tiles(N) + 1) / 2;
  int best = 1;
  double best_cost = 0.0;
  const int64_t smax = std::min<int64_t>(16, chunks);
  for (int64_t S = 1; S <= smax; ++S) {
    const int64_t waves = (pairs * S + kPairSMs - 1) / kPairSMs;
    const int64_t slots = ((chunks + S - 1) / S + cpa - 1) / cpa;
    const double cost = double(waves * (slots + kUnitOverheadSlots)) + 0.3 * double(S);
    if (S == 1 || cost < best_cost - 1e-9) {
      best_cost = cost;
      best = (int)S;
    }
  }
  return best;
}

struct Plan {
  int NACC;     // pair kernel: accumulators per subtile
  bool f16ops;  // widths <= 256
  int NB, R, NMAT, S, n_groups, b_tiles, chunks, XS, WS, AS, tmem_cols;
  size_t smem_bytes;
  uint32_t smem_x, smem_w, smem_bar;
  // workspace layout (bytes)
  size_t off_xh, off_exp, off_cnt, off_ws, ws_total;
};

int next_pow2_cols(int c) {
  int p = 32;
  while (p < c) p <<= 1;
  return p;
}

// Tiling of the CTA-pair kernel.  Only S (and the operand type, by width class) affects the
// arithmetic; NB, R and the ring depths are scheduling choices.
bool make_plan_pair(int fmt, int64_t N, int64_t K, int64_t B, int nmat, Plan* pl) {
  Plan p{};
  p.NMAT = nmat;
  // widths <= 256: f16 operands (x rescaled per row by the preparation kernel, which the GEMM
  // overlaps as its programmatic dependent); above: bf16 straight from the caller.  f16 keeps
  // the Q8_0 products q*d to one f16 rounding, and converts E2M1 codes in one instruction per
  // pair (NVFP4 and MXFP4 weights are exact either way).
  p.f16ops = (B <= 256);
  p.chunks = (int)((K + chunk_k(fmt) - 1) / chunk_k(fmt));
  const int64_t pairs = (row_tiles(N) + 1) / 2;
  if (B <= 256) {
    // plain GEMM: two accumulators per subtile (two concurrent MMA issuers), so NB <= 128;
    // fused gate+up: one accumulator per matrix, one issuer per matrix
    p.S = split_for_pair(fmt, N, K);
    p.NACC = (nmat == 2) ? 1 : 2;
    const int nb_cap = 128;
    const int64_t tiles_b = (B + nb_cap - 1) / nb_cap;  // balanced batch tiles
    p.NB = (int)std::min<int64_t>(((B + tiles_b - 1) / tiles_b + 15) / 16 * 16, nb_cap);
  } else {
    p.S = 1;
    p.NACC = 1;
    p.NB = (nmat == 2) ? 128 : 256;
  }
  p.b_tiles = (int)((B + p.NB - 1) / p.NB);
  p.R = nmat;
  p.n_groups = (int)pairs;
  // A ring: an even number of kPairSlotK slots (each stage half owns AS/2), at most 6, at least
  // 4 -- an issuer's previous slot of the same half lies at most 2 stages back (two issuers
  // alternate groups of one stage, or take alternate matrices), so AS/2 >= 2 keeps that
  // slot's previous use complete before its issuer waits for it
  p.AS = std::min(6, (512 - p.R * p.NACC * p.NB) / kPairACols) & ~1;
  if (p.AS < 4 || (nmat == 1 && p.NACC == 2 && p.R != 1)) return false;
  p.tmem_cols = next_pow2_cols(p.R * p.NACC * p.NB + p.AS * kPairACols);
  if (p.tmem_cols > 512) return false;
  const size_t xstage = (size_t)(p.NB / 2) * 128 * (kPairAK / kSubK);
  const size_t misc = 8 * (2 * 4 + 2 * kMaxWStages + 2 * 6 + 4) + 16 + 8 * kMaxNB + 64;
  const size_t budget = kSmemLimit - 1024 - misc;
  const size_t wstage = (size_t)pair_wstage_bytes(fmt);
  // x ring depth 4 or 2 (even): the two issuers take alternate groups, so an x stage's
  // previous use then belongs to the same issuer, whose wait therefore never aliases a phase
  int XS = 4;
  if (XS * xstage + 4 * wstage > budget) XS = 2;
  if (XS * xstage + 2 * wstage > budget) return false;
  const int WS = (int)std::min<size_t>(kMaxWStages, (budget - XS * xstage) / wstage);
  p.XS = XS;
  p.WS = WS;
  p.smem_x = 0;
  p.smem_w = (uint32_t)(XS * xstage);
  p.smem_bar = p.smem_w + (uint32_t)(WS * wstage);
  // ring barriers, then the accumulator hand-over pair and the issuers' two drain barriers
  const size_t bar_bytes = 8 * (2 * XS + 2 * WS + 2 * p.AS + 4);
  // control words, then per-column exponents and factors (int and float per batch column)
  p.smem_bytes = 1024 + p.smem_bar + bar_bytes + 16 + 8 * p.NB + 64;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  p.off_xh = p.f16ops ? take((size_t)B * pad64(K) * 2) : 0;
  p.off_exp = p.f16ops ? take((size_t)B * 4) : 0;
  p.off_cnt = 0;
  p.off_ws = (p.S > 1) ? take((size_t)p.S * nmat * B * N * 4) : 0;
  p.ws_total = off;
  *pl = p;
  return true;
}

// Plans are pure functions of (fmt, N, K, B, nmat); each host thread keeps its last few.
struct PlanKey {
  int fmt, nmat;
  int64_t N, K, B;
  bool operator==(const PlanKey& o) const {
    return fmt == o.fmt && nmat == o.nmat && N == o.N && K == o.K && B == o.B;
  }
};
constexpr int kCacheEntries = 8;
struct PlanCache {
  PlanKey key[kCacheEntries];
  Plan plan[kCacheEntries];
  bool ok[kCacheEntries];
  int used = 0, next = 0;
};
thread_local PlanCache g_plans;

bool make_plan(int fmt, int64_t N, int64_t K, int64_t B, int nmat, Plan* pl) {
  const PlanKey k{fmt, nmat, N, K, B};
  for (int i = 0; i < g_plans.used; ++i)
    if (g_plans.key[i] == k) {
      *pl = g_plans.plan[i];
      return g_plans.ok[i];
    }
  const bool ok = make_plan_pair(fmt, N, K, B, nmat, pl);
  const int i = g_plans.next;
  g_plans.key[i] = k;
  g_plans.plan[i] = *pl;
  g_plans.ok[i] = ok;
  g_plans.next = (i + 1) % kCacheEntries;
  if (g_plans.used < kCacheEntries) ++g_plans.used;
  return ok;
}

// The x tensor map of a call depends on the operand's address, type and geometry only; each
// host thread keeps its last few encoded maps (a map holds no device state).
struct MapKey {
  int dev, dt, x3d;
  const void* base;
  int64_t rows, pitch, K;
  uint32_t box_rows, box_slices;
  bool operator==(const MapKey& o) const {
    return dev == o.dev && dt == o.dt && x3d == o.x3d && base == o.base && rows == o.rows &&
           pitch == o.pitch && K == o.K && box_rows == o.box_rows && box_slices == o.box_slices;
  }
};
struct MapCache {
  MapKey key[kCacheEntries];
  CUtensorMap map[kCacheEntries];
  int used = 0, next = 0;
};
thread_local MapCache g_maps;

// x operand map: 3-D {64, rows, pitch/64} slices when the row pitch is a multiple of 64
// elements, else 2-D {K, rows} with 64-element boxes.
bool x_map(CUtensorMap* out, int dev, CUtensorMapDataType dt, const void* base, int64_t rows,
           int64_t pitch, int64_t K, bool x3d, uint32_t box_rows, uint32_t box_slices) {
  const MapKey k{dev, (int)dt, x3d ? 1 : 0, base, rows, pitch, K, box_rows, box_slices};
  for (int i = 0; i < g_maps.used; ++i)
    if (g_maps.key[i] == k) {
      *out = g_maps.map[i];
      return true;
    }
  const bool ok = x3d ? make_map3(out, dt, base, (uint64_t)rows, (uint64_t)pitch, box_rows,
                                  box_slices)
                      : make_map(out, dt, 2, base, (uint64_t)K, (uint64_t)rows,
                                 (uint64_t)pitch * 2, kSubK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return false;
  const int i = g_maps.next;
  g_maps.key[i] = k;
  g_maps.map[i] = *out;
  g_maps.next = (i + 1) % kCacheEntries;
  if (g_maps.used < kCacheEntries) ++g_maps.used;
  return true;
}

// Grouped experts: the rows of x are grouped by expert (device offsets), each expert's
// weights come from device pointer tables.
struct MoeArgs {
  const int* off;
  int E;
  int64_t max_rows;
  const void* const* codes[2];
  const void* const* scales[2];
  const float* const* ts[2];
};

// The tiling of a grouped call: the plain plan for max_rows rows (batch tile, rings, operand
// type), with the K split fixed at 1 and a workspace for the f16 copy of all M rows.
bool make_moe_plan(int fmt, int64_t N, int64_t K, int64_t M, int64_t max_rows, int nmat,
                   Plan* pl) {
  if (!make_plan(fmt, N, K, max_rows, nmat, pl)) return false;
  pl->S = 1;
  pl->b_tiles = (int)((max_rows + pl->NB - 1) / pl->NB);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  pl->off_xh = pl->f16ops ? take((size_t)M * pad64(K) * 2) : 0;
  pl->off_exp = pl->f16ops ? take((size_t)M * 4) : 0;
  pl->off_ws = 0;
  pl->ws_total = off;
  return true;
}

int run_impl(int fmt, const void* x, int64_t B, int64_t K, const void* const* codes,
             const void* const* scales, const float* const* ts, int nmat, int64_t N, void* out,
             int out_bf16, void* workspace, size_t ws_bytes, cudaStream_t stream,
             const MoeArgs* moe = nullptr) {
  Plan pl;
  if (moe ? !make_moe_plan(fmt, N, K, B, moe->max_rows, nmat, &pl)
          : !make_plan(fmt, N, K, B, nmat, &pl))
    return QGEMM_ERR_SHAPE;
  if (pl.ws_total > 0 && (workspace == nullptr || ws_bytes < pl.ws_total)) return QGEMM_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return QGEMM_ERR_ALIGN;
  int dev = 0;
  int st = current_device(&dev);
  if (st != QGEMM_OK) return st;
  int* dev_err = error_word();
  if (!dev_err) return cuda_fail(cudaGetLastError(), "cudaGetSymbolAddress");
  uint8_t* wsb = static_cast<uint8_t*>(workspace);

  GemmParams p{};
  p.N = (int)N;
  p.K = (int)K;
  p.B = (int)B;
  p.NB = pl.NB;
  p.R = pl.R;
  p.NMAT = nmat;
  p.S = pl.S;
  p.n_groups = pl.n_groups;
  p.b_tiles = pl.b_tiles;
  p.chunks = pl.chunks;
  p.XS = pl.XS;
  p.WS = pl.WS;
  p.AS = pl.AS;
  p.tmem_cols = pl.tmem_cols;
  p.NACC = pl.NACC;
  p.smem_x = pl.smem_x;
  p.smem_w = pl.smem_w;
  p.smem_bar = pl.smem_bar;
  for (int m = 0; m < 2; ++m) {
    const int mm = (m < nmat) ? m : 0;
    p.ts[m] = ts[mm];
    p.codes[m] = static_cast<const uint8_t*>(codes[mm]);
    p.scales[m] = static_cast<const uint8_t*>(scales[mm]);
  }
  if (moe) {
    p.moe_off = moe->off;
    for (int m = 0; m < 2; ++m) {
      const int mm = (m < nmat) ? m : 0;
      p.moe_codes[m] = reinterpret_cast<const uint8_t* const*>(moe->codes[mm]);
      p.moe_scales[m] = reinterpret_cast<const uint8_t* const*>(moe->scales[mm]);
      p.moe_ts[m] = moe->ts[mm];
    }
  }
  p.x_exp = pl.f16ops ? reinterpret_cast<const int*>(wsb + pl.off_exp) : nullptr;
  p.ws = (pl.S > 1) ? reinterpret_cast<float*>(wsb + pl.off_ws) : nullptr;
  p.out = out;
  p.out_bf16 = out_bf16;
  p.dev_err = dev_err;

  const void* xop = x;
  if (pl.f16ops) {
    PrepParams pp{};
    pp.x = static_cast<const uint16_t*>(x);
    pp.xh = reinterpret_cast<uint16_t*>(wsb + pl.off_xh);
    pp.x_exp = reinterpret_cast<int*>(wsb + pl.off_exp);
    pp.B = (int)B;
    pp.K = (int)K;
    pp.Kp = (int)pad64(K);
    cudaError_t e = launch_prep(pp, stream);
    if (e != cudaSuccess) return cuda_fail(e, "prep kernel launch");
    xop = pp.xh;
  }

  CUtensorMap xmap;
  const CUtensorMapDataType xdt =
      pl.f16ops ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int64_t xpitch = pl.f16ops ? pad64(K) : K;  // elements per row of the x operand
  p.x3d = (xpitch % 64 == 0) ? 1 : 0;
  const bool mapped = x_map(&xmap, dev, xdt, xop, B, xpitch, K, p.x3d != 0,
                            (uint32_t)(pl.NB / 2), (uint32_t)(kPairAK / kSubK));
  if (!mapped) {
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed");
    return QGEMM_ERR_CUDA;
  }
  const int64_t grid64 = (int64_t)pl.n_groups * pl.b_tiles * (moe ? moe->E : pl.S);
  if (grid64 > 0x3FFFFFFF) return QGEMM_ERR_SHAPE;
  const int grid = (int)grid64;
  p.units = grid;
  if (g_prof_begin) cudaEventRecord(g_prof_begin, stream);
  // with f16 operands the GEMM follows the x preparation as its programmatic dependent
  cudaError_t e = launch_pair(fmt, !pl.f16ops, p, pl.smem_bytes, grid, &xmap, pl.f16ops, stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemm kernel launch");
  if (g_prof_end) cudaEventRecord(g_prof_end, stream);
  if (pl.S > 1) {
    ReduceParams rp{};
    rp.ws = p.ws;
    rp.S = pl.S;
    rp.NMAT = nmat;
    rp.B = (int)B;
    rp.N = (int)N;
    rp.out = out;
    rp.out_bf16 = out_bf16;
    e = launch_reduce(rp, stream);
    if (e != cudaSuccess) return cuda_fail(e, "split-K reduce launch");
  }
  return QGEMM_OK;
}

// Device address of g_noalloc_scratch on the current device, looked up once per device (the
// lookup may load this library's device code on that device, so it must not happen inside a
// stream capture).
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return QGEMM_ERR_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return QGEMM_OK;
}

}  // namespace

extern "C" {

int qgemm_packed_size(int fmt, int64_t N, int64_t K, size_t* code_bytes, size_t* scale_bytes) {
  const int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (!code_bytes || !scale_bytes) return QGEMM_ERR_NULL;
  *code_bytes = (size_t)packed_code_bytes(fmt, N, K);
  *scale_bytes = (size_t)packed_scale_bytes(fmt, N, K);
  return QGEMM_OK;
}

int qgemm_packed_geometry(int fmt, int64_t N, int64_t K, int64_t* tiles, int64_t* chunks,
                          int* chunk_elems, int* scale_bytes_per_row) {
  const int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (!tiles || !chunks || !chunk_elems || !scale_bytes_per_row) return QGEMM_ERR_NULL;
  *tiles = row_tiles(N);
  *chunks = k_chunks(fmt, K);
  *chunk_elems = chunk_k(fmt);
  *scale_bytes_per_row = scale_row_bytes(fmt);
  return QGEMM_OK;
}

int qgemm_row_pitches(int fmt, int64_t K, int64_t* cp, int64_t* sp) {
  const int st = check_fmt_shape(fmt, 1, K);
  if (st != QGEMM_OK) return st;
  if (!cp || !sp) return QGEMM_ERR_NULL;
  *cp = rm_code_pitch(fmt, K);
  *sp = rm_scale_pitch(fmt, K);
  return QGEMM_OK;
}

int qgemm_repack_rowmajor(int fmt, int64_t N, int64_t K, const void* codes_rm, int64_t code_pitch,
                          const void* scales_rm, int64_t scale_pitch, void* codes, void* scales,
                          void* stream) {
  const int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (!codes_rm || !codes || (scale_row_bytes(fmt) > 0 && (!scales_rm || !scales)))
    return QGEMM_ERR_NULL;
  if (code_pitch < rm_code_bytes_per_row(fmt, K) || scale_pitch < rm_scale_bytes_per_row(fmt, K))
    return QGEMM_ERR_SHAPE;
  if (!aligned16(codes) || !aligned16(scales)) return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  RepackParams rp{};
  rp.codes_rm = static_cast<const uint8_t*>(codes_rm);
  rp.scales_rm = static_cast<const uint8_t*>(scales_rm);
  rp.code_pitch = code_pitch;
  rp.scale_pitch = scale_pitch;
  rp.codes = static_cast<uint8_t*>(codes);
  rp.scales = static_cast<uint8_t*>(scales);
  rp.N = N;
  rp.K = K;
  rp.fmt = fmt;
  cudaError_t e = launch_repack(rp, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "repack kernel launch");
  return QGEMM_OK;
}

int qgemm_pack(int fmt, const float* W, int64_t N, int64_t K, void* codes, void* scales,
               float* tensor_scale, void* stream) {
  const int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (!W || !weights_given(fmt, codes, scales, tensor_scale)) return QGEMM_ERR_NULL;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return QGEMM_ERR_ALIGN;
  if (has_tensor_scale(fmt) && (reinterpret_cast<uintptr_t>(tensor_scale) & 3u))
    return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  cudaError_t e = launch_pack(fmt, W, N, K, codes, scales, tensor_scale,
                              static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pack kernel launch");
  return QGEMM_OK;
}

int qgemm_split_k(int fmt, int64_t N, int64_t K, int* splits) {
  const int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (!splits) return QGEMM_ERR_NULL;
  *splits = split_for_pair(fmt, N, K);
  return QGEMM_OK;
}

int qgemm_workspace_size(int fmt, int64_t N, int64_t K, int64_t B, size_t* bytes) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (B < 1 || B > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!bytes) return QGEMM_ERR_NULL;
  Plan pl;
  if (!make_plan(fmt, N, K, B, 1, &pl)) return QGEMM_ERR_SHAPE;
  *bytes = pl.ws_total;
  return QGEMM_OK;
}

namespace {
// Fused gate+up above widths of 256.  The single fused kernel would hold two accumulators in
// TMEM and so run N = 128 batch tiles, which dequantize every weight tile twice as often as
// the plain GEMM's N = 256 tiles (measured ~690 against ~1000 TFLOP/s).  Instead, per chunk of
// rows: g = x Wg^T and u = x Wu^T as two plain GEMMs into an fp32 workspace, then the
// fixed-order reduce kernel with S = 1 and both matrices writes h = bf16(SiLU(g) * u), the
// same expression the fused epilogue evaluates on the same fp32 values.  Chunks of at most
// kFfnChunkRows rows bound the workspace; every chunk stays above 256 rows so that both GEMMs
// take the bf16-operand path.
constexpr int64_t kFfnChunkRows = 2048;
struct FfnChunks {
  int64_t rows;    // rows per chunk (the last one may be shorter)
  int64_t count;
  bool ok;
};
FfnChunks ffn_chunks(int64_t M) {
  FfnChunks c{};
  c.count = (M + kFfnChunkRows - 1) / kFfnChunkRows;
  // full chunks keep whole 256-row batch tiles; if that leaves a last chunk of 256 rows or
  // fewer, balance the chunks instead (multiples of 8 rows)
  c.rows = std::min<int64_t>(kFfnChunkRows, (M + 7) / 8 * 8);
  if (M - (c.count - 1) * c.rows <= 256) c.rows = ((M + c.count - 1) / c.count + 7) / 8 * 8;
  const int64_t last = M - (c.count - 1) * c.rows;
  c.ok = (M > 256) && last > 256 && c.rows > 256;
  return c;
}
size_t ffn_gu_bytes(const FfnChunks& c, int64_t N) {
  return ((size_t)2 * (size_t)c.rows * (size_t)N * 4 + 255) / 256 * 256;
}
size_t ffn_two_gemm_bytes(int fmt, int64_t N, int64_t K, const FfnChunks& c) {
  Plan pl;
  if (!make_plan(fmt, N, K, c.rows, 1, &pl)) return 0;
  return ffn_gu_bytes(c, N) + pl.ws_total;
}
}  // namespace

int qgemm_ffn_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!bytes) return QGEMM_ERR_NULL;
  const FfnChunks c = ffn_chunks(M);
  if (c.ok) {
    *bytes = ffn_two_gemm_bytes(fmt, N, K, c);
    return *bytes ? QGEMM_OK : QGEMM_ERR_SHAPE;
  }
  Plan pl;
  if (!make_plan(fmt, N, K, M, 2, &pl)) return QGEMM_ERR_SHAPE;
  *bytes = pl.ws_total;
  return QGEMM_OK;
}

int qgemm_run(int fmt, const void* x, int64_t B, int64_t K, const void* codes, const void* scales,
              const float* tensor_scale, int64_t N, void* y, int y_dtype, void* workspace,
              size_t workspace_bytes, void* stream) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (B < 1 || B > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (y_dtype != QGEMM_Y_F32 && y_dtype != QGEMM_Y_BF16) return QGEMM_ERR_FORMAT;
  if (!x || !y || !weights_given(fmt, codes, scales, tensor_scale)) return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(y))
    return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  const void* cs[1] = {codes};
  const void* ss[1] = {scales};
  const float* tss[1] = {tensor_scale};
  return run_impl(fmt, x, B, K, cs, ss, tss, 1, N, y, y_dtype == QGEMM_Y_BF16, workspace,
                  workspace_bytes, static_cast<cudaStream_t>(stream));
}

int qgemm_run_noalloc(int fmt, const void* x, int64_t B, int64_t K, const void* codes,
                      const void* scales, const float* tensor_scale, int64_t N, void* y,
                      int y_dtype, void* stream) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (B < 1 || B > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (y_dtype != QGEMM_Y_F32 && y_dtype != QGEMM_Y_BF16) return QGEMM_ERR_FORMAT;
  if (!x || !y || !weights_given(fmt, codes, scales, tensor_scale)) return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(y))
    return QGEMM_ERR_ALIGN;
  // the same plan qgemm_run would use; its workspace must fit the fixed scratch
  Plan pl;
  if (!make_plan(fmt, N, K, B, 1, &pl)) return QGEMM_ERR_SHAPE;
  if (pl.ws_total > (size_t)QGEMM_NOALLOC_SCRATCH_BYTES) return QGEMM_ERR_WORKSPACE;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != QGEMM_OK) return st;
  const void* cs[1] = {codes};
  const void* ss[1] = {scales};
  const float* tss[1] = {tensor_scale};
  return run_impl(fmt, x, B, K, cs, ss, tss, 1, N, y, y_dtype == QGEMM_Y_BF16, scratch,
                  (size_t)QGEMM_NOALLOC_SCRATCH_BYTES, static_cast<cudaStream_t>(stream));
}

int qgemm_ffn_gate_up(int fmt, const void* x, int64_t M, int64_t K, const void* g_codes,
                      const void* g_scales, const float* g_ts, const void* u_codes,
                      const void* u_scales, const float* u_ts, int64_t N, void* h,
                      void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!x || !h || !weights_given(fmt, g_codes, g_scales, g_ts) ||
      !weights_given(fmt, u_codes, u_scales, u_ts))
    return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(g_codes) || !aligned16(g_scales) || !aligned16(u_codes) ||
      !aligned16(u_scales) || !aligned16(h))
    return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  const FfnChunks c = ffn_chunks(M);
  if (c.ok) {
    const size_t need = ffn_two_gemm_bytes(fmt, N, K, c);
    if (need == 0) return QGEMM_ERR_SHAPE;
    if (workspace == nullptr || workspace_bytes < need) return QGEMM_ERR_WORKSPACE;
    if (!aligned16(workspace)) return QGEMM_ERR_ALIGN;
    const size_t gu = ffn_gu_bytes(c, N);
    uint8_t* rest = static_cast<uint8_t*>(workspace) + gu;
    const size_t rest_bytes = workspace_bytes - gu;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    for (int64_t r0 = 0; r0 < M; r0 += c.rows) {
      const int64_t mc = std::min<int64_t>(c.rows, M - r0);
      const void* xr = static_cast<const uint8_t*>(x) + (size_t)r0 * (size_t)K * 2;
      float* g = static_cast<float*>(workspace);
      float* u = g + (size_t)mc * (size_t)N;  // the reduce reads matrix 1 at B*N past matrix 0
      int rc = run_impl(fmt, xr, mc, K, &g_codes, &g_scales, &g_ts, 1, N, g, 0, rest,
                        rest_bytes, st);
      if (rc != QGEMM_OK) return rc;
      rc = run_impl(fmt, xr, mc, K, &u_codes, &u_scales, &u_ts, 1, N, u, 0, rest, rest_bytes, st);
      if (rc != QGEMM_OK) return rc;
      ReduceParams rp{};
      rp.ws = g;
      rp.S = 1;
      rp.NMAT = 2;
      rp.B = (int)mc;
      rp.N = (int)N;
      rp.out = static_cast<uint8_t*>(h) + (size_t)r0 * (size_t)N * 2;
      rp.out_bf16 = 1;
      const cudaError_t e = launch_reduce(rp, st);
      if (e != cudaSuccess) return cuda_fail(e, "SiLU(g)*u launch");
    }
    return QGEMM_OK;
  }
  const void* cs[2] = {g_codes, u_codes};
  const void* ss[2] = {g_scales, u_scales};
  const float* tss[2] = {g_ts, u_ts};
  return run_impl(fmt, x, M, K, cs, ss, tss, 2, N, h, 1, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream));
}

int qgemm_device_status(int reset) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int* w = error_word();
  if (!w) return cuda_fail(cudaGetLastError(), "cudaGetSymbolAddress");
  int v = 0;
  e = cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  if (reset && v) {
    const int z = 0;
    e = cudaMemcpy(w, &z, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy");
  }
  return v == kErrArg ? QGEMM_ERR_DEVICE_ARG : v ? QGEMM_ERR_DEVICE_TIMEOUT : QGEMM_OK;
}

const char* qgemm_status_str(int status) {
  switch (status) {
    case QGEMM_OK: return "ok";
    case QGEMM_ERR_FORMAT: return "unknown weight format or output dtype";
    case QGEMM_ERR_SHAPE: return "invalid shape (N, K or B < 1, or too large)";
    case QGEMM_ERR_K_BLOCK: return "K is not a multiple of the format's block size";
    case QGEMM_ERR_NULL: return "a required pointer is NULL";
    case QGEMM_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case QGEMM_ERR_WORKSPACE: return "workspace missing or too small";
    case QGEMM_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case QGEMM_ERR_DEVICE: return "the current device is not an sm_100 GPU";
    case QGEMM_ERR_DEVICE_TIMEOUT: return "a kernel wait hit its time limit";
    case QGEMM_ERR_DEVICE_ARG: return "a kernel refused an argument read from device memory";
    default: return "unknown status";
  }
}

const char* qgemm_last_cuda_error(void) { return g_last_cuda_error; }

namespace {
int check_moe(int fmt, const void* x, int64_t M, int64_t K, int E, const int32_t* off,
              int64_t max_rows, int64_t N) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF || E < 1 || max_rows < 1 || max_rows > 0x7FFFFFFF)
    return QGEMM_ERR_SHAPE;
  if (!x || !off) return QGEMM_ERR_NULL;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(off) & 3u)) return QGEMM_ERR_ALIGN;
  return QGEMM_OK;
}
// a weight pointer table: codes always, scales unless the format has none, tensor scales
// for the formats that have one; each 8-byte aligned
int check_tables(int fmt, const void* const* c, const void* const* sc, const float* const* ts) {
  if (!c || (scale_row_bytes(fmt) > 0 && !sc) || (has_tensor_scale(fmt) && !ts))
    return QGEMM_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(c) & 7u) || (reinterpret_cast<uintptr_t>(sc) & 7u) ||
      (reinterpret_cast<uintptr_t>(ts) & 7u))
    return QGEMM_ERR_ALIGN;
  return QGEMM_OK;
}
}  // namespace

int qgemm_moe_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, int64_t max_rows,
                             size_t* bytes) {
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF || max_rows < 1 || max_rows > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!bytes) return QGEMM_ERR_NULL;
  Plan pl;
  if (!make_moe_plan(fmt, N, K, M, max_rows, 2, &pl)) return QGEMM_ERR_SHAPE;
  Plan p1;
  if (!make_moe_plan(fmt, N, K, M, max_rows, 1, &p1)) return QGEMM_ERR_SHAPE;
  *bytes = std::max(pl.ws_total, p1.ws_total);  // one size serves both grouped entry points
  return QGEMM_OK;
}

int qgemm_moe_run(int fmt, const void* x, int64_t M, int64_t K, int E, const int32_t* off,
                  int64_t max_rows, const void* const* codes_tab, const void* const* scales_tab,
                  const float* const* ts_tab, int64_t N, void* y, int y_dtype, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int st = check_moe(fmt, x, M, K, E, off, max_rows, N);
  if (st != QGEMM_OK) return st;
  if (y_dtype != QGEMM_Y_F32 && y_dtype != QGEMM_Y_BF16) return QGEMM_ERR_FORMAT;
  if (!y) return QGEMM_ERR_NULL;
  if (!aligned16(y)) return QGEMM_ERR_ALIGN;
  st = check_tables(fmt, codes_tab, scales_tab, ts_tab);
  if (st != QGEMM_OK) return st;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  MoeArgs ma{};
  ma.off = off;
  ma.E = E;
  ma.max_rows = max_rows;
  ma.codes[0] = ma.codes[1] = codes_tab;
  ma.scales[0] = ma.scales[1] = scales_tab;
  ma.ts[0] = ma.ts[1] = ts_tab;
  const void* none[1] = {nullptr};
  const float* nts[1] = {nullptr};
  return run_impl(fmt, x, M, K, none, none, nts, 1, N, y, y_dtype == QGEMM_Y_BF16, workspace,
                  workspace_bytes, static_cast<cudaStream_t>(stream), &ma);
}

int qgemm_moe_gate_up(int fmt, const void* x, int64_t M, int64_t K, int E, const int32_t* off,
                      int64_t max_rows, const void* const* g_codes_tab,
                      const void* const* g_scales_tab, const float* const* g_ts_tab,
                      const void* const* u_codes_tab, const void* const* u_scales_tab,
                      const float* const* u_ts_tab, int64_t N, void* h, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int st = check_moe(fmt, x, M, K, E, off, max_rows, N);
  if (st != QGEMM_OK) return st;
  if (!h) return QGEMM_ERR_NULL;
  if (!aligned16(h)) return QGEMM_ERR_ALIGN;
  st = check_tables(fmt, g_codes_tab, g_scales_tab, g_ts_tab);
  if (st == QGEMM_OK) st = check_tables(fmt, u_codes_tab, u_scales_tab, u_ts_tab);
  if (st != QGEMM_OK) return st;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  MoeArgs ma{};
  ma.off = off;
  ma.E = E;
  ma.max_rows = max_rows;
  ma.codes[0] = g_codes_tab;
  ma.codes[1] = u_codes_tab;
  ma.scales[0] = g_scales_tab;
  ma.scales[1] = u_scales_tab;
  ma.ts[0] = g_ts_tab;
  ma.ts[1] = u_ts_tab;
  const void* none[2] = {nullptr, nullptr};
  const float* nts[2] = {nullptr, nullptr};
  return run_impl(fmt, x, M, K, none, none, nts, 2, N, h, 1, workspace, workspace_bytes,
                  static_cast<cudaStream_t>(stream), &ma);
}

// ---------------------------------------------------------------------------------------
// Block-scaled path (MXFP4 / NVFP4 weights with x split into three E2M1 terms, FP8 weights
// with x split into two E4M3 terms)
// ---------------------------------------------------------------------------------------
namespace {
bool bs_fmt(int fmt) {
  return fmt == QGEMM_FMT_MXFP4 || fmt == QGEMM_FMT_NVFP4 || fmt == QGEMM_FMT_FP8;
}
// the kernels' format id: 0 MXFP4, 1 NVFP4, 2 FP8
int bs_id(int fmt) { return fmt == QGEMM_FMT_NVFP4 ? 1 : fmt == QGEMM_FMT_FP8 ? 2 : 0; }
// the per-tensor scale the epilogue applies (NVFP4, FP8), else none
const float* bs_ts(int fmt, const float* ts) { return fmt == QGEMM_FMT_MXFP4 ? nullptr : ts; }
}  // namespace

int qgemm_bs_split_size(int fmt, int64_t M, int64_t K, size_t* code_bytes, size_t* scale_bytes,
                        size_t* exp_bytes) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  if (M < 1 || K < 1 || M > 0x7FFFFFFF || K > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (K % 32 != 0) return QGEMM_ERR_K_BLOCK;
  if (!code_bytes || !scale_bytes || !exp_bytes) return QGEMM_ERR_NULL;
  size_t off_s = 0, off_e = 0, off_p = 0;
  (void)bs_workspace_bytes(bs_id(fmt), M, 0, K, &off_s, &off_e, &off_p);
  const int64_t Mt = (M + 127) / 128;
  *code_bytes = off_s;
  *scale_bytes = off_e - off_s;
  *exp_bytes = (size_t)Mt * 128 * 4;
  return QGEMM_OK;
}

int qgemm_bs_split_x(int fmt, const void* x, int64_t M, int64_t K, void* codes, void* scales,
                     int32_t* x_exp, void* stream) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  if (M < 1 || K < 1 || M > 0x7FFFFFFF || K > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (K % 32 != 0) return QGEMM_ERR_K_BLOCK;
  if (!x || !codes || !scales || !x_exp) return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(x_exp))
    return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  const cudaError_t e = launch_bs_split(bs_id(fmt), static_cast<const uint16_t*>(x), (int)M, (int)K,
                                        static_cast<uint8_t*>(codes), static_cast<uint8_t*>(scales),
                                        reinterpret_cast<int*>(x_exp), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? QGEMM_OK : cuda_fail(e, "split kernel launch");
}

int qgemm_bs_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!bytes) return QGEMM_ERR_NULL;
  *bytes = bs_workspace_bytes(bs_id(fmt), M, N, K, nullptr, nullptr, nullptr);
  return QGEMM_OK;
}

int qgemm_bs_run(int fmt, const void* x, int64_t M, int64_t K, const void* codes,
                 const void* scales, const float* tensor_scale, int64_t N, void* y, int y_dtype,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  const int f = bs_id(fmt);
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (y_dtype != QGEMM_Y_F32 && y_dtype != QGEMM_Y_BF16) return QGEMM_ERR_FORMAT;
  if (!x || !y || !weights_given(fmt, codes, scales, tensor_scale)) return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(y))
    return QGEMM_ERR_ALIGN;
  size_t off_s = 0, off_e = 0, off_p = 0;
  const size_t need = bs_workspace_bytes(f, M, N, K, &off_s, &off_e, &off_p);
  if (!workspace || workspace_bytes < need) return QGEMM_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  int* dev_err = error_word();
  if (!dev_err) return cuda_fail(cudaGetLastError(), "cudaGetSymbolAddress");
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_bs_split(f, static_cast<const uint16_t*>(x), (int)M, (int)K, wsb, wsb + off_s,
                                  reinterpret_cast<int*>(wsb + off_e), s);
  if (e != cudaSuccess) return cuda_fail(e, "split kernel launch");
  if (g_prof_begin) cudaEventRecord(g_prof_begin, s);
  // up to 128 rows the weights are the MMA M operand (decode tiling), above that x is
  const float* ts = bs_ts(fmt, tensor_scale);
  if (M <= 128)
    e = launch_bs_dec(f, (int)M, (int)N, (int)K, wsb, wsb + off_s, reinterpret_cast<const int*>(wsb + off_e),
                      static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales), ts,
                      reinterpret_cast<float*>(wsb + off_p), y, y_dtype == QGEMM_Y_BF16, dev_err, s);
  else
    e = launch_bs_gemm(f, (int)M, (int)N, (int)K, wsb, wsb + off_s, reinterpret_cast<const int*>(wsb + off_e),
                       static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(scales), ts, y,
                       y_dtype == QGEMM_Y_BF16, dev_err, s);
  if (e != cudaSuccess) return cuda_fail(e, "block-scaled gemm launch");
  if (g_prof_end) cudaEventRecord(g_prof_end, s);
  return QGEMM_OK;
}

// Fused gate+up on the block-scaled path: per chunk of up to kBsFfnRows rows, one split of x
// serves both GEMMs; g and u go to an fp32 workspace [2][rows][N] and the split-K reduce
// kernel with S = 1 and both matrices writes h = bf16(SiLU(g) * u), the expression of the other
// fused paths.
namespace {
constexpr int64_t kBsFfnRows = 2048;
size_t bs_ffn_bytes(int f, int64_t N, int64_t K, int64_t M, size_t* off_gu) {
  const int64_t mc = std::min<int64_t>(M, kBsFfnRows);
  const size_t split = (bs_workspace_bytes(f, mc, N, K, nullptr, nullptr, nullptr) + 255) / 256 * 256;
  if (off_gu) *off_gu = split;
  return split + (size_t)2 * (size_t)mc * (size_t)N * 4;
}
}  // namespace

int qgemm_bs_ffn_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!bytes) return QGEMM_ERR_NULL;
  *bytes = bs_ffn_bytes(bs_id(fmt), N, K, M, nullptr);
  return QGEMM_OK;
}

int qgemm_bs_ffn_gate_up(int fmt, const void* x, int64_t M, int64_t K, const void* g_codes,
                         const void* g_scales, const float* g_ts, const void* u_codes,
                         const void* u_scales, const float* u_ts, int64_t N, void* h,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!bs_fmt(fmt)) return QGEMM_ERR_FORMAT;
  int st = check_fmt_shape(fmt, N, K);
  if (st != QGEMM_OK) return st;
  if (M < 1 || M > 0x7FFFFFFF) return QGEMM_ERR_SHAPE;
  if (!x || !h || !weights_given(fmt, g_codes, g_scales, g_ts) ||
      !weights_given(fmt, u_codes, u_scales, u_ts))
    return QGEMM_ERR_NULL;
  if (!aligned16(x) || !aligned16(h) || !aligned16(g_codes) || !aligned16(g_scales) ||
      !aligned16(u_codes) || !aligned16(u_scales))
    return QGEMM_ERR_ALIGN;
  const int f = bs_id(fmt);
  size_t off_gu = 0;
  const size_t need = bs_ffn_bytes(f, N, K, M, &off_gu);
  if (!workspace || workspace_bytes < need) return QGEMM_ERR_WORKSPACE;
  if (!aligned16(workspace)) return QGEMM_ERR_ALIGN;
  if (!device_ok()) return QGEMM_ERR_DEVICE;
  int* dev_err = error_word();
  if (!dev_err) return cuda_fail(cudaGetLastError(), "cudaGetSymbolAddress");
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const float* gts = bs_ts(fmt, g_ts);
  const float* uts = bs_ts(fmt, u_ts);
  for (int64_t r0 = 0; r0 < M; r0 += kBsFfnRows) {
    const int mc = (int)std::min<int64_t>(kBsFfnRows, M - r0);
    size_t off_s = 0, off_e = 0, off_p = 0;
    (void)bs_workspace_bytes(f, mc, N, K, &off_s, &off_e, &off_p);
    const uint16_t* xr = static_cast<const uint16_t*>(x) + (size_t)r0 * (size_t)K;
    cudaError_t e = launch_bs_split(f, xr, mc, (int)K, wsb, wsb + off_s,
                                    reinterpret_cast<int*>(wsb + off_e), s);
    if (e != cudaSuccess) return cuda_fail(e, "split kernel launch");
    float* gbuf = reinterpret_cast<float*>(wsb + off_gu);
    float* ubuf = gbuf + (size_t)mc * (size_t)N;
    for (int m = 0; m < 2 && e == cudaSuccess; ++m) {
      const uint8_t* wc = static_cast<const uint8_t*>(m ? u_codes : g_codes);
      const uint8_t* wsc = static_cast<const uint8_t*>(m ? u_scales : g_scales);
      float* out = m ? ubuf : gbuf;
      if (mc <= 128)
        e = launch_bs_dec(f, mc, (int)N, (int)K, wsb, wsb + off_s, reinterpret_cast<const int*>(wsb + off_e),
                          wc, wsc, m ? uts : gts, reinterpret_cast<float*>(wsb + off_p), out, 0, dev_err, s);
      else
        e = launch_bs_gemm(f, mc, (int)N, (int)K, wsb, wsb + off_s, reinterpret_cast<const int*>(wsb + off_e),
                           wc, wsc, m ? uts : gts, out, 0, dev_err, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "block-scaled gemm launch");
    ReduceParams rp{};
    rp.ws = gbuf;
    rp.S = 1;
    rp.NMAT = 2;
    rp.B = mc;
    rp.N = (int)N;
    rp.out = static_cast<uint8_t*>(h) + (size_t)r0 * (size_t)N * 2;
    rp.out_bf16 = 1;
    e = launch_reduce(rp, s);
    if (e != cudaSuccess) return cuda_fail(e, "SiLU pass launch");
  }
  return QGEMM_OK;
}

int qgemm_profile_events(void* begin_event, void* end_event) {
  g_prof_begin = static_cast<cudaEvent_t>(begin_event);
  g_prof_end = static_cast<cudaEvent_t>(end_event);
  return QGEMM_OK;
}

}  // extern "C"

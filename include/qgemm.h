/*
 * qgemm.h -- C ABI of libqgemm: bf16 activations x block-quantized weights on NVIDIA B200.
 *
 *   y[b][n] = sum_k x[b][k] * dequant(W)[n][k]        b < B, n < N, k < K
 *
 * Operation.  The batched quantized-weight GEMM behind the pages' `gemm_q8_0_batched`
 * (hipfire PR "fix(mtp): chunk scalar Q8 batched GEMM above 64 rows", section "Root
 * cause and fix") and the W4A16 prefill GEMMs (Atlas issue "Qwen3.8-27B on Strix Halo:
 * prefill 2.4x gap + DP4A verify tiers", section "Kernel ranking ...").  Unlike the
 * fixed MAX_BATCH=64 scalar kernel there, every width B >= 1 is accepted in one call,
 * and for 1 <= B <= 256 row b of y is bit-identical whatever the width of the call it
 * belongs to (the PR's chunked-vs-unchunked bit-exactness, generalised).
 *
 * Weight formats (the pages name them; their bit layouts are fixed here):
 *   QGEMM_FMT_Q8_0  int8 codes; one IEEE fp16 scale per 32 consecutive k:  w = q * d.
 *   QGEMM_FMT_NVFP4 E2M1 codes; one E4M3 scale per 16 consecutive k; one fp32 tensor
 *                   scale ts:  w = e2m1 * e4m3 * ts  (ts applied in the epilogue, as on
 *                   the Atlas issue's exact-F16-dequant section).
 *   QGEMM_FMT_MXFP4 E2M1 codes; one E8M0 scale per 32 consecutive k (the MXFP4 model
 *                   card's format, OCP MX v1.0):  w = e2m1 * 2^(e-127).
 *   QGEMM_FMT_FP8   E4M3 codes; no block scales; one fp32 tensor scale ts:  w = e4m3 * ts
 *                   (the FP8 W8A16 layers of the Atlas issue's kernel ranking and verify-tier
 *                   sections; ts applied in the epilogue).  K must be a multiple of 16.
 *
 * Packed layout (tile-major; what qgemm_pack writes and qgemm_run reads).  Rows are grouped
 * in tiles of 128 (T = ceil(N/128)), K in chunks of CK elements (CK = 128 for Q8_0 and FP8,
 * 256 for NVFP4 and MXFP4; C = ceil(K/CK)).  Rows past N and elements past K are zero.
 *   codes  [T][C][128 rows][128 bytes]: the row's CK elements of the chunk (Q8_0: one int8
 *          byte each; FP8: one E4M3 byte each; FP4: element 2j in the low nibble of byte j),
 *          with the row's 16-byte groups permuted: group g of row r is stored at position
 *          g ^ (r & 7).  Size T*C*16384 bytes.
 *   scales [T][C][128 rows][SB bytes], SB = 8 (Q8_0: 4 little-endian fp16; MXFP4: 8 E8M0),
 *          16 (NVFP4: 16 E4M3) or 0 (FP8), the row's block scales of the chunk in K order.
 *          Size T*C*128*SB bytes (0 for FP8: scales_dev may then be NULL everywhere).
 * Each (tile, chunk) is one contiguous block of codes and one of scales, so the kernel
 * streams it with two 1-D bulk copies.
 *
 * Row-major interchange layout (input of qgemm_repack_rowmajor): codes [N][code pitch]
 * (Q8_0, FP8: K bytes; FP4: K/2 bytes, element 2j in the low nibble of byte j), scales
 * [N][scale pitch] (Q8_0: K/32 little-endian fp16; NVFP4: K/16 E4M3; MXFP4: K/32 E8M0;
 * FP8: none, pitch 0);
 * qgemm_row_pitches gives the smallest 16-byte-aligned pitches.
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are device pointers; the caller owns every buffer and the
 *     stream.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - Calls are asynchronous on `stream` and return a status immediately; they never
 *     abort or exit the process.  A status other than QGEMM_OK means nothing was
 *     launched (argument errors) or a launch failed (QGEMM_ERR_CUDA).
 *   - Device pointers must be 16-byte aligned (TMA); x, y and h must be contiguous.
 *   - Device state that outlives a call: the error word read by qgemm_device_status(), and
 *     the fixed scratch of qgemm_run_noalloc (see there).  Host state: each calling thread
 *     keeps its last few tile plans and encoded x tensor maps (TMA descriptors, keyed by
 *     the operand's address and geometry; they hold no device memory).
 *   - qgemm_run and qgemm_ffn_gate_up calls that may overlap on the device need their own
 *     workspaces; qgemm_run_noalloc calls share one scratch and must not overlap.
 *   - The GEMM kernels are programmatic dependents of the small x-preparation kernel
 *     launched just before them and start streaming weights before they wait for it.  x
 *     (and every buffer a call writes) is ordered after all earlier work on the stream; the
 *     packed weights are read assuming the kernel that wrote them has completed, which holds
 *     for every kernel that does not trigger its dependents' launch early (this library's
 *     packers, and any kernel launched without programmatic dependent launch).
 */
#ifndef QGEMM_H
#define QGEMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Weight formats. */
#define QGEMM_FMT_Q8_0 0
#define QGEMM_FMT_NVFP4 1
#define QGEMM_FMT_MXFP4 2
#define QGEMM_FMT_FP8 3

/* Output element types of qgemm_run. */
#define QGEMM_Y_F32 0
#define QGEMM_Y_BF16 1

/* Status codes. */
#define QGEMM_OK 0
#define QGEMM_ERR_FORMAT 1         /* unknown format or output dtype                     */
#define QGEMM_ERR_SHAPE 2          /* N, K or B < 1, or a dimension above 2^31-1        */
#define QGEMM_ERR_K_BLOCK 3        /* K not a multiple of the format's block size       */
#define QGEMM_ERR_NULL 4           /* a required pointer is NULL                         */
#define QGEMM_ERR_ALIGN 5          /* a device pointer is not 16-byte aligned            */
#define QGEMM_ERR_WORKSPACE 6      /* workspace NULL or smaller than the required size   */
#define QGEMM_ERR_CUDA 7           /* a CUDA call or kernel launch failed                */
#define QGEMM_ERR_DEVICE 8         /* the current device is not an sm_100 part           */
#define QGEMM_ERR_DEVICE_TIMEOUT 9 /* a kernel's bounded wait ran out (see device_status) */
#define QGEMM_ERR_DEVICE_ARG 10    /* a kernel refused an argument read from device memory */

/*
 * Sizes of the tile-major packed buffers for an N x K weight matrix.  No device work.
 * Returns QGEMM_ERR_FORMAT / _SHAPE / _K_BLOCK / _NULL.  (No passage: a layout helper for
 * this library's packed layout, described above.)
 */
int qgemm_packed_size(int fmt, int64_t N, int64_t K, size_t* code_bytes, size_t* scale_bytes);

/*
 * Geometry of the tile-major layout: T row tiles, C chunks, CK elements per chunk and SB
 * scale bytes per row per chunk.  No device work.
 */
int qgemm_packed_geometry(int fmt, int64_t N, int64_t K, int64_t* row_tiles, int64_t* k_chunks,
                          int* chunk_elems, int* scale_bytes_per_row);

/* Smallest 16-byte-aligned row pitches (bytes) of the row-major interchange layout. */
int qgemm_row_pitches(int fmt, int64_t K, int64_t* code_pitch, int64_t* scale_pitch);

/*
 * Converts weights packed in the row-major interchange layout (codes_rm_dev with row pitch
 * code_pitch, scales_rm_dev with row pitch scale_pitch, both in bytes) into the tile-major
 * layout (codes_dev / scales_dev of qgemm_packed_size() bytes, 16-byte aligned).  A pure byte
 * permutation; padding is written as zeros.  Asynchronous on `stream`.
 * QGEMM_ERR_SHAPE if a pitch is smaller than the row's packed bytes.
 */
int qgemm_repack_rowmajor(int fmt, int64_t N, int64_t K, const void* codes_rm_dev,
                          int64_t code_pitch, const void* scales_rm_dev, int64_t scale_pitch,
                          void* codes_dev, void* scales_dev, void* stream);

/*
 * Quantize W_dev (fp32, row-major [N][K], contiguous) into the packed layout.
 *   Q8_0 : d = fp16_RNE(max|w|/127) (kept finite), q = clamp(RNE(w/d), -127, 127);
 *          a block whose d is 0 gets q = 0.
 *   NVFP4: ts = fp32_RNE(max|W|/(6*448)); per 16-block s = E4M3_RNE_sat(amax/(6*ts));
 *          code = E2M1_RNE_sat(w/(e4m3(s)*ts)); an all-zero block (or a scale that
 *          rounds to 0) gets scale 0 and codes 0.  Writes ts to *tensor_scale_dev.
 *   MXFP4: e = clamp(floor(log2 amax) - 2 + 127, 0, 254); code = E2M1_RNE_sat(w/2^(e-127));
 *          an all-zero block gets e = 0 and codes 0.
 *   FP8  : ts = fp32_RNE(max|W|/448); code = E4M3_RNE_sat(w/ts); a zero matrix gets ts = 0
 *          and codes 0.  Writes ts to *tensor_scale_dev.
 * Ties round to even.  A negative element whose magnitude rounds to 0 keeps its sign bit.
 * codes_dev / scales_dev: qgemm_packed_size() bytes (tile-major layout), 16-byte aligned.
 * tensor_scale_dev: one float (NVFP4 and FP8; ignored otherwise).
 * Not performance critical (uses fp64 for exact tie decisions).
 */
int qgemm_pack(int fmt, const float* W_dev, int64_t N, int64_t K, void* codes_dev,
               void* scales_dev, float* tensor_scale_dev, void* stream);

/*
 * Bytes of device workspace qgemm_run needs for (fmt, N, K, B).  May be 0.  (No passage: the
 * workspace holds this design's f16 copy of x, its per-row exponents and the split-K
 * partials of the fixed-order reduction.)
 */
int qgemm_workspace_size(int fmt, int64_t N, int64_t K, int64_t B, size_t* bytes);

/*
 * y_dev[B][N] = x_dev[B][K] (bf16) * dequant(W)^T, W given by codes_dev / scales_dev
 * (packed as above) and, for NVFP4 and FP8, the fp32 tensor scale at *tensor_scale_dev.
 *   y_dtype    : QGEMM_Y_F32 (fp32) or QGEMM_Y_BF16 (bf16, round to nearest even).
 *   workspace  : qgemm_workspace_size() bytes of device memory (may be NULL if that
 *                size is 0).  Its contents need no initialisation.
 * Any B >= 1.  For B <= 256 the result row b depends only on x row b, W, and (N, K):
 * the split of K, the order of every sum and the arithmetic do not depend on B.
 * Accuracy: fp32 accumulation of exactly dequantized weights (Q8_0 products are rounded
 * once to the 16-bit operand type).  Up to 256 rows each x row is scaled by a power of two
 * from its own maximum before the f16 conversion (exact for every element within 2^-38 of
 * the row maximum, bf16 subnormals included); the epilogue restores it with the tensor scale
 * applied first, so y is finite whenever the exact result is.
 */
int qgemm_run(int fmt, const void* x_dev, int64_t B, int64_t K, const void* codes_dev,
              const void* scales_dev, const float* tensor_scale_dev, int64_t N, void* y_dev,
              int y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Size in bytes of the fixed device scratch that qgemm_run_noalloc uses in place of a
 * caller-supplied workspace (32 MiB, reserved on every GPU that loads the library).
 */
#define QGEMM_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * qgemm_run without a workspace argument, for callers that cannot allocate device memory:
 * a serving runtime whose memory pool has reserved the GPU's memory up front and forbids
 * allocations outside it, a plugin to which the host framework hands nothing but its input
 * and output buffers, or a latency-critical path where an allocation's cost, its implicit
 * synchronisation or its possible failure cannot be afforded.  The paper has no counterpart;
 * this is a deployment convenience, not part of the method.
 *   Arguments, layouts, results and accuracy: as for qgemm_run (the same kernels run, with
 *   the same K split, so y matches qgemm_run's y for the same inputs).
 *   Scratch: a device global of QGEMM_NOALLOC_SCRATCH_BYTES inside the library, one per GPU.
 *   The call allocates nothing (no cudaMalloc, no library allocator).  A shape whose
 *   qgemm_workspace_size() exceeds QGEMM_NOALLOC_SCRATCH_BYTES is rejected with
 *   QGEMM_ERR_WORKSPACE before any device work; use qgemm_run for it.
 *   Set-up: the first call on each device looks up that device's scratch address (which
 *   may load the library's device code there); make that first call outside any stream
 *   capture, with the device current.
 *   Sharing: every call on a device uses the same scratch, which keeps whatever the last
 *   call left in it.  Nothing needs to start at zero (each call writes every scratch byte
 *   before it reads it), but calls that may overlap on the GPU -- on different streams, or
 *   from several host threads without ordering -- race on the scratch and give wrong
 *   results.  Calls ordered on one stream are safe.
 */
int qgemm_run_noalloc(int fmt, const void* x_dev, int64_t B, int64_t K, const void* codes_dev,
                      const void* scales_dev, const float* tensor_scale_dev, int64_t N,
                      void* y_dev, int y_dtype, void* stream);

/* Bytes of device workspace qgemm_ffn_gate_up needs for (fmt, N, K, M).  Above M = 256 it
 * holds the fp32 g and u of one chunk of rows (at most 2048 rows: 2 * rows * N * 4 bytes). */
int qgemm_ffn_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes);

/*
 * Fused gate+up projection with a SiLU(gate)*up epilogue (Atlas issue, "fused gate+up
 * with dual accumulators ... gate/up are never written to global"):
 *   g = x Wg^T, u = x Wu^T (fp32);
 *   h_dev[M][N] = bf16_RNE( g / (1 + exp(-g)) * u ).
 * Both matrices use the same format and shape [N][K]; x_dev is bf16 [M][K].
 * g_ts_dev / u_ts_dev: NVFP4 / FP8 tensor scales (NULL for the other formats).
 * For M <= 256 one kernel keeps g and u in its accumulators and never stores them, and row m
 * of h depends only on x row m (as for qgemm_run).  Above 256 rows, each chunk of rows runs
 * as two GEMMs into fp32 g and u in the workspace and one SiLU pass (prefill widths, where
 * the single kernel's narrower batch tiles would cost more than the round trip).
 * Asynchronous on `stream`; errors as for qgemm_run.
 */
int qgemm_ffn_gate_up(int fmt, const void* x_dev, int64_t M, int64_t K, const void* g_codes_dev,
                      const void* g_scales_dev, const float* g_ts_dev, const void* u_codes_dev,
                      const void* u_scales_dev, const float* u_ts_dev, int64_t N, void* h_dev,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * Routed mixture-of-experts variants (Atlas issue, "Per-32-K-step hot loop" table: the routed
 * expert kernels moe_w4a16_fused_gate_up_t and its pointer-table twin; Strix Halo prefill
 * journey: "a fused gate/up + SwiGLU for the MoE, and routed down-projections").  Every
 * expert's matrices are packed separately (qgemm_pack) with the same format and shape; the
 * kernel finds them through pointer tables, so they need not be contiguous.
 *   x_dev        bf16 [M][K]: the routed rows grouped by expert -- rows offsets[e] ..
 *                offsets[e+1]-1 belong to expert e (an expert may have none).
 *   offsets_dev  int32 [E+1] in device memory, non-decreasing, offsets[0] = 0, offsets[E] = M
 *                (values are clamped to [0, M], so no row outside x is read or written).
 *   max_rows     an upper bound on any expert's row count (1 <= max_rows); it sizes the
 *                launch, and rows of an expert past it are not computed.
 *   *_codes_tab / *_scales_tab / *_ts_tab: device arrays of E device pointers to each
 *                expert's packed codes, scales (NULL table allowed for FP8) and tensor scale
 *                (NVFP4 and FP8; else NULL).  Each buffer 16-byte aligned (tensor scales 4);
 *                an expert whose entry is NULL or misaligned is skipped and the device status
 *                becomes QGEMM_ERR_DEVICE_ARG.
 * Per expert the arithmetic is that of qgemm_run / qgemm_ffn_gate_up with the K split fixed
 * at 1: for max_rows <= 256 a row's output depends only on that row, its expert's weights
 * and (fmt, N, K) -- not on how many rows the expert or the call has.
 * Workspace: qgemm_moe_workspace_size() bytes (the f16 copy of x and its row exponents).
 */
int qgemm_moe_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, int64_t max_rows,
                             size_t* bytes);

/* y[m][n] = x[m] W_e^T for the rows m of expert e (the routed down projection). */
int qgemm_moe_run(int fmt, const void* x_dev, int64_t M, int64_t K, int E,
                  const int32_t* offsets_dev, int64_t max_rows, const void* const* codes_tab_dev,
                  const void* const* scales_tab_dev, const float* const* ts_tab_dev, int64_t N,
                  void* y_dev, int y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* h[m][n] = bf16(SiLU(x[m] Wg_e^T) * (x[m] Wu_e^T)) for the rows m of expert e (the routed
 * fused gate+up with the SiLU(gate)*up epilogue; g and u never leave the chip). */
int qgemm_moe_gate_up(int fmt, const void* x_dev, int64_t M, int64_t K, int E,
                      const int32_t* offsets_dev, int64_t max_rows,
                      const void* const* g_codes_tab_dev, const void* const* g_scales_tab_dev,
                      const float* const* g_ts_tab_dev, const void* const* u_codes_tab_dev,
                      const void* const* u_scales_tab_dev, const float* const* u_ts_tab_dev,
                      int64_t N, void* h_dev, void* workspace, size_t workspace_bytes,
                      void* stream);

/*
 * Block-scaled path for MXFP4, NVFP4 and FP8 weights (tcgen05.mma.kind::mxf4nvf4, or
 * kind::mxf8f6f4 for FP8, with block scales on both operands; the packed weights feed the
 * tensor cores without a dequantisation pass), with the activations quantised on the fly
 * (Atlas issue, kernel-ranking section: a block-scaled MMA path for prefill).  x is split per
 * row into terms with a power-of-two scale per block, in the MMA's scale type:
 *   MXFP4: three E2M1 terms, 32-element blocks, E8M0 scales, xshift 0, emin -127, top 2;
 *   NVFP4: three E2M1 terms, 16-element blocks, UE4M3 scales (powers of two 2^-9 .. 2^8
 *          only), xshift 10, emin -9, top 2;
 *   FP8:   two E4M3 terms, 32-element blocks, E8M0 scales, xshift 0, emin -127, top 7 (the
 *          weights' block scales are 1);
 *   x_exp = floor(log2 max|x_row|) - xshift,  r_0 = x * 2^-x_exp,
 *   e_j = floor(log2 max_block |r_j|) - top  (a term with e_j < emin and the later ones are
 *   dropped: zero codes, scale 0),  q_j = CODE_RNE_sat(r_j / 2^e_j),  r_{j+1} = r_j - q_j 2^e_j,
 * and y = 2^x_exp * (sum_j (q_j 2^e_j) W^T) [* tensor scale for NVFP4 and FP8], accumulated in
 * fp32.
 * The result differs from qgemm_run by the split's residual (measured normalised error below
 * 2e-4 at the 27B shapes); it is a separate entry point, not a mode of qgemm_run.  Up to 128
 * rows the weights are the MMA M operand and K is split over the SMs by a rule of (N, K)
 * alone (fp32 partials summed in a fixed order); above that x is.
 *
 * qgemm_bs_split_size / qgemm_bs_split_x: the split alone, for fmt MXFP4, NVFP4 or FP8.
 * Layout (device, caller-owned, 16-byte aligned), with Mt = ceil(M/128), CK = 256 (FP4) or
 * 128 (FP8) elements per chunk, C = ceil(K/CK), T = 3 (FP4) or 2 (FP8) terms, sbr = 8 (MXFP4),
 * 16 (NVFP4) or 4 (FP8):
 *   codes  [Mt][C][T][128][128] bytes: row r of block (t, c, j) holds elements
 *          CK c .. CK c + CK-1 of row 128t + r of term j (E2M1: two per byte, even element in
 *          the low nibble; E4M3: one per byte), its 16-byte groups stored at group ^ (r & 7).
 *          Rows past M and elements past K are zero.
 *   scales [Mt][C][T][128][sbr] scale bytes (E8M0 bias 127; UE4M3 bias 7), one per block.
 *   x_exp  [Mt*128] int32 (0 for rows past M and all-zero rows).
 * K must be a multiple of 32.  Errors: QGEMM_ERR_FORMAT, _SHAPE, _K_BLOCK, _NULL, _ALIGN,
 * _DEVICE, _CUDA.
 */
int qgemm_bs_split_size(int fmt, int64_t M, int64_t K, size_t* code_bytes, size_t* scale_bytes,
                        size_t* exp_bytes);
int qgemm_bs_split_x(int fmt, const void* x_dev, int64_t M, int64_t K, void* codes_dev,
                     void* scales_dev, int32_t* x_exp_dev, void* stream);

/*
 * qgemm_bs_workspace_size / qgemm_bs_run: y[M][N] = x W^T on the block-scaled path.  fmt must
 * be QGEMM_FMT_MXFP4, QGEMM_FMT_NVFP4 or QGEMM_FMT_FP8 (else QGEMM_ERR_FORMAT; NVFP4 and FP8
 * need their tensor scale);
 * the other arguments as for qgemm_run, with M the number of x rows.  The workspace
 * (qgemm_bs_workspace_size bytes) holds the split of x and, up to 128 rows, the K-split
 * partials.
 */
int qgemm_bs_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes);
int qgemm_bs_run(int fmt, const void* x_dev, int64_t M, int64_t K, const void* codes_dev,
                 const void* scales_dev, const float* tensor_scale_dev, int64_t N, void* y_dev,
                 int y_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * qgemm_bs_ffn_workspace_size / qgemm_bs_ffn_gate_up: h = bf16(SiLU(x Wg^T) * (x Wu^T)) on the
 * block-scaled path (fmt MXFP4, NVFP4 or FP8), the fused gate+up of the Atlas issue's kernel
 * ranking.  Per chunk of up to 2048 rows one split of x serves both GEMMs; g and u go to an
 * fp32 workspace and one pass writes h (the same SiLU(g) * u expression as
 * qgemm_ffn_gate_up).  Arguments as for qgemm_ffn_gate_up.
 */
int qgemm_bs_ffn_workspace_size(int fmt, int64_t N, int64_t K, int64_t M, size_t* bytes);
int qgemm_bs_ffn_gate_up(int fmt, const void* x_dev, int64_t M, int64_t K, const void* g_codes_dev,
                         const void* g_scales_dev, const float* g_ts_dev, const void* u_codes_dev,
                         const void* u_scales_dev, const float* u_ts_dev, int64_t N, void* h_dev,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * Number of K splits qgemm_run uses for 1 <= B <= 256 (a function of fmt, N, K only).
 */
int qgemm_split_k(int fmt, int64_t N, int64_t K, int* splits);

/*
 * Synchronizes the current device and reports whether any kernel of this library hit a
 * bounded-wait limit (QGEMM_ERR_DEVICE_TIMEOUT) or refused an argument it read from device
 * memory (QGEMM_ERR_DEVICE_ARG) since the last reset, else QGEMM_OK or QGEMM_ERR_CUDA.
 * reset != 0 clears the flag.
 */
int qgemm_device_status(int reset);

/*
 * Instrumentation: when begin_event / end_event are non-NULL (cudaEvent_t handles created by
 * the caller), the next qgemm_run / qgemm_ffn_gate_up calls made by this thread record them
 * on their stream immediately before and after the GEMM kernel (excluding the small x
 * preparation kernel that widths <= 256 run first).  Pass NULL, NULL to stop.  Returns
 * QGEMM_OK.
 */
int qgemm_profile_events(void* begin_event, void* end_event);

/* Static, human-readable text for a status code.  (No passage: error reporting; the pages'
 * only error path is the batch > 64 rejection this library removes.) */
const char* qgemm_status_str(int status);

/* Text of the last CUDA error seen by this library in the calling thread ("" if none). */
const char* qgemm_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QGEMM_H */

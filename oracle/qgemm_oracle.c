/*
 * qgemm_oracle.c -- plain, slow, CPU reference for the block-quantized-weight GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package smoke check and the
 * CPU-baseline leg of the benchmark may load this code.  The CUDA library never
 * links, includes or calls it, and it shares no code, table or helper with it.
 *
 * What it computes (the definition, in fp64, sequential k):
 *     y[b][n] = sum_k  x[b][k] * deq(W)[n][k]
 * with x given as bf16 bit patterns (decoded exactly) and W given in one of four
 * quantized encodings:
 *   Q8_0  : int8 codes, one fp16 scale per 32 consecutive k        (w = q * d16)
 *   NVFP4 : E2M1 codes, one E4M3 scale per 16 consecutive k, plus
 *           one fp32 tensor scale                                   (w = e2m1 * e4m3 * ts)
 *   MXFP4 : E2M1 codes, one E8M0 scale per 32 consecutive k        (w = e2m1 * 2^(e-127))
 *   FP8   : E4M3 codes, one fp32 tensor scale                       (w = e4m3 * ts)
 *
 * Sources (web pages on block-quantized GEMMs):
 *   - hipfire PR "chunk scalar Q8 batched GEMM above 64 rows": the batched Q8_0 GEMM
 *     and its chunked-vs-unchunked bit-exactness matrix (widths 64/65/70/76/256).
 *   - Atlas issue "Qwen3.8-27B on Strix Halo: prefill 2.4x gap": the NVFP4 W4A16 GEMM
 *     (E2M1 codes, E4M3 block scale, fp32 tensor scale applied in the epilogue),
 *     the exhaustive "254 non-NaN scale bytes x 16 codes" exactness argument, the
 *     FP64 host reference with exact weights, and the fused gate+up with a
 *     SiLU(gate)*up epilogue.
 *   - "Qwen3.8-27B MXFP4 (AMD Quark) for RDNA4" model card: the MXFP4 weight format.
 *   - Atlas issue, kernel ranking and verify-tier sections: the FP8 (E4M3) weight layers of
 *     the NVIDIA pack behind w8a16_gemm_n_m128 and w8a16_gemv_batch8.
 * Where the pages are silent (bit layouts, scale recipes, nibble order, rounding of
 * the packers) the readings are stated beside each function.
 *
 * Parity status: every function below is pinned by CPU tests against values fixed
 * by the pages or by the mathematics (enumerated code tables, library float
 * conversions, brute-force rationals, one-hot closed forms, invariants).
 *
 * Packed layout (the library's public layout; this file implements it from its
 * description, independently of the CUDA side):
 *   codes  : row-major [N][cpitch] bytes.  Q8_0: byte k = int8 q_k, cpitch =
 *            roundup(K,16).  NVFP4/MXFP4: byte k/2 holds element k, the even element
 *            in the low nibble, cpitch = roundup(K/2,16).
 *   scales : row-major [N][spitch] bytes.  Q8_0: little-endian fp16 per 32-block,
 *            spitch = roundup(2*K/32,16).  NVFP4: one E4M3 byte per 16-block,
 *            spitch = roundup(K/16,16).  MXFP4: one E8M0 byte per 32-block,
 *            spitch = roundup(K/32,16).  FP8: no block scales, spitch = 0.
 *   FP8 codes: byte k = the E4M3 code of element k, cpitch = roundup(K,16).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_Q8_0 0
#define ORC_NVFP4 1
#define ORC_MXFP4 2
#define ORC_FP8 3

/* ------------------------------------------------------------------------- */
/* Element and scale decoders: each is the format's definition written out.  */
/* ------------------------------------------------------------------------- */

/* E2M1: nibble s e1 e0 m.  Magnitude by the low three bits is
 * {0, 0.5, 1, 1.5, 2, 3, 4, 6}; bit 3 is the sign.  (Atlas issue: "f16 of every
 * E2M1 value"; the code table itself is the standard FP4 E2M1 table.) */
double orc_e2m1(unsigned code) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[code & 7u];
    return (code & 8u) ? -v : v;
}

/* E4M3 (OCP FP8 "fn" variant): sign, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, exponent 15 with mantissa 7 is NaN.  Subnormals: m/8 * 2^-6.
 * The Atlas issue counts "254 non-NaN scale bytes": 256 minus 0x7F and 0xFF. */
double orc_e4m3(unsigned byte) {
    unsigned s = (byte >> 7) & 1u, e = (byte >> 3) & 15u, m = byte & 7u;
    double v;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -v : v;
}

/* E8M0 (OCP MX shared scale): 2^(e-127); e = 255 is NaN. */
double orc_e8m0(unsigned byte) {
    if ((byte & 0xFFu) == 255u) return NAN;
    return ldexp(1.0, (int)(byte & 0xFFu) - 127);
}

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
double orc_f16(unsigned h) {
    unsigned s = (h >> 15) & 1u, e = (h >> 10) & 31u, m = h & 1023u;
    double v;
    if (e == 31u) v = (m == 0u) ? INFINITY : NAN;
    else if (e == 0u) v = ldexp((double)m, -24);
    else v = ldexp(1.0 + (double)m / 1024.0, (int)e - 15);
    return s ? -v : v;
}

/* bfloat16: 1 sign, 8 exponent (bias 127), 7 mantissa bits. */
double orc_bf16(unsigned h) {
    unsigned s = (h >> 15) & 1u, e = (h >> 7) & 255u, m = h & 127u;
    double v;
    if (e == 255u) v = (m == 0u) ? INFINITY : NAN;
    else if (e == 0u) v = ldexp((double)m, -133);
    else v = ldexp(1.0 + (double)m / 128.0, (int)e - 127);
    return s ? -v : v;
}

/* ------------------------------------------------------------------------- */
/* Encoders (round to nearest, ties to even).                                 */
/* ------------------------------------------------------------------------- */

/* E2M1 magnitude code nearest to a >= 0, ties to the even code (the code whose
 * mantissa bit is 0), saturating at 6.  Written as a scan of the 8-entry table. */
static unsigned e2m1_mag_code_rne_sat(double a) {
    unsigned best = 0;
    if (a >= 6.0) return 7u; /* saturate (also keeps huge a away from fp64 distance ties) */
    double bestd = fabs(a - orc_e2m1(0));
    for (unsigned c = 1; c < 8; ++c) {
        double d = fabs(a - orc_e2m1(c));
        if (d < bestd || (d == bestd && (c & 1u) == 0u && (best & 1u) == 1u)) {
            best = c;
            bestd = d;
        }
    }
    return best;
}

/* Full E2M1 code for a value: sign from v (negative values keep the sign bit even
 * when the magnitude rounds to zero), magnitude as above. */
unsigned orc_e2m1_encode(double v) {
    unsigned sign = (v < 0.0) ? 8u : 0u;
    return sign | e2m1_mag_code_rne_sat(fabs(v));
}

/* E4M3 byte nearest to a >= 0 among the 127 finite non-negative values, ties to
 * the even byte, saturating at 448 (0x7E).  The values grow with the byte (0x00..0x7E), so
 * a binary search finds the largest byte lo whose value is <= a; the answer is lo or lo + 1,
 * whichever is nearer, the even one on a tie. */
static double e4m3_pos_table[0x7F];
static int e4m3_pos_table_ready = 0;

unsigned orc_e4m3_encode_pos(double a) {
    unsigned lo = 0, hi = 0x7Eu, mid;
    double dlo, dhi;
    if (!e4m3_pos_table_ready) {  /* the decoder's values, once (callers are single-threaded) */
        for (unsigned c = 0; c < 0x7Fu; ++c) e4m3_pos_table[c] = orc_e4m3(c);
        e4m3_pos_table_ready = 1;
    }
    if (a >= 448.0) return 0x7Eu; /* saturate at the largest finite value */
    while (lo < hi) {             /* invariant: value(lo) <= a (value(0) = 0) */
        mid = (lo + hi + 1u) / 2u;
        if (e4m3_pos_table[mid] <= a) lo = mid;
        else hi = mid - 1u;
    }
    dlo = a - e4m3_pos_table[lo];
    dhi = e4m3_pos_table[lo + 1u] - a;  /* lo < 0x7E here because a < 448 */
    if (dlo < dhi) return lo;
    if (dhi < dlo) return lo + 1u;
    return (lo & 1u) ? lo + 1u : lo;
}

/* Signed E4M3 code of a finite value: the magnitude as orc_e4m3_encode_pos, the sign
 * from v (a negative value whose magnitude rounds to zero keeps the sign bit, 0x80). */
unsigned orc_e4m3_encode(double v) {
    unsigned sign = (v < 0.0) ? 0x80u : 0u;
    return sign | orc_e4m3_encode_pos(fabs(v));
}

/* IEEE binary16 nearest to v, ties to even, saturating to +-65504 (the Q8_0
 * scale is kept finite).  Works by exact power-of-two rescaling and the C
 * library's round-half-even (nearbyint in the default rounding mode). */
unsigned orc_f16_encode_satfinite(double v) {
    unsigned sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x8000u : 0u;
    double a = fabs(v);
    int ex;
    double q, r;
    unsigned e, m;
    if (a == 0.0) return sign;
    (void)frexp(a, &ex);          /* a = f * 2^ex, f in [0.5,1): floor(log2 a) = ex-1 */
    ex -= 1;
    if (ex < -14) ex = -14;       /* subnormal range shares the quantum 2^-24 */
    q = ldexp(1.0, ex - 10);      /* spacing of binary16 values in this binade */
    r = nearbyint(a / q);         /* a/q is exact: division by a power of two */
    a = r * q;
    if (a > 65504.0) a = 65504.0;
    if (a == 0.0) return sign;
    (void)frexp(a, &ex);
    ex -= 1;
    if (ex < -14) { /* subnormal */
        m = (unsigned)(a / ldexp(1.0, -24));
        return sign | m;
    }
    e = (unsigned)(ex + 15);
    m = (unsigned)((a / ldexp(1.0, ex) - 1.0) * 1024.0);
    return sign | (e << 10) | m;
}

/* bfloat16 nearest to v (one rounding from fp64), ties to even; overflow to inf. */
unsigned orc_bf16_encode(double v) {
    unsigned sign = (v < 0.0 || (v == 0.0 && signbit(v))) ? 0x8000u : 0u;
    double a = fabs(v), q, r;
    int ex;
    unsigned e, m;
    if (isnan(v)) return 0x7FC0u;
    if (a == 0.0) return sign;
    (void)frexp(a, &ex);
    ex -= 1;
    if (ex < -126) ex = -126;
    q = ldexp(1.0, ex - 7);
    r = nearbyint(a / q);
    a = r * q;
    if (a == 0.0) return sign;
    if (a >= ldexp(1.0, 128)) return sign | 0x7F80u;
    (void)frexp(a, &ex);
    ex -= 1;
    if (ex < -126) {
        m = (unsigned)(a / ldexp(1.0, -133));
        return sign | m;
    }
    e = (unsigned)(ex + 127);
    m = (unsigned)((a / ldexp(1.0, ex) - 1.0) * 128.0);
    return sign | (e << 7) | m;
}

/* ------------------------------------------------------------------------- */
/* Layout helpers                                                             */
/* ------------------------------------------------------------------------- */

static int64_t roundup16(int64_t v) { return (v + 15) / 16 * 16; }

/* K granularity of each format: its scale block (FP8 has none; 16 keeps x rows aligned). */
int orc_block_size(int fmt) { return (fmt == ORC_NVFP4 || fmt == ORC_FP8) ? 16 : 32; }

int64_t orc_code_pitch(int fmt, int64_t K) {
    return (fmt == ORC_Q8_0 || fmt == ORC_FP8) ? roundup16(K) : roundup16(K / 2);
}

int64_t orc_scale_pitch(int fmt, int64_t K) {
    if (fmt == ORC_Q8_0) return roundup16(2 * (K / 32));
    if (fmt == ORC_NVFP4) return roundup16(K / 16);
    if (fmt == ORC_FP8) return 0;
    return roundup16(K / 32);
}

static void put_nibble(uint8_t *row, int64_t k, unsigned code) {
    uint8_t *p = row + k / 2;
    if (k % 2 == 0) *p = (uint8_t)((*p & 0xF0u) | (code & 0xFu));
    else *p = (uint8_t)((*p & 0x0Fu) | ((code & 0xFu) << 4));
}

/* ORC_MUTATE plants one known mistake (for the tests that show the pins catch it; the
   library build never defines it): 1 nibble order, 2 dropped NVFP4 tensor scale,
   3 dropped last term of each dot product, 4 Q8_0 scale bytes swapped, 5 dropped FP8
   tensor scale, 6 FP8 sign bit ignored. */
#ifndef ORC_MUTATE
#define ORC_MUTATE 0
#endif

static unsigned get_nibble(const uint8_t *row, int64_t k) {
    uint8_t b = row[k / 2];
    if (ORC_MUTATE == 1) return (k % 2 == 0) ? (b >> 4) : (b & 0xFu);
    return (k % 2 == 0) ? (b & 0xFu) : (b >> 4);
}

/* ------------------------------------------------------------------------- */
/* Packers.  Readings (the pages do not define the recipes):                  */
/*  Q8_0 : d16 = fp16_RNE(amax/127) (kept finite); q = clamp(RNE(w/d16),+-127)*/
/*         using the ROUNDED d16, so |w - q*d16| <= d16/2 holds exactly.      */
/*         A block whose d16 is 0 gets q = 0.                                 */
/*  NVFP4: ts = fp32_RNE(amax(W)/(6*448)); s = E4M3_RNE_sat(amax_blk/(6*ts)); */
/*         code = E2M1_RNE_sat(w/(e4m3(s)*ts)).  A block with amax 0, or a    */
/*         zero ts, or a scale that rounds to 0, gets scale 0 and codes 0.    */
/*  MXFP4: e = clamp(floor(log2 amax_blk) - 2 + 127, 0, 254) (OCP MX v1.0);   */
/*         code = E2M1_RNE_sat(w/2^(e-127)); amax 0 gives e = 0, codes 0.     */
/*  FP8  : ts = fp32_RNE(amax(W)/448) (one scale per matrix: the pages' FP8   */
/*         layers come from an NVIDIA pack, whose FP8 recipe scales per       */
/*         tensor); code = E4M3_RNE_sat(w/ts); a zero ts gives codes 0.       */
/* All quotients are formed once in fp64 from exact operands.                 */
/* ------------------------------------------------------------------------- */

void orc_pack_q8_0(const float *W, int64_t N, int64_t K, uint8_t *codes, uint8_t *scales) {
    int64_t cp = orc_code_pitch(ORC_Q8_0, K), sp = orc_scale_pitch(ORC_Q8_0, K);
    memset(codes, 0, (size_t)(N * cp));
    memset(scales, 0, (size_t)(N * sp));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t kb = 0; kb < K / 32; ++kb) {
            const float *w = W + n * K + kb * 32;
            double amax = 0.0, d;
            unsigned h;
            for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs((double)w[i]));
            h = orc_f16_encode_satfinite(amax / 127.0);
            d = orc_f16(h);
            scales[n * sp + 2 * kb] = (uint8_t)(h & 0xFFu);
            scales[n * sp + 2 * kb + 1] = (uint8_t)(h >> 8);
            for (int i = 0; i < 32; ++i) {
                double q = 0.0;
                if (d != 0.0) {
                    q = nearbyint((double)w[i] / d);
                    if (q > 127.0) q = 127.0;
                    if (q < -127.0) q = -127.0;
                }
                codes[n * cp + kb * 32 + i] = (uint8_t)(int8_t)q;
            }
        }
    }
}

/* Returns the fp32 tensor scale through *ts. */
void orc_pack_nvfp4(const float *W, int64_t N, int64_t K, uint8_t *codes, uint8_t *scales,
                    float *ts_out) {
    int64_t cp = orc_code_pitch(ORC_NVFP4, K), sp = orc_scale_pitch(ORC_NVFP4, K);
    double amax = 0.0;
    float ts;
    memset(codes, 0, (size_t)(N * cp));
    memset(scales, 0, (size_t)(N * sp));
    for (int64_t i = 0; i < N * K; ++i) amax = fmax(amax, fabs((double)W[i]));
    ts = (float)(amax / (6.0 * 448.0));
    *ts_out = ts;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t kb = 0; kb < K / 16; ++kb) {
            const float *w = W + n * K + kb * 16;
            double ab = 0.0, sv;
            unsigned s = 0;
            for (int i = 0; i < 16; ++i) ab = fmax(ab, fabs((double)w[i]));
            if (ab != 0.0 && ts != 0.0f) s = orc_e4m3_encode_pos(ab / (6.0 * (double)ts));
            sv = orc_e4m3(s);
            scales[n * sp + kb] = (uint8_t)s;
            for (int i = 0; i < 16; ++i) {
                unsigned c = 0;
                if (sv != 0.0) c = orc_e2m1_encode((double)w[i] / (sv * (double)ts));
                put_nibble(codes + n * cp, kb * 16 + i, c);
            }
        }
    }
}

void orc_pack_mxfp4(const float *W, int64_t N, int64_t K, uint8_t *codes, uint8_t *scales) {
    int64_t cp = orc_code_pitch(ORC_MXFP4, K), sp = orc_scale_pitch(ORC_MXFP4, K);
    memset(codes, 0, (size_t)(N * cp));
    memset(scales, 0, (size_t)(N * sp));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t kb = 0; kb < K / 32; ++kb) {
            const float *w = W + n * K + kb * 32;
            double ab = 0.0, sv;
            int e = 0, ex;
            for (int i = 0; i < 32; ++i) ab = fmax(ab, fabs((double)w[i]));
            if (ab != 0.0) {
                (void)frexp(ab, &ex); /* floor(log2 ab) = ex - 1, exactly */
                e = (ex - 1) - 2 + 127;
                if (e < 0) e = 0;
                if (e > 254) e = 254;
            }
            scales[n * sp + kb] = (uint8_t)e;
            sv = orc_e8m0((unsigned)e);
            for (int i = 0; i < 32; ++i) {
                unsigned c = 0;
                if (ab != 0.0) c = orc_e2m1_encode((double)w[i] / sv);
                put_nibble(codes + n * cp, kb * 32 + i, c);
            }
        }
    }
}

/* Returns the fp32 tensor scale through *ts_out. */
void orc_pack_fp8(const float *W, int64_t N, int64_t K, uint8_t *codes, float *ts_out) {
    int64_t cp = orc_code_pitch(ORC_FP8, K);
    double amax = 0.0;
    float ts;
    memset(codes, 0, (size_t)(N * cp));
    for (int64_t i = 0; i < N * K; ++i) amax = fmax(amax, fabs((double)W[i]));
    ts = (float)(amax / 448.0);
    *ts_out = ts;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            codes[n * cp + k] =
                (uint8_t)(ts != 0.0f ? orc_e4m3_encode((double)W[n * K + k] / (double)ts) : 0u);
}

/* ------------------------------------------------------------------------- */
/* Dequantisation to fp64 (exact).                                            */
/* ------------------------------------------------------------------------- */

void orc_dequant(int fmt, const uint8_t *codes, const uint8_t *scales, float ts, int64_t N,
                 int64_t K, double *Wd) {
    int64_t cp = orc_code_pitch(fmt, K), sp = orc_scale_pitch(fmt, K);
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *cr = codes + n * cp, *sr = scales + n * sp;
        for (int64_t k = 0; k < K; ++k) {
            double v;
            if (fmt == ORC_Q8_0) {
                unsigned h = (unsigned)sr[2 * (k / 32)] | ((unsigned)sr[2 * (k / 32) + 1] << 8);
                if (ORC_MUTATE == 4)
                    h = (unsigned)sr[2 * (k / 32) + 1] | ((unsigned)sr[2 * (k / 32)] << 8);
                v = (double)(int8_t)cr[k] * orc_f16(h);
            } else if (fmt == ORC_NVFP4) {
                v = orc_e2m1(get_nibble(cr, k)) * orc_e4m3(sr[k / 16]) *
                    (ORC_MUTATE == 2 ? 1.0 : (double)ts);
            } else if (fmt == ORC_FP8) {
                v = orc_e4m3(ORC_MUTATE == 6 ? (cr[k] & 0x7Fu) : cr[k]) *
                    (ORC_MUTATE == 5 ? 1.0 : (double)ts);
            } else {
                v = orc_e2m1(get_nibble(cr, k)) * orc_e8m0(sr[k / 32]);
            }
            Wd[n * K + k] = v;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* GEMM: y[b][n] = sum_k x[b][k] * Wd[n][k], fp64, k ascending.               */
/* Threads split the n range only; each dot product is one sequential loop.   */
/* ------------------------------------------------------------------------- */

typedef struct {
    const double *xd;
    const double *Wd;
    double *y;
    int64_t B, K, N, n0, n1;
} gemm_job;

static void *gemm_worker(void *arg) {
    gemm_job *j = (gemm_job *)arg;
    for (int64_t n = j->n0; n < j->n1; ++n) {
        const double *w = j->Wd + n * j->K;
        for (int64_t b = 0; b < j->B; ++b) {
            const double *x = j->xd + b * j->K;
            double acc = 0.0;
            const int64_t kend = (ORC_MUTATE == 3) ? j->K - 1 : j->K;
            for (int64_t k = 0; k < kend; ++k) acc += x[k] * w[k];
            j->y[b * j->N + n] = acc;
        }
    }
    return NULL;
}

/* x16: bf16 bit patterns [B][K]; Wd: dequantised weights [N][K]; y: [B][N]. */
void orc_gemm(const uint16_t *x16, int64_t B, int64_t K, const double *Wd, int64_t N, double *y,
              int nthreads) {
    double *xd = (double *)malloc(sizeof(double) * (size_t)(B * K));
    pthread_t th[256];
    gemm_job jobs[256];
    int t;
    for (int64_t i = 0; i < B * K; ++i) xd[i] = orc_bf16(x16[i]);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > N) nthreads = (int)(N > 0 ? N : 1);
    for (t = 0; t < nthreads; ++t) {
        jobs[t].xd = xd;
        jobs[t].Wd = Wd;
        jobs[t].y = y;
        jobs[t].B = B;
        jobs[t].K = K;
        jobs[t].N = N;
        jobs[t].n0 = N * t / nthreads;
        jobs[t].n1 = N * (t + 1) / nthreads;
        if (nthreads == 1) gemm_worker(&jobs[t]);
        else pthread_create(&th[t], NULL, gemm_worker, &jobs[t]);
    }
    if (nthreads > 1)
        for (t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(xd);
}

/* ------------------------------------------------------------------------- */
/* Activation split for a block-scaled MMA (the "on-the-fly activation          */
/* quantisation" of a kind::mxf8f6f4 / kind::mxf4 path).  Reading: each 32-block */
/* of a row is peeled into `terms` low-precision terms, each with its own E8M0   */
/* (power-of-two) scale from the remaining block maximum:                        */
/*   r_0 = x;  e_j = floor(log2 max|r_j|) - top;  q_j = ENC(r_j / 2^e_j);        */
/*   r_{j+1} = r_j - q_j 2^e_j                                                   */
/* with top = 7 for E4M3 (the maximum lands in [128, 256), below 448) and top = 2 */
/* for E2M1 (the maximum lands in [4, 8), saturating at 6, as the MXFP4 packer).  */
/* xs receives sum_j q_j 2^e_j, the x the block-scaled MMA would multiply.       */
/* elem: 0 = E4M3, 1 = E2M1.                                                     */
/* ------------------------------------------------------------------------- */
void orc_split_x(const uint16_t *x16, int64_t B, int64_t K, int elem, int terms, double *xs) {
    const int top = elem == 0 ? 7 : 2;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t k0 = 0; k0 < K; k0 += 32) {
            double r[32], acc[32];
            const int64_t n = (K - k0 < 32) ? K - k0 : 32;
            for (int64_t i = 0; i < n; ++i) {
                r[i] = orc_bf16(x16[b * K + k0 + i]);
                acc[i] = 0.0;
            }
            for (int j = 0; j < terms; ++j) {
                double amax = 0.0, sc;
                int ex;
                for (int64_t i = 0; i < n; ++i) amax = fmax(amax, fabs(r[i]));
                if (amax == 0.0) break;
                (void)frexp(amax, &ex);           /* floor(log2 amax) = ex - 1 */
                sc = ldexp(1.0, (ex - 1) - top);
                for (int64_t i = 0; i < n; ++i) {
                    double q;
                    if (elem == 0) {
                        unsigned c = orc_e4m3_encode(r[i] / sc);
                        q = orc_e4m3(c);
                    } else {
                        q = orc_e2m1(orc_e2m1_encode(r[i] / sc));
                    }
                    acc[i] += q * sc;
                    r[i] -= q * sc;
                }
            }
            for (int64_t i = 0; i < n; ++i) xs[b * K + k0 + i] = acc[i];
        }
    }
}

/* ------------------------------------------------------------------------- */
/* The activation split of the block-scaled path as the product applies it     */
/* (reading: the split above with a per-row power-of-two prescale and a bounded */
/* range of power-of-two block scales, so that each term's scale is a value of  */
/* the MMA's scale type):                                                       */
/*   xe = floor(log2 max|x_row|) - xshift   (0 for an all-zero row)            */
/*   r_0 = x 2^-xe;  per block of `block` elements and term j:                  */
/*   e_j = floor(log2 max|r_j|) - top; if e_j < emin the term and the later     */
/*   ones are dropped; q_j = ENC(r_j / 2^e_j); r_{j+1} = r_j - q_j 2^e_j,        */
/* with ENC = E2M1_RNE_sat, top = 2 (elem 1) or E4M3_RNE_sat, top = 7 (elem 0). */
/* xs receives 2^xe sum_j q_j 2^e_j.  MXFP4 (E8M0 per 32): block 32, xshift 0,  */
/* emin -127, E2M1.  NVFP4 (UE4M3 per 16, powers of two only): block 16,        */
/* xshift 10, emin -9 (2^-9 is the smallest UE4M3 power of two; the prescale    */
/* puts the row maximum in [2^10, 2^11), so e_j <= 8 and 2^8 is representable), */
/* E2M1.  FP8 weights (E8M0 per 32): block 32, xshift 0, emin -127, E4M3.       */
/* ------------------------------------------------------------------------- */
void orc_split_x_bs(const uint16_t *x16, int64_t B, int64_t K, int block, int xshift, int emin,
                    int elem, int terms, double *xs) {
    const int top = elem == 0 ? 7 : 2;
    for (int64_t b = 0; b < B; ++b) {
        double rmax = 0.0;
        int xe = 0;
        for (int64_t k = 0; k < K; ++k) rmax = fmax(rmax, fabs(orc_bf16(x16[b * K + k])));
        if (rmax > 0.0) {
            int ex;
            (void)frexp(rmax, &ex);
            xe = (ex - 1) - xshift;
        }
        for (int64_t k0 = 0; k0 < K; k0 += block) {
            double r[64], acc[64];
            const int64_t n = (K - k0 < block) ? K - k0 : block;
            for (int64_t i = 0; i < n; ++i) {
                r[i] = ldexp(orc_bf16(x16[b * K + k0 + i]), -xe);
                acc[i] = 0.0;
            }
            for (int j = 0; j < terms; ++j) {
                double amax = 0.0, sc;
                int ex, e;
                for (int64_t i = 0; i < n; ++i) amax = fmax(amax, fabs(r[i]));
                if (amax == 0.0) break;
                (void)frexp(amax, &ex);
                e = (ex - 1) - top;
                if (e < emin) break;
                sc = ldexp(1.0, e);
                for (int64_t i = 0; i < n; ++i) {
                    const double q = elem == 0 ? orc_e4m3(orc_e4m3_encode(r[i] / sc))
                                               : orc_e2m1(orc_e2m1_encode(r[i] / sc));
                    acc[i] += q * sc;
                    r[i] -= q * sc;
                }
            }
            for (int64_t i = 0; i < n; ++i) xs[b * K + k0 + i] = ldexp(acc[i], xe);
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Fused FFN (Atlas issue: fused gate+up with dual accumulators; the pages'    */
/* prefill path writes the activated product as bf16 for the down GEMM).      */
/*   g = x Wg^T, u = x Wu^T (fp64); SiLU(g) = g / (1 + exp(-g));               */
/*   h = bf16_RNE(SiLU(g) * u).  Also returns g and u for error bounds.        */
/* ------------------------------------------------------------------------- */

double orc_silu(double g) { return g / (1.0 + exp(-g)); }

void orc_ffn_gate_up(const uint16_t *x16, int64_t M, int64_t K, const double *Wg,
                     const double *Wu, int64_t N, double *g, double *u, uint16_t *h16,
                     int nthreads) {
    orc_gemm(x16, M, K, Wg, N, g, nthreads);
    orc_gemm(x16, M, K, Wu, N, u, nthreads);
    for (int64_t i = 0; i < M * N; ++i) h16[i] = (uint16_t)orc_bf16_encode(orc_silu(g[i]) * u[i]);
}

/*
 * w4_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU implementation of what the W4-G256
 * quantized-matmul path computes.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it; the product library never
 * links, calls or falls back to it, and it shares no code, header, table or
 * constant with the CUDA sources.
 *
 * Sources (web pages the method is described on):
 *   - "hipfire HFQ4-G256 MMQ prefill" (ai-navigate-news article): HFQ4-G256
 *     weights, activations pre-quantised to a Q8_1-style int8 block layout,
 *     tiled int8 matrix-matrix product with scale application ("What changed"
 *     list).
 *   - "GFX1100-TG200 campaign" (vllm.cpp issue #5, "Goal" and "Working
 *     rules"): batch-1 decode GEMV streaming 4-bit weights; op-level error
 *     against a CPU oracle is the correctness gate.
 *   - "spec(GFX1100-TG150)" (vllm.cpp PR #4, "Design"): the integer core of the
 *     keep-quant path is bit-exact against the CPU.
 * The pages name the formats but print no byte layout; the format used here is
 * the W4-G256 definition: W[N,K], K a multiple of 256, groups of 256 along K,
 * 4-bit codes q in [0,15] with one fp16 scale d and one fp16 min m per group,
 * w = d*q + m; activations for the W4A8 product are int8 per 32-element block
 * with an fp32 scale and an int32 block sum.  The weight quantiser and the
 * dequantised product also take a group size, for the group-32 variant of the
 * same format (one d and m per 32 weights).  Readings where the pages are
 * silent (nibble order, rounding rules, scale formula) are listed in the
 * repository's design notes and restated at each function below.
 *
 * Precision: reductions that define y are carried in fp64 (int64 for integer
 * block dot products).  The weight and activation quantisers are specified in
 * fp32 (compile with -ffp-contract=off and without fast-math) so that a
 * correct GPU implementation reproduces their outputs bit for bit.
 *
 * Parity pins: every function here is pinned by tests against brute force,
 * closed forms, invariants or library routines (no function is "parity
 * unpinned").
 *
 * Mutation hooks: compiling with -DORACLE_MUTANT_<NAME> plants one deliberate
 * mistake; the test-suite builds those variants and checks that its pins
 * catch each one.  A normal build defines none of them.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 256 /* weights per (row, group): one d and one m        */
#define ORACLE_BLOCK 32  /* activations per int8 block: one dx and one S     */

/* ------------------------------------------------------------------------ */
/* scalar conversions (IEEE round-to-nearest-even via the compiler's types) */
/* ------------------------------------------------------------------------ */

static double bf16_bits_to_double(uint16_t b) {
    /* bf16 is the top half of an IEEE binary32 */
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_bits_to_float(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static double f16_bits_to_double(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (double)h;
}

static uint16_t float_to_f16_bits(float f) {
    _Float16 h = (_Float16)f; /* IEEE binary16, round to nearest even */
    uint16_t b;
    memcpy(&b, &h, sizeof b);
    return b;
}

static float f16_bits_to_float(uint16_t b) {
    _Float16 h;
    memcpy(&h, &b, sizeof h);
    return (float)h;
}

/* ------------------------------------------------------------------------ */
/* threads                                                                  */
/* ------------------------------------------------------------------------ */

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------------------ */
/* nibble packing                                                           */
/* ------------------------------------------------------------------------ */

/* One code from a packed row.  Byte j of a row holds element k = 2j in its
 * low four bits and k = 2j+1 in its high four bits (the pages leave the
 * nibble order open; this is the reading adopted). */
static unsigned code_at(const uint8_t *row, int64_t k) {
    uint8_t byte = row[k >> 1];
#ifdef ORACLE_MUTANT_SWAP_NIBBLES
    return (k & 1) ? (byte & 0xFu) : (byte >> 4);
#else
    return (k & 1) ? (byte >> 4) : (byte & 0xFu);
#endif
}

/* q: [N][K] codes 0..15, one per byte  ->  codes: [N][K/2] packed.
 * Returns 0, or -1 on a bad shape or a code above 15. */
int oracle_pack_codes(const uint8_t *q, int64_t N, int64_t K, uint8_t *codes) {
    if (N < 0 || K < 0 || (K & 1)) return -1;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < K / 2; ++j) {
            unsigned lo = q[n * K + 2 * j], hi = q[n * K + 2 * j + 1];
            if (lo > 15 || hi > 15) return -1;
#ifdef ORACLE_MUTANT_SWAP_NIBBLES
            codes[n * (K / 2) + j] = (uint8_t)(hi | (lo << 4));
#else
            codes[n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
#endif
        }
    }
    return 0;
}

/* codes: [N][K/2] packed  ->  q: [N][K], one code per byte. */
int oracle_unpack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *q) {
    if (N < 0 || K < 0 || (K & 1)) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            q[n * K + k] = (uint8_t)code_at(codes + n * (K / 2), k);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* weight quantiser (min/max per group)                                     */
/* ------------------------------------------------------------------------ */

/* w: fp32 [N][K]  ->  codes [N][K/2], d, m: fp16 bits [N][K/group], for a
 * group size `group` that is even and divides K: 256 for W4-G256, 32 for the
 * asymmetric int4 group-32 W4A16 scheme ("ROCM_OCTAVE", "Validation": its
 * models are W4A16, int4, group 32; the sparse-attention evaluation's "Setup"
 * calls the scheme asymmetric, g32), read as the same w = d*q + m form with
 * one d and one m per 32 weights.
 *
 * Per (row, group), in fp32:
 *   mn, mx = min, max of the group's weights
 *   d16 = fp16(RN((mx - mn) / 15)),  m16 = fp16(RN(mn))
 *   q   = 0 for every weight if d16 == 0, else
 *         clamp(rint((w - float(m16)) / float(d16)), 0, 15)   (ties to even)
 * so that w is approximated by float(d16)*q + float(m16), the dequantisation
 * rule w = d*q + m of the format.  Using the fp16-rounded d and m inside the
 * code computation keeps codes consistent with what is stored.
 * A group minimum or maximum that equals zero is taken as +0: -0 and +0 are
 * equal, so which of them a min/max search returns depends on where they sit
 * in the group; storing +0 makes d and m a function of the group's values
 * alone, independent of element order. */
static unsigned weight_code(float w, float df, float mf) {
    if (df == 0.0f) return 0;
    float num = w - mf;
#ifdef ORACLE_MUTANT_ROUND_AWAY
    float qf = roundf(num / df);
#else
    float qf = rintf(num / df);
#endif
    if (qf < 0.0f) qf = 0.0f;
    if (qf > 15.0f) qf = 15.0f;
    return (unsigned)qf;
}

int oracle_w4_pack_grouped(const float *w, int64_t N, int64_t K, int64_t group,
                           uint8_t *codes, uint16_t *d, uint16_t *m) {
    if (N < 0 || K < 0 || group < 2 || (group & 1) || (K % group)) return -1;
    const int64_t G = K / group;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t g = 0; g < G; ++g) {
            const float *wg = w + n * K + g * group;
            float mn = wg[0], mx = wg[0];
            for (int64_t i = 1; i < group; ++i) {
                if (wg[i] < mn) mn = wg[i];
                if (wg[i] > mx) mx = wg[i];
            }
#ifndef ORACLE_MUTANT_SIGNED_ZERO
            if (mn == 0.0f) mn = 0.0f; /* -0 -> +0 */
            if (mx == 0.0f) mx = 0.0f;
#endif
#ifdef ORACLE_MUTANT_RANGE_NO_MIN
            float range = mx;
#else
            float range = mx - mn;
#endif
            uint16_t d16 = float_to_f16_bits(range / 15.0f);
            uint16_t m16 = float_to_f16_bits(mn);
            float df = f16_bits_to_float(d16), mf = f16_bits_to_float(m16);
            uint8_t *crow = codes + n * (K / 2) + g * (group / 2);
            for (int64_t j = 0; j < group / 2; ++j) {
                unsigned lo = weight_code(wg[2 * j], df, mf);
                unsigned hi = weight_code(wg[2 * j + 1], df, mf);
#ifdef ORACLE_MUTANT_SWAP_NIBBLES
                crow[j] = (uint8_t)(hi | (lo << 4));
#else
                crow[j] = (uint8_t)(lo | (hi << 4));
#endif
            }
            d[n * G + g] = d16;
            m[n * G + g] = m16;
        }
    }
    return 0;
}

/* The W4-G256 packer: groups of 256. */
int oracle_w4_pack(const float *w, int64_t N, int64_t K, uint8_t *codes,
                   uint16_t *d, uint16_t *m) {
    return oracle_w4_pack_grouped(w, N, K, ORACLE_GROUP, codes, d, m);
}

/* ------------------------------------------------------------------------ */
/* activation quantiser (int8 per block of 32, Q8_1-style)                  */
/* ------------------------------------------------------------------------ */

/* x: bf16 bits [M][K], K % 32 == 0  ->  qa int8 [M][K], dx fp32 [M][K/32],
 * S int32 [M][K/32].  Per (token, block), in fp32:
 *   amax = max |x|           (exact: bf16 values are binary32 values)
 *   dx   = amax / 127        (IEEE division, round to nearest even)
 *   if amax == 0: dx = 0, qa = 0, S = 0
 *   else qa = clamp(rint(x / dx), -127, 127)  (ties to even),  S = sum of qa.
 * S is the integer sum of the codes, so the min term of the W4A8 product can
 * be formed exactly from it. */
int oracle_q8_quantize(const uint16_t *x, int64_t M, int64_t K, int8_t *qa,
                       float *dx, int32_t *S) {
    if (M < 0 || K < 0 || (K % ORACLE_BLOCK)) return -1;
    const int64_t B = K / ORACLE_BLOCK;
    for (int64_t t = 0; t < M; ++t) {
        for (int64_t b = 0; b < B; ++b) {
            const uint16_t *xb = x + t * K + b * ORACLE_BLOCK;
            float amax = 0.0f;
            for (int i = 0; i < ORACLE_BLOCK; ++i) {
                float a = fabsf(bf16_bits_to_float(xb[i]));
                if (a > amax) amax = a;
            }
#ifdef ORACLE_MUTANT_SCALE_128
            float scale = amax / 128.0f;
#else
            float scale = amax / 127.0f;
#endif
            int32_t sum = 0;
            for (int i = 0; i < ORACLE_BLOCK; ++i) {
                int8_t c = 0;
                if (amax != 0.0f) {
                    float r = bf16_bits_to_float(xb[i]) / scale;
#ifdef ORACLE_MUTANT_ROUND_AWAY
                    float qf = roundf(r);
#else
                    float qf = rintf(r);
#endif
                    if (qf > 127.0f) qf = 127.0f;
                    if (qf < -127.0f) qf = -127.0f;
                    c = (int8_t)qf;
                }
                qa[t * K + b * ORACLE_BLOCK + i] = c;
                sum += c;
            }
#ifdef ORACLE_MUTANT_BLOCKSUM_OFF_BY_ONE
            sum += 1;
#endif
            dx[t * B + b] = (amax == 0.0f) ? 0.0f : scale;
            S[t * B + b] = sum;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* GEMV / GEMM with dequantised weights (the definition, fp64)              */
/* ------------------------------------------------------------------------ */

/* The definition written out:
 *   y[t][n] = sum_k ( d[n][g(k)] * q[n][k] + m[n][g(k)] ) * x[t][k],
 * g(k) = k / group (group = 256 for W4-G256, 32 for the g32 scheme; d and m
 * are [N][K/group]), each weight dequantised on its own, accumulated in fp64
 * in plain k order.  x is fp64 [M][K]; y is fp64 [M][N].  Rows [n0, n1) only
 * (the full product is n0 = 0, n1 = N); y holds M x (n1 - n0) values, row
 * stride (n1 - n0). */
int oracle_gemv_f64_rows_grouped(const uint8_t *codes, const uint16_t *d,
                                 const uint16_t *m, int64_t N, int64_t K,
                                 int64_t group, const double *x, int64_t M,
                                 int64_t n0, int64_t n1, double *y) {
    if (N < 0 || K < 0 || group < 2 || (group & 1) || (K % group) || M < 0) return -1;
    if (n0 < 0 || n1 > N || n0 > n1) return -1;
    const int64_t G = K / group;
    const int64_t W = n1 - n0;
#pragma omp parallel for schedule(static)
    for (int64_t n = n0; n < n1; ++n) {
        const uint8_t *row = codes + n * (K / 2);
        for (int64_t t = 0; t < M; ++t) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
#ifdef ORACLE_MUTANT_GROUP_INDEX
                int64_t g = (k + ORACLE_BLOCK) / group;
                if (g >= G) g = G - 1;
#elif defined(ORACLE_MUTANT_GROUP_FIXED_256)
                int64_t g = k / ORACLE_GROUP;
#else
                int64_t g = k / group;
#endif
                double dd = f16_bits_to_double(d[n * G + g]);
                double mm = f16_bits_to_double(m[n * G + g]);
#ifdef ORACLE_MUTANT_DROP_MIN
                mm = 0.0;
#endif
                double wk = dd * (double)code_at(row, k) + mm;
                acc += wk * x[t * K + k];
            }
            y[t * W + (n - n0)] = acc;
        }
    }
    return 0;
}

int oracle_gemv_f64_rows(const uint8_t *codes, const uint16_t *d,
                         const uint16_t *m, int64_t N, int64_t K,
                         const double *x, int64_t M, int64_t n0, int64_t n1,
                         double *y) {
    return oracle_gemv_f64_rows_grouped(codes, d, m, N, K, ORACLE_GROUP, x, M, n0, n1, y);
}

int oracle_gemv_f64(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
                    int64_t N, int64_t K, const double *x, int64_t M,
                    double *y) {
    return oracle_gemv_f64_rows(codes, d, m, N, K, x, M, 0, N, y);
}

/* Same product with bf16 activations (bf16 bits [M][K]); the bf16 values are
 * widened exactly to fp64 first.  Rows [n0, n1). */
int oracle_gemv_rows_grouped(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
                             int64_t N, int64_t K, int64_t group, const uint16_t *x_bf16,
                             int64_t M, int64_t n0, int64_t n1, double *y) {
    if (M < 0 || K < 0) return -1;
    double *xd = (double *)malloc(sizeof(double) * (size_t)(M * K + 1));
    if (!xd) return -2;
    for (int64_t i = 0; i < M * K; ++i) xd[i] = bf16_bits_to_double(x_bf16[i]);
    int rc = oracle_gemv_f64_rows_grouped(codes, d, m, N, K, group, xd, M, n0, n1, y);
    free(xd);
    return rc;
}

int oracle_gemv_rows(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
                     int64_t N, int64_t K, const uint16_t *x_bf16, int64_t M,
                     int64_t n0, int64_t n1, double *y) {
    return oracle_gemv_rows_grouped(codes, d, m, N, K, ORACLE_GROUP, x_bf16, M, n0, n1, y);
}

int oracle_gemv(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
                int64_t N, int64_t K, const uint16_t *x_bf16, int64_t M,
                double *y) {
    return oracle_gemv_rows(codes, d, m, N, K, x_bf16, M, 0, N, y);
}

/* ------------------------------------------------------------------------ */
/* W4A8 product with int8 activation blocks                                 */
/* ------------------------------------------------------------------------ */

/* Exact integer block dot products:
 *   P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]      (int64)
 * P is int64 [M][N][K/32] (|P| <= 32*15*127, so it also fits int32). */
int oracle_mmq_blockdots(const uint8_t *codes, int64_t N, int64_t K,
                         const int8_t *qa, int64_t M, int64_t *P) {
    if (N < 0 || K < 0 || (K % ORACLE_BLOCK) || M < 0) return -1;
    const int64_t B = K / ORACLE_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t *row = codes + n * (K / 2);
        for (int64_t t = 0; t < M; ++t) {
            for (int64_t b = 0; b < B; ++b) {
                int64_t acc = 0;
                for (int64_t i = 0; i < ORACLE_BLOCK; ++i) {
                    int64_t k = b * ORACLE_BLOCK + i;
                    acc += (int64_t)code_at(row, k) * (int64_t)qa[t * K + k];
                }
                P[(t * N + n) * B + b] = acc;
            }
        }
    }
    return 0;
}

/* y[t][n] = sum_g sum_{b in g} dx[t][b] * ( d[n][g] * P[t][n][b]
 *                                            + m[n][g] * S[t][b] ),
 * the dequantised product with dequantised activations x' = dx * qa: the
 * integer block dot products P are exact, the min term uses the block sums S,
 * and the outer sums are fp64 in plain (g, b) order.  Rows [n0, n1); y holds
 * M x (n1 - n0) values. */
int oracle_mmq_rows(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
                    int64_t N, int64_t K, const int8_t *qa, const float *dx,
                    const int32_t *S, int64_t M, int64_t n0, int64_t n1,
                    double *y) {
    if (N < 0 || K < 0 || (K % ORACLE_GROUP) || M < 0) return -1;
    if (n0 < 0 || n1 > N || n0 > n1) return -1;
    const int64_t G = K / ORACLE_GROUP;
    const int64_t B = K / ORACLE_BLOCK;
    const int64_t BPG = ORACLE_GROUP / ORACLE_BLOCK;
    const int64_t W = n1 - n0;
#pragma omp parallel for schedule(static)
    for (int64_t n = n0; n < n1; ++n) {
        const uint8_t *row = codes + n * (K / 2);
        for (int64_t t = 0; t < M; ++t) {
            double acc = 0.0;
            for (int64_t g = 0; g < G; ++g) {
                double dd = f16_bits_to_double(d[n * G + g]);
                double mm = f16_bits_to_double(m[n * G + g]);
                for (int64_t bi = 0; bi < BPG; ++bi) {
                    int64_t b = g * BPG + bi;
                    int64_t p = 0;
                    for (int64_t i = 0; i < ORACLE_BLOCK; ++i) {
                        int64_t k = b * ORACLE_BLOCK + i;
                        p += (int64_t)code_at(row, k) * (int64_t)qa[t * K + k];
                    }
                    double s = (double)S[t * B + b];
#ifdef ORACLE_MUTANT_MMQ_DROP_BLOCKSUM
                    s = 0.0;
#endif
#ifdef ORACLE_MUTANT_MMQ_NEXT_BLOCK_SCALE
                    const int64_t bs = (bi + 1 < BPG) ? b + 1 : b;
#else
                    const int64_t bs = b;
#endif
                    acc += (double)dx[t * B + bs] * (dd * (double)p + mm * s);
                }
            }
            y[t * W + (n - n0)] = acc;
        }
    }
    return 0;
}

int oracle_mmq(const uint8_t *codes, const uint16_t *d, const uint16_t *m,
               int64_t N, int64_t K, const int8_t *qa, const float *dx,
               const int32_t *S, int64_t M, double *y) {
    return oracle_mmq_rows(codes, d, m, N, K, qa, dx, S, M, 0, N, y);
}

/*
 * Plain CPU oracle for the INT4 group-wise weight-only GEMM (W4A16).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call, link or load
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg use it. It shares no code with the CUDA library.
 *
 * What it computes (Int4GroupwiseGemmPluginV2 page, class description and
 * constructor parameters):
 *     C[m, n] = fp16_rne( sum_{k < K} A[m, k] * q[k, n] * s[floor(k / G), n] )
 * with A fp16 [M, K] row-major, q signed 4-bit codes in [-8, 7] stored two per
 * byte (low nibble = even k), s fp16 [ceil(K/G), N] row-major, C fp16 [M, N].
 * Every operand is widened exactly to double, the sum is taken in double in
 * increasing k, and the double result is rounded once, directly, to binary16
 * with round-to-nearest-even (no intermediate float, which could round twice).
 * The grouped-expert form (Int4MoePlugin page, constructor parameters) applies
 * the same formula to each expert's row segment [off[e], off[e+1]).
 *
 * Encodings defined here, each written from its stated definition:
 *   canonical packed layout  Wp [ceil(K/2), N] uint8, byte (j, n) =
 *       (q[2j, n] & 0xF) | (q[2j+1, n] & 0xF) << 4; a missing odd row packs 0.
 *   tiled layout (the library's weight operand): ceil(N/128) x ceil(K/64)
 *       tiles of 4096 bytes, tile (nt, kt) at byte ((nt * KT) + kt) * 4096.
 *       Inside a tile: half h in {0,1} covers k_local 32h..32h+31; column
 *       j in [0,128) owns 16 bytes at h*2048 + j*16; those 16 bytes are four
 *       little-endian 32-bit words, word w covering k_local 32h+8w+0..7, and
 *       nibble i (bits 4i..4i+3) of word w holds the code of
 *       k_local = 32h + 8w + NIBBLE_K[i], NIBBLE_K = {0,2,4,6,1,3,5,7}.
 *       Codes outside [0,K) x [0,N) are 0.
 *
 * Also the export step before the GEMM: group-wise symmetric int4 quantisation
 * of fp16 weights into codes and fp16 scales (oracle_quantize, at the end).
 *
 * Mutants (ORACLE_MUTANT=1..15) plant one plausible mistake each; they are only
 * compiled by the oracle's own tests to show that its pins catch them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* ---------------------------------------------------------------- binary16 */

/* IEEE 754 binary16 -> double, exact (every binary16 value is a double). */
double oracle_half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0x1F) {
        v = f ? NAN : INFINITY;
    } else if (e == 0) {
        v = ldexp((double)f, -24);            /* subnormal: f * 2^-24 */
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* double -> IEEE 754 binary16, round to nearest, ties to even, in one step. */
uint16_t oracle_double_to_half(double x) {
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7E00;
    if (isinf(x)) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);              /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;             /* a in [2^E, 2^(E+1)) */
    if (E < -14) {
        /* subnormal range: integer multiple of 2^-24 */
        double m = ldexp(a, 24);
#if ORACLE_MUTANT == 7
        double r = floor(m);
#else
        double r = nearbyint(m); /* exact scaled value; default mode rounds half to even */
#endif
        return sign | (uint16_t)r; /* r == 1024 lands on the smallest normal */
    }
    double m = ldexp(a, 10 - E); /* in [1024, 2048) */
#if ORACLE_MUTANT == 7
    double r = floor(m);
#else
    double r = nearbyint(m);
#endif
    if (r == 2048.0) { r = 1024.0; E += 1; }
    if (E > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((E + 15) << 10) | ((int)r - 1024));
}

/* ------------------------------------------------------------ int4 codes */

static inline int decode_nibble(unsigned v) {
    v &= 0xF;
#if ORACLE_MUTANT == 2
    return (int)v;                          /* forgets the sign */
#else
    return (v & 0x8) ? (int)v - 16 : (int)v; /* two's complement nibble */
#endif
}

/* q of row k, column n, read from the canonical packed layout. */
static inline int canonical_code(const uint8_t* wp, int64_t N, int64_t k, int64_t n) {
    uint8_t b = wp[(k >> 1) * N + n];
#if ORACLE_MUTANT == 1
    return decode_nibble((k & 1) ? b : (b >> 4)); /* nibbles swapped */
#else
    return decode_nibble((k & 1) ? (b >> 4) : b);
#endif
}

void oracle_pack(const int8_t* q, int64_t K, int64_t N, uint8_t* wp) {
    int64_t rows = (K + 1) / 2;
    for (int64_t j = 0; j < rows; ++j) {
        for (int64_t n = 0; n < N; ++n) {
            unsigned lo = (unsigned)(uint8_t)q[(2 * j) * N + n];
            unsigned hi = (2 * j + 1 < K) ? (unsigned)(uint8_t)q[(2 * j + 1) * N + n] : 0u;
#if ORACLE_MUTANT == 10
            wp[j * N + n] = (uint8_t)(lo | ((hi & 0xF) << 4)); /* low code not masked */
#else
            wp[j * N + n] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
#endif
        }
    }
}

void oracle_unpack(const uint8_t* wp, int64_t K, int64_t N, int8_t* q) {
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            q[k * N + n] = (int8_t)canonical_code(wp, N, k, n);
}

int64_t oracle_tiled_bytes(int64_t K, int64_t N) {
    return ((N + 127) / 128) * ((K + 63) / 64) * 4096;
}

/* Encode q [K, N] into the tiled layout described in the header comment. */
void oracle_tile(const int8_t* q, int64_t K, int64_t N, uint8_t* wt) {
#if ORACLE_MUTANT == 11
    static const int nibble_k[8] = {0, 1, 2, 3, 4, 5, 6, 7}; /* natural order */
#else
    static const int nibble_k[8] = {0, 2, 4, 6, 1, 3, 5, 7};
#endif
    int64_t NT = (N + 127) / 128, KT = (K + 63) / 64;
    memset(wt, 0, (size_t)(NT * KT * 4096));
    for (int64_t nt = 0; nt < NT; ++nt)
        for (int64_t kt = 0; kt < KT; ++kt) {
            uint8_t* tile = wt + (nt * KT + kt) * 4096;
            for (int h = 0; h < 2; ++h)
                for (int j = 0; j < 128; ++j)
                    for (int w = 0; w < 4; ++w) {
                        uint32_t word = 0;
                        for (int i = 0; i < 8; ++i) {
                            int64_t k = kt * 64 + 32 * h + 8 * w + nibble_k[i];
                            int64_t n = nt * 128 + j;
                            unsigned code = 0;
                            if (k < K && n < N) code = (unsigned)(uint8_t)q[k * N + n] & 0xF;
                            word |= (uint32_t)code << (4 * i);
                        }
                        uint8_t* p = tile + h * 2048 + j * 16 + w * 4;
                        p[0] = (uint8_t)word; p[1] = (uint8_t)(word >> 8);
                        p[2] = (uint8_t)(word >> 16); p[3] = (uint8_t)(word >> 24);
                    }
        }
}

/* --------------------------------------------------------------- the GEMM */

static inline int64_t scale_row(int64_t k, int64_t G) {
#if ORACLE_MUTANT == 3
    return (k + 1) / G;   /* off by one at group boundaries */
#else
    return k / G;
#endif
}

static inline double scale_at(const uint16_t* S, int64_t groups, int64_t N, int64_t g, int64_t n) {
#if ORACLE_MUTANT == 4
    return oracle_half_to_double(S[n * groups + g]); /* reads scales as [N, groups] */
#else
    (void)groups;
    return oracle_half_to_double(S[g * N + n]);
#endif
}

/* One output element; w_col holds the dequantised column n in double. */
static uint16_t dot_round(const double* a_row, const double* w_col, int64_t K) {
#if ORACLE_MUTANT == 5
    float acc = 0.0f;  /* single precision accumulator */
    for (int64_t k = 0; k < K; ++k) acc += (float)(a_row[k] * w_col[k]);
    return oracle_double_to_half((double)acc);
#else
    double acc = 0.0;
    for (int64_t k = 0; k < K; ++k) acc += a_row[k] * w_col[k];
#if ORACLE_MUTANT == 6
    return oracle_double_to_half((double)(float)acc); /* rounds twice */
#else
    return oracle_double_to_half(acc);
#endif
#endif
}

/* Dequantise column n: w[k] = q[k, n] * s[floor(k/G), n], exactly in double. */
static void dequant_column(const uint8_t* wp, const uint16_t* S, int64_t N, int64_t K,
                           int64_t G, int64_t n, double* w) {
    int64_t groups = (K + G - 1) / G;
    for (int64_t k = 0; k < K; ++k) {
        int64_t g = scale_row(k, G);
        if (g >= groups) g = groups - 1;
#if ORACLE_MUTANT == 8
        if (K % G && k >= (K / G) * G) { w[k] = 0.0; continue; } /* drops the last partial group */
#endif
        w[k] = (double)canonical_code(wp, N, k, n) * scale_at(S, groups, N, g, n);
    }
}

static double* widen_rows(const uint16_t* A, int64_t M, int64_t K) {
    double* a = (double*)malloc((size_t)(M * K) * sizeof(double));
    if (!a) return NULL;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k)
#if ORACLE_MUTANT == 9
            a[m * K + k] = oracle_half_to_double(A[k * M + m]); /* reads A as if it were [K, M] */
#else
            a[m * K + k] = oracle_half_to_double(A[m * K + k]);
#endif
    return a;
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* C[M, N] for A [M, K], canonical Wp, S [ceil(K/G), N]. nthreads <= 0: all. Returns 0 on success. */
int oracle_gemm(const uint16_t* A, const uint8_t* wp, const uint16_t* S, int64_t M, int64_t N,
                int64_t K, int64_t G, uint16_t* C, int nthreads) {
    if (M < 0 || N < 0 || K <= 0 || G <= 0) return 1;
    double* a = widen_rows(A, M, K);
    if (!a) return 2;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* w = (double*)malloc((size_t)K * sizeof(double));
        if (!w) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
            for (int64_t n = 0; n < N; ++n) {
                dequant_column(wp, S, N, K, G, n, w);
                for (int64_t m = 0; m < M; ++m) C[m * N + n] = dot_round(a + m * K, w, K);
            }
            free(w);
        }
    }
    free(a);
    return failed ? 2 : 0;
}

/* Only the listed (row, col) elements of the same product, one by one. */
int oracle_gemm_sample(const uint16_t* A, const uint8_t* wp, const uint16_t* S, int64_t M,
                       int64_t N, int64_t K, int64_t G, const int64_t* rows,
                       const int64_t* cols, int64_t count, uint16_t* out) {
    if (M <= 0 || N <= 0 || K <= 0 || G <= 0) return 1;
    double* w = (double*)malloc((size_t)K * sizeof(double));
    double* a = (double*)malloc((size_t)K * sizeof(double));
    if (!w || !a) { free(w); free(a); return 2; }
    for (int64_t i = 0; i < count; ++i) {
        int64_t m = rows[i], n = cols[i];
        if (m < 0 || m >= M || n < 0 || n >= N) { free(w); free(a); return 1; }
        dequant_column(wp, S, N, K, G, n, w);
        for (int64_t k = 0; k < K; ++k) a[k] = oracle_half_to_double(A[m * K + k]);
        out[i] = dot_round(a, w, K);
    }
    free(w); free(a);
    return 0;
}

/* Grouped-expert form: rows [off[e], off[e+1]) of A and C use expert e's
 * canonical weights wp[e] and scales S[e]. Rows of C outside every segment
 * are left untouched. Returns 1 if the offsets are not a valid segmentation. */
int oracle_grouped_gemm(const uint16_t* A, const uint8_t* const* wp, const uint16_t* const* S,
                        const int32_t* off, int64_t E, int64_t total_rows, int64_t N, int64_t K,
                        int64_t G, uint16_t* C, int nthreads) {
    if (E <= 0 || off[0] != 0 || off[E] != total_rows) return 1;
    for (int64_t e = 0; e < E; ++e) if (off[e + 1] < off[e]) return 1;
    for (int64_t e = 0; e < E; ++e) {
        int64_t r0 = off[e];
#if ORACLE_MUTANT == 12
        int64_t r1 = off[e + 1] > r0 ? off[e + 1] - 1 : r0; /* drops each segment's last row */
#else
        int64_t r1 = off[e + 1];
#endif
        if (r1 == r0) continue;
        int rc = oracle_gemm(A + r0 * K, wp[e], S[e], r1 - r0, N, K, G, C + r0 * N, nthreads);
        if (rc) return rc;
    }
    return 0;
}

/* ---------------------------------------------------- weight quantisation */

/*
 * Group-wise symmetric int4 quantisation of fp16 weights W [K, N] row-major:
 * the export step that produces the GEMM's codes and scales.
 *
 * The KV Cache INT8 quantization page (symmetric quantisation kernel) sets
 * scale = max|x| / 127 and x_q = round(x / scale) in float. Here the same rule
 * runs with the 4-bit code range (127 -> 7, the largest positive int4 code)
 * over each group of G rows of one column (Int4 Groupwise GEMM Plugin V2 page:
 * scales [ceil(K/G), N]), and the scale is stored in fp16 as the GEMM reads it:
 *   amax[g, n] = max over the rows k of group g of |W[k, n]|
 *   s[g, n]    = fp16_rne( float(amax) / 7.0f )            (IEEE float division)
 *   q[k, n]    = clamp( round(float(W[k, n]) / float(s[g, n])), -8, 7 ),
 *                q = 0 where s = 0
 * with round() rounding halves away from zero, as C's round does. The codes
 * are written in the canonical packed layout, the scales as fp16 bits.
 * W must be finite.
 */
void oracle_quantize(const uint16_t* W, int64_t K, int64_t N, int64_t G, uint8_t* wp, uint16_t* S) {
    const int64_t groups = (K + G - 1) / G;
    memset(wp, 0, (size_t)(((K + 1) / 2) * N));
    for (int64_t g = 0; g < groups; ++g) {
        const int64_t k0 = g * G;
        const int64_t k1 = k0 + G < K ? k0 + G : K;
        for (int64_t n = 0; n < N; ++n) {
            float amax = 0.0f;
#if ORACLE_MUTANT == 15
            for (int64_t k = 0; k < K; ++k) { /* the whole column instead of the group */
#else
            for (int64_t k = k0; k < k1; ++k) {
#endif
                float a = fabsf((float)oracle_half_to_double(W[k * N + n]));
                if (a > amax) amax = a;
            }
#if ORACLE_MUTANT == 13
            float s32 = amax / 8.0f; /* the int4 range taken as 8 */
#else
            float s32 = amax / 7.0f;
#endif
            uint16_t sh = oracle_double_to_half((double)s32); /* float -> double is exact */
            S[g * N + n] = sh;
            float s = (float)oracle_half_to_double(sh);
            for (int64_t k = k0; k < k1; ++k) {
                int q = 0;
                if (s != 0.0f) {
                    float x = (float)oracle_half_to_double(W[k * N + n]) / s;
#if ORACLE_MUTANT == 14
                    float r = nearbyintf(x); /* halves to even */
#else
                    float r = roundf(x);
#endif
                    q = (int)r;
                    if (q < -8) q = -8;
                    if (q > 7) q = 7;
                }
                unsigned nib = (unsigned)q & 0xF;
                wp[(k >> 1) * N + n] |= (uint8_t)((k & 1) ? nib << 4 : nib);
            }
        }
    }
}

/* ------------------------------------------------ W8A16 (8-bit codes) */

/*
 * The INT8 weight-only variant (the FP8-vs-INT8 TensorRT-LLM comparison page
 * lists INT8 weight-only with an FP16 KV cache among the INT8 configurations):
 * the same group-wise product with signed 8-bit codes in [-128, 127], one per
 * byte, q8 [K, N] row-major (two's complement):
 *     C[m, n] = fp16_rne( sum_{k < K} A[m, k] * q8[k, n] * s[floor(k / G), n] )
 * summed in double in increasing k and rounded once, as oracle_gemm.
 *
 * Tiled layout of 8-bit codes (the library's W8 weight operand):
 * ceil(N/128) x ceil(K/64) tiles of 8192 bytes, tile (nt, kt) at byte
 * ((nt * KT) + kt) * 8192. Inside a tile, quarter h in {0,1,2,3} covers
 * k_local 16h..16h+15; column j in [0,128) owns 16 bytes at h*2048 + j*16,
 * byte b holding the code of k_local = 16h + b. Codes outside [0,K) x [0,N)
 * are 0.
 */
static inline int code8(const int8_t* q8, int64_t N, int64_t k, int64_t n) {
#if ORACLE_MUTANT == 16
    return (int)(uint8_t)q8[k * N + n];  /* codes read as unsigned bytes */
#else
    return (int)q8[k * N + n];
#endif
}

int64_t oracle_tiled_bytes_w8(int64_t K, int64_t N) {
    return ((N + 127) / 128) * ((K + 63) / 64) * 8192;
}

void oracle_tile_w8(const int8_t* q8, int64_t K, int64_t N, uint8_t* wt) {
    int64_t NT = (N + 127) / 128, KT = (K + 63) / 64;
    memset(wt, 0, (size_t)(NT * KT * 8192));
    for (int64_t nt = 0; nt < NT; ++nt)
        for (int64_t kt = 0; kt < KT; ++kt) {
            uint8_t* tile = wt + (nt * KT + kt) * 8192;
            for (int h = 0; h < 4; ++h)
                for (int j = 0; j < 128; ++j)
                    for (int b = 0; b < 16; ++b) {
#if ORACLE_MUTANT == 17
                        int64_t k = kt * 64 + 16 * h + (15 - b); /* bytes in reverse order */
#else
                        int64_t k = kt * 64 + 16 * h + b;
#endif
                        int64_t n = nt * 128 + j;
                        if (k < K && n < N) tile[h * 2048 + j * 16 + b] = (uint8_t)q8[k * N + n];
                    }
        }
}

/* Dequantise column n of the 8-bit codes: w[k] = q8[k, n] * s[floor(k/G), n], exactly in double. */
static void dequant_column_w8(const int8_t* q8, const uint16_t* S, int64_t N, int64_t K, int64_t G,
                              int64_t n, double* w) {
    int64_t groups = (K + G - 1) / G;
    for (int64_t k = 0; k < K; ++k) {
        int64_t g = scale_row(k, G);
        if (g >= groups) g = groups - 1;
        w[k] = (double)code8(q8, N, k, n) * scale_at(S, groups, N, g, n);
    }
}

int oracle_gemm_w8(const uint16_t* A, const int8_t* q8, const uint16_t* S, int64_t M, int64_t N, int64_t K,
                   int64_t G, uint16_t* C, int nthreads) {
    if (M < 0 || N < 0 || K <= 0 || G <= 0) return 1;
    double* a = widen_rows(A, M, K);
    if (!a) return 2;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double* w = (double*)malloc((size_t)K * sizeof(double));
        if (!w) {
            failed = 1;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 16)
#endif
            for (int64_t n = 0; n < N; ++n) {
                dequant_column_w8(q8, S, N, K, G, n, w);
                for (int64_t m = 0; m < M; ++m) C[m * N + n] = dot_round(a + m * K, w, K);
            }
            free(w);
        }
    }
    free(a);
    return failed ? 2 : 0;
}

/*
 * Group-wise symmetric 8-bit quantisation of fp16 weights W [K, N] (the export
 * step of the W8A16 variant): the KV Cache INT8 quantization page's symmetric
 * rule (scale = max|x| / 127, x_q = round(x / scale), in float) over each group
 * of G rows of one column, the scale stored in fp16:
 *   s[g, n] = fp16_rne( float(amax) / 127.0f )
 *   q8[k, n] = clamp( round(float(W[k, n]) / float(s[g, n])), -128, 127 ),
 *              q8 = 0 where s = 0
 * round() takes halves away from zero. Codes are written one per byte, q8
 * [K, N] row-major; the scales as fp16 bits. W must be finite.
 */
void oracle_quantize_w8(const uint16_t* W, int64_t K, int64_t N, int64_t G, int8_t* q8, uint16_t* S) {
    const int64_t groups = (K + G - 1) / G;
    for (int64_t g = 0; g < groups; ++g) {
        const int64_t k0 = g * G;
        const int64_t k1 = k0 + G < K ? k0 + G : K;
        for (int64_t n = 0; n < N; ++n) {
            float amax = 0.0f;
            for (int64_t k = k0; k < k1; ++k) {
                float a = fabsf((float)oracle_half_to_double(W[k * N + n]));
                if (a > amax) amax = a;
            }
#if ORACLE_MUTANT == 18
            float s32 = amax / 128.0f; /* the 8-bit range taken as 128 */
#else
            float s32 = amax / 127.0f;
#endif
            uint16_t sh = oracle_double_to_half((double)s32);
            S[g * N + n] = sh;
            float s = (float)oracle_half_to_double(sh);
            for (int64_t k = k0; k < k1; ++k) {
                int q = 0;
                if (s != 0.0f) {
                    float x = (float)oracle_half_to_double(W[k * N + n]) / s;
#if ORACLE_MUTANT == 19
                    float r = nearbyintf(x); /* halves to even */
#else
                    float r = roundf(x);
#endif
                    q = (int)r;
                    if (q < -128) q = -128;
                    if (q > 127) q = 127;
                }
                q8[k * N + n] = (int8_t)q;
            }
        }
    }
}

/*
 * CPU ORACLE for the weight-only low-bit GEMM -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct fp64 reference used by the parity tests, by the
 * package's smoke check and by the benchmark's CPU-baseline leg. The product path
 * never loads, links or calls this file. It shares no code, header, table or
 * constant with the CUDA library: everything below is written from the definitions
 * stated in this comment.
 *
 * What it computes (Y = X * W^T, X [M][K], W [N][K], Y [M][N]):
 *
 *   ref[m][n] = sum_{k=0}^{K-1} x[m][k] * w[n][k]        accumulated in fp64, k ascending
 *
 * with each weight decoded from its code and its group's scale s (and zero z):
 *   bits 1 (binary): w = s * b, b in {-1,+1}. This is the rule "w_i = scale_g * b_i"
 *          of the bonsai-image-binary-4B-gemlite-1bit model card, section
 *          "Binary Weight Representation: 1-bit g128". Stored bit 1 means +1, 0 means -1.
 *   bits 2 (ternary): w = s * t, t in {-1,0,+1}. The pages name "ternary 2-bit"
 *          weights (mlx-vlm Bonsai article, model overview) but print no formula; the
 *          binary rule with t in place of b is the plainest reading. Stored field
 *          f = t + 1 (0, 1, 2); f == 3 is invalid.
 *   bits 4 (asymmetric uint4): w = (q - z) * s, q in 0..15, z in code units. The pages
 *          give only "bits=4, group_size=64" for the Qwen3 text encoder (mlx-vlm Bonsai
 *          article, component architecture) and "4-bit HQQ" (model card); the
 *          zero-point form is HQQ's affine reading.
 *
 * Groups: g consecutive K elements of one output row n share one scale ("one shared
 * FP16 scale per group of 128 weights", model card). Scales and zeros are fp16 and
 * stored group-major: s(n, k) = scales[(k / g) * N + n].
 *
 * Packed layout (codes packed along K, as the GemLite int2 layout note in
 * Bonsai-Image-Demo PR #20 describes, into uint32 words as the packed MLX checkpoint
 * of image-studio's backend.md stores them):
 *   cpw = 32 / bits codes per word; row n owns words [n * K/cpw, (n+1) * K/cpw).
 *   Offset i of a word (0 .. cpw-1) occupies bits [pos, pos + bits) with
 *   pos = (i % 2) * 16 + (i / 2) * bits: even offsets fill the low 16 bits, odd offsets
 *   the high 16 bits, each half LSB-first, so the offsets 2p and 2p + 1 form pair p.
 *   Which column an offset holds (the pages leave the order inside the packed words open):
 *   - plain order (every binary word, and the words of a 2- or 4-bit row after its last
 *     whole block of four): word j, offset i holds column cpw * j + i;
 *   - block order (2- and 4-bit rows, words taken in blocks of four, so a block spans
 *     4 * cpw columns: 32 for 4-bit, 64 for ternary): in word q (0..3) of block b, pair p
 *     holds columns 4 * cpw * b + 8 * p + 2 * q (low half) and that + 1 (high half).
 *
 * Inputs x are bf16, scales and zeros fp16; both are passed as raw bit patterns and
 * widened to fp64 exactly (IEEE 754 binary16 / bfloat16 definitions below).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_API __attribute__((visibility("default")))

/* Threads an OpenMP loop below will use for a request of `t` (<= 0: the default). */
ORACLE_API int oracle_threads(int t) {
#ifdef _OPENMP
    return t > 0 ? t : omp_get_max_threads();
#else
    (void)t;
    return 1;
#endif
}

/* ---- scalar formats ------------------------------------------------------------------- */

/* bfloat16 is the top half of an IEEE binary32 value. */
ORACLE_API double oracle_bf16_to_f64(uint16_t h) {
    uint32_t b = (uint32_t)h << 16;
    float f;
    memcpy(&f, &b, 4);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
ORACLE_API double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-10 * 2^-14 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp(1024.0 + (double)f, e - 25);      /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round an fp64 value to the nearest bfloat16, ties to even (informational output). */
ORACLE_API uint16_t oracle_f64_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    int sign = signbit(v) ? 1 : 0;
    double a = fabs(v);
    uint16_t s = (uint16_t)(sign << 15);
    if (a == 0.0) return s;
    int e;
    double m = frexp(a, &e);           /* a = m * 2^e, m in [0.5, 1) */
    int E = e - 1;                     /* a = (2m) * 2^E, 2m in [1, 2) */
    if (E < -126) E = -126;            /* subnormal range: fixed quantum 2^-133 */
    double q = ldexp(a, 7 - E);        /* a in units of the last place */
    double r = nearbyint(q);           /* default rounding mode: ties to even */
    double rv = ldexp(r, E - 7);
    if (rv >= ldexp(1.0, 128)) return (uint16_t)(s | 0x7F80);
    /* re-encode rv exactly as binary32, then take its top half (exact by construction) */
    float f = (float)rv;
    uint32_t b;
    memcpy(&b, &f, 4);
    return (uint16_t)(b >> 16) | s;
}

/* ---- packing -------------------------------------------------------------------------- */

static int code_field(int8_t c, int bits, uint32_t* field) {
    if (bits == 1) {
        if (c == 1) { *field = 1; return 0; }
        if (c == -1) { *field = 0; return 0; }
        return 1;
    }
    if (bits == 2) {
        if (c >= -1 && c <= 1) { *field = (uint32_t)(c + 1); return 0; }
        return 1;
    }
    if (bits == 4) {
        if (c >= 0 && c <= 15) { *field = (uint32_t)c; return 0; }
        return 1;
    }
    return 1;
}

static int valid_shape(int64_t N, int64_t K, int bits) {
    if (bits != 1 && bits != 2 && bits != 4) return 0;
    if (N < 0 || K < 0) return 0;
    return K % (32 / bits) == 0;
}

static int bit_pos(int64_t i, int bits) { return (int)((i % 2) * 16 + (i / 2) * bits); }

/* Column held at offset i of word j of a row of wpr words (the order rules above). */
static int64_t column_of(int64_t j, int64_t i, int64_t wpr, int bits) {
    int64_t cpw = 32 / bits;
    if (bits != 1 && j < wpr / 4 * 4) {
        int64_t b = j / 4, q = j % 4, p = i / 2, d = i % 2;
        return 4 * cpw * b + 8 * p + 2 * q + d;
    }
    return cpw * j + i;
}

/* Word j and offset i that hold column k of a row of K columns (the inverse of column_of). */
static void locate(int64_t k, int64_t K, int bits, int64_t* j, int64_t* i) {
    int64_t cpw = 32 / bits, span = 4 * cpw;
    if (bits != 1 && k < (K / cpw) / 4 * span) {
        int64_t b = k / span, r = k % span;
        *j = 4 * b + (r % 8) / 2;
        *i = 2 * (r / 8) + r % 2;
    } else {
        *j = k / cpw;
        *i = k % cpw;
    }
}

/* codes [N][K] int8 -> packed [N][K*bits/32] uint32. Returns the number of invalid
 * codes (their fields are written as 0), or -1 for an invalid shape. */
ORACLE_API int64_t oracle_pack(const int8_t* codes, int64_t N, int64_t K, int bits, uint32_t* packed) {
    if (!valid_shape(N, K, bits)) return -1;
    int64_t cpw = 32 / bits;
    int64_t words = K / cpw;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < words; ++j) {
            uint32_t w = 0;
            for (int64_t i = 0; i < cpw; ++i) {
                uint32_t field = 0;
                if (code_field(codes[n * K + column_of(j, i, words, bits)], bits, &field)) { bad++; field = 0; }
                w |= field << bit_pos(i, bits);
            }
            packed[n * words + j] = w;
        }
    }
    return bad;
}

/* The field of weight (n, k). */
static uint32_t field_at(const uint32_t* packed, int64_t K, int bits, int64_t n, int64_t k) {
    int64_t cpw = 32 / bits, j, i;
    locate(k, K, bits, &j, &i);
    uint32_t word = packed[n * (K / cpw) + j];
    return (word >> bit_pos(i, bits)) & ((1u << bits) - 1u);
}

/* packed -> codes. Returns the number of invalid fields (ternary f == 3, written as 0),
 * or -1 for an invalid shape. */
ORACLE_API int64_t oracle_unpack(const uint32_t* packed, int64_t N, int64_t K, int bits, int8_t* codes) {
    if (!valid_shape(N, K, bits)) return -1;
    int64_t bad = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            uint32_t f = field_at(packed, K, bits, n, k);
            int8_t c;
            if (bits == 1) c = f ? 1 : -1;
            else if (bits == 2) {
                if (f == 3) { bad++; c = 0; } else c = (int8_t)((int)f - 1);
            } else c = (int8_t)f;
            codes[n * K + k] = c;
        }
    }
    return bad;
}

/* ---- decode and GEMM ------------------------------------------------------------------ */

static double weight_at(const uint32_t* packed, const uint16_t* scales, const uint16_t* zeros,
                        int64_t N, int64_t K, int bits, int64_t g, int64_t n, int64_t k) {
    uint32_t f = field_at(packed, K, bits, n, k);
    double s = oracle_f16_to_f64(scales[(k / g) * N + n]);
    if (bits == 1) return f ? s : -s;
    if (bits == 2) {
        if (f == 3) return NAN;                       /* invalid code: poison the result */
        return s * (double)((int)f - 1);
    }
    double z = oracle_f16_to_f64(zeros[(k / g) * N + n]);
    return ((double)f - z) * s;
}

static int valid_problem(int64_t N, int64_t K, int bits, int64_t g, const uint16_t* zeros) {
    if (!valid_shape(N, K, bits)) return 0;
    if (g <= 0 || K % g != 0) return 0;
    if ((bits == 4) != (zeros != NULL)) return 0;
    return 1;
}

/* Dense fp64 weights W [N][K]. Returns 0, or -1 for invalid arguments. */
ORACLE_API int oracle_decode(const uint32_t* packed, const uint16_t* scales, const uint16_t* zeros,
                             int64_t N, int64_t K, int bits, int64_t g, double* W) {
    if (!valid_problem(N, K, bits, g, zeros)) return -1;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            W[n * K + k] = weight_at(packed, scales, zeros, N, K, bits, g, n, k);
    return 0;
}

/* ref [M][N] fp64 = X [M][K] (bf16 bits) times decoded W^T. Rows of X are split over
 * `threads` OpenMP threads (<= 0: the OpenMP default); each output keeps the plain
 * k-ascending fp64 sum. Returns 0, or -1 for invalid arguments / no memory. */
ORACLE_API int oracle_gemm(const uint16_t* X, int64_t M, int64_t K, const uint32_t* packed,
                           const uint16_t* scales, const uint16_t* zeros, int64_t N, int bits,
                           int64_t g, double* ref, int threads) {
    if (!valid_problem(N, K, bits, g, zeros) || M < 0) return -1;
    double* W = (double*)malloc(sizeof(double) * (size_t)(N * K > 0 ? N * K : 1));
    double* Xd = (double*)malloc(sizeof(double) * (size_t)(M * K > 0 ? M * K : 1));
    if (!W || !Xd) { free(W); free(Xd); return -1; }
    oracle_decode(packed, scales, zeros, N, K, bits, g, W);
    for (int64_t i = 0; i < M * K; ++i) Xd[i] = oracle_bf16_to_f64(X[i]);
    int nt = oracle_threads(threads);
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t m = 0; m < M; ++m) {
        const double* xr = Xd + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const double* wr = W + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += xr[k] * wr[k];
            ref[m * N + n] = acc;
        }
    }
    free(W);
    free(Xd);
    return 0;
}

/* The same sum for a list of (m, n) entries only, decoding each weight on the fly:
 * for checking sampled outputs of problems too large to compute whole. */
ORACLE_API int oracle_gemm_entries(const uint16_t* X, int64_t M, int64_t K, const uint32_t* packed,
                                   const uint16_t* scales, const uint16_t* zeros, int64_t N, int bits,
                                   int64_t g, const int64_t* ms, const int64_t* ns, int64_t count,
                                   double* out, int threads) {
    if (!valid_problem(N, K, bits, g, zeros) || M < 0) return -1;
    for (int64_t e = 0; e < count; ++e)
        if (ms[e] < 0 || ms[e] >= M || ns[e] < 0 || ns[e] >= N) return -1;
    int nt = oracle_threads(threads);
#pragma omp parallel for schedule(dynamic, 16) num_threads(nt)
    for (int64_t e = 0; e < count; ++e) {
        int64_t m = ms[e], n = ns[e];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += oracle_bf16_to_f64(X[m * K + k]) * weight_at(packed, scales, zeros, N, K, bits, g, n, k);
        out[e] = acc;
    }
    return 0;
}

/*
 * Seeded synthetic inputs for the low-bit GEMM: activations, weight codes,
 * group scales and zero points.
 *
 * This module holds no arithmetic of the method itself. It only draws random
 * numbers. It is shared by the parity tests, the oracle's callers and the
 * benchmark, so both sides of every comparison see the same bytes.
 *
 * Generator (counter based, so any element can be drawn independently):
 *   x      = seed * 0x9E3779B97F4A7C15 + stream * 0xD1B54A32D192ED03 + index   (mod 2^64)
 *   r(x)   = splitmix64 output function of x (Steele, Lea and Flood, "Fast
 *            splittable pseudorandom number generators", OOPSLA 2014):
 *              z = x + 0x9E3779B97F4A7C15
 *              z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *              z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *              r = z ^ (z >> 31)
 *   u      = (r >> 11) * 2^-53                       uniform on [0, 1)
 *   normal = Box-Muller: element i uses u1 = u(2i), u2 = u(2i+1),
 *            z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2)
 *   bf16   = round-to-nearest-even of (float)z   (double -> float is RNE in C)
 *   fp16   = (_Float16) of the double draw        (correctly rounded, RNE)
 *
 * Codes (int8, one per weight, row-major [N][K]):
 *   bits 1: +1 if u < 0.5 else -1
 *   bits 2: 0 if u < p0; +1 if u < p0 + (1-p0)/2; else -1
 *   bits 4: floor(16 u)  (0..15)
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_API __attribute__((visibility("default")))

static inline uint64_t synth_counter(uint64_t seed, uint64_t stream, uint64_t index) {
    return seed * 0x9E3779B97F4A7C15ULL + stream * 0xD1B54A32D192ED03ULL + index;
}

static inline uint64_t synth_splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline double synth_u01(uint64_t seed, uint64_t stream, uint64_t index) {
    return (double)(synth_splitmix64(synth_counter(seed, stream, index)) >> 11) * 0x1.0p-53;
}

static inline uint16_t synth_f32_to_bf16_rne(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

static inline uint16_t synth_f64_to_f16_rne(double d) {
    _Float16 h = (_Float16)d;
    uint16_t b;
    memcpy(&b, &h, 2);
    return b;
}

SYNTH_API uint64_t synth_raw_u64(uint64_t seed, uint64_t stream, uint64_t index) {
    return synth_splitmix64(synth_counter(seed, stream, index));
}

SYNTH_API void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = synth_u01(seed, stream, (uint64_t)i);
}

static inline double synth_normal_at(uint64_t seed, uint64_t stream, uint64_t i) {
    double u1 = synth_u01(seed, stream, 2 * i);
    double u2 = synth_u01(seed, stream, 2 * i + 1);
    return sqrt(-2.0 * log(1.0 - u1)) * cos(6.283185307179586476925286766559 * u2);
}

SYNTH_API void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = synth_normal_at(seed, stream, (uint64_t)i);
}

/* N(0,1) draws rounded to bf16 (raw bit patterns). */
SYNTH_API void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = synth_f32_to_bf16_rne((float)synth_normal_at(seed, stream, (uint64_t)i));
}

/* U[lo, hi) draws rounded to fp16 (raw bit patterns). */
SYNTH_API void synth_uniform_f16(uint64_t seed, uint64_t stream, uint64_t n, double lo, double hi,
                                 uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = synth_f64_to_f16_rne(lo + (hi - lo) * synth_u01(seed, stream, (uint64_t)i));
}

/* Weight codes as documented in the file header. p0 is used for bits == 2 only. */
SYNTH_API int synth_codes(uint64_t seed, uint64_t stream, uint64_t n, int bits, double p0, int8_t* out) {
    if (bits != 1 && bits != 2 && bits != 4) return -1;
    double p_plus = p0 + 0.5 * (1.0 - p0);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) {
        double u = synth_u01(seed, stream, (uint64_t)i);
        int8_t c;
        if (bits == 1) {
            c = (u < 0.5) ? 1 : -1;
        } else if (bits == 2) {
            c = (u < p0) ? 0 : ((u < p_plus) ? 1 : -1);
        } else {
            int q = (int)(u * 16.0);
            c = (int8_t)(q > 15 ? 15 : q);
        }
        out[i] = c;
    }
    return 0;
}

/*
 * synth.c -- seeded synthetic inputs for the sparse latent-MoE decode layer step.
 *
 * This module draws random numbers and nothing else: it holds none of the layer's
 * arithmetic (no decode, no GEMV, no routing).  Both the CPU oracle's tests and the
 * CUDA path's tests/bench take their inputs from here, so the two see identical bytes.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014).  A stream is named by (seed, layer, tensor id); draw i of a
 * stream is the (i+1)-th SplitMix64 output started from the stream key, so any element
 * can be regenerated on its own (counter-based).
 *
 *   key(seed, layer, tensor) = mix(mix(mix(seed + G) ^ (layer + G)) ^ (tensor + G))
 *   draw(key, i)             = mix(key + (i + 1) * G),   G = 0x9E3779B97F4A7C15
 *
 * Distributions (the five workloads of the Kimi-K3-shaped layer):
 *   uniform bytes  byte j of a stream = byte (j mod 8) (little-endian) of draw(key, j/8);
 *                  packed FP4 codes are such bytes, so each 4-bit code is uniform.
 *   E8M0 scales    byte j = lo + draw(key, j) mod count  (scale exponent uniform in a range).
 *   normals        z_i = sqrt(-2 ln u1) cos(2 pi u2) in double (Box-Muller, cosine branch),
 *                  u1 = ((draw(key,2i) >> 11) + 1) 2^-53 in (0,1],
 *                  u2 =  (draw(key,2i+1) >> 11) 2^-53 in [0,1);
 *                  a bf16 value is bf16_rne(float_rne(sigma * z)).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC synth.c -o libsynth.so -lm
 * Every loop is data-parallel over independent counters, so results do not depend on
 * the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t layer, uint64_t tensor) {
    return mix64(mix64(mix64(seed + SYNTH_G) ^ (layer + SYNTH_G)) ^ (tensor + SYNTH_G));
}

uint64_t synth_draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * SYNTH_G); }

double synth_normal(uint64_t key, uint64_t i) {
    uint64_t d1 = synth_draw(key, 2 * i), d2 = synth_draw(key, 2 * i + 1);
    double u1 = (double)((d1 >> 11) + 1) * 0x1.0p-53;
    double u2 = (double)(d2 >> 11) * 0x1.0p-53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* float -> bf16 bits, round to nearest even (NaN kept quiet). */
static inline uint16_t bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

uint16_t synth_bf16_from_double(double v) { return bf16_rne((float)v); }

/* out[j] = byte of stream `key` at position start + j, j < n. */
void synth_bytes(uint64_t key, uint64_t start, uint64_t n, uint8_t *out) {
    if (n == 0) return;
    uint64_t end = start + n;
    uint64_t w0 = start >> 3, w1 = (end + 7) >> 3;
#pragma omp parallel for schedule(static)
    for (int64_t w = (int64_t)w0; w < (int64_t)w1; ++w) {
        uint64_t d = synth_draw(key, (uint64_t)w);
        for (int b = 0; b < 8; ++b) {
            uint64_t pos = ((uint64_t)w << 3) + (uint64_t)b;
            if (pos >= start && pos < end) out[pos - start] = (uint8_t)(d >> (8 * b));
        }
    }
}

/* out[j] = lo + draw(key, start + j) mod count. */
void synth_scales(uint64_t key, uint64_t start, uint64_t n, uint32_t lo, uint32_t count,
                  uint8_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j)
        out[j] = (uint8_t)(lo + synth_draw(key, start + (uint64_t)j) % count);
}

/* out[j] = bf16(sigma * z_{start+j}). */
void synth_normal_bf16(uint64_t key, uint64_t start, uint64_t n, double sigma, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j)
        out[j] = synth_bf16_from_double(sigma * synth_normal(key, start + (uint64_t)j));
}

/* out[j] = sigma * z_{start+j} in double (used for the router's hot-row bias vector). */
void synth_normal_f64(uint64_t key, uint64_t start, uint64_t n, double sigma, double *out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j) out[j] = sigma * synth_normal(key, start + (uint64_t)j);
}

/*
 * Router rows with a hot set: row e, column j is
 *   bf16(sigma * z_{e*cols+j} + (hot[e] ? beta * bias[j] : 0))
 * where z comes from `key` and bias is a caller-supplied double vector of length cols.
 * With beta = 0 (or no hot rows) this equals synth_normal_bf16 over the whole matrix.
 */
void synth_router_rows(uint64_t key, uint64_t rows, uint64_t cols, double sigma,
                       const uint8_t *hot, double beta, const double *bias, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)rows; ++r) {
        for (uint64_t j = 0; j < cols; ++j) {
            uint64_t i = (uint64_t)r * cols + j;
            double v = sigma * synth_normal(key, i);
            if (hot && hot[r]) v += beta * bias[j];
            out[i] = synth_bf16_from_double(v);
        }
    }
}

/*
 * Second token of the B=2 workload: out[j] = bf16(x0[j] + eps * z_j), x0 given as bf16 bits.
 */
void synth_perturb_bf16(uint64_t key, uint64_t n, const uint16_t *x0, double eps, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < (int64_t)n; ++j) {
        uint32_t u = (uint32_t)x0[j] << 16;
        float f;
        memcpy(&f, &u, 4);
        out[j] = synth_bf16_from_double((double)f + eps * synth_normal(key, (uint64_t)j));
    }
}

/*
 * `count` distinct indices from [0, n) drawn without replacement (partial Fisher-Yates
 * over the identity permutation, swap partner draw(key, i) mod (n - i)).  perm is caller
 * scratch of length n; the chosen indices are perm[0..count).
 */
void synth_choose(uint64_t key, uint32_t n, uint32_t count, uint32_t *perm) {
    for (uint32_t i = 0; i < n; ++i) perm[i] = i;
    for (uint32_t i = 0; i < count && i < n; ++i) {
        uint32_t j = i + (uint32_t)(synth_draw(key, i) % (uint64_t)(n - i));
        uint32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
    }
}

/*
 * synth_host.c -- seeded synthetic inputs, host implementation.
 *
 * This module holds none of the MoE method's arithmetic: it only turns
 * (seed, layer, tensor id, element index) into reproducible F32 numbers.  The
 * CUDA twin (synth_dev.cu) implements the same definition separately, so
 * device-resident weights of any size can be made on the GPU while the oracle
 * regenerates any row it needs on the host.
 *
 * Definition (all integer arithmetic modulo 2^64):
 *   mix64(z): the SplitMix64 output function (G. L. Steele, D. Lea,
 *     C. H. Flood, "Fast splittable pseudorandom number generators",
 *     OOPSLA 2014):  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                    z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31.
 *   G = 0x9E3779B97F4A7C15 (the SplitMix64 increment).
 *   key(seed, layer, tid) = mix64(mix64(seed + G) ^ ((layer << 32) | tid)).
 *   draw(key, c) = mix64(key + (c + 1) * G)  -- the (c+1)-th SplitMix64
 *     output of a generator started at state key.
 *   uniform element i in [a, b):
 *     u = draw(key, i) >> 40  (24 bits);  t = (float)u * 2^-24  (exact);
 *     value = a + (b - a) * t, three binary32 operations, round to nearest.
 *   normal element i, N(0, sigma), Irwin-Hall sum of 12 uniforms:
 *     for j in 0..5: z = draw(key, 6*i + j); S += (z >> 40) + ((z >> 16) & 0xFFFFFF)
 *     n = (float)(int32)(S - 6 * 2^24) * 2^-24   (one rounding in the int->float)
 *     value = sigma * n                         (one binary32 multiply)
 */
#include <stdint.h>

#define SYN_API __attribute__((visibility("default")))

static const uint64_t SYN_G = 0x9E3779B97F4A7C15ull;

static inline uint64_t syn_mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    z ^= z >> 31;
    return z;
}

SYN_API uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t tid) {
    return syn_mix64(syn_mix64(seed + SYN_G) ^ (((uint64_t)layer << 32) | (uint64_t)tid));
}

static inline uint64_t syn_draw(uint64_t key, uint64_t c) { return syn_mix64(key + (c + 1) * SYN_G); }

SYN_API uint64_t synth_draw(uint64_t key, uint64_t c) { return syn_draw(key, c); }

static inline float syn_normal_at(uint64_t key, uint64_t i, float sigma) {
    uint32_t s = 0;
    for (int j = 0; j < 6; ++j) {
        uint64_t z = syn_draw(key, 6 * i + (uint64_t)j);
        s += (uint32_t)(z >> 40) + (uint32_t)((z >> 16) & 0xFFFFFFu);
    }
    float n = (float)((int32_t)s - (int32_t)(6u << 24)) * 0x1p-24f;
    return sigma * n;
}

static inline float syn_uniform_at(uint64_t key, uint64_t i, float a, float b) {
    uint32_t u = (uint32_t)(syn_draw(key, i) >> 40);
    float t = (float)u * 0x1p-24f;
    float range = b - a;
    float scaled = range * t;
    return a + scaled;
}

/* out[j] = normal element (i0 + j), j < n. */
SYN_API void synth_normal(float* out, int64_t n, uint64_t i0, uint64_t key, float sigma) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = syn_normal_at(key, i0 + (uint64_t)j, sigma);
}

/* out[j] = uniform element (i0 + j) in [a, b), j < n. */
SYN_API void synth_uniform(float* out, int64_t n, uint64_t i0, uint64_t key, float a, float b) {
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) out[j] = syn_uniform_at(key, i0 + (uint64_t)j, a, b);
}

/* Rows of a [rows_total x cols] normal matrix: out gets rows r[0..nr). */
SYN_API void synth_normal_rows(float* out, const int64_t* rows, int64_t nr, int64_t cols,
                               uint64_t key, float sigma) {
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < nr; ++k)
        for (int64_t c = 0; c < cols; ++c)
            out[k * cols + c] = syn_normal_at(key, (uint64_t)(rows[k] * cols + c), sigma);
}

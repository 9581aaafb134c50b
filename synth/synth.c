/*
 * synth.c - seeded, counter-based synthetic input generator.
 *
 * This module draws the random inputs (weights, activations, adapter ids,
 * logit offsets) that both the fp64 oracle and the CUDA library consume.  It
 * holds none of the quantisation or MoE arithmetic; it only produces numbers.
 *
 * Generator: SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used in counter mode: the value at index i
 * of stream `key` is mix64(key + (i + 1) * 0x9E3779B97F4A7C15).  Normals come
 * from the Box-Muller transform in fp64 (Box & Muller 1958), one pair per two
 * counters.  Every element depends only on (key, index), so the result is the
 * same for any thread count.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t counter_draw(uint64_t key, uint64_t i) {
    return mix64(key + (i + 1ULL) * GOLDEN);
}

/* Stream key for a named tensor: FNV-1a 64 of the name, folded with the seed. */
uint64_t synth_stream_key(uint64_t seed, const char* name) {
    uint64_t h = 0xCBF29CE484222325ULL;
    for (const unsigned char* p = (const unsigned char*)name; *p; ++p) {
        h ^= (uint64_t)*p;
        h *= 0x100000001B3ULL;
    }
    return mix64(h ^ mix64(seed + GOLDEN));
}

/* Uniform doubles in [0, 1) with 53 random bits. */
void synth_uniform_f64(uint64_t key, int64_t n, double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (double)(counter_draw(key, (uint64_t)i) >> 11) * 0x1.0p-53;
}

/* Normal(mean, std) rounded to fp32. */
void synth_normal_f32(uint64_t key, int64_t n, double mean, double stddev, float* out) {
    const double two_pi = 6.283185307179586476925286766559;
    int64_t pairs = (n + 1) / 2;
    #pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < pairs; ++p) {
        uint64_t a = counter_draw(key, 2ULL * (uint64_t)p);
        uint64_t b = counter_draw(key, 2ULL * (uint64_t)p + 1ULL);
        double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53; /* (0, 1] */
        double u2 = (double)(b >> 11) * 0x1.0p-53;          /* [0, 1) */
        double r = sqrt(-2.0 * log(u1));
        double t = two_pi * u2;
        out[2 * p] = (float)(mean + stddev * r * cos(t));
        if (2 * p + 1 < n) out[2 * p + 1] = (float)(mean + stddev * r * sin(t));
    }
}

/* Multiply each element by `factor` independently with probability `prob`. */
void synth_outliers_f32(uint64_t key, int64_t n, double prob, double factor, float* data) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double u = (double)(counter_draw(key, (uint64_t)i) >> 11) * 0x1.0p-53;
        if (u < prob) data[i] = (float)((double)data[i] * factor);
    }
}

/* Uniform integers in [lo, hi]. */
void synth_uniform_int(uint64_t key, int64_t n, int32_t lo, int32_t hi, int32_t* out) {
    double span = (double)hi - (double)lo + 1.0;
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double u = (double)(counter_draw(key, (uint64_t)i) >> 11) * 0x1.0p-53;
        int64_t v = (int64_t)lo + (int64_t)floor(u * span);
        if (v > hi) v = hi;
        out[i] = (int32_t)v;
    }
}

/* fp32 -> bf16 bit pattern, round to nearest even (finite inputs). */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint32_t u;
        memcpy(&u, &in[i], 4);
        uint32_t lsb = (u >> 16) & 1u;
        u += 0x7FFFu + lsb;
        out[i] = (uint16_t)(u >> 16);
    }
}

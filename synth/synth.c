/*
 * Seeded synthetic inputs shared by the tests, the benchmark and smoke().
 *
 * This module draws random numbers and nothing else: it holds none of the
 * arithmetic of the tree-ordered kernels (no GEMM, no tree, no norm, no exp
 * of the method).  Both the CUDA path and the CPU oracle consume the bytes it
 * writes, so that both sides always see identical inputs.
 *
 * Generator (all counter based, so the output does not depend on the thread
 * count):
 *   - SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014): the i-th output of a stream seeded with s is
 *     mix(s + (i+1) * 0x9e3779b97f4a7c15).
 *   - uniform in (0,1]: ((x >> 11) + 1) * 2^-53.
 *   - standard normals by Box-Muller on consecutive pairs of uniforms
 *     (u1 = U(2p), u2 = U(2p+1)): element 2p gets r*cos(2*pi*u2), element
 *     2p+1 gets r*sin(2*pi*u2), r = sqrt(-2 ln u1), all in binary64.
 *   - bf16 values: mean + std*z rounded to binary32 and then to bfloat16 with
 *     round-to-nearest-even.
 *   - integers in [lo, hi): lo + (x >> 11) % (hi - lo).
 *   - permutations: Fisher-Yates, the draw for position i (from n-1 down to 1)
 *     being output number n-1-i of the stream.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SM64_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/* i-th output (0-based) of the SplitMix64 stream seeded with `seed`. */
static inline uint64_t sm64_at(uint64_t seed, uint64_t i) {
    return sm64_mix(seed + (i + 1) * SM64_GAMMA);
}

static inline double unit_open0(uint64_t x) {
    return (double)((x >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t seed, uint64_t i) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t p = i >> 1;
    double u1 = unit_open0(sm64_at(seed, 2 * p));
    double u2 = unit_open0(sm64_at(seed, 2 * p + 1));
    double r = sqrt(-2.0 * log(u1));
    return (i & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

static inline uint16_t to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

uint64_t synth_splitmix64(uint64_t seed, uint64_t i) { return sm64_at(seed, i); }

void synth_normal_f64(uint64_t seed, uint64_t offset, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = normal_at(seed, offset + (uint64_t)i);
}

void synth_normal_bf16(uint64_t seed, uint64_t offset, int64_t n, double mean, double std,
                       uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        double v = mean + std * normal_at(seed, offset + (uint64_t)i);
        out[i] = to_bf16_rne((float)v);
    }
}

void synth_normal_f32(uint64_t seed, uint64_t offset, int64_t n, double mean, double std,
                      float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(mean + std * normal_at(seed, offset + (uint64_t)i));
}

/* bf16 integers drawn uniformly from [-amp, amp] (used for exactness checks). */
void synth_int_bf16(uint64_t seed, uint64_t offset, int64_t n, int amp, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t x = sm64_at(seed, offset + (uint64_t)i);
        int v = (int)((x >> 11) % (uint64_t)(2 * amp + 1)) - amp;
        out[i] = to_bf16_rne((float)v);
    }
}

void synth_uniform_int32(uint64_t seed, uint64_t offset, int64_t n, int64_t lo, int64_t hi,
                         int32_t* out) {
    uint64_t span = (uint64_t)(hi - lo);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        uint64_t x = sm64_at(seed, offset + (uint64_t)i);
        out[i] = (int32_t)(lo + (int64_t)((x >> 11) % span));
    }
}

void synth_permutation(uint64_t seed, int64_t n, int32_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (int32_t)i;
    for (int64_t i = n - 1; i >= 1; --i) {
        uint64_t x = sm64_at(seed, (uint64_t)(n - 1 - i));
        int64_t j = (int64_t)((x >> 11) % (uint64_t)(i + 1));
        int32_t t = out[i];
        out[i] = out[j];
        out[j] = t;
    }
}

/*
 * Seeded synthetic inputs for the MoE layer: a counter-based generator.
 *
 * This file holds no arithmetic of the MoE method.  It only turns (seed,
 * stream, element index) into numbers, so that the CUDA path and the CPU
 * oracle read the very same input bytes.
 *
 * Generator (published definitions, restated):
 *   - splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014; the constants of Vigna's public-domain
 *     splitmix64): output n of the sequence started at state s is
 *     mix(s + (n + 1) * 0x9E3779B97F4A7C15).
 *   - Box-Muller (Box & Muller 1958): two uniforms u1 in (0,1], u2 in [0,1)
 *     give z0 = r cos(2 pi u2), z1 = r sin(2 pi u2), r = sqrt(-2 ln u1).
 *
 * Stream key of (seed, stream) = output number `stream` of splitmix64
 * started at `seed`.  Element 2p of a stream is z0 of pair p and element
 * 2p+1 is z1, where pair p draws its uniforms from outputs 2p and 2p+1 of
 * splitmix64 started at the stream key.  Every element is thus a pure
 * function of (seed, stream, index): any subset can be regenerated alone.
 *
 * Values are formed in double, scaled by the standard deviation, rounded to
 * float (round to nearest even) and, for bf16 outputs, rounded again from
 * float to bfloat16 (round to nearest even on the bit pattern).
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

static inline uint64_t splitmix_at(uint64_t state, uint64_t n) {
    return mix64(state + (n + 1) * GOLDEN);
}

uint64_t moe_gen_stream_key(uint64_t seed, uint64_t stream) {
    return splitmix_at(seed, stream);
}

uint64_t moe_gen_u64(uint64_t seed, uint64_t stream, uint64_t n) {
    return splitmix_at(moe_gen_stream_key(seed, stream), n);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t p = i >> 1;
    uint64_t b1 = splitmix_at(key, 2 * p);
    uint64_t b2 = splitmix_at(key, 2 * p + 1);
    double u1 = (double)((b1 >> 11) + 1) * 0x1.0p-53; /* (0, 1] */
    double u2 = (double)(b2 >> 11) * 0x1.0p-53;       /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    return (i & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) /* inf / nan: keep, quiet nan */
        return (uint16_t)((u >> 16) | ((u & 0x007FFFFFu) ? 0x40u : 0u));
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* out[i] = float(std * z_i) for i in [first, first + n). */
void moe_gen_normal_f32(uint64_t seed, uint64_t stream, uint64_t first, int64_t n,
                        double std, float* out) {
    uint64_t key = moe_gen_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = (float)(std * normal_at(key, first + (uint64_t)i));
}

/* out[i] = bf16(float(std * z_i)), as raw bfloat16 bit patterns. */
void moe_gen_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, int64_t n,
                         double std, uint16_t* out) {
    uint64_t key = moe_gen_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16_rne((float)(std * normal_at(key, first + (uint64_t)i)));
}

/* Uniform random permutation of 0..n-1 (Fisher-Yates, Durstenfeld form);
 * draw number d picks j = floor(u64 * (i + 1) / 2^64) for i = n-1 .. 1. */
void moe_gen_permutation(uint64_t seed, uint64_t stream, int32_t n, int32_t* out) {
    uint64_t key = moe_gen_stream_key(seed, stream);
    for (int32_t i = 0; i < n; ++i) out[i] = i;
    uint64_t d = 0;
    for (int32_t i = n - 1; i >= 1; --i, ++d) {
        unsigned __int128 m = (unsigned __int128)splitmix_at(key, d) * (uint64_t)(i + 1);
        int32_t j = (int32_t)(m >> 64);
        int32_t t = out[i];
        out[i] = out[j];
        out[j] = t;
    }
}

/* out[i] = byte ((first + i) mod 8) of splitmix64 output (first + i) / 8 of
 * the stream (least significant byte first): uniform random bytes, each a
 * pure function of (seed, stream, index). */
void moe_gen_bytes(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, uint8_t* out) {
    uint64_t key = moe_gen_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        const uint64_t j = first + (uint64_t)i;
        out[i] = (uint8_t)(splitmix_at(key, j >> 3) >> (8 * (j & 7)));
    }
}

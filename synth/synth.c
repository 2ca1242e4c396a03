/*
 * synth.c -- seeded synthetic inputs for the decode workloads.
 *
 * This module draws the random bf16 weights, the pre-filled bf16 KV cache
 * and the random prompt tokens.  It is shared by the fp64 oracle side and the
 * CUDA side so that both see the identical bf16 bytes; it holds none of the
 * decoder's arithmetic (no norm, projection, rotation, attention or routing).
 *
 * Generator: a counter-based stream.  Each tensor has a 64-bit key derived
 * from (seed, FNV-1a-64 of the tensor's name); element pair i draws one
 * SplitMix64 output (Steele, Lea & Flood, "Fast splittable pseudorandom number
 * generators", OOPSLA 2014) of key + i, whose two 24-bit halves become two
 * uniforms in (0,1) and then two N(0,1) draws by the Box-Muller transform
 * (Box & Muller, 1958).  Each draw is scaled by sigma, rounded to fp32 and
 * then to bf16 with round-to-nearest-even.  Because element i depends only on
 * (seed, name, i), the result is independent of thread count and of how the
 * tensor is split.
 */
#include <math.h>
#include <stdio.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t splitmix64(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static uint64_t fnv1a64(const char *s) {
    uint64_t h = 0xCBF29CE484222325ull;
    for (; *s; ++s) {
        h ^= (unsigned char)*s;
        h *= 0x100000001B3ull;
    }
    return h;
}

uint64_t synth_stream_key(uint64_t seed, const char *name) {
    return splitmix64(seed ^ splitmix64(fnv1a64(name)));
}

/* fp32 -> bf16 bit pattern, round to nearest, ties to even (NaN kept quiet). */
uint16_t synth_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* n bf16 draws of N(0, sigma^2) for tensor `name`, written to out[0..n). */
void synth_normal_bf16(uint16_t *out, int64_t n, uint64_t seed, const char *name, float sigma) {
    const uint64_t key = synth_stream_key(seed, name);
    const int64_t pairs = (n + 1) / 2;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < pairs; ++i) {
        const uint64_t r = splitmix64(key + (uint64_t)i);
        const double u1 = ((double)(r >> 40) + 0.5) * (1.0 / 16777216.0);
        const double u2 = ((double)(r & 0xFFFFFFull) + 0.5) * (1.0 / 16777216.0);
        const double rad = sqrt(-2.0 * log(u1));
        const double ang = 6.283185307179586476925 * u2;
        out[2 * i] = synth_f32_to_bf16((float)((double)sigma * rad * cos(ang)));
        if (2 * i + 1 < n) out[2 * i + 1] = synth_f32_to_bf16((float)((double)sigma * rad * sin(ang)));
    }
}

/* n bf16 copies of `value` (e.g. RMSNorm weights of 1.0). */
void synth_const_bf16(uint16_t *out, int64_t n, float value) {
    const uint16_t b = synth_f32_to_bf16(value);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = b;
}

/* n token ids uniform in [0, vocab) for stream `name` (multiply-shift of the
 * high 32 bits; bias below 2^-32 * vocab). */
void synth_tokens(int32_t *out, int64_t n, uint64_t seed, const char *name, int32_t vocab) {
    const uint64_t key = synth_stream_key(seed, name);
    for (int64_t i = 0; i < n; ++i) {
        const uint64_t r = splitmix64(key + (uint64_t)i);
        out[i] = (int32_t)(((r >> 32) * (uint64_t)(uint32_t)vocab) >> 32);
    }
}

/* Pre-filled KV cache region: for each (layer, kv head) the first `filled`
 * positions of a [L][nkv][max_seq][d] bf16 tensor get N(0, sigma^2) draws from
 * stream "<prefix>.<layer>.<head>"; the remaining positions are set to zero.
 * The drawn values do not depend on max_seq. */
void synth_kv_prefill(uint16_t *cache, int n_layers, int n_kv, int max_seq, int d, int filled,
                      uint64_t seed, const char *prefix, float sigma) {
    char name[128];
    for (int l = 0; l < n_layers; ++l) {
        for (int g = 0; g < n_kv; ++g) {
            uint16_t *base = cache + ((int64_t)l * n_kv + g) * (int64_t)max_seq * d;
            snprintf(name, sizeof name, "%s.%d.%d", prefix, l, g);
            if (filled > 0) synth_normal_bf16(base, (int64_t)filled * d, seed, name, sigma);
            memset(base + (int64_t)filled * d, 0, sizeof(uint16_t) * (size_t)(max_seq - filled) * (size_t)d);
        }
    }
}

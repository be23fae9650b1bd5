/*
 * Seeded synthetic inputs for the MoGE layer: normal-distributed tensors,
 * produced on the host, rounded once to the storage type, and handed to
 * BOTH the CPU oracle and the CUDA path (the same bytes go to each side).
 *
 * This file holds no arithmetic of the method itself; it only draws numbers.
 *
 * Generator definition (counter-based, so any slice can be produced alone and
 * the result does not depend on the number of threads):
 *   key      = mix64(seed * 0x9E3779B97F4A7C15 + stream)
 *   u(c)     = ((mix64(key + c) >> 11) + 0.5) * 2^-53         in (0, 1)
 *   pair j   : u1 = u(2j), u2 = u(2j+1)
 *              r  = sqrt(-2 ln u1)
 *              n[2j]   = r cos(2 pi u2)
 *              n[2j+1] = r sin(2 pi u2)                          (Box-Muller)
 *   value[i] = (float)(std * n[i])          then, for bf16 storage,
 *   bf16[i]  = round-to-nearest-even of value[i] to 8 significand bits.
 * mix64 is the SplitMix64 output finaliser (Steele, Lea, Flood 2014).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static inline uint64_t mix64(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

static inline double unit_open(uint64_t key, uint64_t c) {
    return ((double)(mix64(key + c) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * 0x9E3779B97F4A7C15ull + stream);
}

/* normal value number i of the stream, as float (std applied) */
static inline float normal_at(uint64_t key, uint64_t i, double stdv) {
    uint64_t j = i >> 1;
    double u1 = unit_open(key, 2 * j);
    double u2 = unit_open(key, 2 * j + 1);
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    double n = (i & 1) ? r * sin(a) : r * cos(a);
    return (float)(stdv * n);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t b;
    memcpy(&b, &f, 4);
    if ((b & 0x7F800000u) == 0x7F800000u) /* inf / nan: keep, quiet nan */
        return (uint16_t)((b >> 16) | ((b & 0x007FFFFFu) ? 0x40u : 0u));
    uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

/* Fill out[0..n) with elements [first, first+n) of stream (seed, stream). */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                      double stdv, float *out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = normal_at(key, first + (uint64_t)i, stdv);
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, uint64_t n,
                       double stdv, uint16_t *out) {
    uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i)
        out[i] = f32_to_bf16_rne(normal_at(key, first + (uint64_t)i, stdv));
}

/* Round an fp32 array to bf16 (RNE); used to store a residual stream. */
void synth_round_bf16(const float *in, uint64_t n, uint16_t *out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

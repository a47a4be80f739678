/*
 * synth.c - seeded synthetic inputs for the MoE layer workloads.
 *
 * This module only draws random numbers; it holds none of the MoE
 * arithmetic (no routing, no capacity, no permutation, no FFN).  The same
 * bytes feed both the CPU oracle and the CUDA library, so a parity test
 * compares the two on identical inputs.
 *
 * Generator: splitmix64 used as a counter-based generator.  Stream s of
 * seed S has key K(S, s); its i-th 64-bit draw is mix(K + (i + 1) * GAMMA),
 * which is exactly the i-th output of a splitmix64 whose state starts at K
 * (Steele, Lea, Flood, "Fast Splittable Pseudorandom Number Generators",
 * OOPSLA 2014).  Being random access, every draw can be computed in
 * parallel and the result does not depend on the thread count.
 *
 * Normals: Box-Muller in double on the pair (u1, u2) built from draws 2p and
 * 2p+1: u1 in (0, 1], u2 in [0, 1), r = sqrt(-2 ln u1),
 * z0 = r cos(2 pi u2), z1 = r sin(2 pi u2).  Values are rounded to fp32, and
 * to bf16 (round to nearest even) from that fp32 value where bf16 is asked.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SM64_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Key of stream `stream` under `seed`: two rounds of the mixer so that
 * neighbouring (seed, stream) pairs give unrelated keys. */
static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return sm64_mix(sm64_mix(seed + SM64_GAMMA) ^ (stream * 0xD1B54A32D192ED03ULL + 1ULL));
}

static inline uint64_t draw(uint64_t key, uint64_t i) {
    return sm64_mix(key + (i + 1ULL) * SM64_GAMMA);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) {          /* inf / nan: truncate, keep nan quiet */
        uint16_t h = (uint16_t)(u >> 16);
        if (u & 0x007FFFFFu) h |= 0x0040u;
        return h;
    }
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static inline void normal_pair(uint64_t key, int64_t p, double* z0, double* z1) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t a = draw(key, (uint64_t)(2 * p));
    uint64_t b = draw(key, (uint64_t)(2 * p + 1));
    double u1 = ((double)(a >> 11) + 1.0) * 0x1.0p-53;   /* (0, 1] */
    double u2 = (double)(b >> 11) * 0x1.0p-53;           /* [0, 1) */
    double r = sqrt(-2.0 * log(u1));
    *z0 = r * cos(two_pi * u2);
    *z1 = r * sin(two_pi * u2);
}

/* n normals N(mean, std^2) as fp32. */
void synth_normal_f32(uint64_t seed, uint64_t stream, int64_t n, double mean, double std, float* out) {
    const uint64_t key = stream_key(seed, stream);
    const int64_t npair = (n + 1) / 2;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npair; ++p) {
        double z0, z1;
        normal_pair(key, p, &z0, &z1);
        out[2 * p] = (float)(mean + std * z0);
        if (2 * p + 1 < n) out[2 * p + 1] = (float)(mean + std * z1);
    }
}

/* n normals N(mean, std^2) as bf16 bit patterns (fp32 value, then RNE). */
void synth_normal_bf16(uint64_t seed, uint64_t stream, int64_t n, double mean, double std, uint16_t* out) {
    const uint64_t key = stream_key(seed, stream);
    const int64_t npair = (n + 1) / 2;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < npair; ++p) {
        double z0, z1;
        normal_pair(key, p, &z0, &z1);
        out[2 * p] = f32_to_bf16_rne((float)(mean + std * z0));
        if (2 * p + 1 < n) out[2 * p + 1] = f32_to_bf16_rne((float)(mean + std * z1));
    }
}

/* n raw 64-bit draws. */
void synth_u64(uint64_t seed, uint64_t stream, int64_t n, uint64_t* out) {
    const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = draw(key, (uint64_t)i);
}

/* fp32 -> bf16 (round to nearest even), for inputs built from fp32 values. */
void synth_f32_to_bf16(const float* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16_rne(in[i]);
}

/*
 * Seeded, counter-based synthetic inputs for the padding-free varlen GPT-3
 * layer stack.  This file holds no arithmetic of the method itself: it only
 * draws random numbers and rounds them to a storage type.  Both the CUDA path
 * and the fp64 oracle receive the bits it writes, so the two sides always
 * see identical inputs.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014; finaliser constants as published there and
 * in Vigna's reference implementation).  Element c of stream (seed, tensor)
 * is mix(base + (c + 1) * GAMMA) with base = mix(seed ^ mix(tensor + GAMMA)),
 * so any slice of any tensor can be regenerated on its own.
 *
 * Uniform doubles take the top 53 bits: u = (r >> 11) * 2^-53, u in [0, 1).
 * Normals use Box-Muller on the uniform pair (2p, 2p + 1):
 *     rho = sqrt(-2 ln(1 - u0)),  z_even = rho cos(2 pi u1),  z_odd = rho sin(2 pi u1)
 * Element i of a normal tensor is mean + std * z_{i mod 2} of pair p = i / 2.
 * Uniform integers in [lo, hi] are lo + floor(u * (hi - lo + 1)).
 *
 * Storage rounding is round-to-nearest-even, done here by exact scaling and
 * nearbyint() so that it does not depend on compiler half-precision support.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_F32 0
#define SYNTH_F16 1
#define SYNTH_BF16 2
#define SYNTH_F64 3

static const uint64_t GAMMA = 0x9E3779B97F4A7C15ULL;

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_base(uint64_t seed, uint64_t tensor) {
    return mix64(seed ^ mix64(tensor + GAMMA));
}

static inline uint64_t draw(uint64_t base, uint64_t c) { return mix64(base + (c + 1) * GAMMA); }

static inline double to_unit(uint64_t r) { return (double)(r >> 11) * 0x1p-53; }

/* x -> IEEE binary16 bits, round to nearest even. */
static uint16_t round_f16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(a)) return (uint16_t)(sign | 0x7E00u);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    if (a < 0x1p-14) {
        double q = nearbyint(a * 0x1p24); /* subnormal units of 2^-24; 1024 encodes 2^-14 */
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    double m = frexp(a, &e); /* a = m 2^e, m in [0.5, 1) */
    double q = nearbyint(ldexp(m, 11));
    if (q == 2048.0) { q = 1024.0; e += 1; }
    int E = e + 14;
    if (E >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)(E << 10) | (uint16_t)((int)q - 1024));
}

/* x -> bfloat16 bits, round to nearest even. */
static uint16_t round_bf16(double x) {
    uint16_t sign = signbit(x) ? 0x8000u : 0u;
    double a = fabs(x);
    if (isnan(a)) return (uint16_t)(sign | 0x7FC0u);
    if (a < 0x1p-126) {
        double q = nearbyint(a * 0x1p133); /* subnormal units of 2^-133 */
        return (uint16_t)(sign | (uint16_t)q);
    }
    int e;
    double m = frexp(a, &e);
    double q = nearbyint(ldexp(m, 8));
    if (q == 256.0) { q = 128.0; e += 1; }
    int E = e + 126;
    if (E >= 255) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | (uint16_t)(E << 7) | (uint16_t)((int)q - 128));
}

static inline void store(void* out, int dtype, int64_t i, double v) {
    switch (dtype) {
    case SYNTH_F32: ((float*)out)[i] = (float)v; break;
    case SYNTH_F16: ((uint16_t*)out)[i] = round_f16(v); break;
    case SYNTH_BF16: ((uint16_t*)out)[i] = round_bf16(v); break;
    default: ((double*)out)[i] = v; break;
    }
}

/* Elements [offset, offset + n) of the normal stream (seed, tensor), scaled to
 * N(mean, std^2) and rounded to `dtype`, written to out[0 .. n). */
int synth_normal(uint64_t seed, uint64_t tensor, int64_t offset, int64_t n, double mean,
                 double std, int dtype, void* out) {
    if (n < 0 || offset < 0 || !out || dtype < 0 || dtype > 3) return 1;
    const uint64_t base = stream_base(seed, tensor);
    const double two_pi = 6.283185307179586476925286766559;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
        int64_t i = offset + j;
        uint64_t p = (uint64_t)(i >> 1);
        double u0 = to_unit(draw(base, 2 * p));
        double u1 = to_unit(draw(base, 2 * p + 1));
        double rho = sqrt(-2.0 * log(1.0 - u0));
        double z = (i & 1) ? rho * sin(two_pi * u1) : rho * cos(two_pi * u1);
        store(out, dtype, j, mean + std * z);
    }
    return 0;
}

/* Elements [offset, offset + n) of the uniform stream as doubles in [0, 1). */
int synth_uniform(uint64_t seed, uint64_t tensor, int64_t offset, int64_t n, double* out) {
    if (n < 0 || offset < 0 || !out) return 1;
    const uint64_t base = stream_base(seed, tensor);
    for (int64_t j = 0; j < n; ++j) out[j] = to_unit(draw(base, (uint64_t)(offset + j)));
    return 0;
}

/* n integers uniform on [lo, hi] (inclusive), element c = lo + floor(u_c (hi - lo + 1)). */
int synth_uniform_int(uint64_t seed, uint64_t tensor, int64_t n, int32_t lo, int32_t hi,
                      int32_t* out) {
    if (n < 0 || !out || hi < lo) return 1;
    const uint64_t base = stream_base(seed, tensor);
    const double span = (double)hi - (double)lo + 1.0;
    for (int64_t c = 0; c < n; ++c) {
        double u = to_unit(draw(base, (uint64_t)c));
        int64_t v = (int64_t)lo + (int64_t)floor(u * span);
        if (v > hi) v = hi; /* u < 1 makes this unreachable; kept as a guard */
        out[c] = (int32_t)v;
    }
    return 0;
}

/* Raw 64-bit draws, for tests of the generator itself. */
int synth_raw(uint64_t seed, uint64_t tensor, int64_t offset, int64_t n, uint64_t* out) {
    if (n < 0 || offset < 0 || !out) return 1;
    const uint64_t base = stream_base(seed, tensor);
    for (int64_t j = 0; j < n; ++j) out[j] = draw(base, (uint64_t)(offset + j));
    return 0;
}

/* Rounding helpers exposed for tests (double -> storage bits). */
int synth_round(const double* in, int64_t n, int dtype, void* out) {
    if (n < 0 || !in || !out || dtype < 0 || dtype > 3) return 1;
    for (int64_t j = 0; j < n; ++j) store(out, dtype, j, in[j]);
    return 0;
}

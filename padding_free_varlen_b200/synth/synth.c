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
 * Storage rounding is round-to-nearest-even, done on the binary64 bit fields
 * with integer arithmetic so that it does not depend on compiler
 * half-precision support or on the floating-point rounding mode.
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

/* Round a non-negative finite significand m (53 bits, implicit bit set) right
 * by `shift` bits, to nearest, ties to even. */
static inline uint64_t rne_shift(uint64_t m, int shift) {
    if (shift >= 64) return 0;
    if (shift <= 0) return m;
    uint64_t q = m >> shift;
    uint64_t rem = m & ((1ULL << shift) - 1);
    uint64_t half = 1ULL << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) ++q;
    return q;
}

/* x -> IEEE binary16 bits, round to nearest even, from the binary64 fields. */
static uint16_t round_f16(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    int e = (int)((b >> 52) & 0x7FF);
    uint64_t frac = b & ((1ULL << 52) - 1);
    if (e == 0x7FF) return (uint16_t)(sign | (frac ? 0x7E00u : 0x7C00u));
    if (e == 0) return sign; /* binary64 subnormals are far below half the smallest f16 */
    int ue = e - 1023;
    uint64_t m = frac | (1ULL << 52);
    if (ue >= -14) { /* normal f16 range (before rounding) */
        uint64_t q = rne_shift(m, 42);        /* 11-bit significand, in [1024, 2048] */
        if (q == 2048) { q = 1024; ++ue; }
        int E = ue + 15;
        if (E >= 31) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | (uint16_t)(E << 10) | (uint16_t)(q - 1024));
    }
    /* subnormal f16: units of 2^-24; value = m 2^(ue-52) */
    uint64_t q = rne_shift(m, 42 + (-14 - ue));
    return (uint16_t)(sign | (uint16_t)q); /* q == 1024 encodes 2^-14 */
}

/* x -> bfloat16 bits, round to nearest even, from the binary64 fields. */
static uint16_t round_bf16(double x) {
    uint64_t b;
    memcpy(&b, &x, 8);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
    int e = (int)((b >> 52) & 0x7FF);
    uint64_t frac = b & ((1ULL << 52) - 1);
    if (e == 0x7FF) return (uint16_t)(sign | (frac ? 0x7FC0u : 0x7F80u));
    if (e == 0) return sign;
    int ue = e - 1023;
    uint64_t m = frac | (1ULL << 52);
    if (ue >= -126) {
        uint64_t q = rne_shift(m, 45);        /* 8-bit significand, in [128, 256] */
        if (q == 256) { q = 128; ++ue; }
        int E = ue + 127;
        if (E >= 255) return (uint16_t)(sign | 0x7F80u);
        return (uint16_t)(sign | (uint16_t)(E << 7) | (uint16_t)(q - 128));
    }
    uint64_t q = rne_shift(m, 45 + (-126 - ue)); /* units of 2^-133 */
    return (uint16_t)(sign | (uint16_t)q);
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
    /* Pairs p cover elements 2p and 2p + 1; each pair's Box-Muller step runs once. */
    const int64_t p0 = offset >> 1, p1 = (offset + n + 1) >> 1;
#pragma omp parallel for schedule(static)
    for (int64_t p = p0; p < p1; ++p) {
        double u0 = to_unit(draw(base, 2 * (uint64_t)p));
        double u1 = to_unit(draw(base, 2 * (uint64_t)p + 1));
        double rho = sqrt(-2.0 * log(1.0 - u0));
        double ang = two_pi * u1;
        int64_t i0 = 2 * p - offset, i1 = i0 + 1;
        if (i0 >= 0 && i0 < n) store(out, dtype, i0, mean + std * (rho * cos(ang)));
        if (i1 >= 0 && i1 < n) store(out, dtype, i1, mean + std * (rho * sin(ang)));
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

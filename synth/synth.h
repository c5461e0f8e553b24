/*
 * synth.h -- seeded, counter-based generator for the synthetic inputs of the
 * hybrid compressed-attention workloads (raw KV latents, compressor logits,
 * indexer keys, queries, indexer weights, compressor biases, lengths).
 *
 * This module holds no arithmetic of the attention method itself.  It is the
 * one piece of code shared by the fp64 CPU oracle's test harness and the CUDA
 * path's harness: both sides draw identical input bytes from it.  The same
 * definition is compiled for the host (synth_host.c) and for the device
 * (synth_dev.cu); a GPU test checks that the two agree bit for bit.
 *
 * Definition (every step is exact IEEE-754 arithmetic or integer arithmetic,
 * so that any conforming compiler produces the same bits; both builds disable
 * floating-point contraction):
 *
 *   mix64(z)        the SplitMix64 output function (Steele, Lea & Flood,
 *                   "Fast splittable pseudorandom number generators",
 *                   OOPSLA 2014): z ^= z>>30; z *= 0xBF58476D1CE4E5B9;
 *                   z ^= z>>27; z *= 0x94D049BB133111EB; z ^= z>>31.
 *   GAMMA           0x9E3779B97F4A7C15 (the SplitMix64 increment).
 *   stream key      k = mix64(mix64(mix64(seed + GAMMA) + (tensor+1)*GAMMA)
 *                               + (seq+1)*GAMMA)
 *   bits(i)         mix64(k + (i+1)*GAMMA)            (64-bit counter mode)
 *   uniform(i)      (bits(i) >> 11) * 2^-53           in [0, 1)
 *   normal(i)       Box-Muller: u1 = 1 - uniform(2i), u2 = uniform(2i+1),
 *                   sqrt(-2 ln u1) * cos(2 pi u2), with ln and cos evaluated
 *                   by the fixed series below (not by a math library), so the
 *                   host and device agree to the last bit.
 *   bf16(v)         round-to-nearest-even of the double v to bfloat16,
 *                   computed directly from the binary64 pattern (no float
 *                   intermediate, so no double rounding).
 */
#ifndef CSA_SYNTH_H
#define CSA_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#define SYNTH_SQRT(v) sqrt(v)
#else
#include <math.h>
#define SYNTH_FN static inline
#define SYNTH_SQRT(v) sqrt(v)
#endif

/* Tensor identifiers: the 'tensor' coordinate of the stream key. */
enum {
    SYNTH_X = 0,      /* raw KV latent x_t            [tokens, d]      bf16, N(0,1) */
    SYNTH_A = 1,      /* CSA compressor logits a_t    [tokens, d]      bf16, N(0,1) */
    SYNTH_B = 2,      /* HCA compressor logits b_t    [tokens, d]      bf16, N(0,1) */
    SYNTH_KI = 3,     /* raw indexer key k^I_t        [tokens, d_I]    bf16, N(0,1) */
    SYNTH_Q = 4,      /* attention query q_h          [queries, H, d]  bf16, N(0,1) */
    SYNTH_QI = 5,     /* indexer query q^I_h          [queries, H_I, d_I] bf16, N(0,1) */
    SYNTH_W = 6,      /* indexer head weight w_h      [queries, H_I]   fp32, U(0,1) */
    SYNTH_BIAS_C = 7, /* CSA per-offset bias          [2m, d]          fp32, N(0, 0.5^2) */
    SYNTH_BIAS_H = 8, /* HCA per-offset bias          [m', d]          fp32, N(0, 0.5^2) */
    SYNTH_LEN = 9     /* sequence length draw         [B]              integer, uniform */
};

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ULL;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBULL;
    z ^= z >> 31;
    return z;
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t tensor, uint64_t seq) {
    uint64_t k = synth_mix64(seed + SYNTH_GAMMA);
    k = synth_mix64(k + (tensor + 1ULL) * SYNTH_GAMMA);
    return synth_mix64(k + (seq + 1ULL) * SYNTH_GAMMA);
}

SYNTH_FN uint64_t synth_bits(uint64_t key, uint64_t i) {
    return synth_mix64(key + (i + 1ULL) * SYNTH_GAMMA);
}

SYNTH_FN double synth_uniform(uint64_t key, uint64_t i) {
    return (double)(synth_bits(key, i) >> 11) * (1.0 / 9007199254740992.0);
}

SYNTH_FN double synth_as_double(uint64_t u) {
    union { uint64_t u; double d; } c;
    c.u = u;
    return c.d;
}

SYNTH_FN uint64_t synth_as_bits(double d) {
    union { uint64_t u; double d; } c;
    c.d = d;
    return c.u;
}

/* Natural log of u in (0, 1].  Write u = 2^e * f with f in [sqrt(1/2), sqrt(2))
 * (exact, by bit manipulation), then ln u = e ln2 + 2 atanh(s), s = (f-1)/(f+1),
 * |s| < 0.1716, using the odd series of atanh to 14 terms (truncation error
 * below 1e-21 relative).  Only +, -, *, / are used. */
SYNTH_FN double synth_log(double u) {
    uint64_t b = synth_as_bits(u);
    int e = (int)((b >> 52) & 0x7FF) - 1023;
    double f = synth_as_double((b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL); /* [1,2) */
    if (f > 1.4142135623730951) { f = f * 0.5; e = e + 1; }
    double s = (f - 1.0) / (f + 1.0);
    double s2 = s * s;
    double p = 1.0 / 29.0;
    p = p * s2 + 1.0 / 27.0;
    p = p * s2 + 1.0 / 25.0;
    p = p * s2 + 1.0 / 23.0;
    p = p * s2 + 1.0 / 21.0;
    p = p * s2 + 1.0 / 19.0;
    p = p * s2 + 1.0 / 17.0;
    p = p * s2 + 1.0 / 15.0;
    p = p * s2 + 1.0 / 13.0;
    p = p * s2 + 1.0 / 11.0;
    p = p * s2 + 1.0 / 9.0;
    p = p * s2 + 1.0 / 7.0;
    p = p * s2 + 1.0 / 5.0;
    p = p * s2 + 1.0 / 3.0;
    p = p * s2 + 1.0;
    return (double)e * 0.6931471805599453 + 2.0 * s * p;
}

/* Taylor series of cos and sin on [0, pi/4] (17 and 18 terms' worth of
 * accuracy are far beyond what the bf16 output needs). */
SYNTH_FN double synth_cos_small(double x) {
    double x2 = x * x;
    double p = 1.0 / 20922789888000.0;          /* 1/16! */
    p = p * -x2 + 1.0 / 87178291200.0;          /* 1/14! */
    p = p * -x2 + 1.0 / 479001600.0;            /* 1/12! */
    p = p * -x2 + 1.0 / 3628800.0;              /* 1/10! */
    p = p * -x2 + 1.0 / 40320.0;                /* 1/8!  */
    p = p * -x2 + 1.0 / 720.0;                  /* 1/6!  */
    p = p * -x2 + 1.0 / 24.0;                   /* 1/4!  */
    p = p * -x2 + 1.0 / 2.0;                    /* 1/2!  */
    p = p * -x2 + 1.0;
    return p;
}

SYNTH_FN double synth_sin_small(double x) {
    double x2 = x * x;
    double p = 1.0 / 355687428096000.0;         /* 1/17! */
    p = p * -x2 + 1.0 / 1307674368000.0;        /* 1/15! */
    p = p * -x2 + 1.0 / 6227020800.0;           /* 1/13! */
    p = p * -x2 + 1.0 / 39916800.0;             /* 1/11! */
    p = p * -x2 + 1.0 / 362880.0;               /* 1/9!  */
    p = p * -x2 + 1.0 / 5040.0;                 /* 1/7!  */
    p = p * -x2 + 1.0 / 120.0;                  /* 1/5!  */
    p = p * -x2 + 1.0 / 6.0;                    /* 1/3!  */
    p = p * -x2 + 1.0;
    return p * x;
}

/* cos(2 pi t) for t in [0, 1): fold t into [0, 1/8] by the symmetries of cos,
 * all folds being exact subtractions. */
SYNTH_FN double synth_cos2pi(double t) {
    double y = t > 0.5 ? 1.0 - t : t;       /* cos(2pi t) = cos(2pi (1-t)), y in [0, 0.5] */
    double sign = 1.0;
    if (y > 0.25) { y = 0.5 - y; sign = -1.0; } /* cos(pi - a) = -cos(a), y in [0, 0.25] */
    const double two_pi = 6.283185307179586;
    if (y > 0.125) return sign * synth_sin_small(two_pi * (0.25 - y));
    return sign * synth_cos_small(two_pi * y);
}

SYNTH_FN double synth_normal(uint64_t key, uint64_t i) {
    double u1 = 1.0 - synth_uniform(key, 2ULL * i);       /* (0, 1] */
    double u2 = synth_uniform(key, 2ULL * i + 1ULL);      /* [0, 1) */
    double r2 = -2.0 * synth_log(u1);
    double r = r2 > 0.0 ? SYNTH_SQRT(r2) : 0.0;
    return r * synth_cos2pi(u2);
}

/* Round-to-nearest-even of a double to bfloat16, straight from the binary64
 * pattern.  Magnitudes below 2^-126 become signed zero (never reached by the
 * distributions used here); magnitudes that round past the bf16 range
 * become infinity. */
SYNTH_FN uint16_t synth_bf16(double v) {
    uint64_t b = synth_as_bits(v);
    uint16_t sign = (uint16_t)((b >> 48) & 0x8000);
    int e = (int)((b >> 52) & 0x7FF) - 1023;
    uint64_t mant = b & 0x000FFFFFFFFFFFFFULL;
    if (e < -126) return sign;
    uint64_t m7 = mant >> 45;
    uint64_t rest = mant & ((1ULL << 45) - 1ULL);
    const uint64_t half = 1ULL << 44;
    if (rest > half || (rest == half && (m7 & 1ULL))) m7 += 1ULL;
    if (m7 == 128ULL) { m7 = 0ULL; e += 1; }
    if (e > 127) return (uint16_t)(sign | 0x7F80);
    return (uint16_t)(sign | (uint16_t)((e + 127) << 7) | (uint16_t)m7);
}

/* Round-to-nearest-even of a double to binary32 (plain IEEE conversion). */
SYNTH_FN float synth_f32(double v) { return (float)v; }

#endif /* CSA_SYNTH_H */

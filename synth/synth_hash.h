/*
 * synth_hash.h -- counter-based generator for the seeded synthetic inputs.
 *
 * This header is the one piece of code that both the float64 oracle and the
 * device-side input fill use.  It holds NO arithmetic of the attention method:
 * only a hash of (seed, tensor id, element index) and its mapping to an
 * approximately N(0,1) value rounded to bf16.  Every step is integer
 * arithmetic plus one correctly rounded IEEE double multiply, so the host (C)
 * and device (CUDA) compilations give identical bits.
 *
 * Definition (each side implements exactly this):
 *   mix(z)            = the SplitMix64 finaliser (Steele, Lea, Flood, "Fast
 *                       splittable pseudorandom number generators", OOPSLA 2014;
 *                       constants as published by Vigna):
 *                         z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
 *                         z = (z ^ (z >> 27)) * 0x94D049BB133111EB
 *                         z =  z ^ (z >> 31)
 *   key(seed, t)      = mix( mix(seed + G) ^ (t * 0xD1B54A32D192ED03) ),  G = 0x9E3779B97F4A7C15
 *   bits(key, i)      = mix( key + (i + 1) * G )
 *   normal(bits)      = (u0 + u1 + u2 + u3 - 131070) * C,  u_j = 16-bit field j of bits,
 *                       C = 1 / sqrt((65536^2 - 1) / 3)  (Irwin-Hall sum of four
 *                       discrete uniforms scaled to unit variance; |x| <= 3.4641)
 *   bf16(x)           = x rounded to bfloat16, round-to-nearest-even, taken
 *                       directly from the binary64 bits (no float32 step).
 *
 * Tensor ids and element indices are fixed by the callers (synth/__init__.py
 * documents them).
 */
#ifndef SYNTH_HASH_H
#define SYNTH_HASH_H

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GOLDEN 0x9E3779B97F4A7C15ULL
#define SYNTH_TMUL 0xD1B54A32D192ED03ULL
/* 1/sqrt((65536^2-1)/3) as an exact binary64 literal */
#define SYNTH_NORM 0x1.bb67ae86627e7p-16

SYNTH_FN uint64_t synth_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t tensor) {
    return synth_mix(synth_mix(seed + SYNTH_GOLDEN) ^ (tensor * SYNTH_TMUL));
}

SYNTH_FN uint64_t synth_bits(uint64_t key, uint64_t index) {
    return synth_mix(key + (index + 1ULL) * SYNTH_GOLDEN);
}

SYNTH_FN double synth_normal_from_bits(uint64_t b) {
    int64_t s = (int64_t)(b & 0xFFFFULL) + (int64_t)((b >> 16) & 0xFFFFULL) +
                (int64_t)((b >> 32) & 0xFFFFULL) + (int64_t)((b >> 48) & 0xFFFFULL);
#if defined(__CUDA_ARCH__)
    return __dmul_rn((double)(s - 131070), SYNTH_NORM);
#else
    return (double)(s - 131070) * SYNTH_NORM;
#endif
}

/* binary64 -> bfloat16 bits, round to nearest even, from the binary64 bits.
 * Inputs here are finite with |x| < 4; zero maps to +0.  Subnormal binary64
 * inputs cannot occur (the smallest nonzero |x| is C ~ 2.6e-5). */
SYNTH_FN uint16_t synth_bf16_bits(double x) {
    uint64_t u;
#if defined(__CUDA_ARCH__)
    u = (uint64_t)__double_as_longlong(x);
#else
    memcpy(&u, &x, sizeof u);
#endif
    uint64_t sign = u >> 63;
    uint64_t mag = u & 0x7FFFFFFFFFFFFFFFULL;
    if (mag == 0) return (uint16_t)(sign << 15);
    int64_t e = (int64_t)(mag >> 52) - 1023;         /* unbiased exponent */
    uint64_t m = (mag & 0xFFFFFFFFFFFFFULL) | (1ULL << 52); /* 53-bit significand */
    /* keep 8 significant bits (implicit 1 + 7 stored) */
    uint64_t keep = m >> 45;
    uint64_t rem = m & ((1ULL << 45) - 1);
    uint64_t half = 1ULL << 44;
    if (rem > half || (rem == half && (keep & 1ULL))) keep += 1;
    if (keep == (1ULL << 8)) { keep >>= 1; e += 1; }
    uint64_t be = (uint64_t)(e + 127);
    return (uint16_t)((sign << 15) | (be << 7) | (keep & 0x7FULL));
}

/* one bf16 value of stream `key` at element `index` */
SYNTH_FN uint16_t synth_bf16_at(uint64_t key, uint64_t index) {
    return synth_bf16_bits(synth_normal_from_bits(synth_bits(key, index)));
}

/* Logical element index of the per-position key/value streams:
 * request b, position p, kv head g (0 for MLA), feature d; Hkv kv heads, row
 * width W.  Independent of paging, sharding and interleave. */
SYNTH_FN uint64_t synth_kv_index(uint64_t b, uint64_t p, uint64_t g, uint64_t d,
                                 uint64_t Hkv, uint64_t W) {
    return (((b * Hkv + g) << 24) + p) * W + d;
}

/* Tensor ids of the streams */
#define SYNTH_T_Q 1ULL        /* q[b][h][d], plus 64*step for decode step `step` */
#define SYNTH_T_K 2ULL        /* GQA keys */
#define SYNTH_T_V 3ULL        /* GQA values */
#define SYNTH_T_LATENT 4ULL   /* MLA latent rows (576 wide) */

#endif /* SYNTH_HASH_H */

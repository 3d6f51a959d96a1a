/*
 * Seeded, counter-based generator for synthetic decode inputs.
 *
 * This module holds no arithmetic of the decode step itself.  It only draws
 * random numbers: bf16 weights that are approximately N(mean, sigma^2), KV
 * cache contents, token ids and sequence lengths.  Every element is a pure
 * function of (seed, tensor id, element index), so host code and device code
 * produce the same bits and any single element can be regenerated alone.
 *
 * Definition (implemented identically by the host fill in synthetic.c and the
 * device fill in synthetic_fill.cu; both include this header):
 *   mix64(z)      = the SplitMix64 output function (Steele, Lea and Flood,
 *                   "Fast splittable pseudorandom number generators",
 *                   OOPSLA 2014): z += 0x9E3779B97F4A7C15; then two
 *                   xor-shift-multiply rounds and a final xor-shift.
 *   key(seed,tid) = mix64(mix64(seed) ^ tid)
 *   word(i, j)    = mix64(key + 3*i + j),  j in {0, 1, 2}
 *   S             = sum of the twelve 16-bit fields of word(i,0..2)
 *                   (Irwin-Hall sum of 12 uniforms on {0..65535})
 *   n             = 2*S - 786420        (exact integer, |n| <= 786420)
 *   value         = bf16_rne( fp32(n) * fp32(sigma * 2^-17) + mean )
 *                   the product is one correctly rounded fp32 multiply; the
 *                   mean, when nonzero, is added in fp32 before the rounding.
 * Var(n) = 4 * (65536^2 - 1) ~= 2^34, so value has standard deviation
 * sigma * (1 - 2^-32)^(1/2) ~= sigma and is truncated at about +-6 sigma.
 */
#ifndef SYNTHETIC_GEN_H
#define SYNTHETIC_GEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_FN static __host__ __device__ __forceinline__
#else
#define SYN_FN static inline
#endif

SYN_FN uint64_t syn_mix64(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

SYN_FN uint64_t syn_key(uint64_t seed, uint64_t tensor_id) {
    return syn_mix64(syn_mix64(seed) ^ tensor_id);
}

SYN_FN uint64_t syn_word(uint64_t key, uint64_t index, uint64_t j) {
    return syn_mix64(key + 3ull * index + j);
}

/* Irwin-Hall integer n = 2*S - 786420 for element `index`. */
SYN_FN int32_t syn_irwin_hall(uint64_t key, uint64_t index) {
    uint32_t s = 0;
    for (int j = 0; j < 3; ++j) {
        uint64_t w = syn_word(key, index, (uint64_t)j);
        s += (uint32_t)(w & 0xFFFFu) + (uint32_t)((w >> 16) & 0xFFFFu) +
             (uint32_t)((w >> 32) & 0xFFFFu) + (uint32_t)((w >> 48) & 0xFFFFu);
    }
    return (int32_t)(2u * s) - 786420;
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
SYN_FN uint16_t syn_f32_to_bf16(float f) {
    union { float f; uint32_t u; } v;
    v.f = f;
    uint32_t u = v.u;
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* One synthetic bf16 element.  `scale` must be fp32(sigma) * 2^-17. */
SYN_FN uint16_t syn_bf16_value(uint64_t key, uint64_t index, float scale, float mean) {
    float v = (float)syn_irwin_hall(key, index) * scale;
    if (mean != 0.0f) v = v + mean;
    return syn_f32_to_bf16(v);
}

/* Uniform integer in [lo, lo + span) for element `index` (modulo bias < 2^-40). */
SYN_FN int64_t syn_uniform_int(uint64_t key, uint64_t index, int64_t lo, uint64_t span) {
    uint64_t w = syn_word(key, index, 0);
    return lo + (int64_t)((w >> 16) % span);
}

#endif /* SYNTHETIC_GEN_H */

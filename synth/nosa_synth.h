/*
 * nosa_synth.h -- seeded, counter-based synthetic input generator.
 *
 * This module holds only random-number generation: it computes none of the
 * sparse-attention method.  It is the one piece of code that both the CPU
 * oracle and the GPU benchmark harness use, so that both consume identical
 * input bytes.  Every operation below is either integer arithmetic or a
 * single correctly rounded IEEE fp32 multiply/add, so a C compiler (built with
 * -ffp-contract=off) and nvcc (using the explicit _rn intrinsics) produce the
 * same bits.
 *
 * Draws.  An element is addressed by the counter
 *   (seed, stream, layer, seq, head, pos, dim)
 * which is hashed with the SplitMix64 output function (Steele, Lea & Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).  The 64-bit
 * hash is split into four 16-bit uniform integers whose exact integer sum S
 * (0..262140) approximates a normal variate (Irwin-Hall, n = 4).  The centred
 * sum is turned into a float by one fp32 multiply with a constant chosen so
 * the result has unit variance (the variance of one 16-bit uniform draw is
 * (2^32 - 1)/12).  The tails are bounded at +-3.46 sigma.
 *
 * Workload distributions (decode-attention workloads of the NOSA pages: keys
 * and values N(0,1)/sqrt(128), eviction logits N(0,1), queries following
 * q_t = 0.9 q_{t-1} + 0.44 xi_t):
 *   K, V  : z * (1/sqrt(128)), one fp32 multiply with the folded constant,
 *           then round-to-nearest-even to bf16.
 *   e     : z (fp32).
 *   q     : q_0 = z_0, q_t = 0.9f*q_{t-1} + 0.44f*z_t, each product and the
 *           sum rounded to fp32 separately; the kernel input is bf16(q_t).
 *   W1, W2: weights of a synthetic eviction head (random, untrained), per
 *           layer and kv head, fp32: W1 [D][H] (row d, column h) = z, so that
 *           v.W1 has unit variance for v ~ N(0,1)/sqrt(128); W2 [H] =
 *           z * (1/sqrt(128)).
 */
#ifndef NOSA_SYNTH_H
#define NOSA_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define NOSA_SYNTH_FN static __host__ __device__ __forceinline__
#else
#define NOSA_SYNTH_FN static inline
#endif

/* stream identifiers */
#define NOSA_SYNTH_K 1u
#define NOSA_SYNTH_V 2u
#define NOSA_SYNTH_E 3u
#define NOSA_SYNTH_Q 4u
#define NOSA_SYNTH_W1 5u
#define NOSA_SYNTH_W2 6u

/* 1/sqrt((2^32-1)/3): unit-variance scale for the centred 4-draw sum. */
#define NOSA_SYNTH_C_UNIT 0x1.bb67aep-16f   /* 2.6428997e-05, fp32-exact */
/* NOSA_SYNTH_C_UNIT / sqrt(128), rounded once to fp32. */
#define NOSA_SYNTH_C_KV   0x1.3988e2p-19f   /* fp32-exact */
#define NOSA_SYNTH_Q_RHO  0.9f
#define NOSA_SYNTH_Q_SIG  0.44f

NOSA_SYNTH_FN uint64_t nosa_synth_mix(uint64_t z) {
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Hash of everything but the innermost index; one per row of D elements. */
NOSA_SYNTH_FN uint64_t nosa_synth_row(uint64_t seed, uint32_t stream, uint32_t layer,
                                      uint32_t seq, uint32_t head, uint64_t pos) {
    uint64_t h = nosa_synth_mix(seed);
    h = nosa_synth_mix(h ^ ((uint64_t)stream << 32 | layer));
    h = nosa_synth_mix(h ^ ((uint64_t)seq << 32 | head));
    h = nosa_synth_mix(h ^ pos);
    return h;
}

/* Centred Irwin-Hall sum of four 16-bit draws: an integer in [-131070, 131070]. */
NOSA_SYNTH_FN int32_t nosa_synth_centred(uint64_t row, uint32_t dim) {
    uint64_t x = nosa_synth_mix(row + dim);
    int32_t s = (int32_t)(x & 0xFFFFu) + (int32_t)((x >> 16) & 0xFFFFu) +
                (int32_t)((x >> 32) & 0xFFFFu) + (int32_t)(x >> 48);
    return s - 131070;
}

NOSA_SYNTH_FN float nosa_synth_fmul(float a, float b) {
#if defined(__CUDA_ARCH__)
    return __fmul_rn(a, b);
#else
    return a * b;
#endif
}

NOSA_SYNTH_FN float nosa_synth_fadd(float a, float b) {
#if defined(__CUDA_ARCH__)
    return __fadd_rn(a, b);
#else
    return a + b;
#endif
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
NOSA_SYNTH_FN uint16_t nosa_synth_bf16(float f) {
    union { float f; uint32_t u; } c;
    c.f = f;
    uint32_t u = c.u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* unit-variance standard-normal approximation */
NOSA_SYNTH_FN float nosa_synth_normal(uint64_t row, uint32_t dim) {
    return nosa_synth_fmul((float)nosa_synth_centred(row, dim), NOSA_SYNTH_C_UNIT);
}

/* one key or value element, N(0,1)/sqrt(128), as bf16 bits */
NOSA_SYNTH_FN uint16_t nosa_synth_kv(uint64_t row, uint32_t dim) {
    return nosa_synth_bf16(nosa_synth_fmul((float)nosa_synth_centred(row, dim), NOSA_SYNTH_C_KV));
}


/* eviction logit of one token: N(0,1) fp32 */
NOSA_SYNTH_FN float nosa_synth_e(uint64_t seed, uint32_t layer, uint32_t seq, uint32_t kvh,
                                 uint64_t pos) {
    return nosa_synth_normal(nosa_synth_row(seed, NOSA_SYNTH_E, layer, seq, kvh, pos), 0u);
}

/* one step of the query drift recursion, element-wise */
NOSA_SYNTH_FN float nosa_synth_q_next(float prev, float xi) {
    return nosa_synth_fadd(nosa_synth_fmul(NOSA_SYNTH_Q_RHO, prev),
                           nosa_synth_fmul(NOSA_SYNTH_Q_SIG, xi));
}

#endif /* NOSA_SYNTH_H */

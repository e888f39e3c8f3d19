/*
 * synth_host.c -- CPU batch wrappers around the seeded generator in
 * nosa_synth.h.  Used by the oracle-side tests and by the CPU baseline to
 * produce the same input bytes that the GPU-side generator (synth_gpu.cu)
 * writes into device memory.  Build with -ffp-contract=off.
 */
#include "nosa_synth.h"

/* K or V rows of one (layer, seq, kv head): out[T][D] bf16 bits, positions p0..p0+T-1 */
void nosa_synth_kv_rows(uint64_t seed, uint32_t stream, uint32_t layer, uint32_t seq,
                        uint32_t kvh, uint64_t p0, int64_t T, int32_t D, uint16_t *out) {
    for (int64_t t = 0; t < T; ++t) {
        uint64_t row = nosa_synth_row(seed, stream, layer, seq, kvh, p0 + (uint64_t)t);
        for (int32_t d = 0; d < D; ++d) out[t * D + d] = nosa_synth_kv(row, (uint32_t)d);
    }
}

/* eviction logits of one (layer, seq, kv head): out[T] fp32 */
void nosa_synth_e_rows(uint64_t seed, uint32_t layer, uint32_t seq, uint32_t kvh, uint64_t p0,
                       int64_t T, float *out) {
    for (int64_t t = 0; t < T; ++t) out[t] = nosa_synth_e(seed, layer, seq, kvh, p0 + (uint64_t)t);
}

/*
 * Queries of one (layer, seq, q head) for decode steps 0..n-1.
 * out_f32 (nullable) [n][D] fp32 drift state, out_bf16 (nullable) [n][D] bf16 bits.
 */
void nosa_synth_q_steps(uint64_t seed, uint32_t layer, uint32_t seq, uint32_t qh, int64_t n,
                        int32_t D, float *out_f32, uint16_t *out_bf16) {
    float prev[1024];
    if (D > 1024) return;
    for (int64_t t = 0; t < n; ++t) {
        uint64_t row = nosa_synth_row(seed, NOSA_SYNTH_Q, layer, seq, qh, (uint64_t)t);
        for (int32_t d = 0; d < D; ++d) {
            float xi = nosa_synth_normal(row, (uint32_t)d);
            float q = (t == 0) ? xi : nosa_synth_q_next(prev[d], xi);
            prev[d] = q;
            if (out_f32) out_f32[t * D + d] = q;
            if (out_bf16) out_bf16[t * D + d] = nosa_synth_bf16(q);
        }
    }
}

/* Synthetic eviction-head weights of one layer: W1 [Hkv][D][H], W2 [Hkv][H] (fp32). */
void nosa_synth_head_weights(uint64_t seed, uint32_t layer, int32_t Hkv, int32_t D, int32_t H, float *W1,
                             float *W2) {
    for (int32_t g = 0; g < Hkv; ++g) {
        for (int32_t d = 0; d < D; ++d) {
            uint64_t row = nosa_synth_row(seed, NOSA_SYNTH_W1, layer, 0u, (uint32_t)g, (uint64_t)d);
            for (int32_t h = 0; h < H; ++h) W1[((int64_t)g * D + d) * H + h] = nosa_synth_normal(row, (uint32_t)h);
        }
        uint64_t row = nosa_synth_row(seed, NOSA_SYNTH_W2, layer, 0u, (uint32_t)g, 0u);
        for (int32_t h = 0; h < H; ++h)
            W2[(int64_t)g * H + h] = nosa_synth_fmul((float)nosa_synth_centred(row, (uint32_t)h), NOSA_SYNTH_C_KV);
    }
}

/*
 * synth_gpu.cu -- device-side batch wrappers around the seeded generator in
 * nosa_synth.h, so that large synthetic contexts (hundreds of GB over all
 * layers) are produced in device memory at HBM speed instead of on the host.
 * Bytes are identical to synth_host.c.  Exposed through a small C ABI.
 */
#include <cuda_runtime.h>
#include "nosa_synth.h"

/* out[u][T][D] for units u = seq*Hkv + kvh, positions p0.. */
__global__ void synth_kv_kernel(uint64_t seed, uint32_t stream, uint32_t layer, int32_t seq0,
                                int32_t Hkv, int32_t units, uint64_t p0, int64_t T, int32_t D,
                                uint16_t *__restrict__ out) {
    int64_t rows = (int64_t)units * T;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.y + threadIdx.y; r < rows;
         r += (int64_t)gridDim.x * blockDim.y) {
        int32_t u = (int32_t)(r / T);
        int64_t t = r - (int64_t)u * T;
        uint64_t row = nosa_synth_row(seed, stream, layer, (uint32_t)(seq0 + u / Hkv),
                                      (uint32_t)(u % Hkv), p0 + (uint64_t)t);
        for (int32_t d = threadIdx.x; d < D; d += blockDim.x)
            out[r * D + d] = nosa_synth_kv(row, (uint32_t)d);
    }
}

__global__ void synth_e_kernel(uint64_t seed, uint32_t layer, int32_t seq0, int32_t Hkv,
                               int32_t units, uint64_t p0, int64_t T, float *__restrict__ out) {
    int64_t n = (int64_t)units * T;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        int32_t u = (int32_t)(i / T);
        int64_t t = i - (int64_t)u * T;
        out[i] = nosa_synth_e(seed, layer, (uint32_t)(seq0 + u / Hkv), (uint32_t)(u % Hkv),
                              p0 + (uint64_t)t);
    }
}

/* queries of step t for all (seq, q head): state[B*Hq][D] fp32 advanced in place, out bf16 */
__global__ void synth_q_kernel(uint64_t seed, uint32_t layer, int32_t seq0, int32_t Hq, int32_t rows,
                               int64_t t, int32_t D, float *__restrict__ state,
                               uint16_t *__restrict__ out) {
    int32_t r = blockIdx.x;
    if (r >= rows) return;
    uint64_t row = nosa_synth_row(seed, NOSA_SYNTH_Q, layer, (uint32_t)(seq0 + r / Hq),
                                  (uint32_t)(r % Hq), (uint64_t)t);
    for (int32_t d = threadIdx.x; d < D; d += blockDim.x) {
        float xi = nosa_synth_normal(row, (uint32_t)d);
        float q = (t == 0) ? xi : nosa_synth_q_next(state[(int64_t)r * D + d], xi);
        state[(int64_t)r * D + d] = q;
        out[(int64_t)r * D + d] = nosa_synth_bf16(q);
    }
}

static int launch_status(void) { return cudaGetLastError() == cudaSuccess ? 0 : -4; }

extern "C" int nosa_synth_kv_dev(uint64_t seed, uint32_t stream, uint32_t layer, int32_t seq0,
                                 int32_t B, int32_t Hkv, uint64_t p0, int64_t T, int32_t D, void *out,
                                 void *cuda_stream) {
    if (B <= 0 || Hkv <= 0 || T < 0 || D <= 0 || !out) return -1;
    if (T == 0) return 0;
    dim3 blk(32, 8);
    int64_t rows = (int64_t)B * Hkv * T;
    int64_t g = (rows + 7) / 8;
    if (g > 148 * 64) g = 148 * 64;
    synth_kv_kernel<<<(unsigned)g, blk, 0, (cudaStream_t)cuda_stream>>>(
        seed, stream, layer, seq0, Hkv, B * Hkv, p0, T, D, (uint16_t *)out);
    return launch_status();
}

extern "C" int nosa_synth_e_dev(uint64_t seed, uint32_t layer, int32_t seq0, int32_t B, int32_t Hkv,
                                uint64_t p0, int64_t T, void *out, void *cuda_stream) {
    if (B <= 0 || Hkv <= 0 || T < 0 || !out) return -1;
    if (T == 0) return 0;
    int64_t n = (int64_t)B * Hkv * T;
    int64_t g = (n + 255) / 256;
    if (g > 148 * 32) g = 148 * 32;
    synth_e_kernel<<<(unsigned)g, 256, 0, (cudaStream_t)cuda_stream>>>(seed, layer, seq0, Hkv,
                                                                       B * Hkv, p0, T, (float *)out);
    return launch_status();
}

extern "C" int nosa_synth_q_dev(uint64_t seed, uint32_t layer, int32_t seq0, int32_t B, int32_t Hq,
                                int64_t t, int32_t D, void *state, void *out, void *cuda_stream) {
    if (B <= 0 || Hq <= 0 || t < 0 || D <= 0 || !state || !out) return -1;
    synth_q_kernel<<<B * Hq, 128, 0, (cudaStream_t)cuda_stream>>>(seed, layer, seq0, Hq, B * Hq, t, D,
                                                                  (float *)state, (uint16_t *)out);
    return launch_status();
}

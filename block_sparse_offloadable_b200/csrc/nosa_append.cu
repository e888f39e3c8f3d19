// nosa_append.cu -- step a1: append the new token, pool what completes, keep Gamma_e.
//
// NOSA pages: montaan.com summary of arXiv:2510.13602, "Key Design Components"
// item 2 (mean pooling within sub-blocks and max pooling across them, for the
// query-aware and the query-agnostic selection), item 1 (a block dropped by
// the query-agnostic selection is never selected by it again); gist.science
// summary, "ED-DMA" (selection on the pre-exponential eviction score) and
// "Systeme : NOSI" (block-sized KV units on both GPU and CPU).
//
// Decode (T = 1): one warp per unit.  The only HBM traffic is the new rows
// (512 B), one 4 KiB re-read of the keys of a sub-block when it completes,
// and one 256 B read of the eviction logits when a block completes, so the
// kernel is latency-bound by design.
#include "nosa_append_unit.cuh"

namespace nosa {

// ---- eviction head: e_j = sum_h W2[h] softplus(v_j . W1[:, h]) -------------------------
// fp64, every product and sum rounded on its own (no contraction), sums in index
// order (d for the hidden pre-activations, h for the output), rounded once to fp32.
__device__ __forceinline__ double softplus64(double x) {
    return __dadd_rn(x > 0.0 ? x : 0.0, log1p(exp(-fabs(x))));
}

__global__ void __launch_bounds__(128) append_decode_kernel(const AppendParams p) {
    pdl_trigger();  // the select that follows waits for this grid anyway
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x * (blockDim.x >> 5) + warp;
    if (u >= p.units) return;
    append_unit(p, u, lane, p.e_new[u]);
}

// With the fused eviction head: one CTA of kHeadH threads per unit.  One bulk
// copy stages W1 and W2 of the unit's kv head (64.5 KB) in shared memory;
// thread h then runs hidden unit h's pre-activation in order over d, the 128
// terms W2[h] softplus(z_h) are summed in order by one thread, and warp 0
// appends the token with that logit.
constexpr size_t kHeadDecSmem = (size_t)kD * kHeadH * 4 + kHeadH * 4 + kD * 8 + kHeadH * 8 + 16;

__global__ void __launch_bounds__(kHeadH) append_head_decode_kernel(const AppendParams p) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ __align__(16) uint8_t smem[];
    float *w1s = reinterpret_cast<float *>(smem);
    float *w2s = w1s + kD * kHeadH;
    double *vs = reinterpret_cast<double *>(w2s + kHeadH);
    double *ts = vs + kD;
    uint64_t *bar = reinterpret_cast<uint64_t *>(ts + kHeadH);
    __shared__ float s_e;
    const int32_t u = blockIdx.x;
    const int h = threadIdx.x, lane = threadIdx.x & 31;
    const int32_t g = u % p.heads_kv;
    if (h == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (h == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(kD * kHeadH * 4 + kHeadH * 4));
        bulk_load(w1s, p.w1 + (int64_t)g * kD * kHeadH, kD * kHeadH * 4, bar);
        bulk_load(w2s, p.w2 + (int64_t)g * kHeadH, kHeadH * 4, bar);
    }
    {  // the value row as fp64 (exact), while the weights are in flight
        const uint16_t b = p.v_new[(int64_t)u * kD + h];
        vs[h] = (double)__uint_as_float((uint32_t)b << 16);
    }
    const bool ok = mbar_wait(bar, 0);
    if (__syncthreads_or(!ok)) {  // the whole CTA gives up together
        if (!ok) mbar_wait(bar, 0);  // never leave with the copy in flight (bounded again)
        if (h == 0) set_error(p.err, NOSA_EFLAG_TIMEOUT);
        return;
    }
    double z = 0.0;
#pragma unroll 8
    for (int d = 0; d < kD; ++d) z = __dadd_rn(z, __dmul_rn(vs[d], (double)w1s[d * kHeadH + h]));
    ts[h] = __dmul_rn((double)w2s[h], softplus64(z));
    __syncthreads();
    if (h == 0) {
        double e = 0.0;
        for (int i = 0; i < kHeadH; ++i) e = __dadd_rn(e, ts[i]);
        s_e = __double2float_rn(e);
    }
    __syncthreads();
    if (threadIdx.x < 32) append_unit(p, u, lane, s_e);
}

// ---- prefill ----------------------------------------------------------------------

__device__ __forceinline__ int32_t unit_len(const AppendParams &p, int32_t u) {
    return p.lens ? min(p.lens[u / p.heads_kv], p.T) : p.T;
}

// Store the rows of every unit (block-major), their eviction logits, and in
// offload mode the rows of the local block into cache slot 0.  One warp per row.
__global__ void __launch_bounds__(256) prefill_store_kernel(const AppendParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int64_t rows = (int64_t)p.units * p.T;
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
         r += nwarps) {
        const int32_t u = (int32_t)(r / p.T);
        const int32_t t = (int32_t)(r - (int64_t)u * p.T);
        const int32_t len = unit_len(p, u);
        if (t >= len || p.seq_len[u] != 0) continue;
        const int32_t blk = t >> 6, w = t & 63;
        const int chunk = lane & 15;
        const uint16_t *src = (lane < 16 ? p.k_new : p.v_new) + ((int64_t)u * p.T + t) * kD;
        const uint4 val = reinterpret_cast<const uint4 *>(src)[chunk];
        const int64_t off = (lane < 16 ? 0 : kHalfBlockBytes) + (int64_t)w * kRowBytes + chunk * 16;
        *reinterpret_cast<uint4 *>(p.store + ((int64_t)u * p.nblk + blk) * kBlockBytes + off) = val;
        if (p.offload && blk == (len - 1) >> 6)
            *reinterpret_cast<uint4 *>(p.cache + (int64_t)u * p.nslots * kBlockBytes + off) = val;
        if (lane == 0 && !p.w1) p.e_store[(int64_t)u * p.max_ctx + t] = p.e_new[(int64_t)u * p.T + t];
    }
}

// Pool every complete sub-block (mean key) and block (eviction score).  One warp per block.
__global__ void __launch_bounds__(256) prefill_pool_kernel(const AppendParams p) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int32_t bpu = (p.T + kBlock - 1) / kBlock;
    const int64_t items = (int64_t)p.units * bpu;
    for (int64_t it = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
         it += nwarps) {
        const int32_t u = (int32_t)(it / bpu);
        const int32_t blk = (int32_t)(it - (int64_t)u * bpu);
        const int32_t len = unit_len(p, u);
        if (p.seq_len[u] != 0) continue;
        const uint16_t *K = p.k_new + (int64_t)u * p.T * kD;
        for (int s = 0; s < kSubPerBlock; ++s) {
            const int32_t t0 = blk * kBlock + s * kSub;
            if (t0 + kSub > len) break;
            double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
            for (int j = 0; j < kSub; ++j) {
                const uint2 v = reinterpret_cast<const uint2 *>(K + (int64_t)(t0 + j) * kD)[lane];
                a0 += bf16_lo(v.x); a1 += bf16_hi(v.x);
                a2 += bf16_lo(v.y); a3 += bf16_hi(v.y);
            }
            store_ck(p, (int64_t)u * p.nsub + (t0 >> 4), lane, a0 / kSub, a1 / kSub, a2 / kSub, a3 / kSub);
        }
        if ((blk + 1) * kBlock <= len) {
            double m = -__longlong_as_double(0x7FF0000000000000ll);
            if (lane < kSubPerBlock) {
                const float *e = (p.w1 ? p.e_store + (int64_t)u * p.max_ctx : p.e_new + (int64_t)u * p.T) +
                                 (int64_t)blk * kBlock + lane * kSub;
                double acc = 0.0;
                for (int j = 0; j < kSub; ++j) acc += (double)e[j];
                m = acc / kSub;
            }
            m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
            m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
            if (lane == 0) p.blk_evict[(int64_t)u * p.nblk + blk] = m;
        }
    }
}

// Eviction head over the prefilled rows: a CTA stages W1 and W2 of its kv head in
// shared memory and takes kHeadCtaRows rows of one unit; each warp runs 8 rows at
// a time, a lane holding the pre-activations of hidden units lane + 32 i for all
// 8 rows (32 fp64 accumulators); lane r then sums row r's 128 terms in order.
constexpr int kHeadWarpRows = 8;
constexpr int kHeadCtaRows = 256;
constexpr int kHeadTStride = kHeadH + 2;  // doubles per row of t: rows land on distinct banks
constexpr size_t kHeadSmem = (size_t)kD * kHeadH * 4 + kHeadH * 4 + 8 * kHeadWarpRows * kHeadTStride * 8;

__global__ void __launch_bounds__(256) prefill_head_kernel(const AppendParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    float *w1s = reinterpret_cast<float *>(smem);
    float *w2s = w1s + kD * kHeadH;
    double *ts = reinterpret_cast<double *>(w2s + kHeadH);
    const int32_t u = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (p.seq_len[u] != 0) return;  // prefill into a non-empty unit: flagged by prefill_gamma_kernel
    const int32_t len = unit_len(p, u);
    const int32_t r0 = blockIdx.x * kHeadCtaRows, r1 = min(r0 + kHeadCtaRows, len);
    if (r0 >= r1) return;
    const int32_t g = u % p.heads_kv;
    const float4 *w1g = reinterpret_cast<const float4 *>(p.w1 + (int64_t)g * kD * kHeadH);
    for (int i = threadIdx.x; i < kD * kHeadH / 4; i += blockDim.x) reinterpret_cast<float4 *>(w1s)[i] = w1g[i];
    if (threadIdx.x < kHeadH) w2s[threadIdx.x] = p.w2[g * kHeadH + threadIdx.x];
    __syncthreads();
    double *tw = ts + warp * kHeadWarpRows * kHeadTStride;
    for (int32_t rb = r0 + warp * kHeadWarpRows; rb < r1; rb += 8 * kHeadWarpRows) {
        uint2 vv[kHeadWarpRows];
#pragma unroll
        for (int r = 0; r < kHeadWarpRows; ++r)
            vv[r] = (rb + r < r1) ? reinterpret_cast<const uint2 *>(p.v_new + ((int64_t)u * p.T + rb + r) * kD)[lane]
                                  : make_uint2(0u, 0u);
        double z[kHeadWarpRows][4];
#pragma unroll
        for (int r = 0; r < kHeadWarpRows; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) z[r][i] = 0.0;
        for (int d4 = 0; d4 < kD / 4; ++d4) {
            uint32_t wx[kHeadWarpRows], wy[kHeadWarpRows];
#pragma unroll
            for (int r = 0; r < kHeadWarpRows; ++r) {
                wx[r] = __shfl_sync(0xFFFFFFFFu, vv[r].x, d4);
                wy[r] = __shfl_sync(0xFFFFFFFFu, vv[r].y, d4);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                double w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) w[i] = (double)w1s[(4 * d4 + k) * kHeadH + lane + 32 * i];
#pragma unroll
                for (int r = 0; r < kHeadWarpRows; ++r) {
                    const uint32_t word = (k < 2) ? wx[r] : wy[r];
                    const double v = (k & 1) ? bf16_hi(word) : bf16_lo(word);
#pragma unroll
                    for (int i = 0; i < 4; ++i) z[r][i] = __dadd_rn(z[r][i], __dmul_rn(v, w[i]));
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kHeadWarpRows; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tw[r * kHeadTStride + 32 * i + lane] = __dmul_rn((double)w2s[32 * i + lane], softplus64(z[r][i]));
        __syncwarp();
        if (lane < kHeadWarpRows && rb + lane < r1) {
            double e = 0.0;
            for (int h = 0; h < kHeadH; ++h) e = __dadd_rn(e, tw[lane * kHeadTStride + h]);
            p.e_store[(int64_t)u * p.max_ctx + rb + lane] = __double2float_rn(e);
        }
        __syncwarp();
    }
}

// Gamma_e := top-k_e of the candidates by E (ties to the lower block), ascending;
// fill reading: also the pool of every candidate in rank order (nothing is
// dropped before the first decode step).  One CTA per unit; rank counting over
// the candidates held in shared memory (the ranks are a permutation).
__global__ void __launch_bounds__(256) prefill_gamma_kernel(const AppendParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int32_t u = blockIdx.x;
    if (p.seq_len[u] != 0) {
        if (threadIdx.x == 0) set_error(p.err, NOSA_EFLAG_STATE);
        return;
    }
    const int32_t len = unit_len(p, u);
    const int32_t nb_c = len > 0 ? (len - 1) / kBlock : 0;
    double *E = reinterpret_cast<double *>(smem);
    uint8_t *flag = smem + (size_t)p.nblk * sizeof(double);
    for (int i = threadIdx.x; i < nb_c; i += blockDim.x) E[i] = p.blk_evict[(int64_t)u * p.nblk + i];
    __syncthreads();
    const bool pool = p.fill && p.k_e > 0;
    const int32_t stop = pool ? nb_c : p.k_e;
    for (int i = threadIdx.x; i < nb_c; i += blockDim.x) {
        const double ei = E[i];
        int32_t rank = 0;
        for (int j = 0; j < nb_c && rank < stop; ++j) {
            const double ej = E[j];
            rank += (ej > ei) || (ej == ei && j < i);
        }
        flag[i] = rank < p.k_e;
        if (pool) p.pool[(int64_t)u * p.nblk + rank] = i;
    }
    if (pool && threadIdx.x == 0) p.pool_n[u] = nb_c;
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int32_t per = (nb_c + 31) / 32;
        const int32_t b0 = min(lane * per, nb_c), b1 = min(b0 + per, nb_c);
        int32_t cnt = 0;
        for (int i = b0; i < b1; ++i) cnt += flag[i];
        int32_t pre = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            int32_t v = __shfl_up_sync(0xFFFFFFFFu, pre, o);
            if (lane >= o) pre += v;
        }
        int32_t at = pre - cnt;
        int32_t *ge = p.gamma_e + (int64_t)u * p.k_e;
        for (int i = b0; i < b1; ++i)
            if (flag[i]) {
                if (p.offload) {  // Gamma_e starts resident: slot 1 + its place in the ascending list
                    p.slot_block[(int64_t)u * p.nslots + 1 + at] = i;
                    p.block_slot[(int64_t)u * p.nblk + i] = 1 + at;
                }
                ge[at++] = i;
            }
        if (lane == 31) {
            p.gamma_n[u] = pre;
            if (p.offload && len > 0) {
                const int32_t local = (len - 1) / kBlock;
                p.slot_block[(int64_t)u * p.nslots] = local;
                p.block_slot[(int64_t)u * p.nblk + local] = 0;
            }
            p.seq_len[u] = len;
        }
    }
    if (p.offload) {
        // copy the Gamma_e blocks from the prefill input (on the device) into their
        // cache slots: the first decode step then finds Gamma_e resident, as every
        // later step does (Gamma_e(t) lies in S(t-1) plus the previous local block)
        __syncthreads();
        const int32_t n = min(p.gamma_n[u], p.k_e);
        const int32_t *ge = p.gamma_e + (int64_t)u * p.k_e;
        constexpr int kChunks = kBlockBytes / 16, kHalfChunks = kHalfBlockBytes / 16, kRowChunks = kRowBytes / 16;
        for (int j = 0; j < n; ++j) {
            const int32_t b = ge[j];
            uint4 *dst = reinterpret_cast<uint4 *>(p.cache + ((int64_t)u * p.nslots + 1 + j) * kBlockBytes);
            for (int c = threadIdx.x; c < kChunks; c += blockDim.x) {
                const int half = c / kHalfChunks, rem = c % kHalfChunks;
                const int row = rem / kRowChunks, col = rem % kRowChunks;
                const uint16_t *src =
                    (half ? p.v_new : p.k_new) + ((int64_t)u * p.T + (int64_t)b * kBlock + row) * kD;
                dst[c] = reinterpret_cast<const uint4 *>(src)[col];
            }
        }
    }
}

int launch_append(const AppendParams &p, cudaStream_t stream) {
    if (p.T == 1 && p.w1) {
        if (cudaFuncSetAttribute(append_head_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kHeadDecSmem) != cudaSuccess)
            return NOSA_ERR_CUDA;
        return launch_pdl(append_head_decode_kernel, dim3(p.units), dim3(kHeadH), kHeadDecSmem, stream, p) ==
                       cudaSuccess
                   ? NOSA_OK
                   : NOSA_ERR_CUDA;
    }
    if (p.T == 1) {
        const int wpb = 4;
        return launch_pdl(append_decode_kernel, dim3((p.units + wpb - 1) / wpb), dim3(wpb * 32), 0, stream, p) ==
                       cudaSuccess
                   ? NOSA_OK
                   : NOSA_ERR_CUDA;
    }
    const int64_t rows = (int64_t)p.units * p.T;
    int64_t g = (rows + 7) / 8;
    if (g > 148 * 16) g = 148 * 16;
    prefill_store_kernel<<<(unsigned)g, 256, 0, stream>>>(p);
    if (p.w1) {
        if (cudaFuncSetAttribute(prefill_head_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kHeadSmem) != cudaSuccess)
            return NOSA_ERR_CUDA;
        dim3 hg((p.T + kHeadCtaRows - 1) / kHeadCtaRows, p.units);
        prefill_head_kernel<<<hg, 256, kHeadSmem, stream>>>(p);
    }
    const int64_t items = (int64_t)p.units * ((p.T + kBlock - 1) / kBlock);
    g = (items + 7) / 8;
    if (g > 148 * 16) g = 148 * 16;
    prefill_pool_kernel<<<(unsigned)g, 256, 0, stream>>>(p);
    const size_t smem = (size_t)p.nblk * (sizeof(double) + 1);
    if (smem > 48 * 1024) {
        if (cudaFuncSetAttribute(prefill_gamma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem) != cudaSuccess)
            return NOSA_ERR_CUDA;
    }
    prefill_gamma_kernel<<<p.units, 256, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NOSA_OK : NOSA_ERR_CUDA;
}

}  // namespace nosa

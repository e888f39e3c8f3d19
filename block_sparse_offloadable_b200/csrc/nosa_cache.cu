// nosa_cache.cu -- step a4: keep the device block cache equal to this step's selection.
//
// NOSA pages: montaan.com summary of arXiv:2510.13602, "System Optimization
// (NOSI)" item 2 (KV cache in block-sized units on both GPU and CPU, only
// blocks not used in the current step are swapped out) and item 3 (a custom
// host-to-device transfer kernel that reads CPU memory directly through
// Unified Virtual Addressing); gist.science summary, "Systeme : NOSI"
// (set-difference kernels for block swapping, no contiguity requirement).
//
// Two kernels.
//  * plan: one warp per unit computes the set difference against the slot
//    table (free = resident \ S(t), miss = S(t) \ resident), assigns the freed
//    slots in ascending order to the missed blocks in ascending block order,
//    writes the block table and the unit's miss list (slot, block).
//  * gather: every CTA computes the prefix sum of the per-unit miss counts and
//    copies an equal contiguous share of all missed bytes (16-byte loads through
//    the device mapping of pinned host memory, eight in flight per thread), so
//    the PCIe stream stays full until the last byte instead of trailing off with
//    the unit that missed most.
#include "nosa_internal.cuh"

namespace nosa {

namespace {
constexpr int kPlanWarps = 8;             // units per plan CTA
constexpr int kGatherThreads = 256;
constexpr int kGatherCtasPerSm = 2;
constexpr int kUnroll = 8;
constexpr int kChunksPerBlock = kBlockBytes / 16;  // 2048 16-byte chunks per block

__device__ __forceinline__ uint32_t pack_miss(int32_t slot, int32_t blk) {
    return ((uint32_t)slot << 20) | (uint32_t)blk;  // blk < 2^20 / 64, slot < 2^12
}
}  // namespace

__global__ void __launch_bounds__(kPlanWarps * 32) cache_plan_kernel(const CacheParams p) {
    pdl_trigger();  // the gather's CTAs are small; they wait for this grid
    pdl_wait();
    extern __shared__ uint32_t smem_words[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t u = blockIdx.x * kPlanWarps + warp;
    const int32_t nw = p.nblk / 32 + 1;
    uint32_t *bitmap = smem_words + warp * nw;
    int32_t *s_free = reinterpret_cast<int32_t *>(smem_words + kPlanWarps * nw) + warp * (p.nslots + 1);
    if (u >= p.units) return;

    const int32_t n = min(p.nsel[u], p.max_sel);
    const int32_t *S = p.sel + (int64_t)u * p.max_sel;
    int32_t *sb = p.slot_block + (int64_t)u * p.nslots;
    int32_t *bs = p.block_slot + (int64_t)u * p.nblk;
    uint32_t *miss_list = p.miss_list + (int64_t)u * p.max_sel;
    for (int i = lane; i < nw; i += 32) bitmap[i] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int32_t b = S[i];
        if (b >= 0 && b < p.nblk) atomicOr(&bitmap[b >> 5], 1u << (b & 31));
    }
    __syncwarp();
    // free every slot whose block is not needed this step
    for (int s = lane; s < p.nslots; s += 32) {
        const int32_t b = sb[s];
        if (b >= 0 && !((bitmap[b >> 5] >> (b & 31)) & 1u)) {
            bs[b] = -1;
            sb[s] = -1;
        }
    }
    __syncwarp();
    // free slots, ascending
    int32_t nfree = 0;
    for (int s0 = 0; s0 < p.nslots; s0 += 32) {
        const int s = s0 + lane;
        const bool fr = s < p.nslots && sb[s] < 0;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, fr);
        if (fr) s_free[nfree + __popc(m & ((1u << lane) - 1))] = s;
        nfree += __popc(m);
    }
    __syncwarp();
    // hits keep their slot; misses take the next free one
    int32_t nmiss = 0;
    int32_t *bt = p.block_table + (int64_t)u * p.max_sel;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        int32_t b = -1, slot = -1;
        if (i < n) {
            b = S[i];
            slot = (b >= 0 && b < p.nblk) ? bs[b] : -1;
        }
        const bool miss = i < n && b >= 0 && b < p.nblk && slot < 0;
        const unsigned m = __ballot_sync(0xFFFFFFFFu, miss);
        if (miss) {
            const int r = nmiss + __popc(m & ((1u << lane) - 1));
            if (r < nfree) {
                slot = s_free[r];
                bs[b] = slot;
                sb[slot] = b;
                miss_list[r] = pack_miss(slot, b);
            } else {
                set_error(p.err, NOSA_EFLAG_NOSLOT);
            }
        }
        if (i < n) bt[i] = slot;
        nmiss += __popc(m);
    }
    for (int i = n + lane; i < p.max_sel; i += 32) bt[i] = -1;
    if (lane == 0) {
        p.miss_count[u] = min(nmiss, nfree);
        if (p.n_fetched) p.n_fetched[u] = min(nmiss, nfree);
    }
}

__global__ void __launch_bounds__(kGatherThreads) cache_gather_kernel(const CacheParams p) {
    // No early trigger: the decode that follows would hold most of each SM's
    // shared memory for the whole (PCIe-bound) gather.
    pdl_wait();
    extern __shared__ int32_t P[];  // [units + 1] prefix sums of the miss counts
    __shared__ int32_t s_wsum[kGatherThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t U = p.units;
    {
        const int per = (U + kGatherThreads - 1) / kGatherThreads;
        const int u0 = min((int)threadIdx.x * per, U), u1 = min(u0 + per, U);
        int32_t sum = 0;
        for (int u = u0; u < u1; ++u) {
            const int32_t w = p.miss_count[u];
            P[u + 1] = w;
            sum += w;
        }
        int32_t incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += x;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int32_t run = incl - sum;
        for (int w = 0; w < warp; ++w) run += s_wsum[w];
        for (int u = u0; u < u1; ++u) {
            run += P[u + 1];
            P[u + 1] = run;
        }
        if (threadIdx.x == 0) P[0] = 0;
    }
    __syncthreads();
    // this CTA's share of the flattened 16-byte chunks of all missed blocks
    const int64_t total = (int64_t)P[U] * kChunksPerBlock;
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
    int64_t c = lo;
    while (c < hi) {
        // the missed block holding chunk c, and how far this CTA copies into it
        const int32_t m = (int32_t)(c / kChunksPerBlock);
        int32_t u = 0, lo_u = 0, hi_u = U;
        while (hi_u - lo_u > 1) {
            const int32_t mid = (lo_u + hi_u) >> 1;
            if (P[mid] <= m) lo_u = mid;
            else hi_u = mid;
        }
        u = lo_u;
        const uint32_t e = p.miss_list[(int64_t)u * p.max_sel + (m - P[u])];
        const int32_t slot = (int32_t)(e >> 20), blk = (int32_t)(e & 0xFFFFFu);
        const uint8_t *src = p.store + ((int64_t)u * p.nblk + blk) * kBlockBytes;
        uint8_t *dst = p.cache + ((int64_t)u * p.nslots + slot) * kBlockBytes;
        const int64_t bend = min(hi, (int64_t)(m + 1) * kChunksPerBlock);
        const int32_t k0 = (int32_t)(c - (int64_t)m * kChunksPerBlock);
        const int32_t k1 = (int32_t)(bend - (int64_t)m * kChunksPerBlock);
        for (int32_t k = k0 + threadIdx.x; k < k1; k += kGatherThreads * kUnroll) {
            uint4 v[kUnroll];
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                const int32_t kk = k + j * kGatherThreads;
                if (kk < k1) v[j] = ldcg128(src + (int64_t)kk * 16);
            }
#pragma unroll
            for (int j = 0; j < kUnroll; ++j) {
                const int32_t kk = k + j * kGatherThreads;
                if (kk < k1) *reinterpret_cast<uint4 *>(dst + (int64_t)kk * 16) = v[j];
            }
        }
        c = bend;
    }
}

int launch_cache_sync(const CacheParams &p, cudaStream_t stream) {
    const size_t plan_smem = (size_t)kPlanWarps * (((size_t)p.nblk / 32 + 1) * sizeof(uint32_t) +
                                                   ((size_t)p.nslots + 1) * sizeof(int32_t));
    if (plan_smem > 48 * 1024 &&
        cudaFuncSetAttribute(cache_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)plan_smem) != cudaSuccess)
        return NOSA_ERR_CUDA;
    if (launch_pdl(cache_plan_kernel, dim3((p.units + kPlanWarps - 1) / kPlanWarps), dim3(kPlanWarps * 32),
                   plan_smem, stream, p) != cudaSuccess)
        return NOSA_ERR_CUDA;
    const size_t gather_smem = ((size_t)p.units + 1) * sizeof(int32_t);
    return launch_pdl(cache_gather_kernel, dim3(kNumSms * kGatherCtasPerSm), dim3(kGatherThreads), gather_smem,
                      stream, p) == cudaSuccess
               ? NOSA_OK
               : NOSA_ERR_CUDA;
}

}  // namespace nosa

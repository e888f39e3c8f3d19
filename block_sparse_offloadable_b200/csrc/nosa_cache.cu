// nosa_cache.cu -- step a4: keep the device block cache equal to this step's selection.
//
// NOSA pages: montaan.com summary of arXiv:2510.13602, "System Optimization
// (NOSI)" item 2 (KV cache in block-sized units on both GPU and CPU, only
// blocks not used in the current step are swapped out) and item 3 (a custom
// host-to-device transfer kernel that reads CPU memory directly through
// Unified Virtual Addressing); gist.science summary, "Systeme : NOSI"
// (set-difference kernels for block swapping, no contiguity requirement).
//
// One CTA per unit.  Warp 0 computes the set difference against the slot
// table (free = resident \ S(t), miss = S(t) \ resident) and assigns the freed
// slots, in ascending order, to the missed blocks, in ascending block order.
// Then all 8 warps gather the missed 32 KiB blocks from the pinned host store
// with 16-byte loads through the device mapping of host memory (eight loads in
// flight per thread), which turns each warp load into a 512-byte PCIe read.
#include "nosa_internal.cuh"

namespace nosa {

namespace {
constexpr int kSyncThreads = 256;
constexpr int kMaxSel = kMaxKq + kMaxKe + 1;
constexpr int kUnroll = 8;
}

__global__ void __launch_bounds__(kSyncThreads) cache_sync_kernel(const CacheParams p) {
    extern __shared__ uint32_t bitmap[];  // nblk/32 + 1 words
    __shared__ int32_t s_free[kMaxSel + 1];
    __shared__ int32_t s_miss_slot[kMaxSel];
    __shared__ int32_t s_miss_blk[kMaxSel];
    __shared__ int32_t s_nmiss;
    const int32_t u = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 0) {
        const int32_t n = min(p.nsel[u], p.max_sel);
        const int32_t *S = p.sel + (int64_t)u * p.max_sel;
        int32_t *sb = p.slot_block + (int64_t)u * p.nslots;
        int32_t *bs = p.block_slot + (int64_t)u * p.nblk;
        const int32_t nw = p.nblk / 32 + 1;
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
                    s_miss_slot[r] = slot;
                    s_miss_blk[r] = b;
                } else {
                    set_error(p.err, NOSA_EFLAG_NOSLOT);
                }
            }
            if (i < n) bt[i] = slot;
            nmiss += __popc(m);
        }
        for (int i = n + lane; i < p.max_sel; i += 32) bt[i] = -1;
        if (lane == 0) {
            s_nmiss = min(nmiss, nfree);
            if (p.n_fetched) p.n_fetched[u] = min(nmiss, nfree);
        }
    }
    __syncthreads();

    // gather the missed blocks host -> device cache, 16 B per access
    const int32_t nmiss = s_nmiss;
    constexpr int kChunksPerBlock = kBlockBytes / 16;
    const int64_t total = (int64_t)nmiss * kChunksPerBlock;
    for (int64_t c0 = threadIdx.x; c0 < total; c0 += (int64_t)kSyncThreads * kUnroll) {
        uint4 v[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int64_t c = c0 + (int64_t)k * kSyncThreads;
            if (c < total) {
                const int32_t m = (int32_t)(c / kChunksPerBlock);
                const int64_t off = (c - (int64_t)m * kChunksPerBlock) * 16;
                v[k] = ldcg128(p.store + ((int64_t)u * p.nblk + s_miss_blk[m]) * kBlockBytes + off);
            }
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int64_t c = c0 + (int64_t)k * kSyncThreads;
            if (c < total) {
                const int32_t m = (int32_t)(c / kChunksPerBlock);
                const int64_t off = (c - (int64_t)m * kChunksPerBlock) * 16;
                *reinterpret_cast<uint4 *>(p.cache +
                                           ((int64_t)u * p.nslots + s_miss_slot[m]) * kBlockBytes +
                                           off) = v[k];
            }
        }
    }
}

int launch_cache_sync(const CacheParams &p, cudaStream_t stream) {
    const size_t smem = ((size_t)p.nblk / 32 + 1) * sizeof(uint32_t);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(cache_sync_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return NOSA_ERR_CUDA;
    cache_sync_kernel<<<p.units, kSyncThreads, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? NOSA_OK : NOSA_ERR_CUDA;
}

}  // namespace nosa

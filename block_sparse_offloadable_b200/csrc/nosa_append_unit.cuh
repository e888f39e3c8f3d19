// nosa_append_unit.cuh -- the decode-time append of one unit by one warp (step a1),
// shared by the append kernel and the fused append + select kernel.
//
// NOSA pages: montaan.com summary of arXiv:2510.13602, "Key Design Components"
// item 2 (mean pooling within sub-blocks and max pooling across them, for both
// selections) and item 1 (a block dropped by the query-agnostic selection is
// never selected by it again); gist.science summary, "ED-DMA" (selection on the
// pre-exponential eviction score).
#pragma once

#include "nosa_internal.cuh"

namespace nosa {

// Store this lane's 4 pooled-key dims (fp64 means) as fp32, or as bf16 rounded once from fp64.
__device__ __forceinline__ void store_ck(const AppendParams &p, int64_t row, int lane, double a0, double a1,
                                         double a2, double a3) {
    if (p.ck_bf16) {
        __nv_bfloat16 b0 = __double2bfloat16(a0), b1 = __double2bfloat16(a1);
        __nv_bfloat16 b2 = __double2bfloat16(a2), b3 = __double2bfloat16(a3);
        uint2 w;
        w.x = (uint32_t)*reinterpret_cast<uint16_t *>(&b0) | ((uint32_t)*reinterpret_cast<uint16_t *>(&b1) << 16);
        w.y = (uint32_t)*reinterpret_cast<uint16_t *>(&b2) | ((uint32_t)*reinterpret_cast<uint16_t *>(&b3) << 16);
        reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.ck) + row * kD)[lane] = w;
    } else {
        reinterpret_cast<float4 *>(static_cast<float *>(p.ck) + row * kD)[lane] =
            make_float4((float)a0, (float)a1, (float)a2, (float)a3);
    }
}

// Warp-cooperative argmin over Gamma_e by (E ascending, block id descending):
// the member that leaves when a better block arrives.
__device__ __forceinline__ void gamma_e_worst(const int32_t *ge, int32_t ne, const double *E,
                                              int lane, double &wE, int32_t &wid, int32_t &wpos) {
    wE = __longlong_as_double(0x7FF0000000000000ll);  // +inf
    wid = -1;
    wpos = -1;
    for (int j = lane; j < ne; j += 32) {
        int32_t id = ge[j];
        double v = E[id];
        if (v < wE || (v == wE && id > wid)) { wE = v; wid = id; wpos = j; }
    }
    for (int o = 16; o > 0; o >>= 1) {
        double oE = __shfl_xor_sync(0xFFFFFFFFu, wE, o);
        int32_t oid = __shfl_xor_sync(0xFFFFFFFFu, wid, o);
        int32_t opos = __shfl_xor_sync(0xFFFFFFFFu, wpos, o);
        bool take = (oid >= 0) && (wid < 0 || oE < wE || (oE == wE && oid > wid));
        if (take) { wE = oE; wid = oid; wpos = opos; }
    }
}

// One decode append of unit u by one warp, with the token's eviction logit e_tok.
// write_len = false leaves seq_len[u] to the caller (the fused append + select
// writes it once every CTA of the unit has read the old length), and fences the
// device-side writes before the write-through to host memory, which no one
// reads before a later kernel and which can be slow while PCIe is busy.
__device__ __forceinline__ void append_unit(const AppendParams &p, int32_t u, int lane, float e_tok,
                                            bool write_len = true) {
    const int32_t pos = p.seq_len[u];
    if (pos < 0 || pos >= p.max_ctx) {
        if (lane == 0) set_error(p.err, NOSA_EFLAG_CAPACITY);
        return;
    }
    const int32_t blk = pos >> 6, w = pos & 63;
    uint8_t *dst;
    uint8_t *host = nullptr;
    if (p.offload) {
        int32_t slot = -1;
        if (w == 0) {
            // A new local block: take the lowest free cache slot (one is always
            // left free by the previous cache sync).
            for (int s0 = 0; s0 < p.nslots && slot < 0; s0 += 32) {
                int s = s0 + lane;
                bool fr = s < p.nslots && p.slot_block[(int64_t)u * p.nslots + s] < 0;
                unsigned m = __ballot_sync(0xFFFFFFFFu, fr);
                if (m) slot = s0 + __ffs(m) - 1;
            }
            if (slot < 0) {
                if (lane == 0) set_error(p.err, NOSA_EFLAG_NOSLOT);
                return;
            }
            if (lane == 0) {
                p.slot_block[(int64_t)u * p.nslots + slot] = blk;
                p.block_slot[(int64_t)u * p.nblk + blk] = slot;
            }
        } else {
            slot = p.block_slot[(int64_t)u * p.nblk + blk];
            if (slot < 0) {
                if (lane == 0) set_error(p.err, NOSA_EFLAG_STATE);
                return;
            }
        }
        dst = p.cache + ((int64_t)u * p.nslots + slot) * kBlockBytes;
        host = p.store + ((int64_t)u * p.nblk + blk) * kBlockBytes;
    } else {
        dst = p.store + ((int64_t)u * p.nblk + blk) * kBlockBytes;
    }

    // new key row (lanes 0-15) and value row (lanes 16-31), 16 B per lane
    const int chunk = lane & 15;
    const uint16_t *src = (lane < 16 ? p.k_new : p.v_new) + (int64_t)u * kD;
    const uint4 val = reinterpret_cast<const uint4 *>(src)[chunk];
    const int64_t off = (lane < 16 ? 0 : kHalfBlockBytes) + (int64_t)w * kRowBytes + chunk * 16;
    *reinterpret_cast<uint4 *>(dst + off) = val;
    if (lane == 0) p.e_store[(int64_t)u * p.max_ctx + pos] = e_tok;

    // sub-block complete: its compressed key is the mean of its 16 keys (fp64 sum)
    if (((pos + 1) & (kSub - 1)) == 0) {
        const int32_t s = pos >> 4;
        double acc0 = 0.0, acc1 = 0.0, acc2 = 0.0, acc3 = 0.0;
        const uint8_t *rows = dst + (int64_t)(w - (kSub - 1)) * kRowBytes + lane * 8;
        for (int j = 0; j < kSub - 1; ++j) {
            const uint2 v = *reinterpret_cast<const uint2 *>(rows + (int64_t)j * kRowBytes);
            acc0 += bf16_lo(v.x); acc1 += bf16_hi(v.x);
            acc2 += bf16_lo(v.y); acc3 += bf16_hi(v.y);
        }
        const uint2 v = reinterpret_cast<const uint2 *>(p.k_new + (int64_t)u * kD)[lane];
        acc0 += bf16_lo(v.x); acc1 += bf16_hi(v.x);
        acc2 += bf16_lo(v.y); acc3 += bf16_hi(v.y);
        store_ck(p, (int64_t)u * p.nsub + s, lane, acc0 / kSub, acc1 / kSub, acc2 / kSub, acc3 / kSub);
    }

    // block complete: E_b = max over its sub-blocks of the mean eviction logit (fp64)
    if (((pos + 1) & (kBlock - 1)) == 0) {
        double m = -__longlong_as_double(0x7FF0000000000000ll);
        if (lane < kSubPerBlock) {
            const float *e = p.e_store + (int64_t)u * p.max_ctx + (int64_t)blk * kBlock + lane * kSub;
            double acc = 0.0;
            for (int j = 0; j < kSub; ++j)
                acc += (double)((lane == kSubPerBlock - 1 && j == kSub - 1) ? e_tok : e[j]);
            m = acc / kSub;
        }
        m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
        m = fmax(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
        if (lane == 0) p.blk_evict[(int64_t)u * p.nblk + blk] = m;
    }

    // fill reading: the new candidate joins the pool at its rank (E descending;
    // it has the highest id, so it goes after every member with an equal E)
    if (p.fill && w == 0 && blk >= 1 && p.k_e > 0) {
        const int32_t c = blk - 1;
        int32_t *pool = p.pool + (int64_t)u * p.nblk;
        const double *E = p.blk_evict + (int64_t)u * p.nblk;
        const int32_t n = p.pool_n[u];
        const double Ec = E[c];
        int32_t at = 0;
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            at += __popc(__ballot_sync(0xFFFFFFFFu, i < n && E[pool[i]] >= Ec));
        }
        // shift [at, n) up by one, highest chunk first; each chunk is read before it is written
        for (int top = n; top > at; top -= 32) {
            const int i = top - 1 - lane;
            const int32_t v = (i >= at) ? pool[i] : 0;
            __syncwarp();
            if (i >= at) pool[i + 1] = v;
            __syncwarp();
        }
        if (lane == 0) {
            pool[at] = c;
            p.pool_n[u] = n + 1;
        }
    }

    // the previous local block just became a candidate: offer it to Gamma_e
    if (!p.fill && w == 0 && blk >= 1 && p.k_e > 0) {
        const int32_t c = blk - 1;
        int32_t *ge = p.gamma_e + (int64_t)u * p.k_e;
        const double *E = p.blk_evict + (int64_t)u * p.nblk;
        const int32_t ne = p.gamma_n[u];
        if (ne < p.k_e) {
            if (lane == 0) {
                ge[ne] = c;  // c is the largest id: the list stays ascending
                p.gamma_n[u] = ne + 1;
            }
        } else {
            double wE;
            int32_t wid, wpos;
            gamma_e_worst(ge, ne, E, lane, wE, wid, wpos);
            // c has the highest index, so it loses ties: it must be strictly better
            if (wid >= 0 && E[c] > wE) {
                int32_t keep[kMaxKe / 32];
#pragma unroll
                for (int i = 0; i < kMaxKe / 32; ++i) {
                    int j = lane + 32 * i;
                    keep[i] = (j < ne) ? ((j < wpos) ? ge[j] : (j + 1 < ne ? ge[j + 1] : c)) : -1;
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < kMaxKe / 32; ++i) {
                    int j = lane + 32 * i;
                    if (j < ne) ge[j] = keep[i];
                }
            }
        }
    }
    if (write_len && lane == 0) p.seq_len[u] = pos + 1;
    if (!write_len) __threadfence();  // the fused caller hands off to another CTA next
    if (host) *reinterpret_cast<uint4 *>(host + off) = val;  // write-through over PCIe, last
}

}  // namespace nosa

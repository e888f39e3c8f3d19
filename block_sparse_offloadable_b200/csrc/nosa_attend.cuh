// nosa_attend.cuh -- the consumer side of the attention kernels (steps a5, a6 and the fused step):
// the per-warp attention of one staged block and the merges of softmax states.
//
// NOSA pages: gist.science summary of arXiv:2510.13602, "ED-DMA" (the exponent of
// the eviction score is deferred to the attention step: it enters the softmax as
// the additive logit e_j); wmrh.cn NOSA-1B release (exact attention over the
// selected blocks plus the current window).
//
// Consumers are two groups of four warps taking alternate staged blocks; warp w of
// a group owns tokens 16w..16w+15 of a block.  S^T = K Q^T is one m16n8k16 bf16
// tile per 16 dims (M = 16 tokens, N = the <= 8 query heads of the kv head, so
// each K/V byte is read once for all heads); online softmax per head in the log2
// domain; P is rounded to bf16, transposed in registers with movmatrix, and
// O^T += V^T P^T runs as eight more m16n8k16 tiles.  A unit's states end in a
// shared-memory merge of the eight warps, then, when several CTAs share the unit,
// in a merge of their partial (m, l, o) records by the last one to finish.
#pragma once

#include "nosa_internal.cuh"

namespace nosa {

constexpr int kDecW = 4;                  // warps per consumer group (16 tokens of a block each)
constexpr int kGroups = 2;                // consumer groups, taking alternate blocks
constexpr int kConsWarps = kDecW * kGroups;
constexpr int kBoxBytes = 64 * 128;       // one TMA box: 64 rows x 64 bf16
constexpr int kDecThreads = (kConsWarps + 1) * 32;
constexpr int kConsThreads = kConsWarps * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();
// Merge scratch per warp: m[8], l[8], o[8][kHS] with a padded head row and bit 0 of the
// dim XOR-ed with bit 5, so the fragment-order stores of a warp hit 32 distinct banks.
constexpr int kHS = kD + 1;
constexpr int kScr = 2 * kMaxG + kMaxG * kHS;
// Units split into at most this many pieces are merged by their last piece in one pass; with at
// most kFewPieces, all of a thread's loads are issued before any of them is used.
constexpr int kOnePassPieces = 16;
constexpr int kFewPieces = 4;
__device__ __forceinline__ int swz(int x) { return x ^ ((x >> 5) & 1); }

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsThreads) : "memory");
}

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              uint32_t *err) {
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    set_error(err, NOSA_EFLAG_TIMEOUT);
    return false;
}

// Per-lane online-softmax state of one consumer warp (heads 2c, 2c+1 of the group).
struct WarpState {
    float o[8][4];
    float m0, m1, l0, l1;
    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int t = 0; t < 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
        m0 = m1 = kNegInf;
        l0 = l1 = 0.f;
    }
};

// Attention of this warp's 16 tokens of one staged block.
__device__ __forceinline__ void attend_block(WarpState &st, const uint32_t (&qf)[8][2], const uint8_t *t,
                                             const float *eb, int32_t lb, int32_t L, float qk_log2,
                                             int warp, int c, int sig) {
    const int rowA = warp * 16 + sig, rowB = rowA + 8;   // key rows of C rows r, r+8
    const int vt0 = warp * 16 + c;                        // value rows of k = 2c, 2c+1, 2c+8, 2c+9
    const int off0 = ((sig ^ c) << 4), off1 = ((sig ^ (c + 4)) << 4);
    // ---- S^T (16 tokens x 8 heads) = K Q^T, two independent accumulation chains ----
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
    float sacc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint8_t *box = t + (j >> 1) * kBoxBytes;
        const int sw = (((j & 1) << 2) + c) ^ sig;
        const uint4 ka = lds128(box + rowA * 128 + (sw << 4));
        const uint4 kb = lds128(box + rowB * 128 + (sw << 4));
        const uint32_t a0[4] = {ka.x, kb.x, ka.y, kb.y};
        const uint32_t a1[4] = {ka.z, kb.z, ka.w, kb.w};
        mma_16816(sacc, a0, qf[2 * j]);
        mma_16816(sacc2, a1, qf[2 * j + 1]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) sacc[x] += sacc2[x];
    // ---- online softmax over the 16 tokens, per head (2c, 2c+1) ----
    const int64_t posA = (int64_t)lb * kBlock + rowA, posB = posA + 8;
    const float eA = eb[rowA] * kLog2e, eB = eb[rowB] * kLog2e;
    const float x0 = posA < L ? fmaf(sacc[0], qk_log2, eA) : kNegInf;
    const float x1 = posA < L ? fmaf(sacc[1], qk_log2, eA) : kNegInf;
    const float x2 = posB < L ? fmaf(sacc[2], qk_log2, eB) : kNegInf;
    const float x3 = posB < L ? fmaf(sacc[3], qk_log2, eB) : kNegInf;
    float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
    for (int sh = 4; sh < 32; sh <<= 1) {
        bm0 = fmaxf(bm0, __shfl_xor_sync(0xFFFFFFFFu, bm0, sh));
        bm1 = fmaxf(bm1, __shfl_xor_sync(0xFFFFFFFFu, bm1, sh));
    }
    const float mn0 = fmaxf(st.m0, bm0), mn1 = fmaxf(st.m1, bm1);
    const float c0 = (mn0 == kNegInf) ? 1.f : exp2f(st.m0 - mn0);
    const float c1 = (mn1 == kNegInf) ? 1.f : exp2f(st.m1 - mn1);
    const float p0 = (mn0 == kNegInf) ? 0.f : exp2f(x0 - mn0);
    const float p1 = (mn1 == kNegInf) ? 0.f : exp2f(x1 - mn1);
    const float p2 = (mn0 == kNegInf) ? 0.f : exp2f(x2 - mn0);
    const float p3 = (mn1 == kNegInf) ? 0.f : exp2f(x3 - mn1);
    st.m0 = mn0;
    st.m1 = mn1;
    const uint32_t plo = pack_bf16x2(p0, p1), phi = pack_bf16x2(p2, p3);
    st.l0 = fmaf(st.l0, c0, bf16_lo(plo) + bf16_lo(phi));
    st.l1 = fmaf(st.l1, c1, bf16_hi(plo) + bf16_hi(phi));
#pragma unroll
    for (int tt = 0; tt < 8; ++tt) {
        st.o[tt][0] *= c0; st.o[tt][1] *= c1;
        st.o[tt][2] *= c0; st.o[tt][3] *= c1;
    }
    const uint32_t pb[2] = {movmatrix_trans(plo), movmatrix_trans(phi)};
    // ---- O^T (128 dims x 8 heads) += V^T P^T ----
    const bool partial = (int64_t)lb * kBlock + kBlock > L;
#pragma unroll
    for (int bx = 0; bx < 2; ++bx) {
        const uint8_t *vb = t + (2 + bx) * kBoxBytes;
        uint4 v0 = lds128(vb + (vt0 + 0) * 128 + off0);
        uint4 v1 = lds128(vb + (vt0 + 4) * 128 + off1);
        uint4 v2 = lds128(vb + (vt0 + 8) * 128 + off0);
        uint4 v3 = lds128(vb + (vt0 + 12) * 128 + off1);
        if (partial) {  // rows at or beyond L hold stale bits: keep them out of 0 * x
            const int64_t b0 = (int64_t)lb * kBlock + vt0;
            const uint4 z = make_uint4(0, 0, 0, 0);
            if (b0 >= L) v0 = z;
            if (b0 + 4 >= L) v1 = z;
            if (b0 + 8 >= L) v2 = z;
            if (b0 + 12 >= L) v3 = z;
        }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint32_t x = word(v0, wi), y = word(v1, wi);
            const uint32_t x2 = word(v2, wi), y2 = word(v3, wi);
            const uint32_t a[4] = {__byte_perm(x, y, 0x5410), __byte_perm(x, y, 0x7632),
                                   __byte_perm(x2, y2, 0x5410), __byte_perm(x2, y2, 0x7632)};
            mma_16816(st.o[4 * bx + wi], a, pb);
        }
    }
}

__device__ __forceinline__ void store_bf16(uint16_t *dst, float v) {
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    *dst = *reinterpret_cast<uint16_t *>(&b);
}


// Segment end, first half: group 0 folds its per-lane states into group 1's, lane by lane, and
// each warp of group 1 leaves the folded (m, l, o) of its 16-token slice in its scratch slot
// (padded, swizzled layout).  Called by every consumer thread; two consumer barriers inside.
__device__ __forceinline__ void fold_groups(const WarpState &st, float *scratch, int grp, int wq, int r, int c,
                                            int sig) {
    float l0 = st.l0, l1 = st.l1;
#pragma unroll
    for (int sh = 4; sh < 32; sh <<= 1) {
        l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, sh);
        l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, sh);
    }
    float *mine = scratch + wq * kScr;
    float *oo = mine + 2 * kMaxG;
    if (grp == 0) {
        if (r == 0) {
            mine[2 * c] = st.m0; mine[2 * c + 1] = st.m1;
            mine[kMaxG + 2 * c] = l0; mine[kMaxG + 2 * c + 1] = l1;
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int psi = 64 * (t >> 2) + 8 * sig + 2 * (t & 3);
            oo[(2 * c) * kHS + swz(psi)] = st.o[t][0];
            oo[(2 * c + 1) * kHS + swz(psi)] = st.o[t][1];
            oo[(2 * c) * kHS + swz(psi + 1)] = st.o[t][2];
            oo[(2 * c + 1) * kHS + swz(psi + 1)] = st.o[t][3];
        }
    }
    consumer_sync();
    if (grp == 1) {
        const float ma0 = mine[2 * c], ma1 = mine[2 * c + 1];
        const float la0 = mine[kMaxG + 2 * c], la1 = mine[kMaxG + 2 * c + 1];
        const float M0 = fmaxf(ma0, st.m0), M1 = fmaxf(ma1, st.m1);
        const float fa0 = (ma0 == kNegInf) ? 0.f : exp2f(ma0 - M0);
        const float fa1 = (ma1 == kNegInf) ? 0.f : exp2f(ma1 - M1);
        const float fb0 = (st.m0 == kNegInf) ? 0.f : exp2f(st.m0 - M0);
        const float fb1 = (st.m1 == kNegInf) ? 0.f : exp2f(st.m1 - M1);
        float om[8][4];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int psi = 64 * (t >> 2) + 8 * sig + 2 * (t & 3);
            om[t][0] = fmaf(fa0, oo[(2 * c) * kHS + swz(psi)], fb0 * st.o[t][0]);
            om[t][1] = fmaf(fa1, oo[(2 * c + 1) * kHS + swz(psi)], fb1 * st.o[t][1]);
            om[t][2] = fmaf(fa0, oo[(2 * c) * kHS + swz(psi + 1)], fb0 * st.o[t][2]);
            om[t][3] = fmaf(fa1, oo[(2 * c + 1) * kHS + swz(psi + 1)], fb1 * st.o[t][3]);
        }
        __syncwarp();  // every lane has read m, l before lanes r == 0 overwrite them
        if (r == 0) {
            mine[2 * c] = M0; mine[2 * c + 1] = M1;
            mine[kMaxG + 2 * c] = fmaf(fa0, la0, fb0 * l0);
            mine[kMaxG + 2 * c + 1] = fmaf(fa1, la1, fb1 * l1);
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int psi = 64 * (t >> 2) + 8 * sig + 2 * (t & 3);
            oo[(2 * c) * kHS + swz(psi)] = om[t][0];
            oo[(2 * c + 1) * kHS + swz(psi)] = om[t][1];
            oo[(2 * c) * kHS + swz(psi + 1)] = om[t][2];
            oo[(2 * c + 1) * kHS + swz(psi + 1)] = om[t][3];
        }
    }
    consumer_sync();
}

// Segment end, second half, for head h and dim d: the four warps' slices merged into (M, acc, lsum),
// the state of the whole segment (acc / lsum is its output).
__device__ __forceinline__ void merged_state(const float *scratch, int h, int d, float &M, float &acc, float &lsum) {
    M = kNegInf;
#pragma unroll
    for (int w = 0; w < kDecW; ++w) M = fmaxf(M, scratch[w * kScr + h]);
    acc = 0.f;
    lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kDecW; ++w) {
        const float mw = scratch[w * kScr + h];
        const float f = (mw == kNegInf) ? 0.f : exp2f(mw - M);
        acc = fmaf(f, scratch[w * kScr + 2 * kMaxG + h * kHS + swz(d)], acc);
        lsum = fmaf(f, scratch[w * kScr + kMaxG + h], lsum);
    }
}

// Write the partial record (m[8], l[8], o[8][128]) of head h, dim d.
__device__ __forceinline__ void store_partial(float *part, int h, int d, float M, float acc, float lsum) {
    part[2 * kMaxG + h * kD + d] = acc;
    if (d == 0) {
        part[h] = M;
        part[kMaxG + h] = lsum;
    }
}

__device__ __forceinline__ uint2 pack_out4(float4 acc, float ls) {
    uint2 pk;
    if (ls > 0.f) {
        pk.x = pack_bf16x2(acc.x / ls, acc.y / ls);
        pk.y = pack_bf16x2(acc.z / ls, acc.w / ls);
    } else {
        pk.x = pk.y = 0u;
    }
    return pk;
}

// The last of C <= kOnePassPieces pieces of a unit merges their partial records, piece t at
// src0 + t * stride, in piece order, in one pass: each consumer thread takes 4 dims of one head
// and issues its loads at once (all of them with at most kAtOnce pieces: one round trip; more
// registers).  Writes bf16 out.
template <int kAtOnce = kFewPieces>
__device__ __forceinline__ void merge_pieces_onepass(const float *src0, int64_t stride, int C, int G, uint16_t *out,
                                                     int ctid) {
    static_assert(kAtOnce <= kOnePassPieces, "at most kOnePassPieces pieces");
    for (int v = ctid; v < G * (kD / 4); v += kConsThreads) {
        const int h = v / (kD / 4), d4 = (v % (kD / 4)) * 4;
        float mt[kOnePassPieces];
        float ls = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (C <= kAtOnce) {
            // few pieces: every load at once, one round trip
            float lt[kAtOnce];
            float4 ot[kAtOnce];
#pragma unroll
            for (int t = 0; t < kAtOnce; ++t) {
                const float *st_t = src0 + (int64_t)t * stride;
                mt[t] = t < C ? __ldcg(st_t + h) : kNegInf;
                lt[t] = t < C ? __ldcg(st_t + kMaxG + h) : 0.f;
                ot[t] = t < C ? __ldcg(reinterpret_cast<const float4 *>(st_t + 2 * kMaxG + h * kD + d4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float M = kNegInf;
#pragma unroll
            for (int t = 0; t < kAtOnce; ++t) M = fmaxf(M, mt[t]);
#pragma unroll
            for (int t = 0; t < kAtOnce; ++t) {
                if (t < C) {
                    const float f = (mt[t] == kNegInf) ? 0.f : exp2f(mt[t] - M);
                    ls = fmaf(f, lt[t], ls);
                    acc.x = fmaf(f, ot[t].x, acc.x); acc.y = fmaf(f, ot[t].y, acc.y);
                    acc.z = fmaf(f, ot[t].z, acc.z); acc.w = fmaf(f, ot[t].w, acc.w);
                }
            }
        } else {
#pragma unroll
            for (int t = 0; t < kOnePassPieces; ++t) mt[t] = t < C ? __ldcg(src0 + (int64_t)t * stride + h) : kNegInf;
            float M = kNegInf;
#pragma unroll
            for (int t = 0; t < kOnePassPieces; ++t) M = fmaxf(M, mt[t]);
#pragma unroll
            for (int t = 0; t < kOnePassPieces; ++t) {
                if (t < C) {
                    const float *st_t = src0 + (int64_t)t * stride;
                    const float f = (mt[t] == kNegInf) ? 0.f : exp2f(mt[t] - M);
                    const float4 o4 = __ldcg(reinterpret_cast<const float4 *>(st_t + 2 * kMaxG + h * kD + d4));
                    ls = fmaf(f, __ldcg(st_t + kMaxG + h), ls);
                    acc.x = fmaf(f, o4.x, acc.x); acc.y = fmaf(f, o4.y, acc.y);
                    acc.z = fmaf(f, o4.z, acc.z); acc.w = fmaf(f, o4.w, acc.w);
                }
            }
        }
        *reinterpret_cast<uint2 *>(out + h * kD + d4) = pack_out4(acc, ls);
    }
}

// Merge of nc partial records of one unit, any count, in the order of src[]: the scratch holds
// the weight of each record per head, the merged denominators and maxima, and the nc record
// pointers (which the caller fills, then passes a consumer barrier).
struct MergeScratch {
    float *fac;         // [nc][8]
    float *lsum;        // [8]
    float *Ms;          // [8]
    const float **src;  // [nc]
};

__device__ __forceinline__ MergeScratch merge_scratch(float *scratch, int nc) {
    MergeScratch m;
    m.fac = scratch;
    m.lsum = m.fac + nc * kMaxG;
    m.Ms = m.lsum + kMaxG;
    m.src = reinterpret_cast<const float **>(scratch + ((nc * kMaxG + 2 * kMaxG + 1) & ~1));
    return m;
}

// One warp per head finds the weights, then each consumer thread combines 4 dims of one head.
// res == nullptr: writes the bf16 output; otherwise the merged record (the split decode's state).
__device__ __forceinline__ void merge_general(const MergeScratch &ms, int nc, int G, uint16_t *out, float *res,
                                             int warp, int lane, int ctid) {
    for (int h = warp; h < G; h += kConsWarps) {
        float M = kNegInf;
        for (int t = lane; t < nc; t += 32) M = fmaxf(M, __ldcg(ms.src[t] + h));
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, sh));
        float ls = 0.f;
        for (int t = lane; t < nc; t += 32) {
            const float mc = __ldcg(ms.src[t] + h);
            const float f = (mc == kNegInf) ? 0.f : exp2f(mc - M);
            ms.fac[t * kMaxG + h] = f;
            ls = fmaf(f, __ldcg(ms.src[t] + kMaxG + h), ls);
        }
#pragma unroll
        for (int sh = 16; sh > 0; sh >>= 1) ls += __shfl_xor_sync(0xFFFFFFFFu, ls, sh);
        if (lane == 0) {
            ms.lsum[h] = ls;
            ms.Ms[h] = M;
        }
    }
    consumer_sync();
    for (int v = ctid; v < G * (kD / 4); v += kConsThreads) {  // 4 dims per thread
        const int h = v / (kD / 4), d4 = (v % (kD / 4)) * 4;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int t = 0; t < nc; ++t) {
            const float f = ms.fac[t * kMaxG + h];
            const float4 o4 = __ldcg(reinterpret_cast<const float4 *>(ms.src[t] + 2 * kMaxG + h * kD + d4));
            acc.x = fmaf(f, o4.x, acc.x); acc.y = fmaf(f, o4.y, acc.y);
            acc.z = fmaf(f, o4.z, acc.z); acc.w = fmaf(f, o4.w, acc.w);
        }
        const float ls = ms.lsum[h];
        if (res) {
            *reinterpret_cast<float4 *>(res + 2 * kMaxG + h * kD + d4) = acc;
            if (d4 == 0) {
                res[h] = ms.Ms[h];
                res[kMaxG + h] = ls;
            }
            continue;
        }
        *reinterpret_cast<uint2 *>(out + h * kD + d4) = pack_out4(acc, ls);
    }
}

}  // namespace nosa

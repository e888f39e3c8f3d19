// nosa_decode.cu -- steps a5 (sparse decode) and a6 (dense comparator).
//
// NOSA pages: gist.science summary of arXiv:2510.13602, "ED-DMA" (the
// exponential of the eviction score is deferred to the attention step: here
// it enters the softmax as the additive logit e_j); wmrh.cn NOSA-1B release
// (exact attention over the Top-K blocks plus the current window).
//
// Design (split-K flash decoding with GQA sharing, per unit = (seq, kv head)):
//  * grid = (chunks, units), the chunk count chosen against wave quantisation;
//    a CTA takes a balanced, contiguous range of the
//    unit's selected blocks (or of all blocks for the dense comparator).
//  * One producer thread streams every selected block (keys + values, 32 KiB,
//    plus its 64 eviction logits) into a 3-stage shared-memory ring (two CTAs
//    per SM, so six blocks in flight per SM): four
//    2-D TMA tile loads (64 rows x 64 dims, 128-byte swizzle) and one bulk
//    copy per block, completing on the stage's mbarrier.
//  * Four consumer warps each own 16 of the block's 64 tokens.  S^T = K Q^T is
//    one m16n8k16 bf16 tensor-core tile per 16 dims (M = 16 tokens, N = the
//    <= 8 query heads of the group, so each K/V byte is read once for all
//    heads).  Key rows are read straight into A fragments with one 16-byte
//    shared load per lane per 32 dims: the dims are permuted consistently in
//    K and Q (a dot product does not care), and the token rows each lane
//    loads are permuted (0,4,1,5,2,6,3,7) so that, with the TMA swizzle,
//    every quarter-warp hits 8 distinct bank groups.
//  * Online softmax per head in the log2 domain; P is rounded to bf16,
//    transposed in registers with movmatrix, and O^T += V^T P^T runs as eight
//    more m16n8k16 tiles whose A fragments are built from 16-byte value loads
//    with byte permutes (output dims permuted, undone at the store).
//  * The four warps' (m, l, o) states merge in shared memory; with several
//    chunks per unit the partial states go to the workspace and the last CTA
//    of the unit (atomic counter, no waiting) merges them and writes bf16.
#include "nosa_internal.cuh"

namespace nosa {

namespace {
constexpr int kDecW = 4;                  // consumer warps (16 tokens each)
constexpr int kDecS = 3;                  // ring stages (one block each); two CTAs per SM
constexpr int kBoxBytes = 64 * 128;       // one TMA box: 64 rows x 64 bf16
constexpr int kDecThreads = (kDecW + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr int kCtaPerSm = 2;

// Every consumer warp consumes every stage, in order, so mbarrier waiters see
// their phases in order (parity waits cannot tell phase p from p + 2).
size_t decode_smem_bytes(int32_t max_nb) {
    return 1024 + (size_t)kDecS * kBlockBytes + (size_t)kDecS * kBlock * sizeof(float) +
           2 * kDecS * sizeof(uint64_t) + kDecS * sizeof(int32_t) + 2 * (size_t)max_nb * sizeof(int32_t);
}

__device__ __forceinline__ uint32_t word(const uint4 &v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}
}  // namespace

int decode_chunks(int32_t units, int32_t max_blocks) {
    // per-CTA fixed cost ~ 3 blocks (first TMA round trip, the partial merge)
    return best_chunks(units, max_blocks, (int64_t)kNumSms * kCtaPerSm, 3, max_blocks / 4);
}

__global__ void __launch_bounds__(kDecThreads, kCtaPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *ebuf = reinterpret_cast<float *>(tiles + kDecS * kBlockBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(ebuf + kDecS * kBlock);
    uint64_t *empty = full + kDecS;
    int32_t *s_blk = reinterpret_cast<int32_t *>(empty + kDecS);
    int32_t *s_lid = s_blk + kDecS;         // this CTA's logical block ids
    int32_t *s_pid = s_lid + p.max_nb;      // and their physical (store or cache) blocks
    __shared__ int s_last;

    const int32_t u = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t L = p.seq_len[u];
    int32_t nblocks = p.sel ? min(p.nsel[u], p.max_sel) : (L + kBlock - 1) / kBlock;
    if (L <= 0 || nblocks < 0) nblocks = 0;
    const int32_t i0 = (int32_t)((int64_t)chunk * nblocks / p.nchunks);
    const int32_t i1 = (int32_t)((int64_t)(chunk + 1) * nblocks / p.nchunks);
    const int32_t nb = min(i1 - i0, p.max_nb);  // i1 - i0 <= ceil(max blocks / nchunks) < max_nb

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecW);
        }
        fence_mbar_init();
        prefetch_tmap(&tmap);
    }
    __syncthreads();

    if (warp == kDecW) {
        // ---------------- producer ----------------
        // fetch the CTA's block ids once, 32 at a time, so no global load sits
        // between consecutive TMA issues
        {
            const int32_t *selu = p.sel ? p.sel + (int64_t)u * p.max_sel : nullptr;
            const int32_t *btu = p.block_table ? p.block_table + (int64_t)u * p.max_sel : nullptr;
            for (int i = lane; i < nb; i += 32) {
                const int32_t idx = i0 + i;
                const int32_t lb = selu ? selu[idx] : idx;
                s_lid[i] = lb;
                s_pid[i] = btu ? btu[idx] : lb;
            }
            __syncwarp();
        }
        if (lane == 0) {
            for (int i = 0; i < nb; ++i) {
                const int s = i % kDecS;
                if (i >= kDecS && !mbar_wait(&empty[s], ((i / kDecS) - 1) & 1)) {
                    set_error(p.err, NOSA_EFLAG_TIMEOUT);
                    break;
                }
                const int32_t lb = s_lid[i];
                const int32_t pb = s_pid[i];
                const bool ok = lb >= 0 && (int64_t)lb * kBlock < p.max_ctx && pb >= 0 &&
                                pb < p.blocks_per_unit;
                s_blk[s] = ok ? lb : -1;
                if (ok) {
                    const int32_t y = (int32_t)(((int64_t)u * p.blocks_per_unit + pb) * 2 * kBlock);
                    uint8_t *t = tiles + s * kBlockBytes;
                    mbar_arrive_expect_tx(&full[s], kBlockBytes + kBlock * sizeof(float));
                    tma_load_2d(t, &tmap, &full[s], 0, y);
                    tma_load_2d(t + kBoxBytes, &tmap, &full[s], 64, y);
                    tma_load_2d(t + 2 * kBoxBytes, &tmap, &full[s], 0, y + kBlock);
                    tma_load_2d(t + 3 * kBoxBytes, &tmap, &full[s], 64, y + kBlock);
                    bulk_load(ebuf + s * kBlock, p.e + (int64_t)u * p.max_ctx + (int64_t)lb * kBlock,
                              kBlock * sizeof(float), &full[s]);
                } else {
                    mbar_arrive(&full[s]);
                }
            }
            for (int i = max(0, nb - kDecS); i < nb; ++i)
                if (!mbar_wait(&full[i % kDecS], (i / kDecS) & 1)) set_error(p.err, NOSA_EFLAG_TIMEOUT);
        }
    }

    // per-lane fragment coordinates
    const int r = lane >> 2, c = lane & 3;
    const int sig = (r >> 1) + ((r & 1) << 2);  // row permutation 0,4,1,5,2,6,3,7
    float o[8][4];
#pragma unroll
    for (int t = 0; t < 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    float m0 = kNegInf, m1 = kNegInf, l0 = 0.f, l1 = 0.f;

    if (warp < kDecW) {
        // ---------------- consumers ----------------
        uint32_t qf[8][2];
        {
            const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((int64_t)u * p.G + r) * kD);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 x = (r < p.G) ? qrow[4 * j + c] : make_uint4(0, 0, 0, 0);
                qf[2 * j][0] = x.x; qf[2 * j][1] = x.y;
                qf[2 * j + 1][0] = x.z; qf[2 * j + 1][1] = x.w;
            }
        }
        const int rowA = warp * 16 + sig, rowB = rowA + 8;  // key rows of C rows r, r+8
        const int vt0 = warp * 16 + c;                        // value rows of k = 2c, 2c+1, 2c+8, 2c+9
        const int off0 = ((sig ^ c) << 4), off1 = ((sig ^ (c + 4)) << 4);

        for (int i = 0; i < nb; ++i) {
            const int s = i % kDecS;
            if (!mbar_wait(&full[s], (i / kDecS) & 1)) {
                set_error(p.err, NOSA_EFLAG_TIMEOUT);
                break;
            }
            const int32_t lb = s_blk[s];
            if (lb >= 0) {
                const uint8_t *t = tiles + s * kBlockBytes;
                // ---- S^T (16 tokens x 8 heads) = K Q^T ----
                // two independent accumulation chains halve the serial mma latency
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
                // ---- online softmax over this block's 16 tokens, per head (2c, 2c+1) ----
                const float *eb = ebuf + s * kBlock;
                const int64_t posA = (int64_t)lb * kBlock + rowA, posB = posA + 8;
                const float eA = eb[rowA] * kLog2e, eB = eb[rowB] * kLog2e;
                const float x0 = posA < L ? fmaf(sacc[0], p.qk_log2, eA) : kNegInf;
                const float x1 = posA < L ? fmaf(sacc[1], p.qk_log2, eA) : kNegInf;
                const float x2 = posB < L ? fmaf(sacc[2], p.qk_log2, eB) : kNegInf;
                const float x3 = posB < L ? fmaf(sacc[3], p.qk_log2, eB) : kNegInf;
                float bm0 = fmaxf(x0, x2), bm1 = fmaxf(x1, x3);
#pragma unroll
                for (int sh = 4; sh < 32; sh <<= 1) {
                    bm0 = fmaxf(bm0, __shfl_xor_sync(0xFFFFFFFFu, bm0, sh));
                    bm1 = fmaxf(bm1, __shfl_xor_sync(0xFFFFFFFFu, bm1, sh));
                }
                const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
                const float c0 = (mn0 == kNegInf) ? 1.f : exp2f(m0 - mn0);
                const float c1 = (mn1 == kNegInf) ? 1.f : exp2f(m1 - mn1);
                const float p0 = (mn0 == kNegInf) ? 0.f : exp2f(x0 - mn0);
                const float p1 = (mn1 == kNegInf) ? 0.f : exp2f(x1 - mn1);
                const float p2 = (mn0 == kNegInf) ? 0.f : exp2f(x2 - mn0);
                const float p3 = (mn1 == kNegInf) ? 0.f : exp2f(x3 - mn1);
                m0 = mn0;
                m1 = mn1;
                const uint32_t plo = pack_bf16x2(p0, p1), phi = pack_bf16x2(p2, p3);
                l0 = fmaf(l0, c0, bf16_lo(plo) + bf16_lo(phi));
                l1 = fmaf(l1, c1, bf16_hi(plo) + bf16_hi(phi));
#pragma unroll
                for (int tt = 0; tt < 8; ++tt) {
                    o[tt][0] *= c0; o[tt][1] *= c1;
                    o[tt][2] *= c0; o[tt][3] *= c1;
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
                    if (partial) {  // rows at or beyond L hold stale bits: keep them out of 0*x
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
                                               __byte_perm(x2, y2, 0x5410),
                                               __byte_perm(x2, y2, 0x7632)};
                        mma_16816(o[4 * bx + wi], a, pb);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // full l per head: sum over the 8 lanes that share c
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) {
            l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, sh);
            l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, sh);
        }
    }
    __syncthreads();  // ring no longer in use: reuse it as merge scratch

    float *scr = reinterpret_cast<float *>(tiles);
    if (warp < kDecW) {
        float *mine = scr + warp * kPartFloats;
        if (r == 0) {
            mine[2 * c] = m0; mine[2 * c + 1] = m1;
            mine[kMaxG + 2 * c] = l0; mine[kMaxG + 2 * c + 1] = l1;
        }
        float *oo = mine + 2 * kMaxG;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int psi = 64 * (t >> 2) + 8 * sig + 2 * (t & 3);
            oo[(2 * c) * kD + psi] = o[t][0];
            oo[(2 * c + 1) * kD + psi] = o[t][1];
            oo[(2 * c) * kD + psi + 1] = o[t][2];
            oo[(2 * c + 1) * kD + psi + 1] = o[t][3];
        }
    }
    __syncthreads();

    const int nout = p.G * kD;
    uint16_t *out = p.out + (int64_t)u * p.G * kD;
    float *part = p.part + ((int64_t)u * p.nchunks + chunk) * kPartFloats;
    for (int idx = threadIdx.x; idx < nout; idx += kDecThreads) {
        const int h = idx >> 7, d = idx & (kD - 1);
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < kDecW; ++w) M = fmaxf(M, scr[w * kPartFloats + h]);
        float acc = 0.f, lsum = 0.f;
#pragma unroll
        for (int w = 0; w < kDecW; ++w) {
            const float mw = scr[w * kPartFloats + h];
            const float f = (mw == kNegInf) ? 0.f : exp2f(mw - M);
            acc = fmaf(f, scr[w * kPartFloats + 2 * kMaxG + h * kD + d], acc);
            lsum = fmaf(f, scr[w * kPartFloats + kMaxG + h], lsum);
        }
        if (p.nchunks == 1) {
            const float v = lsum > 0.f ? acc / lsum : 0.f;
            __nv_bfloat16 b = __float2bfloat16_rn(v);
            out[idx] = *reinterpret_cast<uint16_t *>(&b);
        } else {
            part[2 * kMaxG + h * kD + d] = acc;
            if (d == 0) {
                part[h] = M;
                part[kMaxG + h] = lsum;
            }
        }
    }
    if (p.nchunks == 1) return;

    // ---- split-K merge by the last CTA of this unit ----
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(&p.counter[u], 1) == p.nchunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) p.counter[u] = 0;
    const float *parts = p.part + (int64_t)u * p.nchunks * kPartFloats;
    for (int idx = threadIdx.x; idx < nout; idx += kDecThreads) {
        const int h = idx >> 7, d = idx & (kD - 1);
        float M = kNegInf;
        for (int cc = 0; cc < p.nchunks; ++cc) M = fmaxf(M, __ldcg(parts + cc * kPartFloats + h));
        float acc = 0.f, lsum = 0.f;
        for (int cc = 0; cc < p.nchunks; ++cc) {
            const float *pc = parts + cc * kPartFloats;
            const float mc = __ldcg(pc + h);
            const float f = (mc == kNegInf) ? 0.f : exp2f(mc - M);
            acc = fmaf(f, __ldcg(pc + 2 * kMaxG + h * kD + d), acc);
            lsum = fmaf(f, __ldcg(pc + kMaxG + h), lsum);
        }
        const float v = lsum > 0.f ? acc / lsum : 0.f;
        __nv_bfloat16 b = __float2bfloat16_rn(v);
        out[idx] = *reinterpret_cast<uint16_t *>(&b);
    }
}

int launch_decode(const DecodeParams &p, const CUtensorMap &tmap, cudaStream_t stream) {
    const size_t smem = decode_smem_bytes(p.max_nb);
    if (cudaFuncSetAttribute(decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return NOSA_ERR_CUDA;
    dim3 grid(p.nchunks, p.units);
    decode_kernel<<<grid, kDecThreads, smem, stream>>>(tmap, p);
    return cudaGetLastError() == cudaSuccess ? NOSA_OK : NOSA_ERR_CUDA;
}

}  // namespace nosa

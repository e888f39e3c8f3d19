// nosa_select.cu -- steps a2 + a3: two-stage block scores and dual selection.
//
// NOSA pages: wmrh.cn NOSA-1B release (two-stage attention: Top-K blocks are
// chosen with the compressed KV, then attention is exact); montaan.com summary
// of arXiv:2510.13602, "Key Design Components" item 2 (mean pooling inside
// sub-blocks, max pooling across them) and item 4 (Equation 7: a query-aware
// budget k_q and a query-agnostic budget k_e); gist.science summary,
// "Mecanisme de double selection".
//
// Design.  The only large operand is the compressed-key array of a unit (fp32:
// 32 B per token, 4 MiB per unit at 128K context; bf16: half that), read once
// per step: the kernel is a streaming GEMV against q_hat = sum of the group's
// query heads, bound by HBM bandwidth.  Each CTA owns a contiguous chunk of
// candidate blocks.  One producer thread streams the chunk into a ring of
// shared-memory stages with bulk asynchronous copies (cp.async.bulk,
// completion on mbarriers); consumer warps read 32 sub-block rows per stage
// (each lane 4 dims of a row: a 16-byte fp32 or 8-byte bf16 shared load),
// reduce the 32 partial dot products with a 31-shuffle transpose-reduction
// (each lane ends with one sub-block), max-pool groups of four lanes to block
// scores, and keep a warp-wide sorted top-32 list of (score, block) keys.  The
// per-chunk lists go to the workspace; the last CTA of the unit to finish
// (atomic counter, no waiting) merges them into Gamma_q, forms the union with
// Gamma_e through a block bitmap, appends the local block and writes the
// ascending selection.  List merges (a chain of dependent shuffles each) run as
// a tree over the consumer warps: first the CTA's four lists, then, in the
// unit's last CTA, a quarter of the chunk lists per warp.
//
// Fused with the decode-time append (nosa_append_select): a sixth warp of each
// unit's chunk-0 CTA appends the token while the other warps stream.  Nothing
// the scoring reads changes: the pooled key and the eviction score that the
// append may complete belong to the local block, which is not a candidate.
// What does change, Gamma_e (or the fill reading's pool) when a new candidate
// arrives, is read only by the finalizing CTA, after the counter hand-off, and
// that CTA writes the new length once every CTA of the unit has read the old.
#include "nosa_append_unit.cuh"

namespace nosa {

namespace {
constexpr int kSelW = 4;    // consumer warps
constexpr int kSelSB = 8;   // blocks per stage (32 sub-block rows)
constexpr int kCtasPerSm = 3;
constexpr int kMaxChunks = 64;  // select_chunk_blocks keeps chunks per unit below this

// Stage geometry per stored key type: 64 KiB in flight per CTA either way
// (fp32: 4 stages of 16 KiB; bf16: 8 stages of 8 KiB).
template <typename T> struct SelGeo;
template <> struct SelGeo<float> { static constexpr int kElem = 4, kStages = 4; };
template <> struct SelGeo<__nv_bfloat16> { static constexpr int kElem = 2, kStages = 8; };
template <typename T> __host__ __device__ constexpr int stage_bytes() { return kSelSB * kSubPerBlock * kD * SelGeo<T>::kElem; }
// Stage s is always consumed by warp s % kSelW, so every mbarrier waiter waits
// its phases in order (parity waits cannot tell phase p from p + 2).
static_assert(SelGeo<float>::kStages % kSelW == 0, "each stage must have a single consumer warp");
static_assert(SelGeo<__nv_bfloat16>::kStages % kSelW == 0, "each stage must have a single consumer warp");

// Named barrier of the kSelW consumer warps (the producer and append warps have left).
__device__ __forceinline__ void sel_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kSelW * 32) : "memory");
}

// Fill reading, one warp: Gamma_e = the first k_e pool entries (E rank order)
// outside Gamma_q, whose bits are already set in `bitmap`; their bits are set
// too, then the pool keeps only the entries in Sel = Gamma_q + Gamma_e, in
// order.  pf_n / pf_id: pool_n[u] and pool[u][lane], loaded early by this warp.
__device__ __forceinline__ void fill_gamma_e(const SelectParams &p, int32_t u, int32_t nb_c, uint32_t *bitmap,
                                             int lane, int32_t pf_n, int32_t pf_id) {
    int32_t *pool = p.pool + (int64_t)u * p.nblk;
    const int32_t n = pf_n;
    int32_t *ge = p.gamma_e_out + (int64_t)u * p.k_e;
    const unsigned lt = (1u << lane) - 1u;
    int32_t taken = 0;
    bool bad = false;
    for (int i0 = 0; i0 < n && taken < p.k_e; i0 += 32) {
        const int i = i0 + lane;
        const int32_t id = (i < n) ? (i0 == 0 ? pf_id : pool[i]) : -1;
        const bool ok = id >= 0 && id < nb_c;
        bad |= (i < n) && !ok;
        const bool elig = ok && !((bitmap[id >> 5] >> (id & 31)) & 1u);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, elig);
        const int32_t r = taken + __popc(m & lt);
        if (elig && r < p.k_e) {
            ge[r] = id;
            atomicOr(&bitmap[id >> 5], 1u << (id & 31));
        }
        taken = min(taken + __popc(m), p.k_e);
        __syncwarp();
    }
    if (lane == 0) p.gamma_n_out[u] = taken;
    int32_t kept = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int32_t id = (i < n) ? (i0 == 0 ? pf_id : pool[i]) : -1;
        const bool keep = id >= 0 && id < nb_c && ((bitmap[id >> 5] >> (id & 31)) & 1u);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, keep);
        __syncwarp();  // the chunk is read before any lane writes (writes land at or below it)
        if (keep) pool[kept + __popc(m & lt)] = id;
        kept += __popc(m);
    }
    if (lane == 0) p.pool_n[u] = kept;
    if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) set_error(p.err, NOSA_EFLAG_STATE);
}

// Does this launch append a token to a unit of length L_prev (the fused launch, room left)?
__device__ __forceinline__ bool appends(const SelectParams &p, int32_t L_prev) {
    return p.fused && L_prev >= 0 && L_prev < p.ap.max_ctx;
}

// Candidate blocks [b0, b1) of this chunk, for a unit of length L_prev before this launch's
// append, and the number of stages that stream them.
__device__ __forceinline__ int32_t chunk_stages(const SelectParams &p, int32_t chunk, int32_t L_prev, int32_t &b0,
                                                int32_t &b1) {
    const int32_t L = appends(p, L_prev) ? L_prev + 1 : L_prev;
    const int32_t nb_c = L > 0 ? (L - 1) / kBlock : 0;
    b0 = min(chunk * p.chunk_blocks, nb_c);
    b1 = min(b0 + p.chunk_blocks, nb_c);
    return (p.k_q > 0 && b1 > b0) ? (b1 - b0 + kSelSB - 1) / kSelSB : 0;
}

template <typename T>
size_t select_smem_bytes(int32_t nblk) {
    constexpr int S = SelGeo<T>::kStages;
    return (size_t)S * stage_bytes<T>() + 2 * S * sizeof(uint64_t) + kSelW * 32 * sizeof(uint64_t) +
           ((size_t)nblk / 32 + 1) * sizeof(uint32_t);
}
}  // namespace

int select_chunk_blocks(int32_t units, int32_t nblk, bool ck_bf16) {
    // candidates per unit are at most nblk - 1; per-CTA fixed cost (pipeline
    // fill, the list merges, the atomic hand-off) ~ the time of 32 fp32 blocks,
    // i.e. of 64 bf16 blocks; one level of the finalizing CTA's merge tree
    // (ceil(n/4) + 1 levels for n chunk lists) ~ 2 fp32 blocks (measured: it
    // decides the chunk count only for small problems, where every split fits
    // in one wave)
    const int64_t work = nblk > 1 ? nblk - 1 : 1;
    int64_t nmax = (work + kSelSB - 1) / kSelSB;
    if (nmax > kMaxChunks) nmax = kMaxChunks;
    const int n = best_chunks(units, work, (int64_t)kNumSms * kCtasPerSm, ck_bf16 ? 64 : 32, nmax, ck_bf16 ? 4 : 2);
    int64_t per = (work + n - 1) / n;
    per = (per + kSelSB - 1) / kSelSB * kSelSB;
    return (int)per;
}

template <typename T>
__global__ void __launch_bounds__((kSelW + 2) * 32) select_kernel(const SelectParams p) {
    constexpr int kSelS = SelGeo<T>::kStages;
    constexpr int kStageBytes = stage_bytes<T>();
    pdl_trigger();  // the successor (cache plan or decode) waits for this grid anyway
    pdl_wait();
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *tiles = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(tiles + kSelS * kStageBytes);
    uint64_t *empty = full + kSelS;
    uint64_t *lists = empty + kSelS;
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(lists + kSelW * 32);
    __shared__ int s_last;

    const int32_t u = blockIdx.y, chunk = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // (the producer reads the length itself, after its first copies are out)
    const int32_t L_prev = warp == kSelW ? 0 : p.seq_len[u];
    const bool grow = appends(p, L_prev);  // this launch appends a token
    const int32_t L = grow ? L_prev + 1 : L_prev;
    // a block became a candidate with this token: Gamma_e (or the pool) may change
    const bool refresh = grow && L_prev >= kBlock && (L_prev & (kBlock - 1)) == 0;
    const int32_t nb_c = L > 0 ? (L - 1) / kBlock : 0;
    int32_t b0, b1;
    const int32_t nstage = chunk_stages(p, chunk, L_prev, b0, b1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSelS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();

    // warp 0 may finalize this unit: fetch Gamma_e (fill reading: the head of
    // the pool) now, while the stream runs
    int32_t ne = (warp == 0 && !p.fill) ? min(p.gamma_n[u], p.k_e) : 0;
    int32_t pf_n = 0, pf_id = -1;
    if (warp == 0 && p.fill) {
        pf_n = min(max(p.pool_n[u], 0), p.nblk);  // a pool never holds more than nblk - 1 ids
        if (lane < pf_n) pf_id = p.pool[(int64_t)u * p.nblk + lane];
    }
    int32_t ge_reg[kMaxKe / 32];
    if (warp == 0) {
        const int32_t *ge = p.gamma_e + (int64_t)u * p.k_e;
#pragma unroll
        for (int i = 0; i < kMaxKe / 32; ++i) {
            const int j = lane + 32 * i;
            ge_reg[i] = (j < ne) ? ge[j] : -1;
        }
    }

    uint64_t list = 0;
    if (warp == kSelW) {
        if (lane == 0) {
            const T *ck = static_cast<const T *>(p.ck) + (int64_t)u * p.nsub * kD;
            auto issue = [&](int i, int32_t bs, int32_t bend) {
                const int s = i % kSelS;
                const uint32_t bytes = (uint32_t)min(kSelSB, bend - bs) * (kSubPerBlock * kD * SelGeo<T>::kElem);
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_load(tiles + s * kStageBytes, ck + (int64_t)bs * kSubPerBlock * kD, bytes, &full[s]);
            };
            // The first ring of stages goes out before this thread has the context length: the
            // chunk is bounded by the largest candidate count max_ctx allows, and the stages of
            // a longer bound than the real one are only waited for, never consumed.  (Whenever
            // the chunk has real work, its first block is chunk * chunk_blocks either way.)
            const int32_t nbc_max = p.nblk - 1;
            const int32_t b0s = min(chunk * p.chunk_blocks, nbc_max);
            const int32_t b1s = min(b0s + p.chunk_blocks, nbc_max);
            const int nspec = (p.k_q > 0 && b1s > b0s) ? min(kSelS, (b1s - b0s + kSelSB - 1) / kSelSB) : 0;
            for (int i = 0; i < nspec; ++i) issue(i, b0s + i * kSelSB, b1s);
            // the real bounds (the load follows the copies; the asm above keeps it there)
            int32_t rb0, rb1;
            const int32_t nst = chunk_stages(p, chunk, ld_volatile_s32(p.seq_len + u), rb0, rb1);
            int issued = nspec;
            for (int i = nspec; i < nst; ++i) {
                const int s = i % kSelS;
                if (i >= kSelS && !mbar_wait(&empty[s], ((i / kSelS) - 1) & 1)) {
                    set_error(p.err, NOSA_EFLAG_TIMEOUT);
                    break;
                }
                issue(i, rb0 + i * kSelSB, rb1);
                issued = i + 1;
            }
            // never leave with copies in flight
            for (int i = max(0, issued - kSelS); i < issued; ++i)
                if (!mbar_wait(&full[i % kSelS], (i / kSelS) & 1)) set_error(p.err, NOSA_EFLAG_TIMEOUT);
        }
    } else if (warp == kSelW + 1) {
        // the fused append (launched only when fused): chunk 0 of each unit
        if (chunk == 0) append_unit(p.ap, u, lane, p.ap.e_new[u], false);  // fences before its hand-off
    } else {
        // q_hat = sum of the G query heads of this kv head, lane's 4 dims; the
        // loads are issued together while the first stages are in flight
        float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);
        {
            const uint2 *q = reinterpret_cast<const uint2 *>(p.q + (int64_t)u * p.G * kD) + lane;
            uint2 w[kMaxG];
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) w[h] = (h < p.G) ? q[h * (kD / 4)] : make_uint2(0u, 0u);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h < p.G) {
                    qv.x += bf16_lo(w[h].x); qv.y += bf16_hi(w[h].x);
                    qv.z += bf16_lo(w[h].y); qv.w += bf16_hi(w[h].y);
                }
            }
        }
        for (int i = warp; i < nstage; i += kSelW) {
            const int s = i % kSelS;
            if (!mbar_wait(&full[s], (i / kSelS) & 1)) {
                set_error(p.err, NOSA_EFLAG_TIMEOUT);
                break;
            }
            const uint8_t *t = tiles + s * kStageBytes;
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float4 k = row4(t, j, lane, static_cast<T *>(nullptr));
                v[j] = fmaf(qv.w, k.w, fmaf(qv.z, k.z, fmaf(qv.y, k.y, qv.x * k.x)));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            reduce_level<16>(v, lane, 16);
            reduce_level<8>(v, lane, 8);
            reduce_level<4>(v, lane, 4);
            reduce_level<2>(v, lane, 2);
            reduce_level<1>(v, lane, 1);
            // lane holds sub-block (bs*4 + lane); max-pool the four sub-blocks of a block
            float sc = v[0] * p.scale;
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 1));
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 2));
            const int32_t bs = b0 + i * kSelSB;
            const int beta = lane >> 2;
            const uint64_t cand =
                ((lane & 3) == 0 && bs + beta < b1) ? select_key(sc, bs + beta) : 0ull;
            list_offer(list, cand, lane);
        }
        lists[warp * 32 + lane] = list;
    }
    __syncthreads();
    if (warp >= kSelW) return;
    // The consumer warps' lists, then (in the unit's last CTA) the chunk lists, merge as
    // a tree: a merge is a chain of dependent shuffles, so depth is what costs.
    // (the first level reads lists 1 and 3 only, so warp 2 may overwrite list 2 at once)
    if ((warp & 1) == 0) list_merge(list, lists[(warp + 1) * 32 + lane], lane);
    if (warp == 2) lists[2 * 32 + lane] = list;
    sel_sync();
    if (warp == 0) list_merge(list, lists[2 * 32 + lane], lane);

    if (p.nchunks > 1) {
        if (warp == 0) {
            uint64_t *mine = p.part_keys + ((int64_t)u * p.nchunks + chunk) * 32;
            mine[lane] = list;
            __syncwarp();
            // counted with release semantics (the warp's list, and what the CTA wrote before the
            // block barrier above, e.g. the fused append); the last chunk acquires the others' lists
            if (lane == 0) s_last = ((int32_t)atom_add_acq_rel_gpu(p.counter + u, 1u) == p.nchunks - 1);
        }
        sel_sync();  // s_last is known to the four warps, and orders their loads after lane 0's acquire
        if (!s_last) return;
        if (warp == 0 && lane == 0) p.counter[u] = 0;
        // warp w folds chunk lists w, w + 4, ...; the loads are issued four at a time
        const uint64_t *all = p.part_keys + (int64_t)u * p.nchunks * 32;
        list = 0;  // a warp without chunks contributes an empty list
        for (int c0 = warp; c0 < p.nchunks; c0 += 4 * kSelW) {
            uint64_t k[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int cj = c0 + j * kSelW;
                k[j] = cj < p.nchunks ? __ldcg(all + cj * 32 + lane) : 0ull;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {  // conditions uniform over the warp
                if (c0 + j * kSelW >= p.nchunks) break;
                if (c0 == warp && j == 0) list = k[0];
                else list_merge(list, k[j], lane);
            }
        }
        lists[warp * 32 + lane] = list;
        sel_sync();
        if ((warp & 1) == 0) list_merge(list, lists[(warp + 1) * 32 + lane], lane);
        if (warp == 2) lists[2 * 32 + lane] = list;
        sel_sync();
        if (warp == 0) list_merge(list, lists[2 * 32 + lane], lane);
    }
    if (warp != 0) return;
    if (refresh) {  // read again what the fused append may have changed (ordered by the hand-off)
        if (!p.fill) {
            ne = min(__ldcg(p.gamma_n + u), p.k_e);
            const int32_t *ge = p.gamma_e + (int64_t)u * p.k_e;
#pragma unroll
            for (int i = 0; i < kMaxKe / 32; ++i) {
                const int j = lane + 32 * i;
                ge_reg[i] = (j < ne) ? __ldcg(ge + j) : -1;
            }
        } else {
            pf_n = min(max(__ldcg(p.pool_n + u), 0), p.nblk);
            pf_id = (lane < pf_n) ? __ldcg(p.pool + (int64_t)u * p.nblk + lane) : -1;
        }
    }
    if (grow && lane == 0) p.ap.seq_len[u] = L;  // every CTA of the unit has read the old length

    // ---- finalize: Gamma_q, union with Gamma_e, local block ----
    const int32_t myid = (lane < p.k_q && list != 0ull) ? key_block(list) : -1;
    if (p.gq && lane < p.k_q) p.gq[(int64_t)u * p.k_q + lane] = myid;
    int32_t *sel = p.sel + (int64_t)u * p.max_sel;
    if (L <= 0) {
        for (int i = lane; i < p.max_sel; i += 32) sel[i] = -1;
        if (lane == 0) {
            p.nsel[u] = 0;
            if (p.fill) p.gamma_n_out[u] = 0;
        }
        return;
    }
    const int32_t nw = (nb_c + 31) >> 5;
    for (int i = lane; i < nw; i += 32) bitmap[i] = 0;
    __syncwarp();
    if (myid >= 0) atomicOr(&bitmap[myid >> 5], 1u << (myid & 31));
#pragma unroll
    for (int i = 0; i < kMaxKe / 32; ++i) {
        const int32_t id = ge_reg[i];
        if (id >= 0 && id < nb_c) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
    }
    __syncwarp();
    if (p.fill) {
        fill_gamma_e(p, u, nb_c, bitmap, lane, pf_n, pf_id);
        __syncwarp();
    }
    const int32_t per = (nw + 31) / 32;
    const int32_t w0 = min(lane * per, nw), w1 = min(w0 + per, nw);
    int32_t cnt = 0;
    for (int i = w0; i < w1; ++i) cnt += __popc(bitmap[i]);
    int32_t pre = cnt;
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t x = __shfl_up_sync(0xFFFFFFFFu, pre, o);
        if (lane >= o) pre += x;
    }
    int32_t at = pre - cnt;
    for (int i = w0; i < w1; ++i) {
        uint32_t m = bitmap[i];
        while (m) {
            const int bit = __ffs(m) - 1;
            m &= m - 1;
            sel[at++] = i * 32 + bit;
        }
    }
    const int32_t total = __shfl_sync(0xFFFFFFFFu, pre, 31);
    if (lane == 0) {
        sel[total] = nb_c;  // the local block, (L-1)/64
        p.nsel[u] = total + 1;
    }
    for (int i = total + 1 + lane; i < p.max_sel; i += 32) sel[i] = -1;
}

template <typename T>
int launch_select_t(const SelectParams &p, cudaStream_t stream) {
    const size_t smem = select_smem_bytes<T>(p.nblk);
    if (cudaFuncSetAttribute(select_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return NOSA_ERR_CUDA;
    dim3 grid(p.nchunks, p.units);
    return launch_pdl(select_kernel<T>, grid, dim3((kSelW + 1 + (p.fused ? 1 : 0)) * 32), smem, stream, p) ==
                   cudaSuccess
               ? NOSA_OK
               : NOSA_ERR_CUDA;
}

int launch_select(const SelectParams &p, cudaStream_t stream) {
    return p.ck_bf16 ? launch_select_t<__nv_bfloat16>(p, stream) : launch_select_t<float>(p, stream);
}

}  // namespace nosa

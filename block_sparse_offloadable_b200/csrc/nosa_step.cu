// nosa_step.cu -- one decode step of a layer in one launch, for a device-resident KV store: the
// append (a1, one token), the two-stage scores and dual selection (a2 + a3) and the sparse decode
// (a5).
//
// NOSA pages: the steps as in nosa_append.cu, nosa_select.cu and nosa_decode.cu.  The split of the
// work follows from the dual selection itself (gist.science summary of arXiv:2510.13602,
// "Mecanisme de double selection"; montaan.com summary, "Key Design Components" item 4): Gamma_e is
// query-agnostic and fixed once the token is appended, so its blocks are attended while the
// query-aware scores that decide Gamma_q are still being computed.
//
// Design.  Each unit (seq, kv head) has a team of C CTAs, one per SM (units * C <= the SM count,
// or C = 1 when the units alone fill the GPU).  Team CTA c
//  * (c = 0, on an extra warp) appends the token exactly as nosa_compress_append does and raises
//    the unit's "appended" flag;
//  * streams its 1/C share of the unit's candidate pooled keys through the stage ring, 16 blocks
//    (fp32) or 32 (bf16) per 32 KiB stage, scores them (q_hat . kbar * scale, max over the four
//    sub-blocks of a block) and keeps a top-32 list per warp; the team's last CTA to publish its
//    list merges the C lists into Gamma_q, writes S(t) exactly as nosa_select does, writes the
//    Gamma_q blocks outside Gamma_e in rank order, and raises the unit's "selected" flag;
//  * attends piece c of the unit's decode list [Gamma_e (k_e slots) | local block | Gamma_q minus
//    Gamma_e (k_q slots)] through the same ring, skipping empty slots: the producer waits for
//    "appended" before its first item and for "selected" before the first Gamma_q item, which
//    come last in the list;
//  * counts its piece; the unit's last piece merges the C partial states and writes the output,
//    then clears the unit's flags and counters for the next launch.
// Stage s of the ring always belongs to consumer group s % 2, in both phases.  Every cross-CTA
// wait is bounded and waits only for CTAs of the same team, which the cooperative launch keeps
// resident together; a wait that runs out sets NOSA_EFLAG_TIMEOUT and the CTA drains.
#include <algorithm>

#include "nosa_append_unit.cuh"
#include "nosa_attend.cuh"

namespace nosa {

namespace {
constexpr int kStepS = 6;                            // ring stages of 32 KiB (+ 256 B of logits)
constexpr int kStepThreads = (kConsWarps + 2) * 32;  // consumers, the producer, the append warp
constexpr int kProducerWarp = kConsWarps;
constexpr int kAppendWarp = kConsWarps + 1;
static_assert(kStepS % kGroups == 0, "stage s must always be consumed by group s % kGroups");

// The consumer warps and the append warp meet here before a team CTA publishes its list, so that
// the append has read the old length before the finalizing CTA writes the new one.
__device__ __forceinline__ void append_barrier_sync() {
    asm volatile("bar.sync 2, %0;" ::"n"(kConsThreads + 32) : "memory");
}
__device__ __forceinline__ void append_barrier_arrive() {
    asm volatile("bar.arrive 2, %0;" ::"n"(kConsThreads + 32) : "memory");
}

// Pooled-key rows per consumer warp per stage: a stage is 32 KiB either way.
template <typename T> struct StepRows;
template <> struct StepRows<float> { static constexpr int kRows = 16; };
template <> struct StepRows<__nv_bfloat16> { static constexpr int kRows = 32; };
template <typename T> __host__ __device__ constexpr int stage_blocks() {
    return kDecW * StepRows<T>::kRows / kSubPerBlock;
}
static_assert(stage_blocks<float>() * kSubPerBlock * kD * 4 == kBlockBytes, "a score stage fills a ring stage");
static_assert(stage_blocks<__nv_bfloat16>() * kSubPerBlock * kD * 2 == kBlockBytes,
              "a score stage fills a ring stage");

// The eight consumer warps' lists (lists[w * 32 + lane], warp w's in `list`) merged as a tree; the
// result is in warp 0's `list`.  Called by every consumer thread.
__device__ __forceinline__ void tree_merge(uint64_t &list, uint64_t *lists, int warp, int lane) {
    lists[warp * 32 + lane] = list;
    consumer_sync();
    if (warp < 4) list_merge(list, lists[(warp + 4) * 32 + lane], lane);
    if (warp < 4 && warp >= 2) lists[warp * 32 + lane] = list;
    consumer_sync();
    if (warp < 2) list_merge(list, lists[(warp + 2) * 32 + lane], lane);
    if (warp == 1) lists[32 + lane] = list;
    consumer_sync();
    if (warp == 0) list_merge(list, lists[32 + lane], lane);
}

// Warp 0 of the unit's finalizing CTA: Gamma_q from the merged list, S(t) = Gamma_q U Gamma_e U
// {local} as nosa_select writes it, the Gamma_q blocks outside Gamma_e for the decode, the new
// length; then the "selected" flag.
__device__ __forceinline__ void finalize_unit(const StepParams &sp, int32_t u, uint64_t list, int32_t L, int32_t nb_c,
                                              bool grow, uint32_t *bitmap, int lane) {
    const DecodeParams &p = sp.d;
    // Gamma_e as this step's append left it
    int ok = 1;
    if (lane == 0) ok = flag_wait(sp.ready + 2 * u);
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (!ok && lane == 0) set_error(p.err, NOSA_EFLAG_TIMEOUT);
    const int32_t ne = L > 0 ? min(max(__ldcg(sp.gamma_n + u), 0), p.k_e) : 0;
    int32_t ge_reg[kMaxKe / 32];
#pragma unroll
    for (int i = 0; i < kMaxKe / 32; ++i) {
        const int j = lane + 32 * i;
        ge_reg[i] = (j < ne) ? __ldcg(sp.gamma_e + (int64_t)u * p.k_e + j) : -1;
    }
    const int32_t myid = (lane < p.k_q && list != 0ull) ? key_block(list) : -1;
    if (sp.gq && lane < p.k_q) sp.gq[(int64_t)u * p.k_q + lane] = myid;
    int32_t *sel = sp.sel + (int64_t)u * p.max_sel;
    int32_t *rest = sp.rest + (int64_t)u * p.k_q;
    if (L <= 0) {
        for (int i = lane; i < p.max_sel; i += 32) sel[i] = -1;
        for (int i = lane; i < p.k_q; i += 32) rest[i] = -1;
        if (lane == 0) sp.nsel[u] = 0;
    } else {
        const int32_t nw = (nb_c + 31) >> 5;
        for (int i = lane; i < nw; i += 32) bitmap[i] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kMaxKe / 32; ++i) {
            const int32_t id = ge_reg[i];
            if (id >= 0 && id < nb_c) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
        }
        __syncwarp();
        // Gamma_q blocks not in Gamma_e, in rank order: the decode list's last k_q slots
        const bool fresh = myid >= 0 && myid < nb_c && !((bitmap[myid >> 5] >> (myid & 31)) & 1u);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, fresh);
        if (fresh) rest[__popc(m & ((1u << lane) - 1u))] = myid;
        for (int i = __popc(m) + lane; i < p.k_q; i += 32) rest[i] = -1;
        __syncwarp();  // every lane has tested its bit before the Gamma_q bits go in
        if (myid >= 0 && myid < nb_c) atomicOr(&bitmap[myid >> 5], 1u << (myid & 31));
        __syncwarp();
        // S(t) ascending: this lane's share of the bitmap words, placed by a prefix count
        const int32_t per = (nw + 31) / 32;
        const int32_t w0 = min(lane * per, nw), w1 = min(w0 + per, nw);
        int32_t cnt = 0;
        for (int i = w0; i < w1; ++i) cnt += __popc(bitmap[i]);
        int32_t pre = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t x = __shfl_up_sync(0xFFFFFFFFu, pre, o);
            if (lane >= o) pre += x;
        }
        int32_t at = pre - cnt;
        for (int i = w0; i < w1; ++i) {
            uint32_t bits = bitmap[i];
            while (bits) {
                const int bit = __ffs(bits) - 1;
                bits &= bits - 1;
                sel[at++] = i * 32 + bit;
            }
        }
        const int32_t total = __shfl_sync(0xFFFFFFFFu, pre, 31);
        if (lane == 0) {
            sel[total] = nb_c;  // the local block, (L-1)/64
            sp.nsel[u] = total + 1;
        }
        for (int i = total + 1 + lane; i < p.max_sel; i += 32) sel[i] = -1;
    }
    // every team CTA has read the old length (each published its list after reading it)
    if (grow && lane == 0) sp.ap.seq_len[u] = L;
    __threadfence();
    __syncwarp();
    if (lane == 0) st_release_gpu(sp.ready + 2 * u + 1, 1);
}
}  // namespace

int step_team_size(int32_t units, int32_t max_sel) {
    if (units > kNumSms) return 1;
    return std::min<int32_t>(kNumSms / units, max_sel);
}

size_t step_smem_bytes(int32_t nblk) {
    return 1024 + (size_t)kStepS * kBlockBytes + (size_t)kStepS * kBlock * sizeof(float) +
           2 * kStepS * sizeof(uint64_t) + kStepS * sizeof(int32_t) + (size_t)kDecW * kScr * sizeof(float) +
           (size_t)kConsWarps * 32 * sizeof(uint64_t) + ((size_t)nblk / 32 + 1) * sizeof(uint32_t);
}

template <typename T>
__global__ void __launch_bounds__(kStepThreads, 1)
    step_kernel(const __grid_constant__ CUtensorMap tmap, const StepParams sp) {
    const DecodeParams &p = sp.d;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *ebuf = reinterpret_cast<float *>(tiles + kStepS * kBlockBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(ebuf + kStepS * kBlock);
    uint64_t *empty = full + kStepS;
    int32_t *s_blk = reinterpret_cast<int32_t *>(empty + kStepS);
    float *scratch = reinterpret_cast<float *>(s_blk + kStepS);
    uint64_t *lists = reinterpret_cast<uint64_t *>(scratch + kDecW * kScr);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(lists + kConsWarps * 32);
    __shared__ int s_last;
    __shared__ volatile int s_abort;
    constexpr int kBPS = stage_blocks<T>();
    constexpr int kRows = StepRows<T>::kRows;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t C = p.pieces;
    const int32_t u = (int32_t)blockIdx.x / C, cidx = (int32_t)blockIdx.x % C;
    // (the append warp reads the length inside the append)
    const int32_t L_prev = warp == kAppendWarp ? 0 : ld_volatile_s32(p.seq_len + u);
    const bool grow = L_prev >= 0 && L_prev < p.max_ctx;
    const int32_t L = grow ? L_prev + 1 : L_prev;
    const int32_t nb_c = L > 0 ? (L - 1) / kBlock : 0;
    // this CTA's score stages [s0, s1) of the unit's ns, covering candidate blocks [s0 * kBPS, b1)
    const int32_t ns = p.k_q > 0 ? (nb_c + kBPS - 1) / kBPS : 0;
    const int32_t s0 = cidx * ns / C, s1 = (cidx + 1) * ns / C;
    const int n_sc = s1 - s0;
    const int32_t b1 = min(s1 * kBPS, nb_c);
    // and its piece [d_lo, d_hi) of the unit's max_sel decode slots (C <= max_sel: never empty)
    const int32_t d_lo = cidx * p.max_sel / C, d_hi = (cidx + 1) * p.max_sel / C;
    const int n_items = d_hi - d_lo;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStepS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecW);
        }
        fence_mbar_init();
        prefetch_tmap(&tmap);
        s_abort = 0;
    }
    __syncthreads();

    if (warp == kAppendWarp) {
        if (cidx == 0) {
            append_unit(sp.ap, u, lane, sp.ap.e_new[u], false);  // fences its writes
            __syncwarp();
            if (lane == 0) st_release_gpu(sp.ready + 2 * u, 1);
        }
        append_barrier_arrive();
        return;
    }

    if (warp == kProducerWarp) {
        // ---------------- producer ----------------
        int it = 0;
        if (lane == 0) {
            const T *ck = static_cast<const T *>(sp.ck) + (int64_t)u * sp.nsub * kD;
            for (int i = 0; i < n_sc && !s_abort; ++i, ++it) {
                const int s = it % kStepS;
                if (it >= kStepS && !wait_or_abort(&empty[s], ((it / kStepS) - 1) & 1, &s_abort, p.err)) break;
                const int32_t bs = (s0 + i) * kBPS;
                const uint32_t bytes = (uint32_t)min(kBPS, b1 - bs) * (kSubPerBlock * kD * (uint32_t)sizeof(T));
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_load(tiles + s * kBlockBytes, ck + (int64_t)bs * kSubPerBlock * kD, bytes, &full[s]);
            }
        }
        it = __shfl_sync(0xFFFFFFFFu, it, 0);
        // decode slots [a, b): the block of each, fetched by the warp 32 at a time; lane 0 issues
        auto issue = [&](int32_t a, int32_t b, int32_t ne) {
            for (int32_t xb = a; xb < b && !s_abort; xb += 32) {
                const int nb = min(32, b - xb);
                const int32_t j = xb + lane;
                int32_t lb = -1;
                if (lane < nb) {
                    if (j < p.k_e) {
                        lb = j < ne ? __ldcg(sp.gamma_e + (int64_t)u * p.k_e + j) : -1;
                        if (lb >= nb_c) lb = -1;  // as S(t): candidates only
                    } else if (j == p.k_e) {
                        lb = L > 0 ? nb_c : -1;
                    } else {
                        lb = __ldcg(sp.rest + (int64_t)u * p.k_q + (j - p.k_e - 1));
                    }
                }
                for (int k = 0; k < nb; ++k, ++it) {
                    const int32_t blk = __shfl_sync(0xFFFFFFFFu, lb, k);
                    if (lane == 0) {
                        const int s = it % kStepS;
                        const bool go = it < kStepS ||
                                        wait_or_abort(&empty[s], ((it / kStepS) - 1) & 1, &s_abort, p.err);
                        if (go) {
                            const bool ok = blk >= 0 && blk < p.nblk;
                            s_blk[s] = ok ? blk : -1;
                            if (ok) {
                                const int32_t y = (int32_t)(((int64_t)u * p.nblk + blk) * 2 * kBlock);
                                uint8_t *t = tiles + s * kBlockBytes;
                                mbar_arrive_expect_tx(&full[s], kBlockBytes + kBlock * sizeof(float));
                                tma_load_2d(t, &tmap, &full[s], 0, y);
                                tma_load_2d(t + kBoxBytes, &tmap, &full[s], 64, y);
                                tma_load_2d(t + 2 * kBoxBytes, &tmap, &full[s], 0, y + kBlock);
                                tma_load_2d(t + 3 * kBoxBytes, &tmap, &full[s], 64, y + kBlock);
                                bulk_load(ebuf + s * kBlock, p.e + (int64_t)u * p.max_ctx + (int64_t)blk * kBlock,
                                          kBlock * sizeof(float), &full[s]);
                            } else {
                                mbar_arrive(&full[s]);
                            }
                        }
                    }
                    __syncwarp();
                }
            }
        };
        // Gamma_e and the local block need the append (its new row, and Gamma_e as it left it)
        int ok = 1;
        if (lane == 0 && !s_abort) {
            ok = flag_wait(sp.ready + 2 * u);
            if (ok) fence_proxy_async_global();  // the copies below read what the append wrote
            else { s_abort = 1; set_error(p.err, NOSA_EFLAG_TIMEOUT); }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok && !s_abort) {
            const int32_t ne = L > 0 ? min(max(__ldcg(sp.gamma_n + u), 0), p.k_e) : 0;
            issue(d_lo, min(d_hi, p.k_e + 1), ne);
            if (d_hi > p.k_e + 1 && !s_abort) {
                // the Gamma_q slots need the selection
                if (lane == 0) {
                    ok = flag_wait(sp.ready + 2 * u + 1);
                    if (!ok) { s_abort = 1; set_error(p.err, NOSA_EFLAG_TIMEOUT); }
                }
                ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
                if (ok) issue(max(d_lo, p.k_e + 1), d_hi, ne);
            }
        }
        // never leave with copies in flight
        if (lane == 0)
            for (int i = max(0, it - kStepS); i < it; ++i) mbar_wait(&full[i % kStepS], (i / kStepS) & 1);
        return;
    }

    // ---------------- consumers ----------------
    const int grp = warp / kDecW, wq = warp % kDecW;
    const int r = lane >> 2, c = lane & 3;
    const int sig = (r >> 1) + ((r & 1) << 2);  // row permutation 0,4,1,5,2,6,3,7
    const int ctid = threadIdx.x;                // 0..kConsThreads-1

    // ---- scores of this CTA's candidate blocks ----
    float4 qv = make_float4(0.f, 0.f, 0.f, 0.f);  // q_hat: the sum of the G query heads, lane's 4 dims
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
    uint64_t list = 0;
    for (int it = grp; it < n_sc; it += kGroups) {
        const int s = it % kStepS;
        if (!wait_or_abort(&full[s], (it / kStepS) & 1, &s_abort, p.err)) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            continue;
        }
        const uint8_t *t = tiles + s * kBlockBytes + wq * kRows * (kD * (int)sizeof(T));
        float v[kRows];
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
            const float4 k = row4(t, j, lane, static_cast<T *>(nullptr));
            v[j] = fmaf(qv.w, k.w, fmaf(qv.z, k.z, fmaf(qv.y, k.y, qv.x * k.x)));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        int32_t beta;
        bool offer;
        float sc;
        if constexpr (kRows == 32) {
            // lane l ends with sub-block row l; a block's four rows are lanes 4b..4b+3
            reduce_level<16>(v, lane, 16);
            reduce_level<8>(v, lane, 8);
            reduce_level<4>(v, lane, 4);
            reduce_level<2>(v, lane, 2);
            reduce_level<1>(v, lane, 1);
            sc = v[0] * sp.scale;
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 1));
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 2));
            beta = lane >> 2;
            offer = (lane & 3) == 0;
        } else {
            // lanes 2r, 2r+1 end with sub-block row r; a block's four rows are lanes 8b..8b+7
            reduce_level<8>(v, lane, 16);
            reduce_level<4>(v, lane, 8);
            reduce_level<2>(v, lane, 4);
            reduce_level<1>(v, lane, 2);
            v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], 1);
            sc = v[0] * sp.scale;
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 2));
            sc = fmaxf(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, 4));
            beta = lane >> 3;
            offer = (lane & 7) == 0;
        }
        const int32_t blk = (s0 + it) * kBPS + wq * (kRows / kSubPerBlock) + beta;
        list_offer(list, (offer && blk < b1) ? select_key(sc, blk) : 0ull, lane);
    }
    tree_merge(list, lists, warp, lane);

    // ---- publish; the team's last CTA forms Gamma_q and S(t) ----
    append_barrier_sync();
    bool fin = true;
    if (C > 1) {
        if (warp == 0) {
            sp.part_keys[((int64_t)u * C + cidx) * 32 + lane] = list;
            __syncwarp();
            // counted with release semantics; the last CTA acquires the others' lists
            if (lane == 0) s_last = ((int32_t)atom_add_acq_rel_gpu(sp.score_ctr + u, 1u) == C - 1);
        }
        consumer_sync();
        fin = s_last;
        if (fin) {
            if (ctid == 0) sp.score_ctr[u] = 0;
            const uint64_t *all = sp.part_keys + (int64_t)u * C * 32;
            list = 0;  // a warp without lists contributes an empty one
            for (int c0 = warp; c0 < C; c0 += 4 * kConsWarps) {
                uint64_t k[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int cj = c0 + j * kConsWarps;
                    k[j] = cj < C ? __ldcg(all + (int64_t)cj * 32 + lane) : 0ull;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {  // conditions uniform over the warp
                    if (c0 + j * kConsWarps >= C) break;
                    if (c0 == warp && j == 0) list = k[0];
                    else list_merge(list, k[j], lane);
                }
            }
            tree_merge(list, lists, warp, lane);
        }
    }
    if (fin && warp == 0) finalize_unit(sp, u, list, L, nb_c, grow, bitmap, lane);

    // ---- attention over this CTA's piece of the decode list ----
    uint32_t qf[8][2];
    {
        const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((int64_t)u * p.G + r) * kD);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint4 x = (r < p.G) ? qrow[4 * jj + c] : make_uint4(0, 0, 0, 0);
            qf[2 * jj][0] = x.x; qf[2 * jj][1] = x.y;
            qf[2 * jj + 1][0] = x.z; qf[2 * jj + 1][1] = x.w;
        }
    }
    WarpState st;
    st.reset();
    for (int it = n_sc + (((n_sc & 1) != grp) ? 1 : 0); it < n_sc + n_items; it += kGroups) {
        const int s = it % kStepS;
        if (wait_or_abort(&full[s], (it / kStepS) & 1, &s_abort, p.err)) {
            const int32_t lb = s_blk[s];
            if (lb >= 0)
                attend_block(st, qf, tiles + s * kBlockBytes, ebuf + s * kBlock, lb, L, p.qk_log2, wq, c, sig);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
    }
    fold_groups(st, scratch, grp, wq, r, c, sig);
    uint16_t *out = p.out + (int64_t)u * p.G * kD;
    float *part = p.part + (int64_t)blockIdx.x * kPartFloats;
    for (int idx = ctid; idx < p.G * kD; idx += kConsThreads) {
        const int h = idx >> 7, d = idx & (kD - 1);
        float M, acc, lsum;
        merged_state(scratch, h, d, M, acc, lsum);
        if (C == 1) store_bf16(out + idx, lsum > 0.f ? acc / lsum : 0.f);
        else store_partial(part, h, d, M, acc, lsum);
    }
    if (C == 1) {
        // this CTA is the whole team: its producer is past both flags
        if (ctid == 0) {
            sp.ready[2 * u] = 0;
            sp.ready[2 * u + 1] = 0;
        }
        return;
    }
    // hand-off of the partial state, as in the decode kernel
    consumer_sync();
    if (ctid == 0) s_last = ((int32_t)atom_add_acq_rel_gpu(p.counter + u, 1u) == C - 1);
    consumer_sync();
    if (!s_last) return;
    // the unit's last piece: every team CTA has finished, so no one reads the flags any more
    if (ctid == 0) {
        p.counter[u] = 0;
        sp.ready[2 * u] = 0;
        sp.ready[2 * u + 1] = 0;
    }
    const float *src0 = p.part + (int64_t)u * C * kPartFloats;
    if (C <= kOnePassPieces) {
        merge_pieces_onepass(src0, kPartFloats, C, p.G, out, ctid);
    } else {
        const MergeScratch ms = merge_scratch(scratch, C);
        for (int t = ctid; t < C; t += kConsThreads) ms.src[t] = src0 + (int64_t)t * kPartFloats;
        consumer_sync();
        merge_general(ms, C, p.G, out, nullptr, warp, lane, ctid);
    }
}

template <typename T>
int launch_step_t(const StepParams &sp, const CUtensorMap &tmap, cudaStream_t stream) {
    const size_t smem = step_smem_bytes(sp.d.nblk);
    if (cudaFuncSetAttribute(step_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return NOSA_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(sp.d.units * sp.d.pieces);
    cfg.blockDim = dim3(kStepThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    // a team of several CTAs waits on itself: keep the whole grid resident together
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = sp.d.pieces > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, step_kernel<T>, tmap, sp) == cudaSuccess ? NOSA_OK : NOSA_ERR_CUDA;
}

int launch_step(const StepParams &sp, const CUtensorMap &tmap, cudaStream_t stream) {
    return sp.ck_bf16 ? launch_step_t<__nv_bfloat16>(sp, tmap, stream) : launch_step_t<float>(sp, tmap, stream);
}

}  // namespace nosa

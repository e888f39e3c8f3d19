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
// or C = 1 when the units alone fill the GPU).  A CTA has eight consumer warps, a producer warp
// and a selection warp.  Team CTA c
//  * (c = 0, selection warp) appends the token exactly as nosa_compress_append does and raises
//    the unit's "appended" flag (a release store: the append wrote what other CTAs then read);
//  * streams its 1/C share of the unit's candidate pooled keys through the stage ring, 16 blocks
//    (fp32) or 32 (bf16) per 32 KiB stage; the consumers score them (q_hat . kbar * scale, max
//    over the four sub-blocks of a block), keep a top-32 list per warp, hand the lists to the
//    selection warp and go straight on to the attention;
//  * (selection warp) merges the eight lists; team CTA 0 gathers the others' lists, merges them
//    into Gamma_q, writes S(t) exactly as nosa_select does and writes the Gamma_q blocks outside
//    Gamma_e in rank order;
//  * attends its piece of the unit's decode slots: a 1/C share of the k_e + 1 slots of Gamma_e
//    and the local block, then a 1/C share of the k_q slots of Gamma_q minus Gamma_e, through the
//    same ring, skipping empty slots; the producer waits for "appended" before its first slot
//    and, for each Gamma_q slot, until team CTA 0 has written it;
//  * counts its piece; the unit's last piece merges the C partial states and writes the output,
//    then clears the unit's flag and piece counter and counts the launch.
// The lists and the Gamma_q slots pass between CTAs without fences: each 64- or 32-bit word
// carries a tag of this launch (from the unit's launch count), and the reader polls until the tag
// is current; a gpu-scope release in mid-stream waits for the SM's copies in flight (~2 us).
// Stage s of the ring always belongs to consumer group s % 2, in both phases.  Every cross-CTA
// wait is bounded and waits only for CTAs of the same team, which the cooperative launch keeps
// resident together; a wait that runs out sets NOSA_EFLAG_TIMEOUT and the CTA drains.
#include <algorithm>

#include "nosa_append_unit.cuh"
#include "nosa_attend.cuh"

namespace nosa {

namespace {
constexpr int kStepS = 6;                            // ring stages of 32 KiB (+ 256 B of logits)
constexpr int kStepThreads = (kConsWarps + 2) * 32;  // consumers, the producer, the selection warp
constexpr int kProducerWarp = kConsWarps;
constexpr int kSelectWarp = kConsWarps + 1;
static_assert(kStepS % kGroups == 0, "stage s must always be consumed by group s % kGroups");

// Named barriers between the consumer warps and the selection warp (one side arrives, the other
// waits): barrier 2, the consumers' lists are in shared memory; barrier 3, the selection warp is
// done (so the flag it raised and its writes come before the CTA counts its piece).
constexpr int kSelBarThreads = kConsThreads + 32;
__device__ __forceinline__ void lists_arrive() { asm volatile("bar.arrive 2, %0;" ::"n"(kSelBarThreads) : "memory"); }
__device__ __forceinline__ void lists_wait() { asm volatile("bar.sync 2, %0;" ::"n"(kSelBarThreads) : "memory"); }
__device__ __forceinline__ void select_done_arrive() {
    asm volatile("bar.arrive 3, %0;" ::"n"(kSelBarThreads) : "memory");
}
__device__ __forceinline__ void select_done_wait() { asm volatile("bar.sync 3, %0;" ::"n"(kSelBarThreads) : "memory"); }

// Tagged words.  A list entry: the key's score order (32 bits), 0x3FFF - block (14 bits: blocks
// < 2^14 at max_ctx <= 2^20) and the tag (18 bits); an empty entry is the tag alone.  A Gamma_q
// slot: (block + 1) << 18 | tag, block -1 for an empty slot.  Tags run 1 .. 2^18 - 1.
constexpr int kTagBits = 18;
constexpr uint32_t kTagMask = (1u << kTagBits) - 1u;
__device__ __forceinline__ uint32_t launch_tag(int32_t launches) { return ((uint32_t)launches % kTagMask) + 1u; }
__device__ __forceinline__ uint64_t pack_key(uint64_t key, uint32_t tag) {
    if (key == 0ull) return tag;
    return (key & 0xFFFFFFFF00000000ull) | ((uint64_t)(0x3FFFu - (uint32_t)key_block(key)) << kTagBits) | tag;
}
__device__ __forceinline__ uint64_t unpack_key(uint64_t w) {
    if ((w >> 32) == 0ull) return 0ull;
    const uint32_t blk = 0x3FFFu - (uint32_t)((w >> kTagBits) & 0x3FFFu);
    return (w & 0xFFFFFFFF00000000ull) | (uint64_t)(0xFFFFFFFFu - blk);
}
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t *p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t *p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u32(uint32_t *p, uint32_t v) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// The best 32 keys of lists l[0..n), n <= 8, merged as a tree; the merges of one level are
// independent, so their shuffle chains interleave.  Conditions are uniform over the warp.
__device__ __forceinline__ uint64_t merge_lists(uint64_t (&l)[8], int n, int lane) {
#pragma unroll
    for (int w = 1; w < 8; w <<= 1) {
#pragma unroll
        for (int i = 0; i < 8; i += 2 * w)
            if (i + w < n) list_merge(l[i], l[i + w], lane);
    }
    return l[0];
}

// The selection warp of team CTA 0: Gamma_q from the merged list, S(t) = Gamma_q U Gamma_e U
// {local} as nosa_select writes it, the Gamma_q blocks outside Gamma_e (tagged) for the decode, the
// new length.  `bitmap` already holds Gamma_e over the words of the nb_c candidates.
__device__ __forceinline__ void finalize_unit(const StepParams &sp, int32_t u, uint64_t list, int32_t L, int32_t nb_c,
                                              bool grow, uint32_t *bitmap, uint32_t tag, int lane) {
    const DecodeParams &p = sp.d;
    const int32_t myid = (lane < p.k_q && list != 0ull) ? key_block(list) : -1;
    if (sp.gq && lane < p.k_q) sp.gq[(int64_t)u * p.k_q + lane] = myid;
    int32_t *sel = sp.sel + (int64_t)u * p.max_sel;
    uint32_t *rest = sp.rest + (int64_t)u * p.k_q;
    if (L <= 0) {
        for (int i = lane; i < p.max_sel; i += 32) sel[i] = -1;
        for (int i = lane; i < p.k_q; i += 32) st_relaxed_u32(rest + i, tag);
        if (lane == 0) sp.nsel[u] = 0;
    } else {
        const int32_t nw = (nb_c + 31) >> 5;
        // Gamma_q blocks not in Gamma_e, in rank order: the decode's Gamma_q slots
        const bool fresh = myid >= 0 && myid < nb_c && !((bitmap[myid >> 5] >> (myid & 31)) & 1u);
        const unsigned m = __ballot_sync(0xFFFFFFFFu, fresh);
        if (fresh) st_relaxed_u32(rest + __popc(m & ((1u << lane) - 1u)), ((uint32_t)(myid + 1) << kTagBits) | tag);
        for (int i = __popc(m) + lane; i < p.k_q; i += 32) st_relaxed_u32(rest + i, tag);
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
    // every team CTA read the old length at its start, before it wrote its list
    if (grow && lane == 0) sp.ap.seq_len[u] = L;
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
    const int32_t L_prev = ld_volatile_s32(p.seq_len + u);
    const int32_t launches = ld_volatile_s32(sp.epoch + u);
    const uint32_t tag = launch_tag(launches);
    const bool grow = L_prev >= 0 && L_prev < p.max_ctx;
    const int32_t L = grow ? L_prev + 1 : L_prev;
    const int32_t nb_c = L > 0 ? (L - 1) / kBlock : 0;
    // this CTA's score stages [s0, s1) of the unit's ns, covering candidate blocks [s0 * kBPS, b1)
    const int32_t ns = p.k_q > 0 ? (nb_c + kBPS - 1) / kBPS : 0;
    const int32_t s0 = cidx * ns / C, s1 = (cidx + 1) * ns / C;
    const int n_sc = s1 - s0;
    const int32_t b1 = min(s1 * kBPS, nb_c);
    // and its piece of the decode slots: [e_lo, e_hi) of the k_e + 1 slots of Gamma_e (slots < k_e)
    // and the local block (slot k_e), then [q_lo, q_hi) of the k_q slots of Gamma_q \ Gamma_e
    const int32_t e_lo = cidx * (p.k_e + 1) / C, e_hi = (cidx + 1) * (p.k_e + 1) / C;
    const int32_t q_lo = cidx * p.k_q / C, q_hi = (cidx + 1) * p.k_q / C;
    const int n_items = (e_hi - e_lo) + (q_hi - q_lo);

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

    if (warp == kSelectWarp) {
        // ---------------- selection warp ----------------
        if (cidx == 0) {
            append_unit(sp.ap, u, lane, sp.ap.e_new[u], false);  // fences its writes
            __syncwarp();
            if (lane == 0) st_release_gpu(sp.appended + u, 1);
        }
        // Gamma_e as this step's append left it, in a bitmap over the candidates, ready for the
        // finalize while the lists are being scored (only the team's last CTA uses it)
        int ok = 1;
        if (lane == 0) {
            ok = flag_wait(sp.appended + u);
            if (!ok) set_error(p.err, NOSA_EFLAG_TIMEOUT);
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        __syncwarp();
        const int32_t ne = L > 0 ? min(max(__ldcg(sp.gamma_n + u), 0), p.k_e) : 0;
        int32_t ge_reg[kMaxKe / 32];
#pragma unroll
        for (int i = 0; i < kMaxKe / 32; ++i) {
            const int j = lane + 32 * i;
            ge_reg[i] = (j < ne) ? __ldcg(sp.gamma_e + (int64_t)u * p.k_e + j) : -1;
        }
        const int32_t nw = (nb_c + 31) >> 5;
        for (int i = lane; i < nw; i += 32) bitmap[i] = 0;
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kMaxKe / 32; ++i) {
            const int32_t id = ge_reg[i];
            if (id >= 0 && id < nb_c) atomicOr(&bitmap[id >> 5], 1u << (id & 31));
        }
        __syncwarp();
        // the consumers' eight lists, merged; then published to the team
        lists_wait();
        uint64_t l8[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) l8[w] = lists[w * 32 + lane];
        uint64_t list = merge_lists(l8, kConsWarps, lane);
        if (cidx > 0) {
            // to team CTA 0, tagged
            st_relaxed_u64(sp.part_keys + ((int64_t)u * C + cidx) * 32 + lane, pack_key(list, tag));
        } else {
            // the other team CTAs' lists, eight at a time, each polled until it carries this tag
            const uint64_t *all = sp.part_keys + (int64_t)u * C * 32;
            bool ok_all = true;
            for (int c0 = 1; c0 < C; c0 += 8) {
                const int n = min(8, C - c0);
                uint64_t w[8];
                bool have[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    w[j] = 0ull;
                    have[j] = j >= n;
                }
                const long long t0 = clock64();
                while (true) {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (!have[j]) {
                            w[j] = ld_relaxed_u64(all + (int64_t)(c0 + j) * 32 + lane);
                            have[j] = (uint32_t)(w[j] & kTagMask) == tag;
                        }
                    }
                    bool mine = true;
#pragma unroll
                    for (int j = 0; j < 8; ++j) mine = mine && have[j];
                    if (__all_sync(0xFFFFFFFFu, mine)) break;
                    if (__shfl_sync(0xFFFFFFFFu, (int)(clock64() - t0 > kWaitCycles), 0)) {
                        ok_all = false;
                        break;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) l8[j] = (j < n && have[j]) ? unpack_key(w[j]) : 0ull;
                list_merge(list, merge_lists(l8, n, lane), lane);
            }
            if (!ok_all && lane == 0) set_error(p.err, NOSA_EFLAG_TIMEOUT);
            finalize_unit(sp, u, list, L, nb_c, grow, bitmap, tag, lane);
        }
        select_done_arrive();
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
        // decode slots [a, b) (slot j < k_e: Gamma_e[j]; k_e: the local block; k_e + 1 + i: the
        // i-th block of Gamma_q \ Gamma_e): the block of each, fetched by the warp 32 at a time;
        // lane 0 issues
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
                        // written (tagged) by team CTA 0's selection warp: poll until current
                        const uint32_t *slot = sp.rest + (int64_t)u * p.k_q + (j - p.k_e - 1);
                        uint32_t w = ld_relaxed_u32(slot);
                        const long long t0 = clock64();
                        while ((w & kTagMask) != tag) {
                            if (clock64() - t0 > kWaitCycles) {
                                set_error(p.err, NOSA_EFLAG_TIMEOUT);
                                s_abort = 1;
                                w = tag;
                                break;
                            }
                            __nanosleep(32);
                            w = ld_relaxed_u32(slot);
                        }
                        lb = (int32_t)(w >> kTagBits) - 1;
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
            ok = flag_wait(sp.appended + u);
            if (ok) fence_proxy_async_global();  // the copies below read what the append wrote
            else { s_abort = 1; set_error(p.err, NOSA_EFLAG_TIMEOUT); }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok && !s_abort) {
            const int32_t ne = L > 0 ? min(max(__ldcg(sp.gamma_n + u), 0), p.k_e) : 0;
            issue(e_lo, e_hi, ne);
            if (q_hi > q_lo && !s_abort) issue(p.k_e + 1 + q_lo, p.k_e + 1 + q_hi, ne);
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
    lists[warp * 32 + lane] = list;  // to the selection warp; the consumers go on
    lists_arrive();

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
    select_done_wait();  // the selection warp's flag and writes come before this CTA's count
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
        // this CTA is the whole team: its producer is past the flag and the Gamma_q slots
        if (ctid == 0) {
            sp.appended[u] = 0;
            sp.epoch[u] = launches + 1;
        }
        return;
    }
    // hand-off of the partial state, as in the decode kernel
    consumer_sync();
    if (ctid == 0) s_last = ((int32_t)atom_add_acq_rel_gpu(p.counter + u, 1u) == C - 1);
    consumer_sync();
    if (!s_last) return;
    // the unit's last piece: every team CTA has finished, so no one reads the flag or the tags any more
    if (ctid == 0) {
        p.counter[u] = 0;
        sp.appended[u] = 0;
        sp.epoch[u] = launches + 1;
    }
    const float *src0 = p.part + (int64_t)u * C * kPartFloats;
    if (C <= kOnePassPieces) {
        merge_pieces_onepass<kOnePassPieces>(src0, kPartFloats, C, p.G, out, ctid);
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

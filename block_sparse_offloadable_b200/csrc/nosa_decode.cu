// nosa_decode.cu -- steps a5 (sparse decode) and a6 (dense comparator).
//
// NOSA pages: gist.science summary of arXiv:2510.13602, "ED-DMA" (the
// exponential of the eviction score is deferred to the attention step: here
// it enters the softmax as the additive logit e_j); wmrh.cn NOSA-1B release
// (exact attention over the Top-K blocks plus the current window).
//
// Design: persistent split-K flash decoding with GQA sharing.
//  * Work items are (unit, selected block) pairs, unit = (seq, kv head).  Each
//    CTA (one per SM) holds the item offsets of the units in shared memory and
//    takes an exactly balanced contiguous range of the flattened item list, so
//    every SM streams the same number of 32 KiB blocks whatever the unit count.
//    The sparse decode gives every unit max_sel items (nsel is max_sel or just
//    below it once the context holds k blocks; the -1 padding past nsel is
//    skipped), which spares a round of global reads before the first block-id
//    load; the other work lists count their items with a prefix sum.  The
//    work lists: S(t) (sparse decode), every block (dense comparator), and the
//    split decode's two passes -- Gamma_e + the local block (its softmax state
//    is kept per unit), then the rest of Gamma_q (merged with that state).
//  * One producer thread streams the range's blocks (keys + values, plus the
//    64 eviction logits) into a 6-stage shared-memory ring: four 2-D TMA tile
//    loads (64 rows x 64 dims, 128-byte swizzle) and one bulk copy per block,
//    completing on the stage's mbarrier.  The block ids of the next 32 items
//    are fetched by the whole producer warp at once.
//  * Two groups of four consumer warps take alternate blocks (stage s always
//    belongs to group s % 2); in a group each warp owns 16 of a block's 64
//    tokens.  S^T = K Q^T is
//    one m16n8k16 bf16 tensor-core tile per 16 dims (M = 16 tokens, N = the
//    <= 8 query heads of the group, so each K/V byte is read once for all
//    heads).  Key rows are read straight into A fragments with one 16-byte
//    shared load per lane per 32 dims: the dims are permuted consistently in
//    K and Q (a dot product does not care), and the token rows each lane loads
//    are permuted (0,4,1,5,2,6,3,7) so that, with the TMA swizzle, every
//    quarter-warp hits 8 distinct bank groups.
//  * Online softmax per head in the log2 domain; P is rounded to bf16,
//    transposed in registers with movmatrix, and O^T += V^T P^T runs as eight
//    more m16n8k16 tiles whose A fragments are built from 16-byte value loads
//    with byte permutes (output dims permuted, undone at the store).
//  * A CTA's range splits into unit segments.  At a segment's end the eight
//    warps merge their (m, l, o) states in shared memory (group 0 folded into
//    group 1, then the four warps, in a padded, swizzled layout that spreads
//    each warp's fragment-order stores over 32 banks; a named barrier, so the
//    producer keeps streaming); a segment covering its whole unit writes bf16
//    output, otherwise the partial state goes to the CTA's workspace slot (only
//    a CTA's first and last segments can be partial) and the last of the
//    unit's contributors to finish (atomic counter, no waiting) merges the
//    partials in CTA order and writes the output.
//  * The consumers derive segment boundaries from the item offsets, not from
//    the stream, so all four always meet at the same barriers; a bounded wait
//    that runs out sets a shared abort flag and the error word, and the rest
//    of the CTA drains without computing.
#include "nosa_attend.cuh"

namespace nosa {

namespace {
// Ring stages (one block each; one CTA per SM).  The resident pass of the
// split decode uses fewer, so that one of its CTAs and one select CTA fit on an
// SM together and the two kernels really run concurrently.
constexpr int kDecS = 6;
constexpr int kDecSResident = 4;
static_assert(kDecS % kGroups == 0 && kDecSResident % kGroups == 0,
              "stage s must always be consumed by group s % kGroups");
// Work items of unit u in the kernel's mode.
__device__ __forceinline__ int32_t unit_work(const DecodeParams &p, int32_t u) {
    const int32_t L = p.seq_len[u];
    if (L <= 0) return 0;
    switch (p.mode) {
    case kModeSel: return max(0, min(p.nsel[u], p.max_sel));
    case kModeResident: return min(max(p.gamma_n[u], 0), p.k_e) + 1;
    case kModeRest: return p.k_q;
    default: return (L + kBlock - 1) / kBlock;
    }
}

// Block id (lb; -1 = nothing to attend) and buffer block index (pb) of item j of unit u.
__device__ __forceinline__ void item_block(const DecodeParams &p, int32_t u, int32_t j, int32_t &lb, int32_t &pb) {
    if (p.mode == kModeSel) {
        lb = p.sel[(int64_t)u * p.max_sel + j];
        pb = p.block_table ? p.block_table[(int64_t)u * p.max_sel + j] : lb;
        return;
    }
    if (p.mode == kModeDense) {
        lb = pb = j;
        return;
    }
    if (p.mode == kModeResident) {
        const int32_t ne = min(max(p.gamma_n[u], 0), p.k_e);
        lb = (j < ne) ? p.gamma_e[(int64_t)u * p.k_e + j] : (p.seq_len[u] - 1) / kBlock;
    } else {  // kModeRest: Gamma_q entries not already attended by the resident pass
        lb = p.gq[(int64_t)u * p.k_q + j];
        if (lb >= 0 && lb < p.nblk &&
            ((p.res_bits[(int64_t)u * p.bits_words + (lb >> 5)] >> (lb & 31)) & 1u))
            lb = -1;
    }
    pb = (p.block_slot && lb >= 0 && lb < p.nblk) ? p.block_slot[(int64_t)u * p.nblk + lb] : lb;
}

// Merge the resident pass's state of unit u (head h, dim d) into (M, acc, lsum) in place.
__device__ __forceinline__ void merge_resident(const DecodeParams &p, int32_t u, int h, int d, float &M, float &acc,
                                               float &lsum) {
    const float *r = p.res_part + (int64_t)u * kPartFloats;
    const float rm = r[h];
    const float Mn = fmaxf(M, rm);
    if (Mn == -__builtin_huge_valf()) return;
    const float fa = (M == -__builtin_huge_valf()) ? 0.f : exp2f(M - Mn);
    const float fr = (rm == -__builtin_huge_valf()) ? 0.f : exp2f(rm - Mn);
    acc = fmaf(fr, r[2 * kMaxG + h * kD + d], fa * acc);
    lsum = fmaf(fr, r[kMaxG + h], fa * lsum);
    M = Mn;
}

// Largest u with P[u] <= x, for 0 <= x < P[U] (skips units without work).
__device__ __forceinline__ int32_t find_unit(const int32_t *P, int32_t U, int64_t x) {
    int32_t lo = 0, hi = U;
    while (hi - lo > 1) {
        const int32_t mid = (lo + hi) >> 1;
        if (P[mid] <= x) lo = mid;
        else hi = mid;
    }
    return lo;
}

// CTA whose range [c*W/G, (c+1)*W/G) holds item x (every range non-empty: W >= G).
__device__ __forceinline__ int32_t cta_of(int64_t x, int64_t W, int32_t G) {
    return (int32_t)(((x + 1) * G - 1) / W);
}

}  // namespace

size_t decode_smem_bytes(int32_t units, int stages) {
    return 1024 + (size_t)stages * kBlockBytes + (size_t)stages * kBlock * sizeof(float) +
           2 * stages * sizeof(uint64_t) + stages * sizeof(int32_t) + (size_t)kDecW * kScr * sizeof(float) +
           ((size_t)units + 1) * sizeof(int32_t);
}

int decode_ctas() { return kNumSms; }

template <int kStages>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p) {
    pdl_trigger();  // the next append's CTAs are tiny; they wait for this grid
    pdl_wait();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *tiles = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *ebuf = reinterpret_cast<float *>(tiles + kStages * kBlockBytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(ebuf + kStages * kBlock);
    uint64_t *empty = full + kStages;
    int32_t *s_blk = reinterpret_cast<int32_t *>(empty + kStages);
    float *scratch = reinterpret_cast<float *>(s_blk + kStages);
    int32_t *P = reinterpret_cast<int32_t *>(scratch + kDecW * kScr);
    __shared__ int32_t s_wsum[kConsWarps + 1];
    __shared__ int s_last;
    __shared__ volatile int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t U = p.units, G = (int32_t)gridDim.x, cta = (int32_t)blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDecW);
        }
        fence_mbar_init();
        prefetch_tmap(&tmap);
        s_abort = 0;
    }
    // ---- P[u] = items of units < u ----
    if (p.mode == kModeSel) {
        // nominal ranges: max_sel items per unit, whatever nsel (sel is -1 padded past nsel,
        // and such items are skipped); no global read stands before the first block-id load
        for (int u = threadIdx.x; u <= U; u += blockDim.x) P[u] = u * p.max_sel;
    } else {  // prefix sum of the per-unit work
        const int per = (U + kDecThreads - 1) / kDecThreads;
        const int u0 = min((int)threadIdx.x * per, U), u1 = min(u0 + per, U);
        int32_t sum = 0;
        for (int u = u0; u < u1; ++u) {
            const int32_t w = unit_work(p, u);
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
    const int64_t W = P[U];
    // Balanced: ranges over Ge <= W CTAs, so that every range holds at least one item.
    // Pieces: unit c / C, piece c % C (the host keeps C <= every unit's item count).
    const int32_t C = p.pieces;
    const int32_t Ge = (int32_t)(W < (int64_t)G ? (W > 0 ? W : 1) : (int64_t)G);
    int64_t lo, hi;
    if (C > 0) {
        const int32_t uc = cta / C, rc = cta % C;
        const int64_t a = uc < U ? P[uc] : W, n = uc < U ? P[uc + 1] - a : 0;
        lo = a + rc * n / C;
        hi = a + (rc + 1) * n / C;
    } else {
        lo = (cta < Ge) ? (int64_t)cta * W / Ge : W;
        hi = (cta < Ge) ? (int64_t)(cta + 1) * W / Ge : W;
    }
    const int32_t n_items = (int32_t)(hi - lo);

    if (warp == kConsWarps) {
        // ---------------- producer ----------------
        int it = 0;
        for (int64_t xb = lo; xb < hi && !s_abort; xb += 32) {
            const int nb = (int)((hi - xb) < 32 ? (hi - xb) : 32);
            int32_t blb = -1, bpb = -1, bu = 0;
            if (lane < nb) {
                const int64_t x = xb + lane;
                bu = find_unit(P, U, x);
                item_block(p, bu, (int32_t)(x - P[bu]), blb, bpb);
            }
            for (int k = 0; k < nb; ++k, ++it) {
                const int32_t u = __shfl_sync(0xFFFFFFFFu, bu, k);
                const int32_t lb = __shfl_sync(0xFFFFFFFFu, blb, k);
                const int32_t pb = __shfl_sync(0xFFFFFFFFu, bpb, k);
                if (lane == 0) {
                    const int s = it % kStages;
                    const bool go =
                        it < kStages || wait_or_abort(&empty[s], ((it / kStages) - 1) & 1, &s_abort, p.err);
                    if (go) {
                        const bool ok = lb >= 0 && (int64_t)lb * kBlock < p.max_ctx && pb >= 0 &&
                                        pb < p.blocks_per_unit;
                        s_blk[s] = ok ? lb : -1;
                        if (!ok && lb >= 0) set_error(p.err, NOSA_EFLAG_STATE);  // a block with no buffer
                        if (ok) {
                            const int32_t y = (int32_t)(((int64_t)u * p.blocks_per_unit + pb) * 2 * kBlock);
                            uint8_t *t = tiles + s * kBlockBytes;
                            mbar_arrive_expect_tx(&full[s], kBlockBytes + kBlock * sizeof(float));
                            tma_load_2d(t, &tmap, &full[s], 0, y);
                            tma_load_2d(t + kBoxBytes, &tmap, &full[s], 64, y);
                            tma_load_2d(t + 2 * kBoxBytes, &tmap, &full[s], 0, y + kBlock);
                            tma_load_2d(t + 3 * kBoxBytes, &tmap, &full[s], 64, y + kBlock);
                            bulk_load(ebuf + s * kBlock,
                                      p.e + (int64_t)u * p.max_ctx + (int64_t)lb * kBlock,
                                      kBlock * sizeof(float), &full[s]);
                        } else {
                            mbar_arrive(&full[s]);
                        }
                    }
                }
                __syncwarp();
            }
        }
        // never leave with copies in flight
        if (lane == 0)
            for (int i = max(0, it - kStages); i < it; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1);
    } else {
        // ---------------- consumers ----------------
        // Group g takes the CTA's items of parity g (stage s = item % 6 is always
        // group s % 2's); warp wq of a group owns tokens 16wq..16wq+15 of a block.
        const int grp = warp / kDecW, wq = warp % kDecW;
        const int r = lane >> 2, c = lane & 3;
        const int sig = (r >> 1) + ((r & 1) << 2);  // row permutation 0,4,1,5,2,6,3,7
        const int ctid = threadIdx.x;                // 0..kConsThreads-1
        WarpState st;
        st.reset();
        uint32_t qf[8][2];
        int32_t L = 0;
        // a unit's queries (B fragments, dims permuted as the key loads) and length
        auto load_unit = [&](int32_t uu) {
            const uint4 *qrow = reinterpret_cast<const uint4 *>(p.q + ((int64_t)uu * p.G + r) * kD);
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const uint4 x = (r < p.G) ? qrow[4 * jj + c] : make_uint4(0, 0, 0, 0);
                qf[2 * jj][0] = x.x; qf[2 * jj][1] = x.y;
                qf[2 * jj + 1][0] = x.z; qf[2 * jj + 1][1] = x.w;
            }
            L = p.seq_len[uu];
        };
        const int32_t first_unit = n_items > 0 ? find_unit(P, U, lo) : 0;
        int32_t u = first_unit;
        if (n_items > 0) load_unit(u);
        for (int64_t x = lo; x < hi;) {
            const int64_t seg_end = min(hi, (int64_t)P[u + 1]);
            const bool whole = (x == P[u]) && (seg_end == P[u + 1]);
            const int slot = (u == first_unit) ? 0 : 1;
            for (int64_t xi = x + ((((x - lo) & 1) != grp) ? 1 : 0); xi < seg_end; xi += kGroups) {
                const int it = (int)(xi - lo);
                const int s = it % kStages;
                if (wait_or_abort(&full[s], (it / kStages) & 1, &s_abort, p.err)) {
                    const int32_t lb = s_blk[s];
                    if (lb >= 0)
                        attend_block(st, qf, tiles + s * kBlockBytes, ebuf + s * kBlock, lb, L, p.qk_log2,
                                     wq, c, sig);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            const int32_t u_next = (seg_end < hi) ? find_unit(P, U, seg_end) : u;

            // ---- segment end: fold group 0 into group 1 lane by lane, merge the four warps ----
            fold_groups(st, scratch, grp, wq, r, c, sig);
            if (seg_end < hi) load_unit(u_next);  // in flight while the merge runs
            const int nout = p.G * kD;
            uint16_t *out = p.out + (int64_t)u * p.G * kD;
            float *part = p.part + ((int64_t)cta * 2 + slot) * kPartFloats;
            for (int idx = ctid; idx < nout; idx += kConsThreads) {
                const int h = idx >> 7, d = idx & (kD - 1);
                float M, acc, lsum;
                merged_state(scratch, h, d, M, acc, lsum);
                if (whole && p.mode == kModeResident) {
                    store_partial(p.res_part + (int64_t)u * kPartFloats, h, d, M, acc, lsum);
                } else if (whole) {
                    if (p.mode == kModeRest) merge_resident(p, u, h, d, M, acc, lsum);
                    store_bf16(out + idx, lsum > 0.f ? acc / lsum : 0.f);
                } else {
                    store_partial(part, h, d, M, acc, lsum);
                }
            }
            if (!whole) {
                // hand-off: the partial is written (barrier), one thread counts it with release
                // semantics; the unit's last contributor acquired the others' partials with the same
                // atomic, and the barrier after it orders every thread's loads below after them
                consumer_sync();
                const int32_t cf = C > 0 ? u * C : cta_of(P[u], W, Ge);
                const int32_t cl = C > 0 ? u * C + C - 1 : cta_of((int64_t)P[u + 1] - 1, W, Ge);
                if (ctid == 0) s_last = ((int32_t)atom_add_acq_rel_gpu(p.counter + u, 1u) == cl - cf);
                consumer_sync();
                if (s_last && C > 0 && C <= kOnePassPieces) {
                    // last piece of the unit: merge the C pieces' partials (piece t: slot 0 of CTA
                    // cf + t) in one pass, every thread loading what its 4 dims need at once
                    if (ctid == 0) p.counter[u] = 0;
                    merge_pieces_onepass(p.part + (int64_t)cf * 2 * kPartFloats, 2 * kPartFloats, C, p.G, out, ctid);
                } else if (s_last) {
                    // last contributor: merge the unit's partials in CTA order
                    if (ctid == 0) p.counter[u] = 0;
                    // the CTA partials (and, merging the rest pass, the resident state)
                    const int nc = cl - cf + 1 + (p.mode == kModeRest ? 1 : 0);  // <= Ge + 1
                    const MergeScratch ms = merge_scratch(scratch, nc);
                    for (int t = ctid; t < nc; t += kConsThreads) {
                        const int32_t cc = cf + t;
                        if (cc > cl) {
                            ms.src[t] = p.res_part + (int64_t)u * kPartFloats;
                        } else {
                            const int sl = (C > 0 || find_unit(P, U, (int64_t)cc * W / Ge) == u) ? 0 : 1;
                            ms.src[t] = p.part + (int64_t)(cc * 2 + sl) * kPartFloats;
                        }
                    }
                    consumer_sync();
                    merge_general(ms, nc, p.G, out,
                                  p.mode == kModeResident ? p.res_part + (int64_t)u * kPartFloats : nullptr, warp,
                                  lane, ctid);
                }
            }
            consumer_sync();  // scratch and s_last are reused by the next segment
            st.reset();
            x = seg_end;
            u = u_next;
        }
        // units without work, one CTA each: zero output (an empty state in the
        // resident pass; the resident state alone in the rest pass)
        for (int32_t uz = cta; uz < U; uz += G) {
            if (P[uz + 1] != P[uz]) continue;
            if (p.mode == kModeResident) {
                float *rp = p.res_part + (int64_t)uz * kPartFloats;
                for (int i = ctid; i < kPartFloats; i += kConsThreads) rp[i] = (i < kMaxG) ? kNegInf : 0.f;
                continue;
            }
            uint16_t *out = p.out + (int64_t)uz * p.G * kD;
            for (int idx = ctid; idx < p.G * kD; idx += kConsThreads) {
                float M = kNegInf, acc = 0.f, lsum = 0.f;
                if (p.mode == kModeRest) merge_resident(p, uz, idx >> 7, idx & (kD - 1), M, acc, lsum);
                store_bf16(out + idx, lsum > 0.f ? acc / lsum : 0.f);
            }
        }
        // the resident pass also leaves, per unit, the set it covered (for the rest pass)
        if (p.mode == kModeResident) {
            for (int32_t uz = cta; uz < U; uz += G) {
                uint32_t *bits = p.res_bits + (int64_t)uz * p.bits_words;
                for (int i = ctid; i < p.bits_words; i += kConsThreads) bits[i] = 0u;
                consumer_sync();
                const int32_t Lz = p.seq_len[uz];
                const int32_t ne = Lz > 0 ? min(max(p.gamma_n[uz], 0), p.k_e) : -1;
                for (int j = ctid; j <= ne; j += kConsThreads) {
                    const int32_t b = (j < ne) ? p.gamma_e[(int64_t)uz * p.k_e + j] : (Lz - 1) / kBlock;
                    if (b >= 0 && b < p.nblk) atomicOr(&bits[b >> 5], 1u << (b & 31));
                }
            }
        }
    }
}

template <int kStages>
int launch_decode_t(const DecodeParams &p, const CUtensorMap &tmap, cudaStream_t stream) {
    const size_t smem = decode_smem_bytes(p.units, kStages);
    if (cudaFuncSetAttribute(decode_kernel<kStages>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return NOSA_ERR_CUDA;
    const int grid = p.pieces > 0 ? p.units * p.pieces : decode_ctas();
    return launch_pdl(decode_kernel<kStages>, dim3(grid), dim3(kDecThreads), smem, stream, tmap, p) ==
                   cudaSuccess
               ? NOSA_OK
               : NOSA_ERR_CUDA;
}

int launch_decode(const DecodeParams &p, const CUtensorMap &tmap, cudaStream_t stream) {
    return p.mode == kModeResident ? launch_decode_t<kDecSResident>(p, tmap, stream)
                                   : launch_decode_t<kDecS>(p, tmap, stream);
}

}  // namespace nosa

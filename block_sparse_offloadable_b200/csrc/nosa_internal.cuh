// nosa_internal.cuh -- kernel parameter blocks and launchers shared by the
// libnosa translation units (not part of the C ABI).
#pragma once

#include <utility>

#include "nosa_common.cuh"

namespace nosa {

struct AppendParams {
    const uint16_t *k_new;   // [u][T][D]
    const uint16_t *v_new;   // [u][T][D]
    const float *e_new;      // [u][T], or null when the eviction head computes e
    const float *w1;         // eviction head: [Hkv][D][kHeadH] or null
    const float *w2;         // [Hkv][kHeadH]
    const int32_t *lens;     // [B] or null (prefill)
    uint8_t *store;          // device address of the KV store (device memory or mapped host)
    uint8_t *cache;          // offload cache or null
    float *e_store;          // [u][max_ctx]
    void *ck;                // [u][nsub][D] fp32, or bf16 when ck_bf16
    double *blk_evict;       // [u][nblk]
    int32_t *gamma_e;        // [u][k_e]
    int32_t *gamma_n;        // [u]
    int32_t *seq_len;        // [u]
    int32_t *slot_block;     // [u][nslots]
    int32_t *block_slot;     // [u][nblk]
    uint32_t *err;
    int64_t max_ctx;
    int32_t *pool;           // [u][nblk] fill reading: not-dropped candidates by E rank
    int32_t *pool_n;         // [u]
    int32_t nblk, nsub, nslots, units, heads_kv, k_e, offload, T, ck_bf16, fill;
};

struct SelectParams {
    const uint16_t *q;        // [B][Hq][D]
    const void *ck;           // [u][nsub][D] fp32, or bf16 when ck_bf16
    const int32_t *gamma_e;   // [u][k_e]
    const int32_t *gamma_n;   // [u]
    const int32_t *seq_len;   // [u]
    int32_t *sel;             // [u][max_sel]
    int32_t *nsel;            // [u]
    int32_t *gq;              // [u][k_q] or null
    uint64_t *part_keys;      // [u][nchunks][32]
    int32_t *counter;         // [u]
    uint32_t *err;
    int32_t *gamma_e_out;     // fill reading: Gamma_e and |Gamma_e| written here
    int32_t *gamma_n_out;
    int32_t *pool;            // [u][nblk] fill reading
    int32_t *pool_n;          // [u]
    int32_t nsub, nblk, G, units, nchunks, chunk_blocks, k_q, k_e, max_sel, ck_bf16, fill;
    float scale;
    int32_t fused;            // append this step's token first (chunk 0's extra warp), see nosa_select.cu
    AppendParams ap;          // the append's parameters when fused (T = 1)
};

struct CacheParams {
    const int32_t *sel;       // [u][max_sel]
    const int32_t *nsel;      // [u]
    const uint8_t *store;     // device address of the host KV store
    uint8_t *cache;           // [u][nslots][2][64][D]
    int32_t *slot_block;      // [u][nslots]
    int32_t *block_slot;      // [u][nblk]
    int32_t *block_table;     // [u][max_sel]
    int32_t *n_fetched;       // [u] or null: copy of miss_count
    int32_t *miss_count;      // [u] workspace: blocks to fetch per unit
    uint32_t *miss_list;      // [u][max_sel] workspace: (slot << 20 | block) of each block to fetch
    uint32_t *err;
    int32_t nblk, nslots, units, max_sel;
};

// Work lists of the decode kernel.
constexpr int kModeSel = 0;       // the blocks of S(t) (sel / nsel)
constexpr int kModeDense = 1;     // every block (the dense comparator)
constexpr int kModeResident = 2;  // Gamma_e + the local block, known right after the append
constexpr int kModeRest = 3;      // the blocks of Gamma_q outside Gamma_e + local, merged with the above

struct DecodeParams {
    const uint16_t *q;          // [B][Hq][D]
    const int32_t *sel;         // [u][max_sel] (kModeSel)
    const int32_t *nsel;        // [u]
    const int32_t *block_table; // [u][max_sel] or null (block id addresses the store)
    const float *e;             // [u][max_ctx]
    const int32_t *seq_len;     // [u]
    uint16_t *out;              // [B][Hq][D]
    float *part;                // [decode CTAs][2][kPartFloats]: first / last segment partials
    int32_t *counter;           // [u]
    uint32_t *err;
    int64_t max_ctx;
    int32_t blocks_per_unit;    // blocks per unit in the tensor-mapped buffer (nblk or nslots)
    int32_t max_sel, G, units;
    float qk_log2;              // scale * log2(e)
    int32_t mode;
    int32_t pieces;             // 0: balanced ranges over decode_ctas() CTAs; C >= 1: U*C CTAs, CTA c
                                // streams piece c % C (of C equal pieces) of unit c / C
    const int32_t *gamma_e;     // kModeResident: [u][k_e] ascending, and gamma_n [u]
    const int32_t *gamma_n;
    const int32_t *gq;          // kModeRest: [u][k_q] Gamma_q, -1 padded
    const int32_t *block_slot;  // kModeResident / kModeRest with offload: [u][nblk] cache slot, else null
    float *res_part;            // [u][kPartFloats] state over Gamma_e + local (written by resident, read by rest)
    uint32_t *res_bits;         // [u][bits_words] membership of Gamma_e + local (same)
    int32_t k_e, k_q, nblk, bits_words;
};

constexpr int kPartFloats = 2 * kMaxG + kMaxG * kD;  // m[8], l[8], o[8][128]

// The fused step (nosa_fused_step): append + select + sparse decode of a device-resident store in
// one launch, a team of C CTAs per unit.  Decode fields: q, e, seq_len, out, err, max_ctx,
// blocks_per_unit (nblk), max_sel, G, units, qk_log2, pieces (C), k_e, k_q, nblk; part holds one
// record per CTA, counter counts a unit's finished pieces.
struct StepParams {
    DecodeParams d;
    AppendParams ap;          // T = 1
    const void *ck;           // [u][nsub][D] fp32, or bf16 when ck_bf16
    const int32_t *gamma_e;   // [u][k_e], read after the unit's append
    const int32_t *gamma_n;   // [u]
    int32_t *sel;             // [u][max_sel] out
    int32_t *nsel;            // [u] out
    int32_t *gq;              // [u][k_q] out or null
    uint64_t *part_keys;      // [u][C][32] workspace: each team CTA's top-32 list, tagged
    int32_t *epoch;           // [u] workspace: launches completed (tags this launch's lists and slots)
    int32_t *appended;        // [u] workspace: 1 = this launch's append is done
    uint32_t *rest;           // [u][k_q] workspace: Gamma_q \ Gamma_e in rank order, tagged
    int32_t nsub, ck_bf16;
    float scale;
};

int launch_append(const AppendParams &p, cudaStream_t stream);
int launch_select(const SelectParams &p, cudaStream_t stream);
int launch_cache_sync(const CacheParams &p, cudaStream_t stream);
int launch_decode(const DecodeParams &p, const CUtensorMap &tmap, cudaStream_t stream);
int launch_step(const StepParams &p, const CUtensorMap &tmap, cudaStream_t stream);

// The argument checks of nosa_select (config, state, pointers, workspace), with
// nothing launched: NOSA_OK or the code nosa_select would return before a launch.
int select_args_ok(const nosa_config *c, const nosa_state *st, const uint16_t *q, int32_t *sel, int32_t *nsel,
                   int32_t *gq, void *ws, size_t ws_bytes);

// Launch geometry, shared by the launchers and the workspace-size queries.
int select_chunk_blocks(int32_t units, int32_t nblk, bool ck_bf16);
int decode_ctas();
// CTAs per unit of the fused step: as many as fit on the SMs at one CTA per SM (at most one per
// decode item), or 1 when the units alone fill the GPU.
int step_team_size(int32_t units, int32_t max_sel);
size_t step_smem_bytes(int32_t nblk);
constexpr int kMaxUnits = 2048;  // (seq, kv head) units per call: the decode kernel's prefix sums live in shared memory

constexpr int kNumSms = 148;

// Split each unit's `work` items into n chunks (one CTA each) to minimise
//   ceil(units*n / slots) * (ceil(work/n) + ovh) + merge * (ceil(n/4) + 1),
// the wave-quantised time plus the merge of the n chunk results by the unit's
// last CTA, a tree over its four consumer warps (ceil(n/4) + 1 levels); `slots`
// CTAs run at once, `ovh` is the per-CTA fixed cost and `merge` the cost of one
// merge level, both in work items.
inline int best_chunks(int64_t units, int64_t work, int64_t slots, int64_t ovh, int64_t nmax, int64_t merge = 0) {
    if (nmax < 1) nmax = 1;
    int64_t best_n = 1, best_cost = -1;
    for (int64_t n = 1; n <= nmax; ++n) {
        const int64_t waves = (units * n + slots - 1) / slots;
        const int64_t cost = waves * ((work + n - 1) / n + ovh) + merge * ((n + 3) / 4 + 1);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best_n = n; }
    }
    return (int)best_n;
}

// Launch with programmatic stream serialization (the kernel must call pdl_wait()
// before touching global memory).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace nosa

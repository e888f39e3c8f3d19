// nosa_api.cu -- the C ABI of libnosa: argument validation, buffer sizes,
// tensor maps and kernel launches.  Declarations and contracts: include/nosa.h.
#include <algorithm>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "nosa_internal.cuh"

using namespace nosa;

namespace {

constexpr int64_t kMaxCtx = 1ll << 20;

struct Geo {
    int64_t units, nblk, nsub, nslots, max_sel, G;
};

bool geo_of(const nosa_config *c, Geo *g) {
    if (nosa_validate_config(c) != NOSA_OK) return false;
    g->units = (int64_t)c->batch * c->heads_kv;
    g->nblk = c->max_ctx / kBlock;
    g->nsub = c->max_ctx / kSub;
    g->nslots = c->k_q + c->k_e + 2;
    g->max_sel = c->k_q + c->k_e + 1;
    g->G = c->heads_q / c->heads_kv;
    return true;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Kind of memory behind p: cudaMemoryTypeDevice / Host / Managed / Unregistered.
int mem_kind(const void *p, void **dev_addr) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return cudaMemoryTypeUnregistered;
    }
    if (dev_addr) *dev_addr = a.devicePointer;
    return a.type;
}

bool is_device(const void *p) {
    const int k = mem_kind(p, nullptr);
    return k == cudaMemoryTypeDevice || k == cudaMemoryTypeManaged;
}

int check_dev(const void *p, bool need16) {
    if (!p) return NOSA_ERR_PTR;
    if (need16 && !aligned16(p)) return NOSA_ERR_PTR;
    return is_device(p) ? NOSA_OK : NOSA_ERR_PTR;
}

// Device address of the KV store: device memory (offload 0) or mapped host memory (offload 1).
int store_addr(const nosa_config *c, const nosa_state *st, uint8_t **out) {
    if (!st->kv_store || !aligned16(st->kv_store)) return NOSA_ERR_PTR;
    void *dev = nullptr;
    const int k = mem_kind(st->kv_store, &dev);
    if (c->offload) {
        if (k != cudaMemoryTypeHost || !dev || !aligned16(dev)) return NOSA_ERR_PTR;
    } else {
        if (k != cudaMemoryTypeDevice && k != cudaMemoryTypeManaged) return NOSA_ERR_PTR;
        dev = st->kv_store;
    }
    *out = static_cast<uint8_t *>(dev);
    return NOSA_OK;
}

int check_state(const nosa_config *c, const nosa_state *st) {
    if (!st) return NOSA_ERR_ARG;
    int rc;
    if ((rc = check_dev(st->evict_logit, true)) || (rc = check_dev(st->ck, true)) ||
        (rc = check_dev(st->blk_evict, true)) || (rc = check_dev(st->gamma_n, false)) ||
        (rc = check_dev(st->seq_len, false)) || (rc = check_dev(st->err, false)))
        return rc;
    if (c->k_e > 0 && (rc = check_dev(st->gamma_e, false))) return rc;
    if (c->offload) {
        if ((rc = check_dev(st->cache, true)) || (rc = check_dev(st->slot_block, false)) ||
            (rc = check_dev(st->block_slot, false)))
            return rc;
    }
    if ((c->flags & NOSA_FLAG_FILL) &&
        ((rc = check_dev(st->pool, false)) || (rc = check_dev(st->pool_n, false))))
        return rc;
    return NOSA_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tensor map over a block-major KV buffer seen as [rows][128] bf16 rows,
// box = 64 rows x 64 dims (128 bytes), 128-byte swizzle.
int kv_tensor_map(CUtensorMap *map, const void *base, int64_t rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
    if (!enc) return NOSA_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kRowBytes};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? NOSA_OK : NOSA_ERR_CUDA;
}

int select_nchunks(const nosa_config *c, const Geo &g) {
    if (c->k_q <= 0) return 1;
    const int cb = select_chunk_blocks((int32_t)g.units, (int32_t)g.nblk, (c->flags & NOSA_FLAG_CK_BF16) != 0);
    int64_t n = (g.nblk - 1 + cb - 1) / cb;
    return n < 1 ? 1 : (int)n;
}

// Words of the per-unit block bitmap in the split-decode buffer.
size_t split_bits_words(const Geo &g) { return (size_t)g.nblk / 32 + 1; }

// Workspace of the fused step: [launch count, piece counter, "appended" flag, spare] per unit, then
// each team CTA's top-32 list, each CTA's partial state, and each unit's Gamma_q \ Gamma_e list.
struct StepWs {
    int32_t C;
    size_t keys, parts, rest, total;
};

StepWs step_ws(const nosa_config *c, const Geo &g) {
    StepWs w;
    w.C = step_team_size((int32_t)g.units, (int32_t)g.max_sel);
    const size_t ctas = (size_t)g.units * w.C;
    w.keys = align256((size_t)g.units * 4 * sizeof(int32_t));
    w.parts = w.keys + align256(ctas * 32 * sizeof(uint64_t));
    w.rest = w.parts + align256(ctas * kPartFloats * sizeof(float));
    w.total = w.rest + (size_t)g.units * (c->k_q > 0 ? c->k_q : 1) * sizeof(int32_t);
    return w;
}

size_t ws_bytes_of(const nosa_config *c, int which) {
    Geo g;
    if (!geo_of(c, &g)) return 0;
    const size_t counters = align256((size_t)g.units * sizeof(int32_t));
    if (which == NOSA_WS_SELECT) {
        const int n = select_nchunks(c, g);
        return n > 1 ? counters + (size_t)g.units * n * 32 * sizeof(uint64_t) : 0;
    }
    if (which == NOSA_WS_SPARSE_DECODE || which == NOSA_WS_DENSE_DECODE)
        return counters + (size_t)decode_ctas() * 2 * kPartFloats * sizeof(float);
    if (which == NOSA_WS_CACHE_SYNC)
        return c->offload ? counters + (size_t)g.units * g.max_sel * sizeof(uint32_t) : 0;
    if (which == NOSA_WS_SPLIT)
        return align256((size_t)g.units * kPartFloats * sizeof(float)) +
               (size_t)g.units * split_bits_words(g) * sizeof(uint32_t);
    if (which == NOSA_WS_FUSED_STEP) {
        if (c->offload || (c->flags & NOSA_FLAG_FILL)) return 0;
        const StepWs w = step_ws(c, g);
        return w.total;
    }
    return 0;
}

int check_ws(const nosa_config *c, int which, void *ws, size_t ws_bytes) {
    const size_t need = ws_bytes_of(c, which);
    if (need == 0) return NOSA_OK;
    if (!ws || ws_bytes < need) return NOSA_ERR_CAPACITY;
    return check_dev(ws, true);
}

// One decode launch in the given mode (kMode*): the work list, where the blocks
// live, and where the result goes differ; see nosa_decode.cu.
int run_decode(const nosa_config *c, const nosa_state *st, const uint16_t *q, int mode, const int32_t *sel,
               const int32_t *nsel, const int32_t *block_table, const int32_t *gq, void *split,
               size_t split_bytes, uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    Geo g;
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    geo_of(c, &g);
    if ((rc = check_state(c, st))) return rc;
    if ((rc = check_dev(q, true))) return rc;
    if (mode != kModeResident && (rc = check_dev(out, true))) return rc;
    if (mode == kModeSel) {
        if ((rc = check_dev(sel, false)) || (rc = check_dev(nsel, false))) return rc;
        if (c->offload && (rc = check_dev(block_table, false))) return rc;
    }
    if (mode == kModeResident || mode == kModeRest) {
        if (c->flags & NOSA_FLAG_FILL) return NOSA_ERR_UNSUPPORTED;  // Gamma_e needs Gamma_q there
        if ((rc = check_ws(c, NOSA_WS_SPLIT, split, split_bytes))) return rc;
        if (mode == kModeRest && c->k_q > 0 && (rc = check_dev(gq, false))) return rc;
    }
    const int which = mode == kModeDense ? NOSA_WS_DENSE_DECODE : NOSA_WS_SPARSE_DECODE;
    if ((rc = check_ws(c, which, ws, ws_bytes))) return rc;

    const void *base;
    int64_t bpu;
    if (c->offload) {
        base = st->cache;
        bpu = g.nslots;
    } else {
        uint8_t *s;
        if ((rc = store_addr(c, st, &s))) return rc;
        base = s;
        bpu = g.nblk;
    }
    CUtensorMap map;
    if ((rc = kv_tensor_map(&map, base, g.units * bpu * 2 * kBlock))) return rc;

    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.q = q;
    p.mode = mode;
    p.sel = mode == kModeSel ? sel : nullptr;
    p.nsel = mode == kModeSel ? nsel : nullptr;
    p.block_table = (mode == kModeSel && c->offload) ? block_table : nullptr;
    if (mode == kModeResident || mode == kModeRest) {
        p.gamma_e = st->gamma_e; p.gamma_n = st->gamma_n; p.k_e = c->k_e;
        p.gq = c->k_q > 0 ? gq : nullptr; p.k_q = c->k_q;
        p.block_slot = c->offload ? st->block_slot : nullptr;
        p.nblk = (int32_t)g.nblk;
        p.bits_words = (int32_t)split_bits_words(g);
        p.res_part = static_cast<float *>(split);
        p.res_bits = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(split) +
                                                  align256((size_t)g.units * kPartFloats * sizeof(float)));
    }
    p.e = st->evict_logit;
    p.seq_len = st->seq_len;
    p.out = out;
    p.err = st->err;
    p.max_ctx = c->max_ctx;
    p.blocks_per_unit = (int32_t)bpu;
    p.max_sel = (int32_t)g.max_sel;
    p.G = (int32_t)g.G;
    p.units = (int32_t)g.units;
    p.qk_log2 = c->scale * 1.4426950408889634f;
    p.counter = static_cast<int32_t *>(ws);
    p.part = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align256((size_t)g.units * sizeof(int32_t)));
    // S(t) gives every unit max_sel nominal items.  With no more units than decode CTAs, each CTA
    // streams one equal piece of one unit: a CTA then ends at most one partial state, at its end,
    // instead of stalling mid-stream on the hand-off of a unit it shares with its neighbour.
    if (mode == kModeSel && g.units <= decode_ctas())
        p.pieces = (int32_t)std::min<int64_t>(decode_ctas() / g.units, g.max_sel);
    return launch_decode(p, map, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int nosa_validate_config(const nosa_config *c) {
    if (!c) return NOSA_ERR_ARG;
    if (c->batch < 1 || c->heads_kv < 1 || c->heads_q < 1 || c->heads_q % c->heads_kv) return NOSA_ERR_ARG;
    if (c->k_q < 0 || c->k_e < 0 || c->k_q + c->k_e < 1 || c->max_ctx <= 0 ||
        c->max_ctx % 64 || (c->flags & ~(NOSA_FLAG_CK_BF16 | NOSA_FLAG_FILL)) != 0 || !(c->scale > 0.f) || !isfinite(c->scale))
        return NOSA_ERR_ARG;
    if (c->offload != 0 && c->offload != 1) return NOSA_ERR_ARG;
    if (c->head_dim != kD || c->block != kBlock || c->sub_block != kSub || c->local_blocks != 1)
        return NOSA_ERR_UNSUPPORTED;
    if (c->heads_q / c->heads_kv > kMaxG || c->k_q > kMaxKq || c->k_e > kMaxKe)
        return NOSA_ERR_UNSUPPORTED;
    if (c->max_ctx > kMaxCtx) return NOSA_ERR_CAPACITY;
    const int64_t units = (int64_t)c->batch * c->heads_kv;
    if (units > kMaxUnits) return NOSA_ERR_CAPACITY;
    const int64_t rows = units * (c->max_ctx / kBlock) * 2 * kBlock;
    if (rows >= (1ll << 31)) return NOSA_ERR_CAPACITY;
    return NOSA_OK;
}

size_t nosa_state_bytes(const nosa_config *c, int which) {
    Geo g;
    if (!geo_of(c, &g)) return 0;
    const size_t u = (size_t)g.units;
    switch (which) {
    case NOSA_BUF_KV_STORE: return u * g.nblk * kBlockBytes;
    case NOSA_BUF_EVICT_LOGIT: return u * c->max_ctx * sizeof(float);
    case NOSA_BUF_CK: return u * g.nsub * kD * ((c->flags & NOSA_FLAG_CK_BF16) ? 2 : sizeof(float));
    case NOSA_BUF_BLK_EVICT: return u * g.nblk * sizeof(double);
    case NOSA_BUF_GAMMA_E: return u * (c->k_e > 0 ? c->k_e : 1) * sizeof(int32_t);
    case NOSA_BUF_GAMMA_N:
    case NOSA_BUF_SEQ_LEN: return u * sizeof(int32_t);
    case NOSA_BUF_CACHE: return c->offload ? u * g.nslots * kBlockBytes : 0;
    case NOSA_BUF_SLOT_BLOCK: return c->offload ? u * g.nslots * sizeof(int32_t) : 0;
    case NOSA_BUF_BLOCK_SLOT: return c->offload ? u * g.nblk * sizeof(int32_t) : 0;
    case NOSA_BUF_ERR: return sizeof(uint32_t);
    case NOSA_BUF_POOL: return (c->flags & NOSA_FLAG_FILL) ? u * g.nblk * sizeof(int32_t) : 0;
    case NOSA_BUF_POOL_N: return (c->flags & NOSA_FLAG_FILL) ? u * sizeof(int32_t) : 0;
    default: return 0;
    }
}

size_t nosa_workspace_bytes(const nosa_config *c, int which) { return ws_bytes_of(c, which); }

int nosa_state_init(const nosa_config *c, const nosa_state *st, void *stream) {
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    if ((rc = check_state(c, st))) return rc;
    uint8_t *s;
    if ((rc = store_addr(c, st, &s))) return rc;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    bool ok = cudaMemsetAsync(st->gamma_n, 0, nosa_state_bytes(c, NOSA_BUF_GAMMA_N), cs) == cudaSuccess &&
              cudaMemsetAsync(st->seq_len, 0, nosa_state_bytes(c, NOSA_BUF_SEQ_LEN), cs) == cudaSuccess &&
              cudaMemsetAsync(st->err, 0, sizeof(uint32_t), cs) == cudaSuccess;
    if (ok && (c->flags & NOSA_FLAG_FILL))
        ok = cudaMemsetAsync(st->pool_n, 0, nosa_state_bytes(c, NOSA_BUF_POOL_N), cs) == cudaSuccess;
    if (ok && c->offload) {
        ok = cudaMemsetAsync(st->slot_block, 0xFF, nosa_state_bytes(c, NOSA_BUF_SLOT_BLOCK), cs) == cudaSuccess &&
             cudaMemsetAsync(st->block_slot, 0xFF, nosa_state_bytes(c, NOSA_BUF_BLOCK_SLOT), cs) == cudaSuccess &&
             cudaMemsetAsync(st->cache, 0, nosa_state_bytes(c, NOSA_BUF_CACHE), cs) == cudaSuccess;
    }
    return ok ? NOSA_OK : NOSA_ERR_CUDA;
}

namespace {
// nosa_compress_append with e_new given, or with the eviction head (w1, w2) computing it.
// Validated parameters of an append (e_new given, or the eviction head w1, w2).
int make_append(const nosa_config *c, const nosa_state *st, const uint16_t *k_new, const uint16_t *v_new,
                const float *e_new, const float *w1, const float *w2, int32_t T, const int32_t *lens,
                AppendParams *out) {
    Geo g;
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    geo_of(c, &g);
    if ((rc = check_state(c, st))) return rc;
    if (T < 1) return NOSA_ERR_ARG;
    if (T > c->max_ctx) return NOSA_ERR_CAPACITY;
    if ((rc = check_dev(k_new, true)) || (rc = check_dev(v_new, true))) return rc;
    if (w1) {
        if ((rc = check_dev(w1, true)) || (rc = check_dev(w2, true))) return rc;
    } else if ((rc = check_dev(e_new, false))) {
        return rc;
    }
    if (lens) {
        if (T == 1) return NOSA_ERR_ARG;
        if ((rc = check_dev(lens, false))) return rc;
    }
    uint8_t *s;
    if ((rc = store_addr(c, st, &s))) return rc;
    AppendParams p;
    memset(&p, 0, sizeof(p));
    p.k_new = k_new; p.v_new = v_new; p.e_new = w1 ? nullptr : e_new; p.lens = lens;
    p.w1 = w1; p.w2 = w1 ? w2 : nullptr;
    p.store = s;
    p.cache = static_cast<uint8_t *>(c->offload ? st->cache : nullptr);
    p.e_store = st->evict_logit; p.ck = st->ck; p.blk_evict = st->blk_evict;
    p.gamma_e = st->gamma_e; p.gamma_n = st->gamma_n; p.seq_len = st->seq_len;
    p.slot_block = st->slot_block; p.block_slot = st->block_slot; p.err = st->err;
    p.max_ctx = c->max_ctx;
    p.nblk = (int32_t)g.nblk; p.nsub = (int32_t)g.nsub; p.nslots = (int32_t)g.nslots;
    p.units = (int32_t)g.units; p.heads_kv = c->heads_kv; p.k_e = c->k_e;
    p.offload = c->offload; p.T = T; p.ck_bf16 = (c->flags & NOSA_FLAG_CK_BF16) != 0;
    p.fill = (c->flags & NOSA_FLAG_FILL) != 0;
    p.pool = p.fill ? st->pool : nullptr; p.pool_n = p.fill ? st->pool_n : nullptr;
    *out = p;
    return NOSA_OK;
}

int append_impl(const nosa_config *c, const nosa_state *st, const uint16_t *k_new, const uint16_t *v_new,
                const float *e_new, const float *w1, const float *w2, int32_t T, const int32_t *lens,
                void *stream) {
    AppendParams p;
    const int rc = make_append(c, st, k_new, v_new, e_new, w1, w2, T, lens, &p);
    return rc ? rc : launch_append(p, static_cast<cudaStream_t>(stream));
}

// Validated parameters of a select.
int make_select(const nosa_config *c, const nosa_state *st, const uint16_t *q, int32_t *sel, int32_t *nsel,
                int32_t *gq, void *ws, size_t ws_bytes, SelectParams *out) {
    Geo g;
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    geo_of(c, &g);
    if ((rc = check_state(c, st))) return rc;
    if ((rc = check_dev(q, true)) || (rc = check_dev(sel, false)) || (rc = check_dev(nsel, false)))
        return rc;
    if (gq && (rc = check_dev(gq, false))) return rc;
    if ((rc = check_ws(c, NOSA_WS_SELECT, ws, ws_bytes))) return rc;
    SelectParams p;
    memset(&p, 0, sizeof(p));
    p.q = q; p.ck = st->ck; p.gamma_e = st->gamma_e; p.gamma_n = st->gamma_n; p.seq_len = st->seq_len;
    p.sel = sel; p.nsel = nsel; p.gq = c->k_q > 0 ? gq : nullptr; p.err = st->err;
    p.nsub = (int32_t)g.nsub; p.nblk = (int32_t)g.nblk; p.G = (int32_t)g.G; p.units = (int32_t)g.units;
    p.nchunks = select_nchunks(c, g);
    p.chunk_blocks = c->k_q > 0 ? select_chunk_blocks(p.units, p.nblk, (c->flags & NOSA_FLAG_CK_BF16) != 0) : p.nblk;
    p.k_q = c->k_q; p.k_e = c->k_e; p.max_sel = (int32_t)g.max_sel; p.scale = c->scale;
    p.ck_bf16 = (c->flags & NOSA_FLAG_CK_BF16) != 0;
    p.fill = (c->flags & NOSA_FLAG_FILL) != 0;
    p.pool = p.fill ? st->pool : nullptr; p.pool_n = p.fill ? st->pool_n : nullptr;
    p.gamma_e_out = p.fill ? st->gamma_e : nullptr; p.gamma_n_out = p.fill ? st->gamma_n : nullptr;
    if (p.nchunks > 1) {
        p.counter = static_cast<int32_t *>(ws);
        p.part_keys = reinterpret_cast<uint64_t *>(static_cast<uint8_t *>(ws) +
                                                   align256((size_t)g.units * sizeof(int32_t)));
    }
    *out = p;
    return NOSA_OK;
}
}  // namespace

int nosa_compress_append(const nosa_config *c, const nosa_state *st, const uint16_t *k_new,
                         const uint16_t *v_new, const float *e_new, int32_t T, const int32_t *lens,
                         void *stream) {
    if (!e_new) return NOSA_ERR_ARG;
    return append_impl(c, st, k_new, v_new, e_new, nullptr, nullptr, T, lens, stream);
}

int nosa_compress_append_head(const nosa_config *c, const nosa_state *st, const uint16_t *k_new,
                              const uint16_t *v_new, const float *w1, const float *w2, int32_t T,
                              const int32_t *lens, void *stream) {
    if (!w1 || !w2) return NOSA_ERR_ARG;
    return append_impl(c, st, k_new, v_new, nullptr, w1, w2, T, lens, stream);
}

int nosa_select(const nosa_config *c, const nosa_state *st, const uint16_t *q, int32_t *sel,
                int32_t *nsel, int32_t *gq, void *ws, size_t ws_bytes, void *stream) {
    SelectParams p;
    const int rc = make_select(c, st, q, sel, nsel, gq, ws, ws_bytes, &p);
    return rc ? rc : launch_select(p, static_cast<cudaStream_t>(stream));
}

int nosa_append_select(const nosa_config *c, const nosa_state *st, const uint16_t *k_new, const uint16_t *v_new,
                       const float *e_new, const uint16_t *q, int32_t *sel, int32_t *nsel, int32_t *gq, void *ws,
                       size_t ws_bytes, void *stream) {
    if (!e_new) return NOSA_ERR_ARG;
    AppendParams a;
    SelectParams p;
    int rc;
    if ((rc = make_append(c, st, k_new, v_new, e_new, nullptr, nullptr, 1, nullptr, &a))) return rc;
    if ((rc = make_select(c, st, q, sel, nsel, gq, ws, ws_bytes, &p))) return rc;
    p.fused = 1;
    p.ap = a;
    return launch_select(p, static_cast<cudaStream_t>(stream));
}

int nosa_fused_step(const nosa_config *c, const nosa_state *st, const uint16_t *k_new, const uint16_t *v_new,
                    const float *e_new, const uint16_t *q, int32_t *sel, int32_t *nsel, int32_t *gq, uint16_t *out,
                    void *ws, size_t ws_bytes, void *stream) {
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    if (c->offload || (c->flags & NOSA_FLAG_FILL)) return NOSA_ERR_UNSUPPORTED;
    if (!e_new) return NOSA_ERR_ARG;
    AppendParams a;
    if ((rc = make_append(c, st, k_new, v_new, e_new, nullptr, nullptr, 1, nullptr, &a))) return rc;
    if ((rc = check_dev(q, true)) || (rc = check_dev(sel, false)) || (rc = check_dev(nsel, false)) ||
        (rc = check_dev(out, true)))
        return rc;
    if (gq && (rc = check_dev(gq, false))) return rc;
    if ((rc = check_ws(c, NOSA_WS_FUSED_STEP, ws, ws_bytes))) return rc;
    Geo g;
    geo_of(c, &g);
    CUtensorMap map;
    if ((rc = kv_tensor_map(&map, a.store, g.units * g.nblk * 2 * kBlock))) return rc;
    const StepWs w = step_ws(c, g);
    uint8_t *wb = static_cast<uint8_t *>(ws);
    StepParams sp;
    memset(&sp, 0, sizeof(sp));
    DecodeParams &p = sp.d;
    p.q = q;
    p.mode = kModeSel;
    p.e = st->evict_logit;
    p.seq_len = st->seq_len;
    p.out = out;
    p.err = st->err;
    p.max_ctx = c->max_ctx;
    p.blocks_per_unit = (int32_t)g.nblk;
    p.max_sel = (int32_t)g.max_sel;
    p.G = (int32_t)g.G;
    p.units = (int32_t)g.units;
    p.qk_log2 = c->scale * 1.4426950408889634f;
    p.pieces = w.C;
    p.k_e = c->k_e;
    p.k_q = c->k_q;
    p.nblk = (int32_t)g.nblk;
    p.counter = reinterpret_cast<int32_t *>(wb) + g.units;
    p.part = reinterpret_cast<float *>(wb + w.parts);
    sp.ap = a;
    sp.ck = st->ck;
    sp.gamma_e = st->gamma_e;
    sp.gamma_n = st->gamma_n;
    sp.sel = sel;
    sp.nsel = nsel;
    sp.gq = c->k_q > 0 ? gq : nullptr;
    sp.epoch = reinterpret_cast<int32_t *>(wb);
    sp.appended = reinterpret_cast<int32_t *>(wb) + 2 * g.units;
    sp.part_keys = reinterpret_cast<uint64_t *>(wb + w.keys);
    sp.rest = reinterpret_cast<uint32_t *>(wb + w.rest);
    sp.nsub = (int32_t)g.nsub;
    sp.ck_bf16 = (c->flags & NOSA_FLAG_CK_BF16) != 0;
    sp.scale = c->scale;
    return launch_step(sp, map, static_cast<cudaStream_t>(stream));
}

int nosa_cache_sync(const nosa_config *c, const nosa_state *st, const int32_t *sel,
                    const int32_t *nsel, int32_t *block_table, int32_t *n_fetched, void *ws,
                    size_t ws_bytes, void *stream) {
    Geo g;
    int rc;
    if ((rc = nosa_validate_config(c))) return rc;
    if (!c->offload) return NOSA_ERR_ARG;
    geo_of(c, &g);
    if ((rc = check_state(c, st))) return rc;
    if ((rc = check_dev(sel, false)) || (rc = check_dev(nsel, false)) ||
        (rc = check_dev(block_table, false)))
        return rc;
    if (n_fetched && (rc = check_dev(n_fetched, false))) return rc;
    if ((rc = check_ws(c, NOSA_WS_CACHE_SYNC, ws, ws_bytes))) return rc;
    uint8_t *s;
    if ((rc = store_addr(c, st, &s))) return rc;
    CacheParams p;
    memset(&p, 0, sizeof(p));
    p.sel = sel; p.nsel = nsel; p.store = s; p.cache = static_cast<uint8_t *>(st->cache);
    p.slot_block = st->slot_block; p.block_slot = st->block_slot; p.block_table = block_table;
    p.n_fetched = n_fetched; p.err = st->err;
    p.miss_count = static_cast<int32_t *>(ws);
    p.miss_list = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) +
                                               align256((size_t)g.units * sizeof(int32_t)));
    p.nblk = (int32_t)g.nblk; p.nslots = (int32_t)g.nslots; p.units = (int32_t)g.units;
    p.max_sel = (int32_t)g.max_sel;
    return launch_cache_sync(p, static_cast<cudaStream_t>(stream));
}

int nosa_sparse_decode(const nosa_config *c, const nosa_state *st, const uint16_t *q,
                       const int32_t *sel, const int32_t *nsel, const int32_t *block_table,
                       uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    return run_decode(c, st, q, kModeSel, sel, nsel, block_table, nullptr, nullptr, 0, out, ws, ws_bytes, stream);
}

int nosa_decode_resident(const nosa_config *c, const nosa_state *st, const uint16_t *q, void *split,
                         size_t split_bytes, void *ws, size_t ws_bytes, void *stream) {
    return run_decode(c, st, q, kModeResident, nullptr, nullptr, nullptr, nullptr, split, split_bytes, nullptr,
                      ws, ws_bytes, stream);
}

int nosa_decode_rest(const nosa_config *c, const nosa_state *st, const uint16_t *q, const int32_t *gq,
                     const void *split, size_t split_bytes, uint16_t *out, void *ws, size_t ws_bytes,
                     void *stream) {
    return run_decode(c, st, q, kModeRest, nullptr, nullptr, nullptr, gq, const_cast<void *>(split), split_bytes,
                      out, ws, ws_bytes, stream);
}

int nosa_dense_decode(const nosa_config *c, const nosa_state *st, const uint16_t *q,
                      uint16_t *out, void *ws, size_t ws_bytes, void *stream) {
    if (c && c->offload) return NOSA_ERR_ARG;
    return run_decode(c, st, q, kModeDense, nullptr, nullptr, nullptr, nullptr, nullptr, 0, out, ws, ws_bytes,
                      stream);
}

int nosa_read_error(const nosa_state *st, uint32_t *flags, int clear, void *stream) {
    if (!st || !flags) return NOSA_ERR_ARG;
    int rc;
    if ((rc = check_dev(st->err, false))) return rc;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, st->err, sizeof(h), cudaMemcpyDeviceToHost, cs) != cudaSuccess ||
        cudaStreamSynchronize(cs) != cudaSuccess)
        return NOSA_ERR_CUDA;
    if (clear && (cudaMemsetAsync(st->err, 0, sizeof(uint32_t), cs) != cudaSuccess ||
                  cudaStreamSynchronize(cs) != cudaSuccess))
        return NOSA_ERR_CUDA;
    *flags = h;
    return h ? NOSA_ERR_DEVICE : NOSA_OK;
}

const char *nosa_strerror(int code) {
    switch (code) {
    case NOSA_OK: return "ok";
    case NOSA_ERR_ARG: return "invalid argument";
    case NOSA_ERR_CAPACITY: return "size exceeds buffer or kernel capacity";
    case NOSA_ERR_PTR: return "pointer of the wrong memory kind or misaligned";
    case NOSA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case NOSA_ERR_TIMEOUT: return "bounded device wait ran out";
    case NOSA_ERR_UNSUPPORTED: return "configuration not supported by this build";
    case NOSA_ERR_DEVICE: return "device error word has bits set";
    default: return "unknown error";
    }
}

}  // extern "C"

int nosa::select_args_ok(const nosa_config *c, const nosa_state *st, const uint16_t *q, int32_t *sel, int32_t *nsel,
                         int32_t *gq, void *ws, size_t ws_bytes) {
    SelectParams p;
    return make_select(c, st, q, sel, nsel, gq, ws, ws_bytes, &p);
}

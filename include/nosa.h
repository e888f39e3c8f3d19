/*
 * nosa.h -- C ABI of libnosa: the per-step decode hot path of NOSA (Native and
 * Offloadable Sparse Attention, arXiv:2510.13602) on one B200 (sm_100a).
 *
 * One decode step of one attention layer is four calls, in this order, on the
 * same CUDA stream:
 *   nosa_compress_append  append the new token; pool what completes; update Gamma_e
 *   nosa_select           two-stage block scores, Gamma_q, union with Gamma_e and local
 *   nosa_cache_sync       (offload mode) swap blocks: fetch misses host -> device cache
 *   nosa_sparse_decode    exact softmax attention over the selected blocks
 * or three, with nosa_append_select doing the first two in one launch; with the KV
 * store in device memory, nosa_fused_step does the whole step in one launch.  Also:
 * nosa_compress_append_head (the eviction logits from the fused eviction head),
 * nosa_decode_resident + nosa_decode_rest (the attention split around the
 * select and the cache sync), nosa_dense_decode (the full-attention
 * comparator), nosa_select_noalloc, and the nosa_check_wait_timeout diagnostic.
 *
 * Units.  A "unit" is one (sequence b, kv head g) pair, u = b * heads_kv + g.
 * Blocks are 64 tokens, sub-blocks 16 tokens; block j holds positions
 * 64j..64j+63.  With L tokens in a unit, blocks 0 .. (L-1)/64 - 1 are the
 * candidates and block (L-1)/64 is the local block (always kept, never
 * scored, not counted in k = k_q + k_e).
 *
 * Memory.  The caller allocates every buffer (sizes from nosa_state_bytes and
 * nosa_workspace_bytes).  The library allocates nothing and keeps no state
 * besides a cached driver entry point (and the fixed scratch array of
 * nosa_select_noalloc).  Every call is asynchronous on the
 * given stream and validates its arguments on the host before launching
 * anything; a non-zero return means nothing was launched.  Conditions only
 * the device can see (a sequence outgrowing max_ctx, a bounded wait running
 * out) set bits in the device error word (nosa_state.err) and the kernel skips
 * the affected unit; read them with nosa_read_error.
 *
 * Pointers are plain addresses: "device" means device global memory; "host"
 * means page-locked host memory that the device can address (cudaHostAlloc /
 * cudaMallocHost, or cudaHostRegister with cudaHostRegisterMapped).  bf16
 * tensors are passed as uint16_t bit patterns.  Streams are cudaStream_t
 * values passed as void* (NULL = legacy default stream).
 */
#ifndef NOSA_H
#define NOSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define NOSA_OK 0
#define NOSA_ERR_ARG (-1)          /* bad argument or inconsistent configuration */
#define NOSA_ERR_CAPACITY (-2)     /* a size exceeds what the buffers or the kernels hold */
#define NOSA_ERR_PTR (-3)          /* pointer of the wrong kind or misaligned */
#define NOSA_ERR_CUDA (-4)         /* a CUDA call or kernel launch failed */
#define NOSA_ERR_TIMEOUT (-5)      /* reserved: a bounded device wait ran out */
#define NOSA_ERR_UNSUPPORTED (-6)  /* valid but not built (e.g. head_dim != 128) */
#define NOSA_ERR_DEVICE (-7)       /* nosa_read_error found device error bits */

/* Device error-word bits (nosa_state.err). */
#define NOSA_EFLAG_CAPACITY 0x1u   /* append beyond max_ctx: token dropped */
#define NOSA_EFLAG_TIMEOUT 0x2u    /* a bounded mbarrier wait gave up: output of that tile invalid */
#define NOSA_EFLAG_NOSLOT 0x4u     /* offload cache had no free slot: token dropped */
#define NOSA_EFLAG_STATE 0x8u      /* state inconsistent (prefill into a non-empty unit, lost local block,
                                       a block to attend that has no cache slot) */

/*
 * Problem configuration.  Built: head_dim 128, block 64, sub_block 16,
 * local_blocks 1, 1 <= heads_q/heads_kv <= 8, 0 <= k_q <= 32,
 * 0 <= k_e <= 256, max_ctx a positive multiple of 64 and <= 2^20, and
 * batch * heads_kv <= 2048, and batch * heads_kv * max_ctx * 2 < 2^31
 * (tensor-map row coordinates).
 */
typedef struct nosa_config {
    int32_t batch;        /* B sequences */
    int32_t heads_q;      /* Hq query heads */
    int32_t heads_kv;     /* Hkv kv heads; G = Hq / Hkv query heads share one kv head */
    int32_t head_dim;     /* D */
    int32_t block;        /* tokens per block (64) */
    int32_t sub_block;    /* tokens per sub-block (16) */
    int32_t k_q;          /* query-aware budget: Gamma_q = top-k_q blocks by query score */
    int32_t k_e;          /* query-agnostic budget: Gamma_e = top-k_e blocks by eviction score */
    int32_t local_blocks; /* local window in blocks (1) */
    int32_t offload;      /* 0: KV store in device memory; 1: KV store in host memory + device block cache */
    int64_t max_ctx;      /* capacity in tokens per sequence */
    float scale;          /* softmax scale of q.k (normally 1/sqrt(D)) */
    int32_t flags;        /* NOSA_FLAG_* bits; 0 = defaults */
} nosa_config;

/*
 * Pooled keys stored as bf16 (the fp64 sub-block mean rounded to the nearest
 * bf16, ties to even) instead of fp32: half the bytes nosa_select streams.
 */
#define NOSA_FLAG_CK_BF16 0x1

/*
 * "Fill" combination of the two selections (montaan.com summary of
 * 2510.13602, "Key Design Components" item 4: query-aware blocks first, the
 * remainder filled with query-agnostic ones; item 1: a block the selection
 * lets go is never selected by the query-agnostic part again).  Gamma_e is
 * then the top-k_e by E among the candidates outside Gamma_q that have been
 * selected at every step since they became candidates (or since the
 * prefill); Sel = Gamma_q and Gamma_e are disjoint, |Sel| <= k.  Without the
 * flag Gamma_e is the independent top-k_e and Sel their union.
 */
#define NOSA_FLAG_FILL 0x2

/*
 * Per-layer state.  Every buffer is caller-owned; nosa_state_bytes(cfg, NOSA_BUF_x)
 * gives its size.  Layouts (u = unit, nblk = max_ctx/64, nsub = max_ctx/16,
 * nslots = k_q + k_e + 2):
 *   kv_store    bf16 [u][nblk][2][64][D]; [..][0] = keys, [..][1] = values.
 *               Device memory if offload == 0, host memory if offload == 1.
 *   evict_logit fp32 [u][max_ctx]   per-token eviction logit e_j (device)
 *   ck          fp32 [u][nsub][D]   compressed keys: mean of each 16-token sub-block (device);
 *               bf16 [u][nsub][D] with NOSA_FLAG_CK_BF16
 *   blk_evict   fp64 [u][nblk]      block eviction score E_b, pre-exponential (device)
 *   gamma_e     int32 [u][k_e]      Gamma_e block ids, ascending; in E-rank order with
 *                                   NOSA_FLAG_FILL (device)
 *   gamma_n     int32 [u]           |Gamma_e| (device)
 *   seq_len     int32 [u]           tokens held, L (device)
 *   cache       bf16 [u][nslots][2][64][D]  offload block cache (device; NULL if offload == 0)
 *   slot_block  int32 [u][nslots]   block held by each cache slot, -1 = free (device; offload only)
 *   block_slot  int32 [u][nblk]     cache slot of each block, -1 = not resident (device; offload only)
 *   err         uint32 [1]          device error word (device)
 *   pool        int32 [u][nblk]     NOSA_FLAG_FILL only: the candidates not yet dropped,
 *               sorted by E descending, ties to the lower block (device; NULL otherwise)
 *   pool_n      int32 [u]           NOSA_FLAG_FILL only: entries in pool (device)
 * nosa_state_init must run once before the first append.
 */
typedef struct nosa_state {
    void *kv_store;
    float *evict_logit;
    void *ck;
    double *blk_evict;
    int32_t *gamma_e;
    int32_t *gamma_n;
    int32_t *seq_len;
    void *cache;
    int32_t *slot_block;
    int32_t *block_slot;
    uint32_t *err;
    int32_t *pool;
    int32_t *pool_n;
} nosa_state;

enum nosa_buffer {
    NOSA_BUF_KV_STORE = 0,
    NOSA_BUF_EVICT_LOGIT,
    NOSA_BUF_CK,
    NOSA_BUF_BLK_EVICT,
    NOSA_BUF_GAMMA_E,
    NOSA_BUF_GAMMA_N,
    NOSA_BUF_SEQ_LEN,
    NOSA_BUF_CACHE,
    NOSA_BUF_SLOT_BLOCK,
    NOSA_BUF_BLOCK_SLOT,
    NOSA_BUF_ERR,
    NOSA_BUF_POOL,
    NOSA_BUF_POOL_N,
    NOSA_BUF_COUNT
};

enum nosa_call {
    NOSA_WS_SELECT = 0,
    NOSA_WS_SPARSE_DECODE = 1,
    NOSA_WS_DENSE_DECODE = 2,
    NOSA_WS_CACHE_SYNC = 3,
    NOSA_WS_SPLIT = 4,  /* the buffer nosa_decode_resident fills and nosa_decode_rest reads */
    NOSA_WS_FUSED_STEP = 5
};

/* Validate a configuration: NOSA_OK or a negative code. */
int nosa_validate_config(const nosa_config *cfg);

/* Bytes of one state buffer (0 if the buffer is unused in this mode, or cfg invalid). */
size_t nosa_state_bytes(const nosa_config *cfg, int which);

/*
 * Bytes of scratch workspace a call needs (device memory).  A workspace must
 * be zero-filled once after allocation; every completed call leaves its
 * counters at zero again, so it can be reused by later calls on the same
 * stream.  Two calls that overlap on the GPU must not share a workspace.
 */
size_t nosa_workspace_bytes(const nosa_config *cfg, int which_call);

/* Reset a state: empty sequences, empty Gamma_e, empty cache, error word 0. */
int nosa_state_init(const nosa_config *cfg, const nosa_state *st, void *stream);

/*
 * a1 -- append + compress.  NOSA pages: montaan.com summary of 2510.13602,
 * "Key Design Components" item 2 (mean pooling within sub-blocks, max pooling
 * across them, for both selections); gist.science summary, "Mecanisme de
 * double selection" (Gamma_e and its eviction rule) and "ED-DMA" (the
 * eviction score stays pre-exponential).
 *
 *   k_new, v_new  device bf16 [u][T][D]   keys / values of the appended tokens
 *   e_new         device fp32 [u][T]      their eviction logits
 *   T             1 = decode (append one token to every unit);
 *                 T > 1 = prefill of empty units (every seq_len must be 0)
 *   lens          device int32 [B] or NULL: prefill only, tokens of sequence b
 *                 (<= T; ragged batches); NULL = T for every sequence
 *
 * For each unit: stores the rows at position L (offload: into the device cache
 * slot of the local block, and written through to the host store); when a
 * 16-token sub-block completes, stores its mean key (fp64 sum of the bf16
 * keys, stored fp32, or rounded to bf16 with NOSA_FLAG_CK_BF16); when a 64-token block completes, stores E_b = max over
 * its sub-blocks of the mean eviction logit (fp64); when a block becomes a
 * candidate, it enters Gamma_e if |Gamma_e| < k_e, or replaces the member with
 * the lowest E if its E is strictly higher (the member is then dropped for
 * good).  With NOSA_FLAG_FILL the candidate instead joins the pool at its
 * rank, and nosa_select forms Gamma_e.  Prefill builds the pooled arrays and
 * Gamma_e = top-k_e by E (ties to the lower block), with NOSA_FLAG_FILL the
 * pool of every candidate in rank order, and, in offload mode, puts the local
 * block and the Gamma_e blocks in the cache (from the prefill input, without a
 * host transfer), so that Gamma_e is resident from the first decode step on.
 * Device errors: NOSA_EFLAG_CAPACITY (L + T > max_ctx; unit skipped),
 * NOSA_EFLAG_STATE (prefill into a non-empty unit), NOSA_EFLAG_NOSLOT.
 */
int nosa_compress_append(const nosa_config *cfg, const nosa_state *st, const uint16_t *k_new,
                         const uint16_t *v_new, const float *e_new, int32_t T, const int32_t *lens,
                         void *stream);

/* Hidden width of the eviction head of nosa_compress_append_head. */
#define NOSA_EVICT_HIDDEN 128

/*
 * a1 with the eviction head fused in.  NOSA pages: montaan.com summary of
 * 2510.13602, "Key Design Components" item 3 (Equation 4: the eviction score
 * of token j is tau(v_j W1) W2 with tau = softplus) and "System Optimization
 * (NOSI)" item 1 (the eviction head fused into the kernel that splits QKV).
 *
 *   w1  device fp32 [Hkv][D][NOSA_EVICT_HIDDEN]   one head per kv head (row d, column h),
 *       16-byte aligned
 *   w2  device fp32 [Hkv][NOSA_EVICT_HIDDEN], 16-byte aligned
 *
 * As nosa_compress_append, but the eviction logit of every appended token is
 * computed from its value row in the same launch instead of being passed in:
 *   e_j = sum_h w2[g][h] * softplus( sum_d v_j[d] * w1[g][d][h] ),
 * in fp64 with each product and sum rounded on its own, sums in index order,
 * softplus(x) = max(x, 0) + log1p(exp(-|x|)), rounded once to fp32 and stored
 * in evict_logit.  Same device errors as nosa_compress_append.
 */
int nosa_compress_append_head(const nosa_config *cfg, const nosa_state *st, const uint16_t *k_new,
                              const uint16_t *v_new, const float *w1, const float *w2, int32_t T,
                              const int32_t *lens, void *stream);

/*
 * a2 + a3 -- two-stage block scoring and dual selection.  NOSA pages:
 * wmrh.cn NOSA-1B release ("two-stage attention: select Top-K blocks with
 * compressed KV, then exact attention"); montaan.com items 2 and 4
 * (Equation 7, the k_q / k_e budgets); gist.science "Mecanisme de double
 * selection".
 *
 *   q      device bf16 [B][Hq][D]  this step's queries
 *   sel    device int32 [u][k_q+k_e+1] out: S(t) = (Gamma_q U Gamma_e) U {local},
 *          ascending (the local block, the largest id, last), -1 padded
 *   nsel   device int32 [u] out: |S(t)|
 *   gq     device int32 [u][k_q] out or NULL: Gamma_q in rank order, -1 padded
 *   ws     device workspace of nosa_workspace_bytes(cfg, NOSA_WS_SELECT) bytes
 *
 * s_b = max over the four sub-blocks s of b of  (sum over the G query heads h
 * of kv head g of q_h) . kbar_s * scale, in fp32, for every candidate b;
 * Gamma_q = the k_q highest (ties to the lower block).  Uses Gamma_e as left
 * by nosa_compress_append; with NOSA_FLAG_FILL, takes Gamma_e = the first
 * k_e pool entries outside Gamma_q (written to gamma_e in rank order, and
 * gamma_n), then keeps in the pool only the entries in Sel.
 */
int nosa_select(const nosa_config *cfg, const nosa_state *st, const uint16_t *q, int32_t *sel,
                int32_t *nsel, int32_t *gq, void *ws, size_t ws_bytes, void *stream);

/*
 * a1 (decode, T = 1) and a2 + a3 in one launch: nosa_compress_append(T = 1)
 * followed by nosa_select, with the same arguments, results and device errors,
 * but without a launch between them.  The append runs on an extra warp of
 * one CTA per unit while the pooled keys stream (the scoring reads nothing the
 * append writes: the pooled key and eviction score it may complete belong to
 * the local block, which is never a candidate).  The new Gamma_e (or fill
 * pool) and length are read and written by the unit's finalizing CTA, after
 * every CTA of the unit is done.  Eviction logits given (not the fused head).
 */
int nosa_append_select(const nosa_config *cfg, const nosa_state *st, const uint16_t *k_new,
                       const uint16_t *v_new, const float *e_new, const uint16_t *q, int32_t *sel,
                       int32_t *nsel, int32_t *gq, void *ws, size_t ws_bytes, void *stream);

/*
 * a1 (decode, T = 1) + a2 + a3 + a5 in one launch, for a KV store in device
 * memory: nosa_append_select followed by nosa_sparse_decode, with the same
 * arguments, results and device errors (out equal up to the order of
 * floating-point sums), but one kernel.  NOSA pages: as those calls; the
 * overlap follows from the dual selection (gist.science summary of
 * 2510.13602, "Mecanisme de double selection"; montaan.com "Key Design
 * Components" item 4): Gamma_e needs no query, so its blocks and the local
 * block are attended while the query-aware scores are being computed, and only
 * the blocks of Gamma_q outside Gamma_e wait for the selection.
 *
 *   k_new, v_new, e_new, q, sel, nsel, gq   as nosa_append_select
 *   out   device bf16 [B][Hq][D] out, as nosa_sparse_decode
 *   ws    device workspace of nosa_workspace_bytes(cfg, NOSA_WS_FUSED_STEP) bytes
 *
 * Each unit is served by a team of CTAs that wait on one another (bounded
 * waits); with several CTAs per unit the kernel is launched cooperatively, so
 * the whole grid (at most one CTA per SM) must be able to run at once:
 * NOSA_ERR_CUDA if it cannot.  The workspace keeps a count of launches per
 * unit (it tags what the team's CTAs pass to one another), so after the
 * one-time zero fill it must serve only this state's nosa_fused_step calls.  NOSA_ERR_UNSUPPORTED with offload == 1 (the
 * cache sync runs between the selection and the decode) or NOSA_FLAG_FILL
 * (Gamma_e is formed after Gamma_q there).
 */
int nosa_fused_step(const nosa_config *cfg, const nosa_state *st, const uint16_t *k_new, const uint16_t *v_new,
                    const float *e_new, const uint16_t *q, int32_t *sel, int32_t *nsel, int32_t *gq, uint16_t *out,
                    void *ws, size_t ws_bytes, void *stream);

/*
 * a4 -- block cache synchronisation (offload mode).  NOSA pages: montaan.com
 * "System Optimization (NOSI)" item 2 (block-sized KV units on GPU and CPU;
 * only blocks unused in the current step are swapped out) and item 3 (a
 * transfer kernel reading host memory directly through UVA); gist.science
 * "Systeme : NOSI" (set-difference kernels for block swapping).
 *
 *   sel, nsel    from nosa_select
 *   block_table  device int32 [u][k_q+k_e+1] out: cache slot of each sel entry, -1 padded
 *   n_fetched    device int32 [u] out or NULL: blocks fetched from the host this step
 *   ws           device workspace of nosa_workspace_bytes(cfg, NOSA_WS_CACHE_SYNC) bytes
 *
 * Frees every slot whose block is not in S(t), assigns the freed slots (in
 * ascending order) to the blocks of S(t) that are not resident (in ascending
 * block order), and copies each such block (32 KiB: keys and values) from the
 * host store into its slot with 16-byte loads through the device mapping of
 * host memory, the copy split evenly over all SMs.  Offload mode only
 * (NOSA_ERR_ARG otherwise).
 */
int nosa_cache_sync(const nosa_config *cfg, const nosa_state *st, const int32_t *sel,
                    const int32_t *nsel, int32_t *block_table, int32_t *n_fetched, void *ws,
                    size_t ws_bytes, void *stream);

/*
 * a5 -- sparse decode.  NOSA pages: gist.science "ED-DMA" (the exponent of
 * the eviction score is applied in the attention step) and wmrh.cn (exact
 * attention over the selected blocks).
 *
 *   q            device bf16 [B][Hq][D]
 *   sel, nsel    from nosa_select
 *   block_table  device int32 [u][k_q+k_e+1] from nosa_cache_sync (offload), or NULL
 *                (device store: block ids address the store directly)
 *   out          device bf16 [B][Hq][D] out
 *   ws           device workspace of nosa_workspace_bytes(cfg, NOSA_WS_SPARSE_DECODE) bytes
 *
 * For every query head h of kv head g: o_h = sum_j p_j v_j with
 * p = softmax_j(q_h . k_j * scale + e_j) over the tokens j < L of the blocks
 * in sel; bf16 inputs, fp32 accumulation, bf16 output (round to nearest even).
 */
int nosa_sparse_decode(const nosa_config *cfg, const nosa_state *st, const uint16_t *q,
                       const int32_t *sel, const int32_t *nsel, const int32_t *block_table,
                       uint16_t *out, void *ws, size_t ws_bytes, void *stream);

/*
 * a6 -- dense comparator (FullAttn of the NOSA pages, montaan.com "The
 * gist"): the same attention, with the same e_j bias, over all L tokens.
 * Device store only (offload == 0; NOSA_ERR_ARG otherwise).
 */
int nosa_dense_decode(const nosa_config *cfg, const nosa_state *st, const uint16_t *q,
                      uint16_t *out, void *ws, size_t ws_bytes, void *stream);

/*
 * a5 split in two, so that the blocks already on the GPU are attended while
 * the missed ones are fetched.  NOSA pages: montaan.com summary of
 * 2510.13602, "Empirical Results and Analysis" item 4 (the wall-time
 * breakdown: decoding is bound by KV loading) and "System Optimization
 * (NOSI)" item 2 (only blocks unused in the current step are swapped out).
 * Union reading only (NOSA_ERR_UNSUPPORTED with NOSA_FLAG_FILL, where Gamma_e
 * depends on Gamma_q).
 *
 * nosa_decode_resident: right after nosa_compress_append of the step, and
 * concurrently with nosa_select / nosa_cache_sync (another stream).  Attends
 * over R(t) = Gamma_e(t) + {local block} as left by the append; every block of
 * R(t) is on the GPU already (Gamma_e(t) lies in S(t-1) plus the previous
 * local block, and a cache sync never frees a block of S(t)).  Writes into
 * `split` (nosa_workspace_bytes(cfg, NOSA_WS_SPLIT) bytes, device) each unit's
 * softmax state over R(t) and the set R(t).
 *
 * nosa_decode_rest: after nosa_select (its gq output), nosa_cache_sync and
 * nosa_decode_resident.  Attends over Gamma_q(t) minus R(t), merges with the
 * state in `split`, and writes `out` exactly as nosa_sparse_decode would (up
 * to the order of floating-point sums).
 *
 *   ws  device workspace of nosa_workspace_bytes(cfg, NOSA_WS_SPARSE_DECODE) bytes each;
 *       the two calls may share one, as they never overlap
 */
int nosa_decode_resident(const nosa_config *cfg, const nosa_state *st, const uint16_t *q, void *split,
                         size_t split_bytes, void *ws, size_t ws_bytes, void *stream);
int nosa_decode_rest(const nosa_config *cfg, const nosa_state *st, const uint16_t *q, const int32_t *gq,
                     const void *split, size_t split_bytes, uint16_t *out, void *ws, size_t ws_bytes,
                     void *stream);

/*
 * Read the device error word (synchronises the stream).  *flags receives the
 * bits; if clear != 0 the word is reset to 0.  Returns NOSA_OK if no bit was
 * set, NOSA_ERR_DEVICE if some was, or another negative code.
 */
int nosa_read_error(const nosa_state *st, uint32_t *flags, int clear, void *stream);

/*
 * Diagnostic (the pages have no counterpart): runs the library's bounded
 * mbarrier wait, with a bound of max_cycles SM clock cycles (1 .. 2^32), on a
 * phase that no thread completes, and sets NOSA_EFLAG_TIMEOUT in the device
 * word *err when the bound runs out -- the path every pipeline wait of the
 * library takes if its copies never land.  The kernel then returns normally.
 *   err  device uint32 [1]
 */
int nosa_check_wait_timeout(uint32_t *err, int64_t max_cycles, void *stream);

/*
 * nosa_select without a caller-provided workspace, for callers that cannot
 * allocate device memory (a plug-in that is handed only its inputs and
 * outputs, or a path that must not call cudaMalloc because it may
 * synchronise the device).  The NOSA paper has no counterpart of this entry
 * point; it exists for such integrations.
 *
 * Same arguments, outputs and results as nosa_select, minus ws/ws_bytes.  The
 * scratch lives in a fixed __device__ array of NOSA_NOALLOC_SELECT_SCRATCH
 * bytes inside the library (every GPU that loads the library holds it until
 * the process exits); configurations whose nosa_workspace_bytes(cfg,
 * NOSA_WS_SELECT) exceeds that size are rejected with NOSA_ERR_CAPACITY.  The
 * function allocates nothing.  Its first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, that device current); make
 * that first call before any stream capture.  Each call clears the array's
 * counters on the stream before the kernel, after every argument check has
 * passed: a refused call queues nothing.  `stream` must belong to the current
 * device: the array's address is looked up for the current device, and the
 * call does not check the stream's device.  All calls on a device
 * share the one array, which keeps the last call's contents: calls that
 * overlap on the GPU (other streams, other threads) race and must not be
 * issued.
 */
#define NOSA_NOALLOC_SELECT_SCRATCH (1u << 20)
int nosa_select_noalloc(const nosa_config *cfg, const nosa_state *st, const uint16_t *q,
                        int32_t *sel, int32_t *nsel, int32_t *gq, void *stream);

/*
 * Test hook of nosa_select_noalloc (no paper counterpart): fill the whole
 * shared scratch array of the current device with `byte`, on `stream`, as an
 * interrupted earlier call could have left it.  A following
 * nosa_select_noalloc must still give nosa_select's results.  `stream` must
 * belong to the current device; allocates nothing.
 */
int nosa_noalloc_scratch_poison(uint8_t byte, void *stream);

/* Human-readable text of a return code. */
const char *nosa_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* NOSA_H */

/*
 * nosa_oracle.c -- plain, slow, single-threaded CPU oracle of one NOSA decode
 * step, in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this file.  It shares no code with the
 * CUDA library (no headers, helpers or constants); the only thing both sides
 * have in common is the seeded input generator, whose bytes they consume.
 *
 * Source: "NOSA: Native and Offloadable Sparse Attention" (arXiv:2510.13602)
 * as summarised on the montaan.com and gist.science pages:
 *   - two-stage block scoring: mean pooling of keys inside 16-token
 *     sub-blocks, q.k over the pooled keys, max pooling to 64-token blocks
 *     (montaan.com, "Key Design Components" item 2; gist.science,
 *     "Implementation par blocs");
 *   - dual selection: query-aware top-k_q (Gamma_q) and query-agnostic
 *     top-k_e (Gamma_e) by an eviction score that is kept pre-exponential
 *     (gist.science, "Mecanisme de double selection", "ED-DMA");
 *   - budgeted union of the two, at most k = k_q + k_e blocks (montaan.com,
 *     item 4, Equation 7), plus the current window (wmrh.cn: only the current
 *     window and the Top-K blocks stay on the GPU);
 *   - eviction rule: a block not selected by Gamma_e at step t is never
 *     selected by it again (montaan.com item 1; gist.science);
 *   - locality bound gamma(t) >= k_e/k (montaan.com, Equation 3;
 *     gist.science, "Garantie de localite");
 *   - exact attention over the selected blocks with the eviction exponent
 *     applied inside the softmax (gist.science, "ED-DMA").
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - Gamma_q and Gamma_e are independent top-k's whose union is taken.
 *     Alternative reading, "fill" (item 4 of the same summary: query-aware
 *     blocks first, the remainder filled by query-agnostic ones): Gamma_e is
 *     the top-k_e by E among the candidates that are neither in Gamma_q nor
 *     dropped, where a block is dropped for good at the first step at which
 *     no component selects it.  Sel then has up to k blocks, disjoint parts.
 *   - A query-group (GQA) score is the sum over its q heads of q_h . kbar.
 *   - Sub-blocks are 16 aligned, non-overlapping tokens; 4 per block.  The
 *     eviction score of a block is the same two-stage pooling applied to the
 *     per-token eviction logits (mean inside a sub-block, max over the
 *     block's sub-blocks).
 *   - The eviction exponent enters the softmax as an additive logit bias
 *     e_j, i.e. weight ~ exp(q.k * scale) * exp(e_j).
 *   - The local window is the block holding the newest token (truncated at L);
 *     it is always kept and not counted in k.
 *   - Ties in any top-k go to the lower block index.
 *   - After a prefill, Gamma_e is the plain top-k_e; nothing is marked
 *     dropped before the first decode step; the block cache holds Gamma_e and
 *     the local block (the prefill has them at hand, so no transfer).
 *   - Decode order: append the token, then select, then attend (the new token
 *     attends to itself).
 *
 * Pins: see tests/test_oracle_pins.py.  Parity of the GQA-sum reading and of
 * the union reading is not fixed by the pages (parity unpinned for those two
 * readings; both sides follow them).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t D, G, block, sub, k_q, k_e;
    int32_t ck_bf16;         /* pooled keys stored as bf16 (nearest, ties to even) */
    int32_t fill;            /* "fill" reading of the Gamma_q / Gamma_e combination */
    double scale;
    int64_t cap, L;
    uint16_t *K, *V;         /* [cap][D] bf16 bits */
    float *e;                /* [cap] eviction logits */
    double *ck;              /* [cap/sub][D] compressed (mean-pooled) keys */
    double *E;               /* [cap/block] block eviction scores */
    unsigned char *dropped;  /* [cap/block] dropped from Gamma_e once */
    unsigned char *ge_inc;   /* [cap/block] incrementally maintained Gamma_e */
    int32_t n_ge_inc;
    int32_t *prevS;          /* S(t-1), ascending */
    int32_t n_prevS, have_prev;
    unsigned char *resident; /* simulated GPU block cache */
    int64_t viol_gamma, viol_reselect, viol_incremental, viol_fetch, steps;
} nosa_oracle_unit;

typedef struct {
    int32_t nb_c;       /* candidate (complete, non-local) blocks */
    int32_t local;      /* local block id */
    int32_t n_fetch;    /* simulated cache misses this step */
    int32_t n_sel;      /* |Sel| (without local) */
    int32_t n_overlap;  /* |Sel(t) ∩ S(t-1)| */
    double gamma;       /* n_overlap / n_sel, or -1 if undefined */
} nosa_oracle_stats;

static double bf16_to_double(uint16_t b) {
    union { uint32_t u; float f; } c;
    c.u = (uint32_t)b << 16;
    return (double)c.f;
}

nosa_oracle_unit *nosa_oracle_unit_new(int32_t D, int32_t G, int32_t block, int32_t sub,
                                       int32_t k_q, int32_t k_e, double scale, int64_t cap) {
    if (D <= 0 || G <= 0 || block <= 0 || sub <= 0 || block % sub || cap <= 0 || cap % block)
        return NULL;
    nosa_oracle_unit *u = (nosa_oracle_unit *)calloc(1, sizeof(*u));
    if (!u) return NULL;
    u->D = D; u->G = G; u->block = block; u->sub = sub; u->k_q = k_q; u->k_e = k_e;
    u->scale = scale; u->cap = cap;
    int64_t nb = cap / block;
    u->K = (uint16_t *)calloc((size_t)(cap * D), sizeof(uint16_t));
    u->V = (uint16_t *)calloc((size_t)(cap * D), sizeof(uint16_t));
    u->e = (float *)calloc((size_t)cap, sizeof(float));
    u->ck = (double *)calloc((size_t)(cap / sub * D), sizeof(double));
    u->E = (double *)calloc((size_t)nb, sizeof(double));
    u->dropped = (unsigned char *)calloc((size_t)nb, 1);
    u->ge_inc = (unsigned char *)calloc((size_t)nb, 1);
    u->resident = (unsigned char *)calloc((size_t)nb, 1);
    u->prevS = (int32_t *)calloc((size_t)nb, sizeof(int32_t));
    if (!u->K || !u->V || !u->e || !u->ck || !u->E || !u->dropped || !u->ge_inc || !u->resident ||
        !u->prevS) {
        free(u->K); free(u->V); free(u->e); free(u->ck); free(u->E); free(u->dropped);
        free(u->ge_inc); free(u->resident); free(u->prevS); free(u);
        return NULL;
    }
    return u;
}

void nosa_oracle_unit_free(nosa_oracle_unit *u) {
    if (!u) return;
    free(u->K); free(u->V); free(u->e); free(u->ck); free(u->E); free(u->dropped);
    free(u->ge_inc); free(u->resident); free(u->prevS); free(u);
}

/*
 * x rounded to the nearest bf16 value (8 significant bits, fp32 exponent
 * range), ties to even: the mantissa scaled to [128, 256) is rounded with
 * rint (the default rounding mode is to nearest, ties to even).
 */
double nosa_oracle_round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    if (fabs(x) < ldexp(1.0, -126)) return ldexp(rint(ldexp(x, 133)), -133); /* subnormal spacing 2^-133 */
    int e;
    double m = frexp(x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
    return ldexp(rint(ldexp(m, 8)), e - 8);
}

/* Compressed key of sub-block s: the fp64 mean of its keys (rounded to bf16 in that mode). */
static void compress_sub_block(nosa_oracle_unit *u, int64_t s) {
    for (int32_t d = 0; d < u->D; ++d) {
        double acc = 0.0;
        for (int32_t j = 0; j < u->sub; ++j)
            acc += bf16_to_double(u->K[(s * u->sub + j) * u->D + d]);
        double mean = acc / u->sub;
        u->ck[s * u->D + d] = u->ck_bf16 ? nosa_oracle_round_bf16(mean) : mean;
    }
}

/* Store pooled keys as bf16 from now on (set before the first append). */
void nosa_oracle_set_ck_bf16(nosa_oracle_unit *u, int32_t on) { u->ck_bf16 = on != 0; }

void nosa_oracle_set_fill(nosa_oracle_unit *u, int32_t on) { u->fill = on != 0; }

/*
 * Eviction head (montaan.com summary of 2510.13602, "Key Design Components"
 * item 3, Equation 4; the nonlinearity is softplus, as in DMA's design):
 *   e_j = sum_h W2[h] * softplus( sum_d v_j[d] * W1[d][h] ),
 * for the value rows V [T][D] (bf16 bits) of one kv head, W1 [D][H], W2 [H]
 * (fp32 values).  fp64 throughout, sums in index order, each product and sum
 * rounded on its own; the result is rounded once to fp32 (the logits' storage
 * type).  softplus(x) = max(x, 0) + log1p(exp(-|x|)), which neither overflows
 * nor loses the small values.  Reading where the pages are silent: one head per
 * layer and kv head, with hidden size H.
 */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

void nosa_oracle_evict_head(const uint16_t *V, int64_t T, int32_t D, int32_t H, const float *W1,
                            const float *W2, float *e_out) {
    for (int64_t j = 0; j < T; ++j) {
        double e = 0.0;
        for (int32_t h = 0; h < H; ++h) {
            double z = 0.0;
            for (int32_t d = 0; d < D; ++d) z += bf16_to_double(V[j * D + d]) * (double)W1[(int64_t)d * H + h];
            e += (double)W2[h] * softplus(z);
        }
        e_out[j] = (float)e;
    }
}

/* Block eviction score: max over the block's sub-blocks of the mean eviction logit. */
static void evict_score_block(nosa_oracle_unit *u, int64_t b) {
    int32_t per = u->block / u->sub;
    double best = -INFINITY;
    for (int32_t s = 0; s < per; ++s) {
        double acc = 0.0;
        int64_t t0 = b * u->block + (int64_t)s * u->sub;
        for (int32_t j = 0; j < u->sub; ++j) acc += (double)u->e[t0 + j];
        double m = acc / u->sub;
        if (m > best) best = m;
    }
    u->E[b] = best;
}

/* Append T tokens (K, V rows [T][D] bf16 bits, e [T]); pool what completes. */
static int append_tokens(nosa_oracle_unit *u, const uint16_t *K, const uint16_t *V,
                         const float *e, int64_t T) {
    if (T < 0 || u->L + T > u->cap) return -2;
    memcpy(u->K + u->L * u->D, K, (size_t)(T * u->D) * sizeof(uint16_t));
    memcpy(u->V + u->L * u->D, V, (size_t)(T * u->D) * sizeof(uint16_t));
    memcpy(u->e + u->L, e, (size_t)T * sizeof(float));
    int64_t L0 = u->L, L1 = u->L + T;
    for (int64_t s = L0 / u->sub; s < L1 / u->sub; ++s) compress_sub_block(u, s);
    for (int64_t b = L0 / u->block; b < L1 / u->block; ++b) evict_score_block(u, b);
    u->L = L1;
    return 0;
}

typedef struct { double score; int32_t idx; } scored_t;

/* descending score, ties to the lower block index */
static int cmp_scored(const void *a, const void *b) {
    const scored_t *x = (const scored_t *)a, *y = (const scored_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int cmp_int(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Top-k of n scored entries by full sort; writes ids in rank order; returns count. */
static int32_t top_k(const double *score, int32_t n, int32_t k, int32_t *out) {
    if (k <= 0 || n <= 0) return 0;
    scored_t *tmp = (scored_t *)malloc((size_t)n * sizeof(scored_t));
    for (int32_t i = 0; i < n; ++i) { tmp[i].score = score[i]; tmp[i].idx = i; }
    qsort(tmp, (size_t)n, sizeof(scored_t), cmp_scored);
    int32_t m = k < n ? k : n;
    for (int32_t i = 0; i < m; ++i) out[i] = tmp[i].idx;
    free(tmp);
    return m;
}

/* number of candidate blocks at length L: the complete blocks before the local one */
static int32_t n_candidates(const nosa_oracle_unit *u) {
    return u->L <= 0 ? 0 : (int32_t)((u->L - 1) / u->block);
}

/* Prefill: append T tokens, then Gamma_e := plain top-k_e of the candidates. */
int nosa_oracle_prefill(nosa_oracle_unit *u, const uint16_t *K, const uint16_t *V,
                        const float *e, int64_t T) {
    int rc = append_tokens(u, K, V, e, T);
    if (rc) return rc;
    int32_t nb_c = n_candidates(u);
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(nb_c + 1));
    int32_t n = top_k(u->E, nb_c, u->k_e, ids);
    memset(u->ge_inc, 0, (size_t)(u->cap / u->block));
    for (int32_t i = 0; i < n; ++i) u->ge_inc[ids[i]] = 1;
    u->n_ge_inc = n;
    /* the block cache starts holding Gamma_e and the local block: the prefill has
       every block at hand, so these cost no transfer */
    memset(u->resident, 0, (size_t)(u->cap / u->block));
    for (int32_t i = 0; i < n; ++i) u->resident[ids[i]] = 1;
    if (u->L > 0) u->resident[(u->L - 1) / u->block] = 1;
    free(ids);
    u->have_prev = 0;
    return 0;
}

/*
 * Incremental Gamma_e maintenance when block b becomes a candidate: it
 * enters if there is room, or if it beats the worst member (lowest score,
 * ties: the higher index is worse), which then leaves.  Checked every step
 * against the brute-force top-k_e.
 */
static void gamma_e_insert(nosa_oracle_unit *u, int32_t b) {
    if (u->k_e <= 0) return;
    if (u->n_ge_inc < u->k_e) { u->ge_inc[b] = 1; u->n_ge_inc++; return; }
    int32_t worst = -1;
    for (int32_t i = 0; i < b; ++i) {
        if (!u->ge_inc[i]) continue;
        if (worst < 0 || u->E[i] < u->E[worst] || (u->E[i] == u->E[worst] && i > worst)) worst = i;
    }
    if (worst >= 0 && (u->E[b] > u->E[worst] || (u->E[b] == u->E[worst] && b < worst))) {
        u->ge_inc[worst] = 0;
        u->ge_inc[b] = 1;
    }
}

/* Softmax attention of the G query heads over the token list tok[0..n). */
static void attend(const nosa_oracle_unit *u, const uint16_t *q, const int64_t *tok, int64_t n,
                   double *o) {
    double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int32_t h = 0; h < u->G; ++h) {
        double m = -INFINITY;
        for (int64_t i = 0; i < n; ++i) {
            int64_t j = tok[i];
            double dot = 0.0;
            for (int32_t d = 0; d < u->D; ++d)
                dot += bf16_to_double(q[h * u->D + d]) * bf16_to_double(u->K[j * u->D + d]);
            z[i] = dot * u->scale + (double)u->e[j];
            if (z[i] > m) m = z[i];
        }
        double l = 0.0;
        for (int32_t d = 0; d < u->D; ++d) o[h * u->D + d] = 0.0;
        for (int64_t i = 0; i < n; ++i) {
            double p = exp(z[i] - m);
            l += p;
            for (int32_t d = 0; d < u->D; ++d)
                o[h * u->D + d] += p * bf16_to_double(u->V[tok[i] * u->D + d]);
        }
        for (int32_t d = 0; d < u->D; ++d) o[h * u->D + d] = n > 0 ? o[h * u->D + d] / l : 0.0;
    }
    free(z);
}

/*
 * Block scores of the candidates for query heads q[G][D] (bf16 bits):
 * s_b = max over sub-blocks s of b of  sum_h (q_h . kbar_s) * scale.
 */
static void block_scores(const nosa_oracle_unit *u, const uint16_t *q, int32_t nb_c,
                         double *s_out) {
    int32_t per = u->block / u->sub;
    for (int32_t b = 0; b < nb_c; ++b) {
        double best = -INFINITY;
        for (int32_t s = 0; s < per; ++s) {
            const double *kb = u->ck + ((int64_t)b * per + s) * u->D;
            double acc = 0.0;
            for (int32_t h = 0; h < u->G; ++h) {
                double dot = 0.0;
                for (int32_t d = 0; d < u->D; ++d) dot += bf16_to_double(q[h * u->D + d]) * kb[d];
                acc += dot;
            }
            double v = acc * u->scale;
            if (v > best) best = v;
        }
        s_out[b] = best;
    }
}

/*
 * One decode step: append the token (k, v: [D] bf16 bits; e), select, simulate
 * the block cache, attend.  Outputs (all caller-allocated):
 *   sel[k_q+k_e+1], *nsel : S(t) = (Gamma_q ∪ Gamma_e) ∪ {local}, ascending
 *   gq[k_q], *ngq         : Gamma_q in rank order
 *   ge[k_e], *nge         : Gamma_e ascending
 *   scores[nb_c] (nullable): query block scores;  o[G][D]: attention output
 */
int nosa_oracle_step(nosa_oracle_unit *u, const uint16_t *k, const uint16_t *v, float e,
                     const uint16_t *q, int32_t *sel, int32_t *nsel, int32_t *gq, int32_t *ngq,
                     int32_t *ge, int32_t *nge, double *scores, double *o,
                     nosa_oracle_stats *st) {
    int rc = append_tokens(u, k, v, &e, 1);
    if (rc) return rc;
    int32_t nb_c = n_candidates(u);
    int32_t local = (int32_t)((u->L - 1) / u->block);
    int new_local = ((u->L - 1) % u->block) == 0;
    if (new_local && local >= 1 && !u->fill) gamma_e_insert(u, local - 1);

    double *s = (double *)malloc(sizeof(double) * (size_t)(nb_c + 1));
    block_scores(u, q, nb_c, s);
    if (scores) memcpy(scores, s, sizeof(double) * (size_t)nb_c);

    int32_t n_q = top_k(s, nb_c, u->k_q, gq);
    int32_t *ge_rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)(u->k_e + 1));
    int32_t n_e;
    if (!u->fill) {
        n_e = top_k(u->E, nb_c, u->k_e, ge_rank);
    } else {
        /* fill: top-k_e by E over the candidates outside Gamma_q not yet dropped */
        double *Ef = (double *)malloc(sizeof(double) * (size_t)(nb_c + 1));
        unsigned char *in_q = (unsigned char *)calloc((size_t)(nb_c + 1), 1);
        for (int32_t i = 0; i < n_q; ++i) in_q[gq[i]] = 1;
        int32_t n_elig = 0;
        for (int32_t b = 0; b < nb_c; ++b) {
            int elig = !in_q[b] && !u->dropped[b];
            Ef[b] = elig ? u->E[b] : -INFINITY;
            n_elig += elig;
        }
        n_e = top_k(Ef, nb_c, u->k_e < n_elig ? u->k_e : n_elig, ge_rank);
        free(Ef); free(in_q);
    }
    memcpy(ge, ge_rank, sizeof(int32_t) * (size_t)n_e);
    qsort(ge, (size_t)n_e, sizeof(int32_t), cmp_int);

    /* invariant (iii), union reading: incremental Gamma_e equals the brute-force one */
    if (!u->fill) {
        int32_t cnt = 0, mismatch = 0;
        for (int32_t b = 0; b < nb_c; ++b) cnt += u->ge_inc[b];
        if (cnt != n_e) mismatch = 1;
        for (int32_t i = 0; i < n_e; ++i)
            if (!u->ge_inc[ge[i]]) mismatch = 1;
        if (mismatch) u->viol_incremental++;
    }
    /* invariant (ii): no dropped block re-enters Gamma_e; then mark the new drops
       (union: every candidate outside Gamma_e; fill: every candidate outside Sel) */
    {
        unsigned char *keep = (unsigned char *)calloc((size_t)(nb_c + 1), 1);
        for (int32_t i = 0; i < n_e; ++i) {
            if (u->dropped[ge[i]]) u->viol_reselect++;
            keep[ge[i]] = 1;
        }
        if (u->fill)
            for (int32_t i = 0; i < n_q; ++i) keep[gq[i]] = 1;
        for (int32_t b = 0; b < nb_c; ++b)
            if (!keep[b]) u->dropped[b] = 1;
        free(keep);
    }

    /* Sel = Gamma_q ∪ Gamma_e, ascending; S = Sel ∪ {local} */
    unsigned char *mark = (unsigned char *)calloc((size_t)(local + 1), 1);
    for (int32_t i = 0; i < n_q; ++i) mark[gq[i]] = 1;
    for (int32_t i = 0; i < n_e; ++i) mark[ge[i]] = 1;
    int32_t n_sel = 0;
    for (int32_t b = 0; b < nb_c; ++b)
        if (mark[b]) sel[n_sel++] = b;
    sel[n_sel] = local;
    int32_t n_S = n_sel + 1;

    /* invariant (i): gamma(t) = |Sel(t) ∩ S(t-1)| / |Sel(t)| >= k_e / k */
    int32_t overlap = 0;
    if (u->have_prev) {
        for (int32_t i = 0, j = 0; i < n_sel && j < u->n_prevS;) {
            if (sel[i] == u->prevS[j]) { overlap++; i++; j++; }
            else if (sel[i] < u->prevS[j]) i++;
            else j++;
        }
        int32_t kk = u->k_q + u->k_e;
        if (nb_c >= u->k_e && n_sel > 0 && (int64_t)overlap * kk < (int64_t)u->k_e * n_sel)
            u->viol_gamma++;
    }

    /* simulated block cache: the new local block is written, not fetched */
    if (new_local) u->resident[local] = 1;
    int32_t n_fetch = 0;
    for (int32_t i = 0; i < n_S; ++i)
        if (!u->resident[sel[i]]) n_fetch++;
    /* invariant (iv): misses only come from Gamma_q \ S(t-1) */
    if (u->have_prev) {
        int32_t fresh_q = 0;
        for (int32_t i = 0; i < n_q; ++i) {
            int found = 0;
            for (int32_t j = 0; j < u->n_prevS; ++j)
                if (u->prevS[j] == gq[i]) { found = 1; break; }
            if (!found) fresh_q++;
        }
        if (n_fetch > fresh_q) u->viol_fetch++;
    }
    memset(u->resident, 0, (size_t)(u->cap / u->block));
    for (int32_t i = 0; i < n_S; ++i) u->resident[sel[i]] = 1;

    /* exact attention over the tokens of S(t) that exist (positions < L) */
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)n_S * (size_t)u->block);
    int64_t n_tok = 0;
    for (int32_t i = 0; i < n_S; ++i)
        for (int32_t j = 0; j < u->block; ++j) {
            int64_t p = (int64_t)sel[i] * u->block + j;
            if (p < u->L) tok[n_tok++] = p;
        }
    attend(u, q, tok, n_tok, o);

    memcpy(u->prevS, sel, sizeof(int32_t) * (size_t)n_S);
    u->n_prevS = n_S;
    u->have_prev = 1;
    u->steps++;

    *nsel = n_S; *ngq = n_q; *nge = n_e;
    if (st) {
        st->nb_c = nb_c; st->local = local; st->n_fetch = n_fetch; st->n_sel = n_sel;
        st->n_overlap = overlap;
        st->gamma = (u->steps > 1 && n_sel > 0) ? (double)overlap / n_sel : -1.0;
    }
    free(tok); free(mark); free(ge_rank); free(s);
    return 0;
}

/* Dense comparator: softmax attention (with the same bias) over all L tokens. */
int nosa_oracle_dense(const nosa_oracle_unit *u, const uint16_t *q, double *o) {
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(u->L > 0 ? u->L : 1));
    for (int64_t i = 0; i < u->L; ++i) tok[i] = i;
    attend(u, q, tok, u->L, o);
    free(tok);
    return 0;
}

/* Accessors for tests. */
int64_t nosa_oracle_len(const nosa_oracle_unit *u) { return u->L; }
const double *nosa_oracle_ck(const nosa_oracle_unit *u) { return u->ck; }
const double *nosa_oracle_E(const nosa_oracle_unit *u) { return u->E; }
void nosa_oracle_violations(const nosa_oracle_unit *u, int64_t out[5]) {
    out[0] = u->viol_gamma; out[1] = u->viol_reselect; out[2] = u->viol_incremental;
    out[3] = u->viol_fetch; out[4] = u->steps;
}

/*
 * Attention of the G heads over the tokens (< L) of an arbitrary ascending
 * block list: used to evaluate the output on another selection (e.g. one that
 * differs from this unit's by an excused near-tie).
 */
int nosa_oracle_attend_blocks(const nosa_oracle_unit *u, const uint16_t *q, const int32_t *blocks,
                              int32_t n, double *o) {
    int64_t *tok = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1) * (size_t)u->block);
    int64_t n_tok = 0;
    for (int32_t i = 0; i < n; ++i)
        for (int32_t j = 0; j < u->block; ++j) {
            int64_t p = (int64_t)blocks[i] * u->block + j;
            if (blocks[i] >= 0 && p < u->L) tok[n_tok++] = p;
        }
    attend(u, q, tok, n_tok, o);
    free(tok);
    return 0;
}

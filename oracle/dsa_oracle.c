/*
 * dsa_oracle.c -- plain, slow, single-threaded CPU oracle for the DeepSeek
 * Sparse Attention (DSA) prefill path: lightning-indexer scores, exact top-k
 * selection, and absorbed-MLA softmax attention over the selected keys.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA path: it decodes its own inputs from the raw bf16 / fp8-e4m3 bytes and
 * computes every quantity in IEEE fp64 with a fixed, documented loop order.
 *
 * Sources (each function names the passage it follows):
 *   [MLX]  mlx-lm PR #1997, "GLM prefill now attends only to the keys its
 *          indexer picks", section "How it works" (32-head indexer over all
 *          keys, top-k per query, one gathered 576-wide block per query shared
 *          by all heads, absorbed latent-space attention, 4,096-key blocked
 *          top-k fold that selects the same keys as a full sort).
 *   [LITE] "LiteTopK / LiteDSA" (arXiv 2607.11976), Abstract (Indexer-TopK:
 *          score, then select the exact top-k).
 *   [LCPP] llama.cpp PR #25917, "cuda : support for sparse KV indices in MMA
 *          flash attention kernel", discussion (an int32 index mask, -1 for a
 *          masked entry; causality applied to the indices).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - the lightning-indexer score is I[t,s] = sum_h w[t,h] * max(0, q[t,h,:].k[s,:]),
 *     ReLU per head before the signed head weight, one indexer key per position
 *     shared by all indexer heads;
 *   - causality is inclusive: query t sits at position p_t = q_pos0 + t and sees
 *     keys s <= p_t; with general causality (an index mask) query t sees the
 *     keys of its own half-open range [lo_t, hi_t);
 *   - ties in I are broken toward the smaller key index;
 *   - the selected set is emitted in ascending key order, then -1 padding when
 *     fewer than topk keys are visible;
 *   - fp8 inputs are OCP E4M3FN with unit scale.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* Data-type codes of the indexer operands (the same numeric meaning as the
 * library's public enum, restated here on purpose so the two share nothing). */
#define ORACLE_IDX_BF16 0
#define ORACLE_IDX_E4M3 1

#define MLA_LAT 512
#define MLA_ROPE 64
#define MLA_DIM (MLA_LAT + MLA_ROPE)

int oracle_version(void) { return 1; }

/* bfloat16: the upper 16 bits of an IEEE binary32; every value is exact in fp64. */
double oracle_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3FN: 1 sign bit, 4 exponent bits (bias 7),
 * 3 mantissa bits, no infinities, S.1111.111 is NaN; exponent field 0 encodes
 * subnormals m/8 * 2^-6. */
double oracle_e4m3_value(uint8_t bits) {
    int sign = bits >> 7;
    int e = (bits >> 3) & 0xF;
    int m = bits & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

static double idx_value(const void *base, int dtype, int64_t i) {
    if (dtype == ORACLE_IDX_BF16) return oracle_bf16_value(((const uint16_t *)base)[i]);
    return oracle_e4m3_value(((const uint8_t *)base)[i]);
}

/*
 * Lightning-indexer scores of one query row t over every visible key
 * s = 0 .. p_t (p_t = q_pos0 + t), [MLX] "How it works" (the indexer scores
 * each query against every cached key with 32 heads) and [LITE] Abstract.
 *
 *   I[t,s] = sum_{h < H_I} w[t,h] * max(0, sum_{d < D_I} q_idx[t,h,d] * k_idx[s,d])
 *
 * Loop order: h ascending, and inside it d ascending, in fp64.
 * q_idx: [L, H_I, D_I] raw bits; k_idx: [N, D_I] raw bits; w: [L, H_I] fp32.
 * out receives p_t + 1 doubles.
 */
int oracle_indexer_scores(const void *q_idx, const void *k_idx, const float *w, int dtype,
                          int L, int N, int H_I, int D_I, int q_pos0, int t, double *out) {
    if (t < 0 || t >= L || q_pos0 < 0 || q_pos0 + L > N || H_I <= 0 || D_I <= 0) return ORACLE_EINVAL;
    if (dtype != ORACLE_IDX_BF16 && dtype != ORACLE_IDX_E4M3) return ORACLE_EINVAL;
    int p_t = q_pos0 + t;
    double *q = (double *)malloc(sizeof(double) * (size_t)H_I * D_I);
    double *k = (double *)malloc(sizeof(double) * (size_t)D_I);
    if (!q || !k) { free(q); free(k); return ORACLE_ENOMEM; }
    for (int h = 0; h < H_I; ++h)
        for (int d = 0; d < D_I; ++d)
            q[h * D_I + d] = idx_value(q_idx, dtype, ((int64_t)t * H_I + h) * D_I + d);
    for (int s = 0; s <= p_t; ++s) {
        for (int d = 0; d < D_I; ++d) k[d] = idx_value(k_idx, dtype, (int64_t)s * D_I + d);
        double score = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double dot = 0.0;
            for (int d = 0; d < D_I; ++d) dot += q[h * D_I + d] * k[d];
            double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w[(int64_t)t * H_I + h] * relu;
        }
        out[s] = score;
    }
    free(q);
    free(k);
    return ORACLE_OK;
}

/*
 * Lightning-indexer scores of query row t over the keys of a half-open range
 * [lo, hi): general causality carried by the index mask, [LCPP] discussion
 * (causality applied to the indices rather than assumed triangular, so that
 * a unified cache holding several sequences, or a non-triangular mask, is
 * expressed per query).  The same formula and loop order as
 * oracle_indexer_scores; out receives hi - lo doubles, out[j] for key lo + j.
 * Requires 0 <= lo <= hi <= N; positions play no further role.
 */
int oracle_indexer_scores_range(const void *q_idx, const void *k_idx, const float *w, int dtype,
                                int L, int N, int H_I, int D_I, int lo, int hi, int t, double *out) {
    if (t < 0 || t >= L || lo < 0 || hi < lo || hi > N || H_I <= 0 || D_I <= 0) return ORACLE_EINVAL;
    if (dtype != ORACLE_IDX_BF16 && dtype != ORACLE_IDX_E4M3) return ORACLE_EINVAL;
    double *q = (double *)malloc(sizeof(double) * (size_t)H_I * D_I);
    double *k = (double *)malloc(sizeof(double) * (size_t)D_I);
    if (!q || !k) { free(q); free(k); return ORACLE_ENOMEM; }
    for (int h = 0; h < H_I; ++h)
        for (int d = 0; d < D_I; ++d)
            q[h * D_I + d] = idx_value(q_idx, dtype, ((int64_t)t * H_I + h) * D_I + d);
    for (int s = lo; s < hi; ++s) {
        for (int d = 0; d < D_I; ++d) k[d] = idx_value(k_idx, dtype, (int64_t)s * D_I + d);
        double score = 0.0;
        for (int h = 0; h < H_I; ++h) {
            double dot = 0.0;
            for (int d = 0; d < D_I; ++d) dot += q[h * D_I + d] * k[d];
            double relu = dot > 0.0 ? dot : 0.0;
            score += (double)w[(int64_t)t * H_I + h] * relu;
        }
        out[s - lo] = score;
    }
    free(q);
    free(k);
    return ORACLE_OK;
}

typedef struct {
    double v;
    int32_t i;
} scored_key;

/* Total order of the selection: larger score first, equal scores by smaller index. */
static int by_score_desc_index_asc(const void *pa, const void *pb) {
    const scored_key *a = (const scored_key *)pa, *b = (const scored_key *)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->i > b->i) - (a->i < b->i);
}

static int int32_asc(const void *pa, const void *pb) {
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * Exact top-k by a full sort, [MLX] "How it works" (the stock indexer sorts
 * the whole score row) and [LITE] Abstract (exact Top-k).  Sorting the
 * index-ordered row by score with ties kept in index order is the same as
 * sorting by (score desc, index asc), which is what the comparator does.
 * idx_out[topk]: selected keys ascending, then -1 padding ([LCPP] discussion).
 * kth_out (may be NULL): the k-th best score, or -inf when nvis <= topk.
 */
int oracle_topk_fullsort(const double *scores, int nvis, int topk, int32_t *idx_out, double *kth_out) {
    if (nvis < 0 || topk <= 0) return ORACLE_EINVAL;
    if (nvis <= topk) {
        for (int j = 0; j < topk; ++j) idx_out[j] = j < nvis ? j : -1;
        if (kth_out) *kth_out = -INFINITY;
        return ORACLE_OK;
    }
    scored_key *all = (scored_key *)malloc(sizeof(scored_key) * (size_t)nvis);
    if (!all) return ORACLE_ENOMEM;
    for (int s = 0; s < nvis; ++s) { all[s].v = scores[s]; all[s].i = s; }
    qsort(all, (size_t)nvis, sizeof(scored_key), by_score_desc_index_asc);
    for (int j = 0; j < topk; ++j) idx_out[j] = all[j].i;
    if (kth_out) *kth_out = all[topk - 1].v;
    qsort(idx_out, (size_t)topk, sizeof(int32_t), int32_asc);
    free(all);
    return ORACLE_OK;
}

/*
 * Exact top-k by the blocked fold of [MLX] "How it works": score the keys in
 * blocks, fold each block into a running list of the best topk, so that each
 * selection step only looks at topk + block rows.  Must select the same set
 * as oracle_topk_fullsort: by the page, folding block by block can only
 * differ from selecting over the whole row where equal scores compete for
 * the last places, and the index tie-break removes that freedom.
 */
int oracle_topk_blocked_fold(const double *scores, int nvis, int topk, int block, int32_t *idx_out) {
    if (nvis < 0 || topk <= 0 || block <= 0) return ORACLE_EINVAL;
    scored_key *run = (scored_key *)malloc(sizeof(scored_key) * ((size_t)topk + (size_t)block));
    if (!run) return ORACLE_ENOMEM;
    int n = 0;
    for (int b0 = 0; b0 < nvis; b0 += block) {
        int b1 = b0 + block < nvis ? b0 + block : nvis;
        for (int s = b0; s < b1; ++s) { run[n].v = scores[s]; run[n].i = s; ++n; }
        qsort(run, (size_t)n, sizeof(scored_key), by_score_desc_index_asc);
        if (n > topk) n = topk;
    }
    for (int j = 0; j < topk; ++j) idx_out[j] = j < n ? run[j].i : -1;
    qsort(idx_out, (size_t)n, sizeof(int32_t), int32_asc);
    free(run);
    return ORACLE_OK;
}

/* Softmax attention of one query head over an explicit list of keys, in the
 * order given.  Shared by the sparse and dense entry points below. */
static void attend_keys(const uint16_t *qrow, const uint16_t *kv, const int32_t *keys, int nkeys,
                        double scale, double *z, double *out, double *lse) {
    double m = -INFINITY;
    for (int j = 0; j < nkeys; ++j) {
        const uint16_t *kr = kv + (int64_t)keys[j] * MLA_DIM;
        double lat = 0.0, rope = 0.0;
        for (int d = 0; d < MLA_LAT; ++d) lat += oracle_bf16_value(qrow[d]) * oracle_bf16_value(kr[d]);
        for (int d = 0; d < MLA_ROPE; ++d)
            rope += oracle_bf16_value(qrow[MLA_LAT + d]) * oracle_bf16_value(kr[MLA_LAT + d]);
        z[j] = scale * (lat + rope);
        if (z[j] > m) m = z[j];
    }
    for (int d = 0; d < MLA_LAT; ++d) out[d] = 0.0;
    if (nkeys == 0) {
        if (lse) *lse = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (int j = 0; j < nkeys; ++j) { z[j] = exp(z[j] - m); Z += z[j]; }
    for (int j = 0; j < nkeys; ++j) {
        const uint16_t *kr = kv + (int64_t)keys[j] * MLA_DIM;
        double p = z[j] / Z;
        for (int d = 0; d < MLA_LAT; ++d) out[d] += p * oracle_bf16_value(kr[d]);
    }
    if (lse) *lse = m + log(Z);
}

/*
 * Absorbed-MLA attention of query row t over its selected keys, [MLX] "How it
 * works": every key is the 576-wide joined row (512 latent + 64 rope) of the
 * cache, the gathered block is shared by all H heads, and the value is the
 * 512-wide latent part of the same row.
 *
 *   z_j = scale * (q_lat[t,h].kv_lat[i_j] + q_rope[t,h].k_rope[i_j])
 *   out[t,h] = sum_j softmax(z)_j * kv_lat[i_j],  lse[t,h] = log sum_j exp(z_j)
 *
 * q: [L, H, 576] bf16 bits; kv: [N, 576] bf16 bits; idx: [topk] for this row,
 * -1 entries are skipped ([LCPP] discussion).  out: [H, 512]; lse: [H] or NULL.
 */
int oracle_sparse_mla(const uint16_t *q, const uint16_t *kv, const int32_t *idx, int L, int N, int H,
                      int topk, double scale, int t, double *out, double *lse) {
    if (t < 0 || t >= L || H <= 0 || topk <= 0) return ORACLE_EINVAL;
    int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)topk);
    double *z = (double *)malloc(sizeof(double) * (size_t)topk);
    if (!keys || !z) { free(keys); free(z); return ORACLE_ENOMEM; }
    int n = 0;
    for (int j = 0; j < topk; ++j) {
        if (idx[j] < 0) continue;
        if (idx[j] >= N) { free(keys); free(z); return ORACLE_EINVAL; }
        keys[n++] = idx[j];
    }
    for (int h = 0; h < H; ++h)
        attend_keys(q + ((int64_t)t * H + h) * MLA_DIM, kv, keys, n, scale, z, out + (int64_t)h * MLA_LAT,
                    lse ? lse + h : NULL);
    free(keys);
    free(z);
    return ORACLE_OK;
}

/*
 * Dense causal attention of query row t over every visible key 0 .. p_t, the
 * masked dense prefill that [MLX] "The change" describes as the baseline.  It
 * is the brute-force check for the sparse path: when the selection holds every
 * visible key in ascending order the two are the same arithmetic.
 */
int oracle_dense_causal_mla(const uint16_t *q, const uint16_t *kv, int L, int N, int H, int q_pos0,
                            double scale, int t, double *out, double *lse) {
    if (t < 0 || t >= L || q_pos0 < 0 || q_pos0 + L > N || H <= 0) return ORACLE_EINVAL;
    int nvis = q_pos0 + t + 1;
    int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)nvis);
    double *z = (double *)malloc(sizeof(double) * (size_t)nvis);
    if (!keys || !z) { free(keys); free(z); return ORACLE_ENOMEM; }
    for (int s = 0; s < nvis; ++s) keys[s] = s;
    for (int h = 0; h < H; ++h)
        attend_keys(q + ((int64_t)t * H + h) * MLA_DIM, kv, keys, nvis, scale, z, out + (int64_t)h * MLA_LAT,
                    lse ? lse + h : NULL);
    free(keys);
    free(z);
    return ORACLE_OK;
}

/*
 * One whole row of the path: scores, full-sort top-k, attention over the
 * selection.  Used by the CPU baseline timing so that one call is one query
 * token of work.  scores_scratch holds at least p_t + 1 doubles.
 */
int oracle_prefill_row(const void *q_idx, const void *k_idx, const float *w, int dtype, int L, int N,
                       int H_I, int D_I, int q_pos0, int topk, const uint16_t *q, const uint16_t *kv, int H,
                       double scale, int t, double *scores_scratch, int32_t *idx_out, double *out, double *lse) {
    int rc = oracle_indexer_scores(q_idx, k_idx, w, dtype, L, N, H_I, D_I, q_pos0, t, scores_scratch);
    if (rc) return rc;
    rc = oracle_topk_fullsort(scores_scratch, q_pos0 + t + 1, topk, idx_out, NULL);
    if (rc) return rc;
    return oracle_sparse_mla(q, kv, idx_out, L, N, H, topk, scale, t, out, lse);
}

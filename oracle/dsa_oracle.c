/*
 * dsa_oracle.c -- CPU oracle for the DSA (DeepSeek-style Sparse Attention) hot path
 * with IndexShare, as described for GLM-5.2.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct reference that
 * the CUDA library is checked against.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  It shares no code, header, table or helper
 * with the CUDA path, and it never calls into it.
 *
 * Plain C11, single threaded, double precision for every floating-point result.
 * Sources (page title, section):
 *   [p1] "GLM-5.2 MTP IndexShare inference" (4sapi.ai blog): "Indexer Share",
 *        "Indexer Share in the MTP layer", "KV Share".
 *   [p2] "GLM-5.2 1M architecture teardown" (clawlihai.cn): "Cut 1: DSA" (index_topk
 *        2048, index_head_dim 128, index_n_heads 32), "Cut 2: IndexShare"
 *        (index_topk_freq 4), "Cut 3: MLA" (kv_lora_rank 512).
 *   [p3] "GLM-5.2 speculative decoding" (yun88.com news 9578): "GLM-5.2's MTP improvement".
 *   [p5] "Le contexte d'un million de tokens" (glmmodel.cn): "Attention sparse IndexShare",
 *        "MTP avec IndexShare et KVShare".
 * The pages name the lightweight indexer and its sizes but print no formula; the
 * score used here is the standard DSA lightweight-indexer form
 *     I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]),
 * and the attention is the absorbed-MLA form over a 576-wide compressed row whose
 * first 512 entries are the value (512 latent + 64 rope).  Both readings are listed
 * with the other readings of the pages in the design notes.
 *
 * Data types at the boundary: bf16 tensors arrive as raw uint16 bit patterns, weights
 * as float32, scores for the selection step as float32 (the selection is an integer
 * decision and is taken in the precision the GPU kernel produces, fp32).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG -1
#define OR_ERR_NOMEM -2
#define OR_ERR_INVARIANT -3

/* bf16 -> double: a bf16 value is the upper half of an IEEE binary32 pattern. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Number of cached tokens query t may look at: positions s <= q_pos0 + t, s < N
 * (causal mask).  For decode the query is the newest cached token, q_pos0 = N-1. */
static long visible_count(long N, long q_pos0, long t)
{
    long v = q_pos0 + t + 1;
    if (v < 0) v = 0;
    if (v > N) v = N;
    return v;
}

/* ------------------------------------------------------------------------------- */
/* Step 1: lightweight indexer score  ([p2] Cut 1; [p5] Attention sparse IndexShare)   */
/* ------------------------------------------------------------------------------- */
/*
 * q      [B, T, n_heads, head_dim]  bf16 bits   (indexer queries)
 * w      [B, T, n_heads]            float32     (per-query head weights)
 * k      [B, N, head_dim]           bf16 bits   (one shared index key per cached token)
 * scores [B, T, N]                  double      out; -inf where s is not visible to t
 */
int oracle_index_score(const uint16_t *q, const float *w, const uint16_t *k,
                       int B, int T, int N, int n_heads, int head_dim, long q_pos0,
                       double *scores)
{
    if (!q || !w || !k || !scores || B < 0 || T < 0 || N < 0 || n_heads <= 0 || head_dim <= 0)
        return OR_ERR_ARG;
    for (long b = 0; b < B; ++b) {
        for (long t = 0; t < T; ++t) {
            const uint16_t *qt = q + ((b * T + t) * (long)n_heads) * head_dim;
            const float *wt = w + (b * T + t) * (long)n_heads;
            double *row = scores + (b * T + t) * (long)N;
            long vis = visible_count(N, q_pos0, t);
            for (long s = 0; s < N; ++s) {
                if (s >= vis) {
                    row[s] = -INFINITY;
                    continue;
                }
                const uint16_t *ks = k + (b * (long)N + s) * head_dim;
                double total = 0.0;
                for (int h = 0; h < n_heads; ++h) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += bf16_to_double(qt[(long)h * head_dim + d]) * bf16_to_double(ks[d]);
                    double relu = dot > 0.0 ? dot : 0.0;
                    total += (double)wt[h] * relu;
                }
                row[s] = total;
            }
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------------- */
/* Step 2: per-query top-k select  ([p2] Cut 1: keep the best 2048 of N)               */
/* ------------------------------------------------------------------------------- */
/*
 * The k selected tokens are the first k of the visible positions under the strict
 * total order "higher score first; on equal scores, lower token index first".
 * Equal scores compare equal under IEEE rules (so -0 == +0); a NaN score ranks below
 * every number.  The selected indices are written in ascending token order; when fewer
 * than k positions are visible, all of them are kept and the rest of the row is -1.
 */
typedef struct {
    float score;
    int32_t index;
} scored_t;

static int rank_before(const scored_t *a, const scored_t *b)
{
    int an = isnan(a->score), bn = isnan(b->score);
    if (an != bn) return bn;              /* the number ranks before the NaN */
    if (!an && a->score != b->score) return a->score > b->score;
    return a->index < b->index;           /* tie: lower token index first */
}

static int cmp_rank(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (rank_before(a, b)) return -1;
    if (rank_before(b, a)) return 1;
    return 0;
}

static int cmp_int32(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* scores [B, T, N] float32 -> idx [B, T, k] int32 */
int oracle_topk(const float *scores, int B, int T, int N, long q_pos0, int k, int32_t *idx)
{
    if (!scores || !idx || B < 0 || T < 0 || N < 0 || k <= 0) return OR_ERR_ARG;
    scored_t *buf = (scored_t *)malloc(sizeof(scored_t) * (size_t)(N > 0 ? N : 1));
    if (!buf) return OR_ERR_NOMEM;
    for (long r = 0; r < (long)B * T; ++r) {
        long t = r % T;
        const float *row = scores + r * (long)N;
        int32_t *out = idx + r * (long)k;
        long vis = visible_count(N, q_pos0, t);
        long take = vis < k ? vis : k;
        if (vis <= k) {
            for (long j = 0; j < vis; ++j) out[j] = (int32_t)j;
        } else {
            for (long s = 0; s < vis; ++s) {
                buf[s].score = row[s];
                buf[s].index = (int32_t)s;
            }
            qsort(buf, (size_t)vis, sizeof(scored_t), cmp_rank);
            for (long j = 0; j < take; ++j) out[j] = buf[j].index;
            qsort(out, (size_t)take, sizeof(int32_t), cmp_int32);
        }
        for (long j = take; j < k; ++j) out[j] = -1;
    }
    free(buf);
    return OR_OK;
}

/* ------------------------------------------------------------------------------- */
/* Step 3: sparse MLA attention over the selected rows  ([p2] Cut 1 and Cut 3)         */
/* ------------------------------------------------------------------------------- */
/*
 * For one query head with query vector qh (dqk wide) and the selected cache rows
 * c[idx_j] (dqk wide each; the value is the first dv entries):
 *     z_j   = scale * (qh . c[idx_j])           over the valid j (idx_j >= 0)
 *     p_j   = exp(z_j - max z) / sum_i exp(z_i - max z)
 *     out   = sum_j p_j * c[idx_j][0:dv]
 * With no valid index the output is zero.
 *
 * q   [B, T, H, dqk] bf16 bits, kv [B, N, dqk] bf16 bits, idx [B, T, k] int32,
 * out [B, T, H, dv] double.
 */
int oracle_sparse_attn(const uint16_t *q, const uint16_t *kv, const int32_t *idx,
                       int B, int T, int N, int H, int k, int dqk, int dv, double scale,
                       double *out)
{
    if (!q || !kv || !idx || !out || B < 0 || T < 0 || N < 0 || H <= 0 || k <= 0 ||
        dqk <= 0 || dv <= 0 || dv > dqk)
        return OR_ERR_ARG;
    double *z = (double *)malloc(sizeof(double) * (size_t)k);
    if (!z) return OR_ERR_NOMEM;
    for (long b = 0; b < B; ++b) {
        for (long t = 0; t < T; ++t) {
            const int32_t *sel = idx + (b * T + t) * (long)k;
            for (long j = 0; j < k; ++j)
                if (sel[j] >= N) { free(z); return OR_ERR_ARG; }
            for (long h = 0; h < H; ++h) {
                const uint16_t *qh = q + ((b * T + t) * (long)H + h) * dqk;
                double *o = out + ((b * T + t) * (long)H + h) * dv;
                double zmax = -INFINITY;
                for (long j = 0; j < k; ++j) {
                    if (sel[j] < 0) continue;
                    const uint16_t *c = kv + (b * (long)N + sel[j]) * dqk;
                    double dot = 0.0;
                    for (int d = 0; d < dqk; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(c[d]);
                    z[j] = scale * dot;
                    if (z[j] > zmax) zmax = z[j];
                }
                for (int d = 0; d < dv; ++d) o[d] = 0.0;
                if (zmax == -INFINITY) continue; /* nothing selected */
                double denom = 0.0;
                for (long j = 0; j < k; ++j)
                    if (sel[j] >= 0) denom += exp(z[j] - zmax);
                for (long j = 0; j < k; ++j) {
                    if (sel[j] < 0) continue;
                    double p = exp(z[j] - zmax) / denom;
                    const uint16_t *c = kv + (b * (long)N + sel[j]) * dqk;
                    for (int d = 0; d < dv; ++d) o[d] += p * bf16_to_double(c[d]);
                }
            }
        }
    }
    free(z);
    return OR_OK;
}

/*
 * The same attention written densely: softmax over all N cached positions with the
 * logit set to -inf for every position that is not in the selected set.  Used only
 * to pin oracle_sparse_attn (the two must agree up to rounding).
 */
int oracle_dense_masked_attn(const uint16_t *q, const uint16_t *kv, const int32_t *idx,
                             int B, int T, int N, int H, int k, int dqk, int dv, double scale,
                             double *out)
{
    if (!q || !kv || !idx || !out || B < 0 || T < 0 || N <= 0 || H <= 0 || k <= 0 ||
        dqk <= 0 || dv <= 0 || dv > dqk)
        return OR_ERR_ARG;
    double *z = (double *)malloc(sizeof(double) * (size_t)N);
    unsigned char *allowed = (unsigned char *)malloc((size_t)N);
    if (!z || !allowed) { free(z); free(allowed); return OR_ERR_NOMEM; }
    for (long b = 0; b < B; ++b) {
        for (long t = 0; t < T; ++t) {
            const int32_t *sel = idx + (b * T + t) * (long)k;
            memset(allowed, 0, (size_t)N);
            for (long j = 0; j < k; ++j) {
                if (sel[j] >= N) { free(z); free(allowed); return OR_ERR_ARG; }
                if (sel[j] >= 0) allowed[sel[j]] = 1;
            }
            for (long h = 0; h < H; ++h) {
                const uint16_t *qh = q + ((b * T + t) * (long)H + h) * dqk;
                double *o = out + ((b * T + t) * (long)H + h) * dv;
                double zmax = -INFINITY;
                for (long s = 0; s < N; ++s) {
                    if (!allowed[s]) { z[s] = -INFINITY; continue; }
                    const uint16_t *c = kv + (b * (long)N + s) * dqk;
                    double dot = 0.0;
                    for (int d = 0; d < dqk; ++d) dot += bf16_to_double(qh[d]) * bf16_to_double(c[d]);
                    z[s] = scale * dot;
                    if (z[s] > zmax) zmax = z[s];
                }
                for (int d = 0; d < dv; ++d) o[d] = 0.0;
                if (zmax == -INFINITY) continue;
                double denom = 0.0;
                for (long s = 0; s < N; ++s) denom += exp(z[s] - zmax); /* exp(-inf) = 0 */
                for (long s = 0; s < N; ++s) {
                    if (!allowed[s]) continue;
                    double p = exp(z[s] - zmax) / denom;
                    const uint16_t *c = kv + (b * (long)N + s) * dqk;
                    for (int d = 0; d < dv; ++d) o[d] += p * bf16_to_double(c[d]);
                }
            }
        }
    }
    free(z);
    free(allowed);
    return OR_OK;
}

/* ------------------------------------------------------------------------------- */
/* Step 4: IndexShare group  ([p1] Indexer Share; [p2] Cut 2; [p5] IndexShare)         */
/* ------------------------------------------------------------------------------- */
/*
 * One group of L layers shares one indexer: the indexer and the top-k run once (in
 * the group's first layer) and every layer of the group attends over the same index
 * list.  With compute_indices == 0 the caller's idx_shared is used as it is (this is
 * also the MTP draft-step reuse of [p1] and [p5]: steps 2.. reuse the step-1 indices,
 * so no draft-token position can be selected).
 *
 * The index buffer must come out of every layer byte-identical; the oracle checks it
 * and returns OR_ERR_INVARIANT otherwise.
 *
 * iq [B,T,n_heads,head_dim], w [B,T,n_heads], ik [B,N,head_dim]: indexer inputs;
 * q[l] [B,T,H,dqk], kv[l] [B,N,dqk]: layer l's queries and compressed cache;
 * idx_shared [B,T,k]; out[l] [B,T,H,dv] double.
 * The scores are rounded to float32 before the selection (the selection is taken in the
 * precision the GPU kernel produces).
 */
int oracle_group_forward(const uint16_t *iq, const float *w, const uint16_t *ik,
                         const uint16_t *const *q, const uint16_t *const *kv, int L,
                         int B, int T, int N, int n_heads, int head_dim, long q_pos0,
                         int H, int k, int dqk, int dv, double scale, int compute_indices,
                         int32_t *idx_shared, double *const *out)
{
    if (!q || !kv || !idx_shared || !out || L <= 0) return OR_ERR_ARG;
    size_t nidx = (size_t)B * T * k;
    if (compute_indices) {
        size_t ns = (size_t)B * T * N;
        double *sd = (double *)malloc(sizeof(double) * (ns ? ns : 1));
        float *sf = (float *)malloc(sizeof(float) * (ns ? ns : 1));
        if (!sd || !sf) { free(sd); free(sf); return OR_ERR_NOMEM; }
        int rc = oracle_index_score(iq, w, ik, B, T, N, n_heads, head_dim, q_pos0, sd);
        for (size_t i = 0; rc == OR_OK && i < ns; ++i) sf[i] = (float)sd[i];
        if (rc == OR_OK) rc = oracle_topk(sf, B, T, N, q_pos0, k, idx_shared);
        free(sd);
        free(sf);
        if (rc != OR_OK) return rc;
    }
    int32_t *before = (int32_t *)malloc(sizeof(int32_t) * (nidx ? nidx : 1));
    if (!before) return OR_ERR_NOMEM;
    memcpy(before, idx_shared, sizeof(int32_t) * nidx);
    int rc = OR_OK;
    for (int l = 0; l < L && rc == OR_OK; ++l) {
        rc = oracle_sparse_attn(q[l], kv[l], idx_shared, B, T, N, H, k, dqk, dv, scale, out[l]);
        if (rc == OR_OK && memcmp(before, idx_shared, sizeof(int32_t) * nidx) != 0)
            rc = OR_ERR_INVARIANT;
    }
    free(before);
    return rc;
}

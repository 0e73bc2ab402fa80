/*
 * shard_oracle.c -- CPU oracle for the context-sharded decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Like dsa_oracle.c (and compiled into the same liboracle.so),
 * this is the slow, obviously-correct reference that the CUDA library is checked against;
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * Source (page title, section): "Le contexte d'un million de tokens" (glmmodel.cn), "Service
 * efficace pour un million de contextes": a million-token context is served by spreading
 * it over several GPUs.  The pages give no algorithm; the reading taken is the plain one
 * that keeps the result identical to the unsharded path: every GPU holds a contiguous
 * range of the cached tokens (index keys and compressed rows), scores and selects its own
 * best k, the k best of all candidates are the row's top-k (a token in the global top-k is
 * in its own shard's top-k), and each GPU attends over the selected rows it holds; the
 * partial results combine exactly by their log-sum-exp:
 *     out = sum_w exp(lse_w - LSE) out_w,   LSE = ln sum_w exp(lse_w),
 * where out_w is the softmax-weighted value sum over shard w's selected rows and lse_w the
 * natural log of the sum of exp(logit) over them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG -1
#define OR_ERR_NOMEM -2

static double sh_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Attention over the selected rows one shard holds.
 *   q      [B, T, H, dqk] bf16 bits
 *   kv     [B, Ns, dqk]   bf16 bits: global positions [offset, offset + Ns) of the cache
 *   idx    [B, T, k]      global positions (entries < 0 or outside the shard are skipped)
 *   out    [B, T, H, dv]  double out: sum_j p_j kv[j, :dv], p = softmax over the shard's rows
 *                         (0 when the shard holds none of them)
 *   lse    [B, T, H]      double out: ln sum_j exp(scale * q . kv[j]) over those rows
 *                         (-inf when none)
 */
int oracle_sparse_attn_partial(const uint16_t *q, const uint16_t *kv, const int32_t *idx, int B, int T, int Ns,
                               long offset, int H, int k, int dqk, int dv, double scale, double *out, double *lse)
{
    if (!q || !kv || !idx || !out || !lse || B < 0 || T < 0 || Ns < 0 || H <= 0 || k <= 0 || dqk <= 0 || dv <= 0 ||
        dv > dqk)
        return OR_ERR_ARG;
    double *z = (double *)malloc(sizeof(double) * (size_t)k);
    if (!z) return OR_ERR_NOMEM;
    for (long b = 0; b < B; ++b) {
        for (long t = 0; t < T; ++t) {
            const int32_t *sel = idx + (b * T + t) * (long)k;
            for (long h = 0; h < H; ++h) {
                const uint16_t *qh = q + ((b * T + t) * (long)H + h) * dqk;
                double *o = out + ((b * T + t) * (long)H + h) * dv;
                double zmax = -INFINITY;
                for (long j = 0; j < k; ++j) {
                    const long g = sel[j];
                    if (g < offset || g >= offset + Ns) continue;
                    const uint16_t *c = kv + (b * (long)Ns + (g - offset)) * dqk;
                    double dot = 0.0;
                    for (int d = 0; d < dqk; ++d) dot += sh_bf16(qh[d]) * sh_bf16(c[d]);
                    z[j] = scale * dot;
                    if (z[j] > zmax) zmax = z[j];
                }
                for (int d = 0; d < dv; ++d) o[d] = 0.0;
                if (zmax == -INFINITY) {
                    lse[(b * T + t) * (long)H + h] = -INFINITY;
                    continue;
                }
                double denom = 0.0;
                for (long j = 0; j < k; ++j) {
                    const long g = sel[j];
                    if (g >= offset && g < offset + Ns) denom += exp(z[j] - zmax);
                }
                for (long j = 0; j < k; ++j) {
                    const long g = sel[j];
                    if (g < offset || g >= offset + Ns) continue;
                    const double p = exp(z[j] - zmax) / denom;
                    const uint16_t *c = kv + (b * (long)Ns + (g - offset)) * dqk;
                    for (int d = 0; d < dv; ++d) o[d] += p * sh_bf16(c[d]);
                }
                lse[(b * T + t) * (long)H + h] = zmax + log(denom);
            }
        }
    }
    free(z);
    return OR_OK;
}

/*
 * Combines W partial attentions of the same queries over disjoint row sets.
 *   outs [W, R, dv] double, lses [W, R] double (R = B*T*H rows) -> out [R, dv] double
 * out = sum_w exp(lse_w - LSE) outs_w with LSE = ln sum_w exp(lse_w); a row whose every
 * lse is -inf is 0.
 */
int oracle_merge_partials(const double *outs, const double *lses, int W, long R, int dv, double *out)
{
    if (!outs || !lses || !out || W <= 0 || R < 0 || dv <= 0) return OR_ERR_ARG;
    for (long r = 0; r < R; ++r) {
        double m = -INFINITY;
        for (int w = 0; w < W; ++w)
            if (lses[(long)w * R + r] > m) m = lses[(long)w * R + r];
        double *o = out + r * dv;
        for (int d = 0; d < dv; ++d) o[d] = 0.0;
        if (m == -INFINITY) continue;
        double s = 0.0;
        for (int w = 0; w < W; ++w) s += exp(lses[(long)w * R + r] - m);
        for (int w = 0; w < W; ++w) {
            const double c = exp(lses[(long)w * R + r] - m) / s;
            const double *ow = outs + ((long)w * R + r) * dv;
            for (int d = 0; d < dv; ++d) o[d] += c * ow[d];
        }
    }
    return OR_OK;
}

typedef struct {
    float score;
    int32_t pos;
} sh_cand_t;

/* a ranks before b: higher score first, equal scores (-0 == +0) to the lower position, NaN last */
static int sh_before(const sh_cand_t *a, const sh_cand_t *b)
{
    const int an = isnan(a->score), bn = isnan(b->score);
    if (an != bn) return bn;
    if (!an && a->score != b->score) return a->score > b->score;
    return a->pos < b->pos;
}

static int sh_cmp(const void *pa, const void *pb)
{
    const sh_cand_t *a = (const sh_cand_t *)pa, *b = (const sh_cand_t *)pb;
    if (sh_before(a, b)) return -1;
    if (sh_before(b, a)) return 1;
    return 0;
}

static int sh_cmp_i32(const void *pa, const void *pb)
{
    const int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/*
 * The k best of M candidates per query row.
 *   score [R, M] f32, pos [R, M] global positions (< 0: no candidate) -> idx [R, k]: the
 *   selected positions ascending, -1 padding when fewer than k candidates exist.
 */
int oracle_merge_candidates(const float *score, const int32_t *pos, long R, int M, int k, int32_t *idx)
{
    if (!score || !pos || !idx || R < 0 || M < 0 || k <= 0) return OR_ERR_ARG;
    sh_cand_t *c = (sh_cand_t *)malloc(sizeof(sh_cand_t) * (size_t)(M > 0 ? M : 1));
    if (!c) return OR_ERR_NOMEM;
    for (long r = 0; r < R; ++r) {
        int n = 0;
        for (int j = 0; j < M; ++j) {
            if (pos[r * M + j] < 0) continue;
            c[n].score = score[r * M + j];
            c[n].pos = pos[r * M + j];
            ++n;
        }
        qsort(c, (size_t)n, sizeof(sh_cand_t), sh_cmp);
        const int take = n < k ? n : k;
        int32_t *o = idx + r * (long)k;
        for (int j = 0; j < take; ++j) o[j] = c[j].pos;
        qsort(o, (size_t)take, sizeof(int32_t), sh_cmp_i32);
        for (int j = take; j < k; ++j) o[j] = -1;
    }
    free(c);
    return OR_OK;
}

/*
 * fp8_oracle.c -- CPU oracle for the indexer score over an FP8 index-key cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Like dsa_oracle.c (and compiled into the same liboracle.so),
 * this is the slow, obviously-correct reference that the CUDA library is checked against;
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * Source (page title, section): "Le contexte d'un million de tokens" (glmmodel.cn),
 * "Entraînement par renforcement de l'agent intelligent": an FP8 KV cache keeps the
 * rollout memory within budget.  The page names no FP8 format; the reading taken is
 * E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals, no
 * infinities, S.1111.111 = NaN) for the index keys and the indexer queries.  The score is
 * the same lightweight-indexer form as dsa_oracle.c,
 *     I(t,s) = sum_h w[t,h] * ReLU(q[t,h] . k[s]),
 * on the decoded values, in double precision.
 */
#include <math.h>
#include <stdint.h>

#define OR_OK 0
#define OR_ERR_ARG -1

/* E4M3 byte -> double, from the format's definition. */
double oracle_e4m3_to_double(uint8_t b)
{
    const int sign = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Number of cached tokens query t may look at: positions s <= q_pos0 + t, s < N. */
static long visible(long N, long q_pos0, long t)
{
    long v = q_pos0 + t + 1;
    return v < 0 ? 0 : (v > N ? N : v);
}

/*
 * q      [B, T, n_heads, head_dim]  E4M3 bytes  (indexer queries)
 * w      [B, T, n_heads]            float32     (per-query head weights)
 * k      [B, N, head_dim]           E4M3 bytes  (one shared index key per cached token)
 * scores [B, T, N]                  double      out; -inf where s is not visible to t
 */
int oracle_index_score_e4m3(const uint8_t *q, const float *w, const uint8_t *k, int B, int T, int N, int n_heads,
                            int head_dim, long q_pos0, double *scores)
{
    if (!q || !w || !k || !scores || B < 0 || T < 0 || N < 0 || n_heads <= 0 || head_dim <= 0) return OR_ERR_ARG;
    for (long b = 0; b < B; ++b) {
        for (long t = 0; t < T; ++t) {
            const uint8_t *qt = q + ((b * T + t) * (long)n_heads) * head_dim;
            const float *wt = w + (b * T + t) * (long)n_heads;
            double *row = scores + (b * T + t) * (long)N;
            const long vis = visible(N, q_pos0, t);
            for (long s = 0; s < N; ++s) {
                if (s >= vis) {
                    row[s] = -INFINITY;
                    continue;
                }
                const uint8_t *ks = k + (b * (long)N + s) * head_dim;
                double total = 0.0;
                for (int h = 0; h < n_heads; ++h) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += oracle_e4m3_to_double(qt[(long)h * head_dim + d]) * oracle_e4m3_to_double(ks[d]);
                    total += (double)wt[h] * (dot > 0.0 ? dot : 0.0);
                }
                row[s] = total;
            }
        }
    }
    return OR_OK;
}

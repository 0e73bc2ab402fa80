/*
 * verify_oracle.c -- CPU oracle for the MTP verify step: rejection sampling of the draft
 * tokens against the target model's distributions.
 *
 * TEST INFRASTRUCTURE ONLY.  Like dsa_oracle.c (and compiled into the same liboracle.so),
 * this is the slow, obviously-correct reference that the CUDA library is checked against;
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or helper with the CUDA path.
 *
 * Source (page title, section): "GLM-5.2 MTP IndexShare inference" (4sapi.ai), "Rejection
 * Sampling: from 'pick the champion' to 'look at agreement'": for every vocabulary entry
 * take the smaller of the two models' probabilities and add them up; that sum is the
 * acceptance rate, the probability that the draft token is taken.  "GLM-5.2 speculative
 * decoding" (yun88.com news 9578) and the MTP sections of the other pages: the draft
 * tokens are verified in order and the sequence is cut at the first rejection.
 *
 * The pages give the acceptance rate but not the accept / resample procedure.  The
 * reading taken is the standard speculative-sampling rule whose acceptance probability is
 * exactly that sum:
 *   - the draft token x (drawn from the draft distribution q) is accepted iff
 *     u * q[x] < p[x] for a uniform u in [0, 1), i.e. with probability min(1, p[x] / q[x]);
 *   - otherwise a token is drawn from the residual r_v = max(0, p_v - q_v), normalised.
 * Summed over x ~ q, the acceptance probability is sum_v min(p_v, q_v).
 *
 * Both decisions are integers, so both are taken exactly, in the precision of the inputs
 * (float32):
 *   - accept: the product u * q[x] is one float32 multiplication, compared with p[x];
 *   - resample: r_v = p_v - q_v in float32 (one rounding), negatives to 0; integer weights
 *     W_v = floor(r_v * 2^40) (exact: a power-of-two scale of a value below 1, truncated);
 *     S = sum_v W_v (exact in 64 bits for a vocabulary below 2^24); target
 *     T = floor(floor(u2 * 2^24) * S / 2^24) in exact integer arithmetic; the token is the
 *     smallest v whose inclusive prefix sum of W exceeds T.  When S = 0 (no residual mass)
 *     the draft token is kept.
 * The acceptance rate itself is reported in double precision.
 */
#include <stdint.h>
#include <stdlib.h>

#define OR_OK 0
#define OR_ERR_ARG -1

/* Acceptance rate of one row: sum_v min(p_v, q_v), accumulated in double. */
static double acceptance_rate(const float *p, const float *q, int V)
{
    double a = 0.0;
    for (int v = 0; v < V; ++v) a += (double)(p[v] < q[v] ? p[v] : q[v]);
    return a;
}

/* Residual token of one row (see the header): exact integer inverse CDF. */
static int32_t resample(const float *p, const float *q, int V, float u2, int32_t fallback)
{
    uint64_t S = 0;
    for (int v = 0; v < V; ++v) {
        float r = p[v] - q[v];
        if (r > 0.0f) S += (uint64_t)(r * 1099511627776.0f); /* 2^40 */
    }
    if (S == 0) return fallback;
    const uint64_t u24 = (uint64_t)(u2 * 16777216.0f); /* 2^24 */
    const uint64_t T = (uint64_t)(((unsigned __int128)u24 * S) >> 24);
    uint64_t run = 0;
    for (int v = 0; v < V; ++v) {
        float r = p[v] - q[v];
        if (r > 0.0f) run += (uint64_t)(r * 1099511627776.0f);
        if (run > T) return v;
    }
    return fallback; /* not reached: T < S */
}

/*
 * Verify B sequences of S draft tokens each (row r = b * S + j is draft position j of
 * sequence b):
 *   p, q   [B*S, V] float32: target and draft probabilities of each position
 *   draft  [B*S] the draft tokens; u, u2 [B*S] uniform numbers in [0, 1) for the accept
 *          test and for the resample
 *   alpha  [B*S] out: acceptance rate sum_v min(p_v, q_v) (double)
 *   accept [B*S] out: 1 if the draft token is accepted, else 0
 *   token  [B*S] out: the draft token if accepted, else the residual sample
 *   accepted_len [B] out: how many leading positions of the sequence are accepted (the
 *          sequence is cut at its first rejection, whose resampled token follows them)
 */
int oracle_verify(const float *p, const float *q, const int32_t *draft, const float *u, const float *u2, int B,
                  int S, int V, double *alpha, int32_t *accept, int32_t *token, int32_t *accepted_len)
{
    if (!p || !q || !draft || !u || !u2 || !alpha || !accept || !token || !accepted_len) return OR_ERR_ARG;
    if (B <= 0 || S <= 0 || V <= 0 || V >= (1 << 24)) return OR_ERR_ARG;
    for (long r = 0; r < (long)B * S; ++r) {
        const float *pr = p + r * (long)V, *qr = q + r * (long)V;
        const int32_t x = draft[r];
        if (x < 0 || x >= V) return OR_ERR_ARG;
        alpha[r] = acceptance_rate(pr, qr, V);
        const float uq = u[r] * qr[x];
        accept[r] = uq < pr[x] ? 1 : 0;
        token[r] = accept[r] ? x : resample(pr, qr, V, u2[r], x);
    }
    for (int b = 0; b < B; ++b) {
        int n = 0;
        while (n < S && accept[(long)b * S + n]) ++n;
        accepted_len[b] = n;
    }
    return OR_OK;
}

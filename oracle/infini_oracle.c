/*
 * Plain, slow, single-threaded fp64 CPU oracle of the Infini-attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline / reference leg may load this code.  The product path
 * (the CUDA library) shares nothing with it: no headers, helpers, tables or kernels.
 *
 * Sources (page title, then section):
 *   [blk] AI Wiki "Infini-Attention", "What happens inside the Infini-attention block?"
 *         -- local causal attention A_dot = softmax(Q_s K_s^T / sqrt(d)) V_s, the feature
 *            map sigma(x) = ELU(x) + 1, the retrieval A_mem = sigma(Q_s) M_{s-1} /
 *            (sigma(Q_s) z_{s-1}) and the gate A = sigmoid(beta) A_mem + (1 - sigmoid(beta)) A_dot.
 *   [mem] AI Wiki "Infini-Attention", "How does the compressive memory work?"
 *         -- delta rule M_s = M_{s-1} + sigma(K_s)^T (V_s - sigma(K_s) M_{s-1} / (sigma(K_s) z_{s-1})),
 *            z_s = z_{s-1} + sum_t sigma(K_{s,t}), and the additive ("linear") variant
 *            M_s = M_{s-1} + sigma(K_s)^T V_s.
 *   [hf]  "Hugging Face Infini-Attention Reproduction Analysis", "Infini-Attention Mechanism",
 *         steps 1-6: fixed-size segments processed in order; only the memory is carried.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - softmax scale 1/sqrt(d) with d the head dimension; sigma is applied to raw q and k;
 *   - ELU alpha = 1, so sigma(x) = x + 1 for x > 0 and exp(x) otherwise;
 *   - the causal mask keeps j <= i (a token sees itself); no key of an earlier segment
 *     enters the local softmax;
 *   - a quotient whose denominator is exactly 0 is 0 (A_mem while z = 0, and the delta
 *     residual's prediction while z = 0);
 *   - the delta rule is one batch update per segment: every token of segment s reads M_{s-1};
 *   - beta is one scalar per query head; query head h reads key/value head h / (H / Hkv);
 *   - d_key = d_value = d;
 *   - a final segment shorter than N (L % N != 0) is processed the same way, shorter.
 *
 * Layouts (row-major, contiguous):  q, out [B,H,L,d];  k, v [B,Hkv,L,d];  beta [H];
 * M0, M_out [B,Hkv,d,d] (row = key feature, column = value feature);  z0, z_out [B,Hkv,d].
 * Inputs are float (bf16 inputs arrive widened, which is exact); all arithmetic and all
 * outputs are double.  M0 / z0 may be NULL, meaning zeros.  seg_out, when not NULL, is a
 * [ceil(L/N)] byte mask: the output rows of segment s are computed only where seg_out[s]
 * is nonzero (the memory chain always runs over every segment); rows not computed are
 * left untouched.
 *
 * Returns 0 on success, 1 on an invalid argument, 2 on an allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* [blk]: sigma(x) = ELU(x) + 1 with alpha = 1. */
static double feature_map(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* [blk]: the gate is the logistic sigmoid of the per-head scalar beta. */
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

int oracle_infini_attn_fwd(const float *q, const float *k, const float *v, const float *beta,
                           const float *M0, const float *z0, double *out, double *M_out,
                           double *z_out, int64_t B, int64_t H, int64_t Hkv, int64_t L,
                           int64_t N, int64_t d, int update_rule, const unsigned char *seg_out)
{
    if (!q || !k || !v || !beta || !out || !M_out || !z_out) return 1;
    if (B <= 0 || H <= 0 || Hkv <= 0 || L <= 0 || N <= 0 || d <= 0) return 1;
    if (H % Hkv != 0 || (update_rule != 0 && update_rule != 1)) return 1;

    const int64_t G = H / Hkv;
    const int64_t S = (L + N - 1) / N;
    const double scale = 1.0 / sqrt((double)d);

    double *M = malloc(sizeof(double) * d * d);       /* memory M_{s-1}            */
    double *z = malloc(sizeof(double) * d);           /* normaliser z_{s-1}        */
    double *sk = malloc(sizeof(double) * N * d);      /* sigma(K_s), one row/token */
    double *resid = malloc(sizeof(double) * N * d);   /* value written per token   */
    double *logit = malloc(sizeof(double) * N);
    double *sq = malloc(sizeof(double) * d);
    double *adot = malloc(sizeof(double) * d);
    double *num = malloc(sizeof(double) * d);
    if (!M || !z || !sk || !resid || !logit || !sq || !adot || !num) {
        free(M); free(z); free(sk); free(resid); free(logit); free(sq); free(adot); free(num);
        return 2;
    }

    for (int64_t b = 0; b < B; ++b) {
        for (int64_t kvh = 0; kvh < Hkv; ++kvh) {
            const int64_t st = b * Hkv + kvh;
            const float *K = k + st * L * d;
            const float *V = v + st * L * d;
            for (int64_t i = 0; i < d * d; ++i) M[i] = M0 ? (double)M0[st * d * d + i] : 0.0;
            for (int64_t i = 0; i < d; ++i) z[i] = z0 ? (double)z0[st * d + i] : 0.0;

            for (int64_t s = 0; s < S; ++s) {            /* [hf] step 1: segments in order */
                const int64_t t0 = s * N;
                const int64_t n = (L - t0 < N) ? (L - t0) : N;

                if (!seg_out || seg_out[s]) {
                    for (int64_t hh = 0; hh < G; ++hh) {
                        const int64_t h = kvh * G + hh;
                        const double g = sigmoid((double)beta[h]);
                        const float *Q = q + ((b * H + h) * L) * d;
                        double *O = out + ((b * H + h) * L) * d;
                        for (int64_t i = 0; i < n; ++i) {
                            const float *qi = Q + (t0 + i) * d;
                            /* [blk] A_dot: causal softmax over keys t0..t0+i of this segment. */
                            double mx = -INFINITY;
                            for (int64_t j = 0; j <= i; ++j) {
                                const float *kj = K + (t0 + j) * d;
                                double a = 0.0;
                                for (int64_t c = 0; c < d; ++c) a += (double)qi[c] * (double)kj[c];
                                logit[j] = a * scale;
                                if (logit[j] > mx) mx = logit[j];
                            }
                            double den_soft = 0.0;
                            for (int64_t e = 0; e < d; ++e) adot[e] = 0.0;
                            for (int64_t j = 0; j <= i; ++j) {
                                const double p = exp(logit[j] - mx);
                                const float *vj = V + (t0 + j) * d;
                                den_soft += p;
                                for (int64_t e = 0; e < d; ++e) adot[e] += p * (double)vj[e];
                            }
                            /* [blk] A_mem = sigma(q) M_{s-1} / (sigma(q) . z_{s-1}); 0 when the
                             * denominator is exactly 0 (empty memory). */
                            double den_mem = 0.0;
                            for (int64_t c = 0; c < d; ++c) {
                                sq[c] = feature_map((double)qi[c]);
                                den_mem += sq[c] * z[c];
                            }
                            for (int64_t e = 0; e < d; ++e) num[e] = 0.0;
                            for (int64_t c = 0; c < d; ++c)
                                for (int64_t e = 0; e < d; ++e) num[e] += sq[c] * M[c * d + e];
                            double *oi = O + (t0 + i) * d;
                            for (int64_t e = 0; e < d; ++e) {
                                const double amem = (den_mem == 0.0) ? 0.0 : num[e] / den_mem;
                                const double ad = adot[e] / den_soft;
                                oi[e] = g * amem + (1.0 - g) * ad;      /* [blk] gate */
                            }
                        }
                    }
                }

                /* [mem] memory update with this segment's keys and values. */
                for (int64_t t = 0; t < n; ++t)
                    for (int64_t c = 0; c < d; ++c)
                        sk[t * d + c] = feature_map((double)K[(t0 + t) * d + c]);

                for (int64_t t = 0; t < n; ++t) {
                    const float *vt = V + (t0 + t) * d;
                    double *rt = resid + t * d;
                    if (update_rule == 0) {
                        /* additive variant: write V_s itself */
                        for (int64_t e = 0; e < d; ++e) rt[e] = (double)vt[e];
                    } else {
                        /* delta rule: write V_s minus what M_{s-1} already returns for k_t */
                        double den = 0.0;
                        for (int64_t c = 0; c < d; ++c) den += sk[t * d + c] * z[c];
                        for (int64_t e = 0; e < d; ++e) num[e] = 0.0;
                        for (int64_t c = 0; c < d; ++c)
                            for (int64_t e = 0; e < d; ++e) num[e] += sk[t * d + c] * M[c * d + e];
                        for (int64_t e = 0; e < d; ++e)
                            rt[e] = (double)vt[e] - ((den == 0.0) ? 0.0 : num[e] / den);
                    }
                }
                /* M_s = M_{s-1} + sigma(K_s)^T R_s  (every token read M_{s-1} above) */
                for (int64_t t = 0; t < n; ++t)
                    for (int64_t c = 0; c < d; ++c) {
                        const double a = sk[t * d + c];
                        for (int64_t e = 0; e < d; ++e) M[c * d + e] += a * resid[t * d + e];
                    }
                /* z_s = z_{s-1} + sum_t sigma(K_{s,t}) */
                for (int64_t t = 0; t < n; ++t)
                    for (int64_t c = 0; c < d; ++c) z[c] += sk[t * d + c];
            }
            memcpy(M_out + st * d * d, M, sizeof(double) * d * d);
            memcpy(z_out + st * d, z, sizeof(double) * d);
        }
    }
    free(M); free(z); free(sk); free(resid); free(logit); free(sq); free(adot); free(num);
    return 0;
}

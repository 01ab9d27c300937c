/*
 * Gated delta rule oracle: a plain, slow, fp64 CPU restatement of the
 * recurrence, used ONLY as test infrastructure (tests, the package's smoke
 * check and the benchmark's CPU baseline).  Nothing on the product path links
 * or calls this file, and it shares no code with the CUDA kernels.
 *
 * What it computes (per sequence b and head h, independently):
 *
 *     alpha_t = exp(g_t)
 *     S_t     = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t     = S_t q_t
 *
 * with S in R^{Dv x Dk} stored row-major ([Dv][Dk], row i contiguous in Dk),
 * starting from S_0 (zeros when the caller passes NULL).  The recurrence is the
 * gated delta rule of the linear-attention layers of the hybrid Qwen 3.5
 * models; the ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev
 * article d2880479, opening post) fixes the setting it is used in: a scalar
 * gate per token and head, head dim 128, single-sequence prefill, and a state
 * kept in F32 accumulators on the device.  The note itself prints no formula
 * and no worked example.
 *
 * The update is evaluated in the PRODUCT form as written above, term by term:
 *     u      = S_{t-1} k_t                       (Dv vector)
 *     S_t    = alpha_t*S_{t-1} - alpha_t*beta_t*u k_t^T + beta_t*v_t k_t^T
 * so that it shares no algebra (delta form, chunking, WY/UT transform) with
 * the GPU path.  Every value is widened to double before use; no fused or
 * reordered arithmetic beyond the loops below.
 *
 * Layouts (all contiguous, last index fastest):
 *   q, k : [B][T][H][Dk]   (float; callers pass the bf16 inputs widened exactly)
 *   v    : [B][T][H][Dv]
 *   g, beta : [B][T][H]
 *   S0   : [B][H][Dv][Dk]  or NULL (zeros)
 *   o    : [B][T][H][Dv]   double, written
 *   S_T  : [B][H][Dv][Dk]  double, written
 *
 * Returns 0 on success, -1 on bad sizes, -2 on allocation failure.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int64_t idx4(int64_t a, int64_t b, int64_t c, int64_t d,
                    int64_t nb, int64_t nc, int64_t nd) {
    return ((a * nb + b) * nc + c) * nd + d;
}

/* One token of the recurrence on the state S ([Dv][Dk], updated in place),
 * evaluated in the product form; writes o_t = S_t q_t. */
static void gdn_step(double *S, const float *qt, const float *kt, const float *vt,
                     double gt, double bt, double *ot, int Dk, int Dv, double *u) {
    const double alpha = exp(gt);
    /* u = S_{t-1} k_t */
    for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        const double *Si = S + (int64_t)i * Dk;
        for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)kt[j];
        u[i] = acc;
    }
    /* S_t = alpha*S_{t-1} - alpha*beta*u k^T + beta*v k^T */
    for (int i = 0; i < Dv; ++i) {
        double *Si = S + (int64_t)i * Dk;
        const double vi = (double)vt[i];
        for (int j = 0; j < Dk; ++j) {
            const double kj = (double)kt[j];
            Si[j] = alpha * Si[j] - alpha * bt * u[i] * kj + bt * vi * kj;
        }
    }
    /* o_t = S_t q_t */
    for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        const double *Si = S + (int64_t)i * Dk;
        for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)qt[j];
        ot[i] = acc;
    }
}

/* One (b, h) chain, t in [0, T). */
static void run_chain(const float *q, const float *k, const float *v,
                      const float *g, const float *beta, const float *S0,
                      double *o, double *S_T, int b, int h, int T, int H,
                      int Dk, int Dv, double *S, double *u) {
    const int64_t s_off = ((int64_t)b * H + h) * (int64_t)Dv * Dk;
    if (S0) {
        for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) S[e] = (double)S0[s_off + e];
    } else {
        memset(S, 0, sizeof(double) * (size_t)Dv * (size_t)Dk);
    }
    for (int t = 0; t < T; ++t) {
        const int64_t gi = ((int64_t)b * T + t) * H + h;
        gdn_step(S, q + idx4(b, t, h, 0, T, H, Dk), k + idx4(b, t, h, 0, T, H, Dk),
                 v + idx4(b, t, h, 0, T, H, Dv), (double)g[gi], (double)beta[gi],
                 o + idx4(b, t, h, 0, T, H, Dv), Dk, Dv, u);
    }
    if (S_T) memcpy(S_T + s_off, S, sizeof(double) * (size_t)Dv * (size_t)Dk);
}

int oracle_gdn_prefill_f64(const float *q, const float *k, const float *v,
                           const float *g, const float *beta, const float *S0,
                           double *o, double *S_T, int B, int T, int H,
                           int Dk, int Dv) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return -1;
    const int chains = B * H;
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)Dv * (size_t)Dk);
        double *u = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!S || !u) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int c = 0; c < chains; ++c) {
                run_chain(q, k, v, g, beta, S0, o, S_T, c / H, c % H, T, H, Dk, Dv, S, u);
            }
        }
        free(S);
        free(u);
    }
    return failed ? -2 : 0;
}

/* Restricted to the chains listed in `chain_ids` (each b*H + h): used to check
 * sampled chains of workloads too large for a full fp64 pass.  Outputs use the
 * full [B][T][H][Dv] / [B][H][Dv][Dk] layouts; entries of unlisted chains are
 * left untouched. */
int oracle_gdn_prefill_chains_f64(const float *q, const float *k, const float *v,
                                  const float *g, const float *beta, const float *S0,
                                  double *o, double *S_T, int B, int T, int H,
                                  int Dk, int Dv, const int *chain_ids, int n_ids) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0 || n_ids < 0) return -1;
    for (int n = 0; n < n_ids; ++n)
        if (chain_ids[n] < 0 || chain_ids[n] >= B * H) return -1;
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)Dv * (size_t)Dk);
        double *u = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!S || !u) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int n = 0; n < n_ids; ++n) {
                const int c = chain_ids[n];
                run_chain(q, k, v, g, beta, S0, o, S_T, c / H, c % H, T, H, Dk, Dv, S, u);
            }
        }
        free(S);
        free(u);
    }
    return failed ? -2 : 0;
}

/* One decode step: the recurrence above with T = 1, the state updated in place.
 * q, k: [B][H][Dk]; v: [B][H][Dv]; g, beta: [B][H]; S: [B][H][Dv][Dk] (inout);
 * o: [B][H][Dv]. */
int oracle_gdn_decode_step_f64(const float *q, const float *k, const float *v,
                               const float *g, const float *beta, double *S,
                               double *o, int B, int H, int Dk, int Dv) {
    if (B < 0 || H < 0 || Dk <= 0 || Dv <= 0) return -1;
    const int chains = B * H;
    int failed = 0;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * (size_t)Dv);
        if (!u) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(static)
            for (int c = 0; c < chains; ++c) {
                gdn_step(S + (int64_t)c * Dv * Dk, q + (int64_t)c * Dk, k + (int64_t)c * Dk,
                         v + (int64_t)c * Dv, (double)g[c], (double)beta[c],
                         o + (int64_t)c * Dv, Dk, Dv, u);
            }
        }
        free(u);
    }
    return failed ? -2 : 0;
}

/* ------------------------------------------------------------------------
 * Per-channel gate (KDA, the "next" variant the ROCmFPX gated-delta-net
 * prefill note names among the cases its fused kernel did not cover).  The
 * scalar gate becomes one decay per key channel, applied where the scalar one
 * is:
 *
 *     alpha_t = exp(g_t)                       (a vector over Dk)
 *     S_t     = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t     = S_t q_t
 *
 * evaluated, as above, in the product form term by term:
 *     u       = S_{t-1} diag(alpha_t) k_t                          (Dv vector)
 *     S_t[i][j] = alpha_t[j] S_{t-1}[i][j] - beta_t u[i] k_t[j] + beta_t v_t[i] k_t[j]
 *
 * g is [B][T][H][Dk] (natural-log decays, fp32); everything else is laid out
 * as for the scalar gate.
 */
static void kda_step(double *S, const float *qt, const float *kt, const float *vt,
                     const float *gt, double bt, double *ot, int Dk, int Dv, double *u,
                     double *a) {
    for (int j = 0; j < Dk; ++j) a[j] = exp((double)gt[j]);
    /* u = S_{t-1} diag(alpha) k */
    for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        const double *Si = S + (int64_t)i * Dk;
        for (int j = 0; j < Dk; ++j) acc += Si[j] * a[j] * (double)kt[j];
        u[i] = acc;
    }
    for (int i = 0; i < Dv; ++i) {
        double *Si = S + (int64_t)i * Dk;
        const double vi = (double)vt[i];
        for (int j = 0; j < Dk; ++j) {
            const double kj = (double)kt[j];
            Si[j] = a[j] * Si[j] - bt * u[i] * kj + bt * vi * kj;
        }
    }
    for (int i = 0; i < Dv; ++i) {
        double acc = 0.0;
        const double *Si = S + (int64_t)i * Dk;
        for (int j = 0; j < Dk; ++j) acc += Si[j] * (double)qt[j];
        ot[i] = acc;
    }
}

int oracle_kda_prefill_f64(const float *q, const float *k, const float *v,
                           const float *g, const float *beta, const float *S0,
                           double *o, double *S_T, int B, int T, int H,
                           int Dk, int Dv) {
    if (B < 0 || T < 0 || H < 0 || Dk <= 0 || Dv <= 0) return -1;
    const int chains = B * H;
    int failed = 0;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)Dv * (size_t)Dk);
        double *u = (double *)malloc(sizeof(double) * (size_t)Dv);
        double *a = (double *)malloc(sizeof(double) * (size_t)Dk);
        if (!S || !u || !a) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int c = 0; c < chains; ++c) {
                const int b = c / H, h = c % H;
                const int64_t s_off = ((int64_t)b * H + h) * (int64_t)Dv * Dk;
                if (S0) {
                    for (int64_t e = 0; e < (int64_t)Dv * Dk; ++e) S[e] = (double)S0[s_off + e];
                } else {
                    memset(S, 0, sizeof(double) * (size_t)Dv * (size_t)Dk);
                }
                for (int t = 0; t < T; ++t) {
                    const int64_t gi = ((int64_t)b * T + t) * H + h;
                    kda_step(S, q + idx4(b, t, h, 0, T, H, Dk), k + idx4(b, t, h, 0, T, H, Dk),
                             v + idx4(b, t, h, 0, T, H, Dv), g + idx4(b, t, h, 0, T, H, Dk),
                             (double)beta[gi], o + idx4(b, t, h, 0, T, H, Dv), Dk, Dv, u, a);
                }
                if (S_T) memcpy(S_T + s_off, S, sizeof(double) * (size_t)Dv * (size_t)Dk);
            }
        }
        free(S);
        free(u);
        free(a);
    }
    return failed ? -2 : 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

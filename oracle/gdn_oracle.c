/*
 * gdn_oracle.c -- plain fp64 CPU oracle for the FG^2-GDN recurrence and the
 * DeltaProduct n_h variant.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only tests/, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference arm of bench.py use it.  It shares no code, header,
 * table or helper with the CUDA library under gated_delta_rule_fg_b200/.
 *
 * What it computes (token by token, one (batch, head) pair at a time):
 *
 *   FG^2-GDN update rule -- "FG^2-GDN: Enhancing Long-Context Gated Delta
 *   Networks with Doubly Fine-Grained Control", sec. 2 "FG2-GDN Update Rule",
 *   and the reading notes of the same paper, sec. 2.2, eq. (11):
 *       k~_t = sqrt(beta_t) (.) k_t,   v~_t = sqrt(beta_t) (.) v_t
 *       S_t  = (I - k~_t k~_t^T) Diag(alpha_t) S_{t-1} + k~_t v~_t^T
 *       o_t  = S_t^T q_t                      (the UPDATED state is read)
 *   with S in R^{dk x dv}.  Written as
 *       X   = Diag(alpha_t) S_{t-1}
 *       S_t = X + k~_t (v~_t - X^T k~_t)^T
 *   which is the same matrix (expand (I - k~ k~^T) X + k~ v~^T).
 *
 *   Readings where the pages leave a step open:
 *     - q and k arrive raw and are L2-normalised per token and head,
 *       x / sqrt(sum x^2 + eps), before k is scaled by sqrt(beta); no 1/sqrt(d)
 *       query scale is applied (none is mentioned).
 *     - alpha and beta arrive already activated (alpha in (0,1], beta >= 0).
 *     - the decay is applied first, then the erase/write, as eq. (11) is
 *       written.
 *     - scalar alpha (GDN) and scalar beta (KDA, DeltaNet) broadcast over the
 *       channels (reading notes, sec. 1 table of GDN / KDA / FG^2-GDN).
 *     - channel-wise beta multiplies v, so it needs dk == dv (eq. (11)).
 *
 *   FG^2-GDN+ -- same paper, "FG2-GDN+ Variant"; reading notes sec. 2.3,
 *   eq. (13): the key side and the value side get their own rates,
 *       k^_t = sqrt(beta^k_t) (.) k_t,   v~_t = sqrt(beta^v_t) (.) v_t
 *       S_t  = (I - k^_t k^_t^T) Diag(alpha_t) S_{t-1} + k^_t v~_t^T
 *   with beta^k in R^{dk} and beta^v in R^{dv} (so dk may differ from dv).
 *   gdn_head takes an optional beta_v; when it is given, v is scaled by it.
 *
 *   DeltaProduct -- "DeltaProduct: Improving State-Tracking in Linear RNNs via
 *   Householder Products", "Approach": n_h generalized Householder steps per
 *   token, each one online gradient step on one (k, v, beta) triple,
 *       S <- (I - beta_{t,m} k_{t,m} k_{t,m}^T) S + beta_{t,m} k_{t,m} v_{t,m}^T,
 *   with a scalar forget gate gamma_t ("Add a forget gate", the Gated
 *   DeltaProduct row of the ablation table).  The page gives no placement for
 *   the gate; this oracle multiplies S by gamma_t once per token, before the
 *   first Householder step (the decay-first order of eq. (11)).  The output is
 *   read once per token after the last step: o_t = S^T q_t.
 *
 * Inputs are float32 arrays (bf16 inputs are passed exactly upcast); every
 * operation is done in double.  Layouts are row-major:
 *   q, k [B,T,H,dk]   v [B,T,H,dv]   alpha/beta [B,T,H,dk] or [B,T,H]
 *   S0, S_final [B,H,dk,dv]   o [B,T,H,dv]
 * DeltaProduct: k [B,T,H,nh,dk], v [B,T,H,nh,dv], beta [B,T,H,nh],
 * gamma [B,T,H].
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* x / sqrt(sum x^2 + eps), in double. */
static void l2_normalise(const float* x, int n, double eps, double* out) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
    double inv = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) out[i] = (double)x[i] * inv;
}

/* One (batch, head) pair of the FG^2-GDN recurrence, eq. (11). */
static void gdn_head(const float* q, const float* k, const float* v,
                     const float* alpha, const float* beta, const float* beta_v, const float* S0,
                     double* o, double* S_final,
                     int b, int h, int B, int H, int T, int dk, int dv,
                     int alpha_scalar, int beta_scalar, double eps) {
    (void)B;
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* X = (double*)malloc((size_t)dk * dv * sizeof(double));
    double* qh = (double*)malloc((size_t)dk * sizeof(double));
    double* kt = (double*)malloc((size_t)dk * sizeof(double));
    double* vt = (double*)malloc((size_t)dv * sizeof(double));
    double* e = (double*)malloc((size_t)dv * sizeof(double));
    if (S0) {
        const float* s0 = S0 + ((size_t)b * H + h) * dk * dv;
        for (size_t i = 0; i < (size_t)dk * dv; ++i) S[i] = (double)s0[i];
    }
    for (int t = 0; t < T; ++t) {
        size_t tok = ((size_t)b * T + t) * H + h;          /* token-head row */
        const float* qr = q + tok * dk;
        const float* kr = k + tok * dk;
        const float* vr = v + tok * dv;
        l2_normalise(qr, dk, eps, qh);
        l2_normalise(kr, dk, eps, kt);
        /* k~ = sqrt(beta) (.) k^ ; v~ = sqrt(beta) (.) v */
        for (int i = 0; i < dk; ++i) {
            double bi = beta_scalar ? (double)beta[tok] : (double)beta[tok * dk + i];
            kt[i] *= sqrt(bi);
        }
        for (int j = 0; j < dv; ++j) {
            double bj;
            if (beta_v) bj = beta_scalar ? (double)beta_v[tok] : (double)beta_v[tok * dv + j];
            else bj = beta_scalar ? (double)beta[tok] : (double)beta[tok * dk + j];
            vt[j] = (double)vr[j] * sqrt(bj);
        }
        /* X = Diag(alpha_t) S_{t-1} */
        for (int i = 0; i < dk; ++i) {
            double ai = alpha_scalar ? (double)alpha[tok] : (double)alpha[tok * dk + i];
            for (int j = 0; j < dv; ++j) X[(size_t)i * dv + j] = ai * S[(size_t)i * dv + j];
        }
        /* e = v~ - X^T k~ */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += X[(size_t)i * dv + j] * kt[i];
            e[j] = vt[j] - acc;
        }
        /* S_t = X + k~ e^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = X[(size_t)i * dv + j] + kt[i] * e[j];
        /* o_t = S_t^T q^ */
        double* orow = o + tok * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qh[i];
            orow[j] = acc;
        }
    }
    if (S_final) {
        double* sf = S_final + ((size_t)b * H + h) * dk * dv;
        memcpy(sf, S, (size_t)dk * dv * sizeof(double));
    }
    free(S); free(X); free(qh); free(kt); free(vt); free(e);
}

/* Whole tensor, or the (b,h) pairs listed in `pairs` (2*npairs ints) when
 * npairs > 0.  Rows of o / S_final for pairs not listed are left untouched. */
int oracle_gdn_seq(const float* q, const float* k, const float* v,
                   const float* alpha, const float* beta, const float* beta_v, const float* S0,
                   double* o, double* S_final,
                   int B, int H, int T, int dk, int dv,
                   int alpha_scalar, int beta_scalar, double eps,
                   const int* pairs, int npairs, int nthreads) {
    if (!beta_scalar && !beta_v && dk != dv) return 1;
    int n = npairs > 0 ? npairs : B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int p = 0; p < n; ++p) {
        int b = npairs > 0 ? pairs[2 * p] : p / H;
        int h = npairs > 0 ? pairs[2 * p + 1] : p % H;
        gdn_head(q, k, v, alpha, beta, beta_v, S0, o, S_final, b, h, B, H, T, dk, dv,
                 alpha_scalar, beta_scalar, eps);
    }
    return 0;
}

/* One (batch, head) pair of DeltaProduct n_h with the scalar forget gate. */
static void dp_head(const float* q, const float* k, const float* v,
                    const float* gamma, const float* beta, const float* S0,
                    double* o, double* S_final,
                    int b, int h, int H, int T, int nh, int dk, int dv, double eps) {
    double* S = (double*)calloc((size_t)dk * dv, sizeof(double));
    double* qh = (double*)malloc((size_t)dk * sizeof(double));
    double* kh = (double*)malloc((size_t)dk * sizeof(double));
    double* e = (double*)malloc((size_t)dv * sizeof(double));
    if (S0) {
        const float* s0 = S0 + ((size_t)b * H + h) * dk * dv;
        for (size_t i = 0; i < (size_t)dk * dv; ++i) S[i] = (double)s0[i];
    }
    for (int t = 0; t < T; ++t) {
        size_t tok = ((size_t)b * T + t) * H + h;
        double g = (double)gamma[tok];
        for (size_t i = 0; i < (size_t)dk * dv; ++i) S[i] *= g;
        for (int m = 0; m < nh; ++m) {
            size_t sub = tok * nh + m;
            l2_normalise(k + sub * dk, dk, eps, kh);
            double bm = (double)beta[sub];
            const float* vr = v + sub * dv;
            /* S <- S + beta k (v - S^T k)^T  ==  (I - beta k k^T) S + beta k v^T */
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * kh[i];
                e[j] = (double)vr[j] - acc;
            }
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += bm * kh[i] * e[j];
        }
        l2_normalise(q + tok * dk, dk, eps, qh);
        double* orow = o + tok * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * qh[i];
            orow[j] = acc;
        }
    }
    if (S_final) {
        double* sf = S_final + ((size_t)b * H + h) * dk * dv;
        memcpy(sf, S, (size_t)dk * dv * sizeof(double));
    }
    free(S); free(qh); free(kh); free(e);
}

int oracle_deltaproduct_seq(const float* q, const float* k, const float* v,
                            const float* gamma, const float* beta, const float* S0,
                            double* o, double* S_final,
                            int B, int H, int T, int nh, int dk, int dv, double eps,
                            const int* pairs, int npairs, int nthreads) {
    int n = npairs > 0 ? npairs : B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int p = 0; p < n; ++p) {
        int b = npairs > 0 ? pairs[2 * p] : p / H;
        int h = npairs > 0 ? pairs[2 * p + 1] : p % H;
        dp_head(q, k, v, gamma, beta, S0, o, S_final, b, h, H, T, nh, dk, dv, eps);
    }
    return 0;
}

/* Number of threads an OpenMP region of this library would use. */
int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * KDA oracle -- TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.
 *
 * A plain, slow, obviously-correct fp64 CPU restatement of Kimi Delta
 * Attention (KDA).  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline / reference arm may load it.  It shares no code, header, table or
 * helper with the CUDA library, and the CUDA library never calls it.
 *
 * Sources (page title, then section / equation):
 *  [RN]  "Kimi Linear: An Expressive, Efficient Attention Architecture"
 *        (research-notes page on arXiv 2510.26692), section Method,
 *        "From Linear Attention to KDA": the DeltaNet update, its residual
 *        form, the KDA recurrence S_t = (I - b_t k_t k_t^T) Diag(a_t) S_{t-1}
 *        + b_t k_t v_t^T with o_t = S_t^T q_t, and the implementation reading
 *        S~ = Diag(a_t) S_{t-1}, S_t = S~ + b_t k_t (v_t - S~^T k_t)^T.
 *  [RN-CV] same page, section "Code Verification": the naive recurrent KDA
 *        first multiplies the state by exp(g), then writes b k (v - k^T S).
 *  [RN-CA] same page, section "Chunkwise Algorithm": KDA as a constrained
 *        DPLR transition D = Diag(a), a = b k, b = k (.) a; the untied generic
 *        DPLR form is the comparison point.
 *
 * Conventions shared by every entry point here:
 *   token tensors are packed as [Ttot][H][D] (row-major, D fastest);
 *   sequences are the half-open token ranges [cu[n], cu[n+1]), n < N;
 *   states are [N][H][DK][DV] (row = key channel, column = value channel);
 *   g is the log of the per-channel decay (a = exp(g), g <= 0), beta is [Ttot][H];
 *   scale multiplies q (scale = 1 is the pages' o_t = S_t^T q_t).
 * s0 may be NULL (zero initial state); sT may be NULL (not wanted).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int kda_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Residual ("read, then write the error back") form of one KDA step,
 * [RN] / [RN-CV]:  S~ = Diag(exp(g)) S;  S = S~ + beta k (v - S~^T k)^T;
 * o = scale * S^T q.  y is a DV-long scratch vector. */
static void kda_step_residual(double *S, const double *q, const double *k,
                              const double *v, const double *g, double beta,
                              double scale, double *o, double *y, int DK, int DV)
{
    for (int i = 0; i < DK; ++i) {
        double a = exp(g[i]);
        double *row = S + (size_t)i * DV;
        for (int j = 0; j < DV; ++j) row[j] *= a;
    }
    for (int j = 0; j < DV; ++j) y[j] = 0.0;
    for (int i = 0; i < DK; ++i) {
        const double *row = S + (size_t)i * DV;
        for (int j = 0; j < DV; ++j) y[j] += row[j] * k[i];
    }
    for (int i = 0; i < DK; ++i) {
        double *row = S + (size_t)i * DV;
        double bk = beta * k[i];
        for (int j = 0; j < DV; ++j) row[j] += bk * (v[j] - y[j]);
    }
    if (o) {
        for (int j = 0; j < DV; ++j) {
            double acc = 0.0;
            for (int i = 0; i < DK; ++i) acc += S[(size_t)i * DV + j] * q[i];
            o[j] = scale * acc;
        }
    }
}

/* Product form of one step, [RN] eq. (KDA), for the general diagonal-plus-
 * low-rank transition of [RN-CA]:
 *   S = (I - a b^T) Diag(exp(g)) S + beta k v^T.
 * With a = beta k and b = k this is exactly the KDA step.  The transition
 * matrix M = (I - a b^T) Diag(exp(g)) is built explicitly (DK x DK) and
 * multiplied in, so this route shares no algebra with kda_step_residual. */
static void dplr_step_product(double *S, const double *q, const double *k,
                              const double *v, const double *g,
                              const double *a, const double *b, double beta,
                              double scale, double *o, double *M, double *tmp,
                              int DK, int DV)
{
    for (int r = 0; r < DK; ++r)
        for (int c = 0; c < DK; ++c)
            M[(size_t)r * DK + c] = ((r == c) ? 1.0 : 0.0) - a[r] * b[c];
    for (int r = 0; r < DK; ++r)
        for (int c = 0; c < DK; ++c)
            M[(size_t)r * DK + c] *= exp(g[c]);           /* right-multiply by Diag */
    for (int r = 0; r < DK; ++r)
        for (int j = 0; j < DV; ++j) {
            double acc = 0.0;
            for (int c = 0; c < DK; ++c) acc += M[(size_t)r * DK + c] * S[(size_t)c * DV + j];
            tmp[(size_t)r * DV + j] = acc + beta * k[r] * v[j];
        }
    memcpy(S, tmp, sizeof(double) * (size_t)DK * DV);
    if (o) {
        for (int j = 0; j < DV; ++j) {
            double acc = 0.0;
            for (int i = 0; i < DK; ++i) acc += S[(size_t)i * DV + j] * q[i];
            o[j] = scale * acc;
        }
    }
}

/* Token-by-token KDA over packed sequences, residual form.  Parallel over
 * (sequence, head) pairs, which the recurrence keeps independent. */
void kda_oracle_recurrent(const double *q, const double *k, const double *v,
                          const double *g, const double *beta,
                          const double *s0, double *o, double *sT,
                          const long long *cu, int N, int H, int DK, int DV,
                          double scale)
{
    const size_t SS = (size_t)DK * DV;
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
#endif
    for (int n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * SS);
            double *y = (double *)malloc(sizeof(double) * DV);
            if (s0) memcpy(S, s0 + ((size_t)n * H + h) * SS, sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (long long t = cu[n]; t < cu[n + 1]; ++t) {
                size_t th = (size_t)t * H + h;
                kda_step_residual(S, q + th * DK, k + th * DK, v + th * DV,
                                  g + th * DK, beta[th], scale,
                                  o ? o + th * DV : NULL, y, DK, DV);
            }
            if (sT) memcpy(sT + ((size_t)n * H + h) * SS, S, sizeof(double) * SS);
            free(S);
            free(y);
        }
    }
}

/* Token-by-token generic DPLR recurrence, product form:
 *   S_t = (I - a_t b_t^T) Diag(exp(g_t)) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = scale * S_t^T q_t.
 * a and b are [Ttot][H][DK].  KDA is the special case a = beta k, b = k. */
void kda_oracle_dplr_product(const double *q, const double *k, const double *v,
                             const double *g, const double *beta,
                             const double *a, const double *b,
                             const double *s0, double *o, double *sT,
                             const long long *cu, int N, int H, int DK, int DV,
                             double scale)
{
    const size_t SS = (size_t)DK * DV;
#ifdef _OPENMP
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
#endif
    for (int n = 0; n < N; ++n) {
        for (int h = 0; h < H; ++h) {
            double *S = (double *)malloc(sizeof(double) * SS);
            double *M = (double *)malloc(sizeof(double) * (size_t)DK * DK);
            double *tmp = (double *)malloc(sizeof(double) * SS);
            if (s0) memcpy(S, s0 + ((size_t)n * H + h) * SS, sizeof(double) * SS);
            else memset(S, 0, sizeof(double) * SS);
            for (long long t = cu[n]; t < cu[n + 1]; ++t) {
                size_t th = (size_t)t * H + h;
                dplr_step_product(S, q + th * DK, k + th * DK, v + th * DV,
                                  g + th * DK, a + th * DK, b + th * DK, beta[th],
                                  scale, o ? o + th * DV : NULL, M, tmp, DK, DV);
            }
            if (sT) memcpy(sT + ((size_t)n * H + h) * SS, S, sizeof(double) * SS);
            free(S);
            free(M);
            free(tmp);
        }
    }
}

/*
 * Float64 CPU oracle for causal kernelized linear attention.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the package smoke check and
 * the benchmark's CPU-baseline leg, never by the product path.
 *
 * Sources:
 *   "What Is Linear Attention?" (xutianle.me): §4 recurrence S_t, z_t, o_t;
 *       §5.1 gamma decay; §5.2 delta rule; §5.3 gate on the write.
 *   "Efficient attention variants" (bailixisu.com): §4 phi = ELU+1;
 *       §5 write-then-read causal recurrence; §7.1 RetNet decay;
 *       §7.4 gated delta rule alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T;
 *       §10 NumPy verification program (the loop order used here).
 *   "Transformers Are RNNs" notes (myhz0606.com): eps added to the denominator.
 *
 * Parity pins live in the test suite (hand example, dense masked form, closed
 * forms for the final state, decay and delta examples).
 */
#include "la_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ELU(x)+1 with alpha = 1 ("Efficient attention variants" §4 and §10). */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* One (b,h) chain of the kernelized recurrence.  a, b: scratch of length d. */
static void kernelized_chain(const double* q, const double* k, const double* v,
                             double gamma, const double* S0, const double* z0,
                             double* o, double* S, double* z,
                             int N, int d, int dv, double eps, int apply_phi,
                             double* a, double* b)
{
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)d * dv);
    else memset(S, 0, sizeof(double) * (size_t)d * dv);
    if (z0) memcpy(z, z0, sizeof(double) * (size_t)d);
    else memset(z, 0, sizeof(double) * (size_t)d);

    for (int t = 0; t < N; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        double* ot = o + (size_t)t * dv;
        for (int i = 0; i < d; ++i) {
            a[i] = apply_phi ? phi(qt[i]) : qt[i];
            b[i] = apply_phi ? phi(kt[i]) : kt[i];
        }
        /* write: S_t = gamma S_{t-1} + phi(k_t) v_t^T ; z_t = gamma z_{t-1} + phi(k_t) */
        for (int i = 0; i < d; ++i) {
            double* Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] = gamma * Si[j] + b[i] * vt[j];
            z[i] = gamma * z[i] + b[i];
        }
        /* read: o_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps) */
        double den = 0.0;
        for (int i = 0; i < d; ++i) den += a[i] * z[i];
        den += eps;
        for (int j = 0; j < dv; ++j) {
            double num = 0.0;
            for (int i = 0; i < d; ++i) num += a[i] * S[(size_t)i * dv + j];
            ot[j] = num / den;
        }
    }
}

void la_oracle_kernelized(const double* q, const double* k, const double* v,
                          const double* gamma, const double* S0, const double* z0,
                          double* o, double* S_out, double* z_out,
                          int B, int H, int N, int d, int dv,
                          double eps, int apply_phi)
{
    const int chains = B * H;
#pragma omp parallel
    {
        double* a = (double*)malloc(sizeof(double) * (size_t)d);
        double* b = (double*)malloc(sizeof(double) * (size_t)d);
        double* S = (double*)malloc(sizeof(double) * (size_t)d * dv);
        double* z = (double*)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < chains; ++c) {
            const int h = c % H;
            const size_t qo = (size_t)c * N * d, vo = (size_t)c * N * dv;
            const size_t so = (size_t)c * d * dv, zo = (size_t)c * d;
            kernelized_chain(q + qo, k + qo, v + vo, gamma ? gamma[h] : 1.0,
                             S0 ? S0 + so : NULL, z0 ? z0 + zo : NULL,
                             o + vo, S, z, N, d, dv, eps, apply_phi, a, b);
            if (S_out) memcpy(S_out + so, S, sizeof(double) * (size_t)d * dv);
            if (z_out) memcpy(z_out + zo, z, sizeof(double) * (size_t)d);
        }
        free(a); free(b); free(S); free(z);
    }
}

/* One (b,h) chain of the gated delta rule.  vhat: scratch of length dv. */
static void gated_delta_chain(const double* q, const double* k, const double* v,
                              const double* alpha, const double* g, const double* S0,
                              double* o, double* S, int N, int d, int dv, double* vhat)
{
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)d * dv);
    else memset(S, 0, sizeof(double) * (size_t)d * dv);

    for (int t = 0; t < N; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        double* ot = o + (size_t)t * dv;
        const double at = alpha[t], gt = g[t];
        /* old prediction read from the previous state: vhat = S_{t-1}^T k_t */
        for (int j = 0; j < dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += S[(size_t)i * dv + j] * kt[i];
            vhat[j] = s;
        }
        /* decay, then write the error measured on the decayed state:
         * S_t = alpha S_{t-1} + g k (v - alpha vhat)^T */
        for (int i = 0; i < d; ++i) {
            double* Si = S + (size_t)i * dv;
            for (int j = 0; j < dv; ++j) Si[j] = at * Si[j] + gt * kt[i] * (vt[j] - at * vhat[j]);
        }
        /* read: o_t = S_t^T q_t */
        for (int j = 0; j < dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += S[(size_t)i * dv + j] * qt[i];
            ot[j] = s;
        }
    }
}

void la_oracle_gated_delta(const double* q, const double* k, const double* v,
                           const double* alpha, const double* g, const double* S0,
                           double* o, double* S_out,
                           int B, int H, int N, int d, int dv)
{
    const int chains = B * H;
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)d * dv);
        double* vhat = (double*)malloc(sizeof(double) * (size_t)dv);
#pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < chains; ++c) {
            const size_t qo = (size_t)c * N * d, vo = (size_t)c * N * dv;
            const size_t so = (size_t)c * d * dv, ao = (size_t)c * N;
            gated_delta_chain(q + qo, k + qo, v + vo, alpha + ao, g + ao,
                              S0 ? S0 + so : NULL, o + vo, S, N, d, dv, vhat);
            if (S_out) memcpy(S_out + so, S, sizeof(double) * (size_t)d * dv);
        }
        free(S); free(vhat);
    }
}

/* GLA with a per-key-channel gate ("Efficient attention variants" §7.2): each
 * entry of alpha_t says how much of the matching row of the state (one key
 * channel) is kept, broadcast along the value dimension; then the usual write
 * and read.  No feature map, no normaliser (the §7 recurrences leave both out).
 *     S_t[i][:] = alpha_t[i] * S_{t-1}[i][:] + k_t[i] * v_t[:]
 *     o_t = S_t^T q_t
 * alpha [B,H,N,d]; S0 NULL means a zero start state. */
void la_oracle_gla(const double* q, const double* k, const double* v, const double* alpha,
                   const double* S0, double* o, double* S_out, int B, int H, int N, int d, int dv)
{
    const int chains = B * H;
#pragma omp parallel
    {
        double* S = (double*)malloc(sizeof(double) * (size_t)d * dv);
#pragma omp for schedule(dynamic, 1)
        for (int c = 0; c < chains; ++c) {
            const size_t qo = (size_t)c * N * d, vo = (size_t)c * N * dv, so = (size_t)c * d * dv;
            for (size_t e = 0; e < (size_t)d * dv; ++e) S[e] = S0 ? S0[so + e] : 0.0;
            for (int t = 0; t < N; ++t) {
                const double* qt = q + qo + (size_t)t * d;
                const double* kt = k + qo + (size_t)t * d;
                const double* at = alpha + qo + (size_t)t * d;
                const double* vt = v + vo + (size_t)t * dv;
                for (int i = 0; i < d; ++i) {
                    double* Si = S + (size_t)i * dv;
                    for (int j = 0; j < dv; ++j) Si[j] = at[i] * Si[j] + kt[i] * vt[j];
                }
                double* ot = o + vo + (size_t)t * dv;
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < d; ++i) acc += qt[i] * S[(size_t)i * dv + j];
                    ot[j] = acc;
                }
            }
            if (S_out) memcpy(S_out + so, S, sizeof(double) * (size_t)d * dv);
        }
        free(S);
    }
}

/* Short causal convolution ("What Is Linear Attention?" §5.4): a window of the
 * last w tokens, one filter per (head, channel), no activation.  With the
 * previous w-1 inputs of the chain as the window's history (cache; zero when
 * absent), xh = [cache; x] and
 *     y_t[c] = sum_{i=0}^{w-1} W[h][c][i] * xh[t + i][c]      (xh[t + w-1] = x_t)
 * and the new cache is the last w-1 rows of xh. */
void la_oracle_causal_conv(const double* x, const double* W, const double* cache,
                           double* y, double* cache_out, int B, int H, int N, int d, int w)
{
    const int chains = B * H, hist = w - 1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int ch = 0; ch < chains; ++ch) {
        const int h = ch % H;
        const double* xc = x + (size_t)ch * N * d;
        const double* cc = cache ? cache + (size_t)ch * hist * d : NULL;
        /* row r of the history-extended sequence, channel c */
#define XH(r, c) ((r) < hist ? (cc ? cc[(size_t)(r) * d + (c)] : 0.0) : xc[(size_t)((r) - hist) * d + (c)])
        for (int t = 0; t < N; ++t)
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int i = 0; i < w; ++i) acc += W[((size_t)h * d + c) * w + i] * XH(t + i, c);
                y[((size_t)ch * N + t) * d + c] = acc;
            }
        if (cache_out)
            for (int r = 0; r < hist; ++r)
                for (int c = 0; c < d; ++c)
                    cache_out[((size_t)ch * hist + r) * d + c] = XH(N + r, c);
#undef XH
    }
}

int la_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Float64 CPU oracle for causal kernelized linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This library exists to check the CUDA path; only
 * the test suite, the package smoke check and the benchmark's CPU-baseline
 * leg may load it.  It shares no code, header or constant with the CUDA path.
 *
 * Every function is the plain token-by-token recurrence, in float64, in the
 * order the pages write it; OpenMP runs independent (batch, head) chains on
 * separate threads and nothing else is reordered.
 *
 * Layouts (row-major, contiguous, float64):
 *   q, k [B,H,N,d]; v, o [B,H,N,dv]; S [B,H,d,dv] (rows = key feature,
 *   columns = value); z [B,H,d]; gamma [H]; alpha, g [B,H,N].
 */
#ifndef LA_ORACLE_H
#define LA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

/* Causal kernelized linear attention with normaliser and optional per-head
 * decay ("What Is Linear Attention?" §4 and §5.1; "Efficient attention
 * variants" §5 and §7.1):
 *     a = phi(q_t), b = phi(k_t)
 *     S_t = gamma_h S_{t-1} + b v_t^T,   z_t = gamma_h z_{t-1} + b
 *     o_t = (a^T S_t) / (a^T z_t + eps)
 * phi(x) = elu(x)+1 = (x > 0 ? x + 1 : exp(x)) when apply_phi != 0, else the
 * identity (the pages' hand example feeds features directly).
 * gamma: NULL means gamma = 1 for every head.  S0/z0: NULL means a zero start
 * state.  S_out/z_out receive the final state (may be NULL). */
void la_oracle_kernelized(const double* q, const double* k, const double* v,
                          const double* gamma, const double* S0, const double* z0,
                          double* o, double* S_out, double* z_out,
                          int B, int H, int N, int d, int dv,
                          double eps, int apply_phi);

/* Gated delta rule ("Efficient attention variants" §7.4; "What Is Linear
 * Attention?" §5.2-5.3):
 *     S_t = alpha_t S_{t-1} + g_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T
 *     o_t = S_t^T q_t
 * No feature map, no normaliser.  S0 NULL means a zero start state. */
void la_oracle_gated_delta(const double* q, const double* k, const double* v,
                           const double* alpha, const double* g, const double* S0,
                           double* o, double* S_out,
                           int B, int H, int N, int d, int dv);

/* GLA, per-key-channel gate ("Efficient attention variants" §7.2):
 *     S_t = diag(alpha_t) S_{t-1} + k_t v_t^T,  o_t = S_t^T q_t
 * alpha [B,H,N,d].  No feature map, no normaliser.  S0 NULL: zero start. */
void la_oracle_gla(const double* q, const double* k, const double* v, const double* alpha,
                   const double* S0, double* o, double* S_out, int B, int H, int N, int d, int dv);

/* Short causal convolution ("What Is Linear Attention?" §5.4): x [B,H,N,d],
 * W [H,d,w], cache [B,H,w-1,d] or NULL (zero history) -> y [B,H,N,d] and, if
 * cache_out is not NULL, the last w-1 inputs [B,H,w-1,d].  Weight i multiplies
 * the input w-1-i tokens back (the last weight the current token). */
void la_oracle_causal_conv(const double* x, const double* W, const double* cache,
                           double* y, double* cache_out, int B, int H, int N, int d, int w);

/* Number of OpenMP threads the oracle will use. */
int la_oracle_threads(void);

#ifdef __cplusplus
}
#endif
#endif

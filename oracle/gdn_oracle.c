/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness yardstick for the
 * CUDA library: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark may build, load or call it.  It shares no code, header,
 * table or helper with the CUDA path.
 *
 * What it computes is the plain definition, token by token, in fp64:
 *
 *   token-wise gated delta rule (SANA-WM summary, paper-graph-ui, section 3.2
 *   "Memory-Efficient Long-Context Modeling", paragraph "Frame-wise Gated
 *   DeltaNet (GDN)", the standard token-wise update; restated on the SANA-WM
 *   teardown, thesatyajit, section "The linear part: a gated delta rule, one
 *   frame per step"):
 *
 *       S_i = gamma_i S_{i-1} + (v_i - gamma_i S_{i-1} k_i) beta_i k_i^T
 *       o_i = S_i q_i
 *
 *   which is the same map as S_i = alpha_i S_{i-1} (I - beta_i k_i k_i^T)
 *   + beta_i v_i k_i^T with alpha = gamma.  S is d_v x d_k (S k ~ v), the
 *   output reads the state AFTER the token's own update.
 *
 *   frame-wise SANA-WM operator (same page and section, the frame-wise
 *   update equations for M_t, U_t, S_t and O_t):
 *
 *       M_t = gamma_t (I - K_t beta_t K_t^T),  U_t = V_t beta_t K_t^T
 *       S_t = S_{t-1} M_t + U_t,               O_t = S_t Q_t
 *
 * Layouts (row-major, contiguous): q,k [B,T,H,d_k]; v,o [B,T,H,d_v];
 * alpha,beta [B,T,H]; frame-wise gamma [B,F,H]; states [B,H,d_v,d_k].
 * The (b,h) chains are independent and are spread over OpenMP threads;
 * within a chain the loop over tokens is strictly sequential.
 */
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Returns the number of threads a parallel region would use. */
int gdn_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Token-wise recurrence for all (b,h) chains.
 *   reverse      : 0 walks t = 0..T-1, 1 walks t = T-1..0 (the reversed-time
 *                  scan of the bidirectional variant: same update, tokens
 *                  visited backwards, each gate applied at its own token).
 *   reset_every  : if > 0, the state is set to zero at the start of every
 *                  run of reset_every tokens except the first (chunk-causal
 *                  reversed scan: reset at chunk boundaries).
 *   S_in         : may be NULL (zero initial state).
 *   S_out        : may be NULL (final state not returned).
 *   nthreads     : <= 0 keeps the OpenMP default.
 * Returns 0, or -1 on a bad argument.
 */
int gdn_oracle_token(const double *q, const double *k, const double *v,
                     const double *alpha, const double *beta,
                     const double *S_in, double *S_out, double *o,
                     int B, int H, long long T, int d_k, int d_v,
                     int reverse, long long reset_every, int nthreads)
{
    if (!q || !k || !v || !alpha || !beta || !o) return -1;
    if (B < 0 || H < 0 || T < 0 || d_k <= 0 || d_v <= 0) return -1;
    const long long chains = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (long long c = 0; c < chains; ++c) {
        const int b = (int)(c / H), h = (int)(c % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)d_v * d_k);
        double *x = (double *)malloc(sizeof(double) * (size_t)d_v);
        if (S_in) memcpy(S, S_in + c * (long long)d_v * d_k, sizeof(double) * (size_t)d_v * d_k);
        else memset(S, 0, sizeof(double) * (size_t)d_v * d_k);

        for (long long n = 0; n < T; ++n) {
            const long long t = reverse ? (T - 1 - n) : n;
            if (reset_every > 0 && n > 0) {
                const int boundary = reverse ? ((t + 1) % reset_every == 0) : (t % reset_every == 0);
                if (boundary) memset(S, 0, sizeof(double) * (size_t)d_v * d_k);
            }
            const long long row = ((long long)b * T + t) * H + h;   /* token-head index */
            const double *kt = k + row * d_k, *qt = q + row * d_k, *vt = v + row * d_v;
            const double a = alpha[row], be = beta[row];
            /* x = S k_t : what the state currently returns for this key */
            for (int i = 0; i < d_v; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d_k; ++j) acc += S[(size_t)i * d_k + j] * kt[j];
                x[i] = acc;
            }
            /* S <- a (S - be x k^T) + be v k^T */
            for (int i = 0; i < d_v; ++i) {
                const double xi = be * x[i], vi = be * vt[i];
                for (int j = 0; j < d_k; ++j) {
                    double s = S[(size_t)i * d_k + j];
                    S[(size_t)i * d_k + j] = a * (s - xi * kt[j]) + vi * kt[j];
                }
            }
            /* o_t = S q_t, read from the updated state */
            double *ot = o + row * d_v;
            for (int i = 0; i < d_v; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d_k; ++j) acc += S[(size_t)i * d_k + j] * qt[j];
                ot[i] = acc;
            }
        }
        if (S_out) memcpy(S_out + c * (long long)d_v * d_k, S, sizeof(double) * (size_t)d_v * d_k);
        free(S);
        free(x);
    }
    return 0;
}

/*
 * Frame-wise SANA-WM operator: one rank-L update per frame of frame_len
 * tokens, every token of frame t reads the state after frame t's update.
 *   gamma : [B,F,H], the scalar decay of each frame (F = T / frame_len).
 *   beta  : [B,T,H], the per-token update gates (the diagonal of beta_t).
 * M_t and U_t are formed explicitly, as the equations write them.
 */
int gdn_oracle_framewise(const double *q, const double *k, const double *v,
                         const double *gamma, const double *beta,
                         const double *S_in, double *S_out, double *o,
                         int B, int H, long long T, int frame_len, int d_k, int d_v,
                         int nthreads)
{
    if (!q || !k || !v || !gamma || !beta || !o) return -1;
    if (B < 0 || H < 0 || T < 0 || frame_len <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (T % frame_len != 0) return -1;
    const long long F = T / frame_len;
    const long long chains = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (long long c = 0; c < chains; ++c) {
        const int b = (int)(c / H), h = (int)(c % H);
        double *S = (double *)malloc(sizeof(double) * (size_t)d_v * d_k);
        double *Sn = (double *)malloc(sizeof(double) * (size_t)d_v * d_k);
        double *M = (double *)malloc(sizeof(double) * (size_t)d_k * d_k);
        double *U = (double *)malloc(sizeof(double) * (size_t)d_v * d_k);
        if (S_in) memcpy(S, S_in + c * (long long)d_v * d_k, sizeof(double) * (size_t)d_v * d_k);
        else memset(S, 0, sizeof(double) * (size_t)d_v * d_k);

        for (long long f = 0; f < F; ++f) {
            const double g = gamma[((long long)b * F + f) * H + h];
            /* M = g (I - sum_s beta_s k_s k_s^T),  U = sum_s beta_s v_s k_s^T */
            for (int i = 0; i < d_k; ++i)
                for (int j = 0; j < d_k; ++j) M[(size_t)i * d_k + j] = (i == j) ? 1.0 : 0.0;
            memset(U, 0, sizeof(double) * (size_t)d_v * d_k);
            for (int s = 0; s < frame_len; ++s) {
                const long long row = ((long long)b * T + f * frame_len + s) * H + h;
                const double *ks = k + row * d_k, *vs = v + row * d_v;
                const double be = beta[row];
                for (int i = 0; i < d_k; ++i)
                    for (int j = 0; j < d_k; ++j) M[(size_t)i * d_k + j] -= be * ks[i] * ks[j];
                for (int i = 0; i < d_v; ++i)
                    for (int j = 0; j < d_k; ++j) U[(size_t)i * d_k + j] += be * vs[i] * ks[j];
            }
            for (size_t e = 0; e < (size_t)d_k * d_k; ++e) M[e] *= g;
            /* S <- S M + U */
            for (int i = 0; i < d_v; ++i)
                for (int j = 0; j < d_k; ++j) {
                    double acc = U[(size_t)i * d_k + j];
                    for (int m = 0; m < d_k; ++m) acc += S[(size_t)i * d_k + m] * M[(size_t)m * d_k + j];
                    Sn[(size_t)i * d_k + j] = acc;
                }
            memcpy(S, Sn, sizeof(double) * (size_t)d_v * d_k);
            /* O_t = S_t Q_t */
            for (int s = 0; s < frame_len; ++s) {
                const long long row = ((long long)b * T + f * frame_len + s) * H + h;
                const double *qs = q + row * d_k;
                double *os = o + row * d_v;
                for (int i = 0; i < d_v; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < d_k; ++j) acc += S[(size_t)i * d_k + j] * qs[j];
                    os[i] = acc;
                }
            }
        }
        if (S_out) memcpy(S_out + c * (long long)d_v * d_k, S, sizeof(double) * (size_t)d_v * d_k);
        free(S);
        free(Sn);
        free(M);
        free(U);
    }
    return 0;
}

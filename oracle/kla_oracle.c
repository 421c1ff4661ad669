/*
 * kla_oracle.c -- plain, slow, sequential fp64 CPU oracle for the per-channel
 * Kalman filter of Kalman Linear Attention (KLA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * What it computes (one independent scalar filter per channel):
 *
 *   dynamics      x_t = a_t x_{t-1} + w_t,   Var w_t = p_t
 *                 (scalar, diagonal case of the linear state-space model,
 *                  "Kalman filter" primer Part 1, section 2, eq. 2.1-2.2)
 *   predict       P-_t = a_t^2 P_{t-1} + p_t,    m-_t = a_t m_{t-1}
 *                 (the predict half of the predict-update cycle, primer
 *                  section 5.1 / Figure 5; the printed equations are missing
 *                  from the extracted page, so the textbook scalar form is used)
 *   update        lambda_t = 1/P-_t + phi_t,      eta_t = m-_t/P-_t + b_t
 *                 (information-form update of the KLA review, "Circularity
 *                  Check": prior precision plus token-evidence precision
 *                  phi_t = k_t^2 Lambda^v_t; the information mean adds the
 *                  token information b_t)
 *   emit          lambda_t, eta_t, mu_t = eta_t/lambda_t, var_t = 1/lambda_t
 *
 * The state before token 1 is the prior (lambda_0, eta_0): P_0 = 1/lambda_0,
 * m_0 = eta_0/lambda_0.  Output row t-1 holds the posterior after token t.
 *
 * This is the covariance form of the filter, written out step by step.  The
 * Moebius / affine-scan form that the CUDA path uses is an algebraic
 * rearrangement of it (KLA review, "What carries the argument"); the tests
 * pin this file against closed forms and exact rational arithmetic.
 *
 * Layout: a, p, phi, b, lambda, eta, mu, var are [B, T, H, N] row-major
 * (N fastest); lambda0, eta0 are [B, H, N].  All arrays are host fp64.
 * Compile with -ffp-contract=off so that every operation rounds once.
 */
#include <stdint.h>
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* One token of the filter for one channel: posterior (P, m) before the token,
 * inputs (a, p, phi, b), posterior (lambda, eta) after it. */
static void kf_token(double a, double p, double phi, double b,
                     double P_prev, double m_prev,
                     double *lam_out, double *eta_out)
{
    /* predict */
    const double P_pred = a * a * P_prev + p;
    const double m_pred = a * m_prev;
    /* update, information form */
    *lam_out = 1.0 / P_pred + phi;
    *eta_out = m_pred / P_pred + b;
}

/* Sequential filter over T tokens of one channel.  `stride` is the distance
 * in elements between consecutive tokens of the channel. */
static void kf_channel(const double *a, const double *p, const double *phi,
                       const double *b, int64_t T, int64_t stride,
                       double lam0, double eta0,
                       double *lam, double *eta, double *mu, double *var)
{
    double P = 1.0 / lam0;
    double m = eta0 / lam0;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t i = t * stride;
        double lam_t, eta_t;
        kf_token(a[i], p[i], phi[i], b[i], P, m, &lam_t, &eta_t);
        lam[i] = lam_t;
        eta[i] = eta_t;
        mu[i] = eta_t / lam_t;
        var[i] = 1.0 / lam_t;
        P = 1.0 / lam_t;
        m = eta_t / lam_t;
    }
}

/* Whole-sequence filter for B*H*N channels.  Returns 0 on success, -1 on a
 * bad argument.  `nthreads` <= 0 means one thread; channels are independent,
 * so threads split channels and never the time axis. */
int kla_oracle_forward(const double *a, const double *p, const double *phi,
                       const double *b, const double *lam0, const double *eta0,
                       double *lam, double *eta, double *mu, double *var,
                       int64_t B, int64_t T, int64_t H, int64_t N, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || N < 0) return -1;
    const int64_t HN = H * N;
    const int64_t C = B * HN;
    if (C == 0 || T == 0) return 0;
    if (!a || !p || !phi || !b || !lam0 || !eta0 || !lam || !eta || !mu || !var)
        return -1;
    if (nthreads <= 0) nthreads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (int64_t ch = 0; ch < C; ++ch) {
        const int64_t bi = ch / HN;
        const int64_t hn = ch % HN;
        const int64_t base = bi * T * HN + hn;
        kf_channel(a + base, p + base, phi + base, b + base, T, HN,
                   lam0[ch], eta0[ch],
                   lam + base, eta + base, mu + base, var + base);
    }
    return 0;
}

/* One token for C channels (recurrent decode).  The state (lambda, eta) is
 * read and overwritten in place; mu and var receive the token's outputs. */
int kla_oracle_step(const double *a, const double *p, const double *phi,
                    const double *b, double *lam_state, double *eta_state,
                    double *mu, double *var, int64_t C)
{
    if (C < 0) return -1;
    if (C == 0) return 0;
    if (!a || !p || !phi || !b || !lam_state || !eta_state || !mu || !var)
        return -1;
    for (int64_t ch = 0; ch < C; ++ch) {
        const double P = 1.0 / lam_state[ch];
        const double m = eta_state[ch] / lam_state[ch];
        double lam_t, eta_t;
        kf_token(a[ch], p[ch], phi[ch], b[ch], P, m, &lam_t, &eta_t);
        lam_state[ch] = lam_t;
        eta_state[ch] = eta_t;
        mu[ch] = eta_t / lam_t;
        var[ch] = 1.0 / lam_t;
    }
    return 0;
}

/* Number of threads an OpenMP region may use here (1 without OpenMP). */
int kla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

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
#include <stdlib.h>
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

/*
 * Gradients (reverse mode) of the whole-sequence filter above.
 *
 * Given the gradients of a scalar loss with respect to every output
 * (g_lambda, g_eta, g_mu, g_var, each [B, T, H, N]; a NULL array means a zero
 * gradient), return the gradients with respect to every input: a, p, phi, b
 * ([B, T, H, N]) and the prior lambda0, eta0 ([B, H, N]).  The KLA review
 * claims end-to-end training of the layer ("parallel training" of the filter)
 * without giving the backward pass; this is the chain rule taken through the
 * covariance-form steps of kf_token / kf_channel, one token at a time in
 * reverse, nothing else:
 *
 *   state entering token t:  P (variance), m (mean)
 *   P- = a^2 P + p,  m- = a m,  lambda = 1/P- + phi,  eta = m-/P- + b,
 *   mu = eta/lambda,  var = 1/lambda,  and the state leaving the token is
 *   P' = 1/lambda, m' = eta/lambda (the same expressions as var and mu).
 *
 * Walking back, (gP', gm') is the gradient flowing into the state that leaves
 * token t from every later token (zero after the last one).  The prior enters
 * as P = 1/lambda0, m = eta0/lambda0.  The forward pass is recomputed for each
 * channel (the states entering every token are kept in a scratch array).
 * Returns 0 on success, -1 on a bad argument, -2 when scratch memory cannot be
 * allocated.
 */
static void kf_channel_backward(const double *a, const double *p, const double *phi,
                                const double *b, int64_t T, int64_t stride,
                                double lam0, double eta0,
                                const double *g_lam, const double *g_eta,
                                const double *g_mu, const double *g_var,
                                double *ga, double *gp, double *gphi, double *gb,
                                double *g_lam0, double *g_eta0,
                                double *P_in, double *m_in)
{
    /* forward: the state entering each token */
    double P = 1.0 / lam0, m = eta0 / lam0;
    for (int64_t t = 0; t < T; ++t) {
        const int64_t k = t * stride;
        P_in[t] = P;
        m_in[t] = m;
        double lam_t, eta_t;
        kf_token(a[k], p[k], phi[k], b[k], P, m, &lam_t, &eta_t);
        const double P_out = 1.0 / lam_t, m_out = eta_t / lam_t;
        P = P_out;
        m = m_out;
    }
    /* reverse */
    double gP_next = 0.0, gm_next = 0.0;
    for (int64_t t = T - 1; t >= 0; --t) {
        const int64_t i = t * stride;
        const double at = a[i], pt = p[i];
        const double P_prev = P_in[t], m_prev = m_in[t];
        /* recompute the token */
        const double P_pred = at * at * P_prev + pt;
        const double m_pred = at * m_prev;
        const double lam = 1.0 / P_pred + phi[i];
        const double eta = m_pred / P_pred + b[i];
        /* gradients reaching var (= P') and mu (= m') */
        const double g_v = (g_var ? g_var[i] : 0.0) + gP_next;
        const double g_m = (g_mu ? g_mu[i] : 0.0) + gm_next;
        /* mu = eta / lambda, var = 1 / lambda */
        const double g_l = (g_lam ? g_lam[i] : 0.0)
                           - g_v / (lam * lam) - g_m * eta / (lam * lam);
        const double g_e = (g_eta ? g_eta[i] : 0.0) + g_m / lam;
        /* lambda = 1/P- + phi, eta = m-/P- + b */
        gphi[i] = g_l;
        gb[i] = g_e;
        const double g_Pp = -g_l / (P_pred * P_pred) - g_e * m_pred / (P_pred * P_pred);
        const double g_mp = g_e / P_pred;
        /* P- = a^2 P + p, m- = a m */
        ga[i] = g_Pp * 2.0 * at * P_prev + g_mp * m_prev;
        gp[i] = g_Pp;
        gP_next = g_Pp * at * at;
        gm_next = g_mp * at;
    }
    /* P = 1/lambda0, m = eta0/lambda0 */
    *g_lam0 = -gP_next / (lam0 * lam0) - gm_next * eta0 / (lam0 * lam0);
    *g_eta0 = gm_next / lam0;
}

int kla_oracle_backward(const double *a, const double *p, const double *phi,
                        const double *b, const double *lam0, const double *eta0,
                        const double *g_lam, const double *g_eta,
                        const double *g_mu, const double *g_var,
                        double *ga, double *gp, double *gphi, double *gb,
                        double *g_lam0, double *g_eta0,
                        int64_t B, int64_t T, int64_t H, int64_t N, int nthreads)
{
    if (B < 0 || T < 0 || H < 0 || N < 0) return -1;
    const int64_t HN = H * N;
    const int64_t C = B * HN;
    if (C == 0) return 0;
    if (!lam0 || !eta0 || !g_lam0 || !g_eta0) return -1;
    if (T > 0 && (!a || !p || !phi || !b || !ga || !gp || !gphi || !gb)) return -1;
    if (nthreads <= 0) nthreads = 1;
    int failed = 0;
#ifdef _OPENMP
#pragma omp parallel num_threads(nthreads)
#endif
    {
        double *scratch = (double *)malloc(sizeof(double) * (size_t)(2 * (T > 0 ? T : 1)));
        if (!scratch) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            failed = 1;
        }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t ch = 0; ch < C; ++ch) {
            if (!scratch) continue;
            const int64_t bi = ch / HN;
            const int64_t hn = ch % HN;
            const int64_t base = (bi * T) * HN + hn;  /* token 0 of the channel */
            const double prior_lam = lam0[ch], prior_eta = eta0[ch];
            kf_channel_backward(a + base, p + base, phi + base, b + base, T, HN,
                                prior_lam, prior_eta,
                                g_lam ? g_lam + base : NULL, g_eta ? g_eta + base : NULL,
                                g_mu ? g_mu + base : NULL, g_var ? g_var + base : NULL,
                                ga + base, gp + base, gphi + base, gb + base,
                                g_lam0 + ch, g_eta0 + ch, scratch, scratch + (T > 0 ? T : 1));
        }
        free(scratch);
    }
    return failed ? -2 : 0;
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

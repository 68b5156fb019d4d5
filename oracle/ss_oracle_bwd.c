/*
 * Selective-scan backward: plain fp64 CPU oracle of the gradients.
 *
 * TEST INFRASTRUCTURE ONLY, like ss_oracle.c: only the test suite and the
 * benchmark's CPU legs load it; it shares no code with the CUDA library.
 *
 * The forward it differentiates is the one of ss_oracle.c (the
 * selective_scan_ref walkthrough, "Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑
 * （附避坑指南）", §2.2-§3.3, state starting at zero):
 *   x_l = delta_l + bias,  d_l = softplus(x_l) (or exp(x_l)),
 *   a_ln = exp(d_l A_n),   h_ln = a_ln h_(l-1)n + d_l B_nl u_l,
 *   s_l = sum_n C_nl h_ln + D u_l,   y_l = s_l silu(z_l)  (y_l = s_l without z).
 * The walkthrough trains it through autograd (§6 mentions the gradient only
 * in passing); the gradients here are the chain rule of that loop, written
 * out.  With g_l = dL/ds_l = dy_l silu(z_l) and the adjoint state
 *   lam_ln = dL/dh_ln = g_l C_nl + a_(l+1)n lam_(l+1)n   (lam past the end = 0),
 * per row (b, d):
 *   dz_l     = dy_l s_l silu'(z_l),  silu'(z) = sig(z) (1 + z (1 - sig(z)))
 *   dD      += g_l u_l
 *   dC_nl   += g_l h_ln                         (summed over the rows d of batch b)
 *   dB_nl   += lam_ln d_l u_l                   (summed over d)
 *   du_l     = g_l D + sum_n lam_ln d_l B_nl
 *   dd_l     = sum_n lam_ln (B_nl u_l + h_(l-1)n a_ln A_n)
 *   dA_n    += sum_l lam_ln h_(l-1)n a_ln d_l   (summed over b and l)
 *   ddelta_l = dd_l softplus'(x_l) = dd_l sig(x_l)  (1 above torch's threshold 20;
 *              dd_l d_l in exp mode),   dbias += ddelta_l (summed over b and l).
 * Sums over rows are done in a fixed order, so results do not depend on the
 * thread count.
 * With sequence starts (the reset mask of ss_oracle.c: the state entering a
 * start is zero), h_(l-1) has no part in h_l at a start l, so there the
 * h_(l-1) terms of dd_l and dA vanish and no adjoint passes from l to l-1.
 * With a given state h0 before step 0 (the initial state of ss_oracle.c),
 * h_(-1) = h0 in the loop above and its gradient is the adjoint carried past
 * step 0:  dh0_n = a_0n lam_0n  (0 when a sequence starts at step 0).
 * With a gradient dlast of the loss with respect to the last state h_(L-1)
 * (the loss is then sum(dy * y) + sum(dlast * h_(L-1)), as when the last
 * state feeds the next piece of a sequence), the adjoint past the end is
 * dlast instead of zero: lam_(L-1)n = g_(L-1) C_n,L-1 + dlast_n.
 *
 * Optionally, for every gradient that is a sum over rows or steps (dA, dB,
 * dC, dD, ddelta_bias), the sum of the absolute values of its terms.  The
 * state and the adjoint in a term are themselves sums built by their
 * recursions, whose terms can cancel; a finite-precision value of either
 * carries an error of the order of the sum of the absolute values of its own
 * terms.  So each term is taken with h and lam replaced by those magnitudes,
 *   hm_ln = |a_ln| hm_(l-1)n + |d_l B_nl u_l|,   lam_m_ln = |g_l C_nl| + |a_(l+1)n| lam_m_(l+1)n
 * (hm before step 0 = |h0|, lam_m past the end = |dlast|, both cut at a
 * sequence start like h and lam), and the other factors with |.|; a step's
 * ddelta term with the magnitudes of its terms over the states.  These scale
 * the tolerance of a finite-precision sum per element; they are not
 * gradients, and the gradients above do not depend on them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* Returns 0 on success, -1 on a bad argument or allocation failure.
 * Required: u, delta, A, B, C, dy, du, ddelta, dA, dB, dC.  dD is required
 * when D is given, dz when z is, ddelta_bias when delta_bias is, dh0 when h0
 * is.  h0 (batch, dim, N): the state before step 0 (NULL: zero).  dlast
 * (batch, dim, N): the gradient with respect to the last state (NULL: zero).
 * mA, mB, mC, mD, mbias: NULL, or the sums of |terms| of dA, dB, dC, dD,
 * ddelta_bias (shapes of those). */
int ss_oracle_bwd_full(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                       const double *u, const double *delta, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *z, const double *delta_bias, int delta_softplus,
                       const uint8_t *reset, const double *h0, const double *dlast,
                       const double *dy, double *du,
                       double *ddelta, double *dA, double *dB, double *dC, double *dD,
                       double *dz, double *ddelta_bias, double *dh0, double *mA, double *mB,
                       double *mC, double *mD, double *mbias, int nthreads)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1)
        return -1;
    if (!A || !dA || (batch * dim > 0 && seqlen > 0 &&
                      (!u || !delta || !B || !C || !dy || !du || !ddelta || !dB || !dC)))
        return -1;
    if ((D && !dD) || (z && !dz) || (delta_bias && !ddelta_bias) || (h0 && !dh0))
        return -1;
    const int64_t N = dstate, L = seqlen;
    /* per-row partial sums over l, reduced over b afterwards in order */
    double *pA = calloc((size_t)(batch * dim * N + 1), sizeof(double));
    double *pD = calloc((size_t)(batch * dim + 1), sizeof(double));
    double *pbias = calloc((size_t)(batch * dim + 1), sizeof(double));
    double *qA = calloc((size_t)(batch * dim * N + 1), sizeof(double)); /* the same, of |terms| */
    double *qD = calloc((size_t)(batch * dim + 1), sizeof(double));
    double *qbias = calloc((size_t)(batch * dim + 1), sizeof(double));
    if (!pA || !pD || !pbias || !qA || !qD || !qbias) {
        free(pA), free(pD), free(pbias), free(qA), free(qD), free(qbias);
        return -1;
    }
    if (batch > 0 && L > 0) {
        memset(dB, 0, sizeof(double) * (size_t)(batch * N * L));
        memset(dC, 0, sizeof(double) * (size_t)(batch * N * L));
        if (mB)
            memset(mB, 0, sizeof(double) * (size_t)(batch * N * L));
        if (mC)
            memset(mC, 0, sizeof(double) * (size_t)(batch * N * L));
    }
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
#endif
    for (int64_t b = 0; b < batch; ++b) {
        double *h = malloc(sizeof(double) * (size_t)((L + 1) * N)); /* h[(l+1)N + n]: after step l */
        double *dl = malloc(sizeof(double) * (size_t)(L + 1));
        double *xs = malloc(sizeof(double) * (size_t)(L + 1));
        double *s = malloc(sizeof(double) * (size_t)(L + 1));
        double *carry = malloc(sizeof(double) * (size_t)N);
        double *hm = malloc(sizeof(double) * (size_t)((L + 1) * N)); /* magnitudes of h */
        double *cm = malloc(sizeof(double) * (size_t)N);              /* magnitudes of carry */
        if (!h || !dl || !xs || !s || !carry || !hm || !cm) {
            bad |= 1;
            free(h), free(dl), free(xs), free(s), free(carry), free(hm), free(cm);
            continue;
        }
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            /* forward, keeping every state (h[0..N-1]: the state before step 0) */
            for (int64_t n = 0; n < N; ++n) {
                h[n] = h0 ? h0[row * N + n] : 0.0;
                hm[n] = fabs(h[n]);
            }
            for (int64_t l = 0; l < L; ++l) {
                const int64_t idx = row * L + l;
                const int keep = !(reset && reset[b * L + l]); /* 0 at a sequence start */
                double x = delta[idx];
                if (delta_bias)
                    x += delta_bias[d];
                xs[l] = x;
                dl[l] = delta_softplus ? (x > 20.0 ? x : log1p(exp(x))) : exp(x);
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const int64_t bn = (b * N + n) * L + l;
                    const double a = exp(dl[l] * A[d * N + n]);
                    h[(l + 1) * N + n] = a * (keep ? h[l * N + n] : 0.0) + dl[l] * B[bn] * u[idx];
                    hm[(l + 1) * N + n] = fabs(a) * (keep ? hm[l * N + n] : 0.0) + fabs(dl[l] * B[bn] * u[idx]);
                    acc += C[bn] * h[(l + 1) * N + n];
                }
                if (D)
                    acc += D[d] * u[idx];
                s[l] = acc;
            }
            /* reverse sweep with the adjoint state */
            for (int64_t n = 0; n < N; ++n) { /* a_(l+1) lam_(l+1); past the end: dlast */
                carry[n] = dlast ? dlast[row * N + n] : 0.0;
                cm[n] = fabs(carry[n]);
            }
            for (int64_t l = L - 1; l >= 0; --l) {
                const int64_t idx = row * L + l;
                const int keep = !(reset && reset[b * L + l]);
                double g = dy[idx];
                if (z) {
                    const double sg = sigmoid(z[idx]);
                    dz[idx] = dy[idx] * s[l] * sg * (1.0 + z[idx] * (1.0 - sg));
                    g = dy[idx] * z[idx] * sg;
                }
                double dui = D ? g * D[d] : 0.0;
                if (D)
                    pD[row] += g * u[idx], qD[row] += fabs(g * u[idx]);
                double ddl = 0.0, ddl_m = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const int64_t bn = (b * N + n) * L + l;
                    const double a = exp(dl[l] * A[d * N + n]);
                    const double lam = g * C[bn] + carry[n];
                    const double lam_m = fabs(g * C[bn]) + cm[n];
                    dC[bn] += g * h[(l + 1) * N + n];
                    dB[bn] += lam * dl[l] * u[idx];
                    if (mC)
                        mC[bn] += fabs(g) * hm[(l + 1) * N + n];
                    if (mB)
                        mB[bn] += lam_m * fabs(dl[l] * u[idx]);
                    dui += lam * dl[l] * B[bn];
                    const double da = keep ? lam * h[l * N + n] : 0.0;
                    const double da_m = keep ? lam_m * hm[l * N + n] : 0.0;
                    ddl += lam * B[bn] * u[idx] + da * a * A[d * N + n];
                    ddl_m += lam_m * fabs(B[bn] * u[idx]) + da_m * fabs(a * A[d * N + n]);
                    pA[row * N + n] += da * a * dl[l];
                    qA[row * N + n] += da_m * fabs(a * dl[l]);
                    carry[n] = keep ? a * lam : 0.0;
                    cm[n] = keep ? fabs(a) * lam_m : 0.0;
                }
                du[idx] = dui;
                const double dx = delta_softplus ? ddl * (xs[l] > 20.0 ? 1.0 : sigmoid(xs[l]))
                                                 : ddl * dl[l];
                const double fx = delta_softplus ? (xs[l] > 20.0 ? 1.0 : sigmoid(xs[l])) : dl[l];
                ddelta[idx] = dx;
                pbias[row] += dx;
                qbias[row] += ddl_m * fabs(fx);
            }
            if (h0) /* the adjoint passed on past step 0 (zero after a start at step 0) */
                for (int64_t n = 0; n < N; ++n)
                    dh0[row * N + n] = L > 0 ? carry[n] : (dlast ? dlast[row * N + n] : 0.0);
        }
        free(h), free(dl), free(xs), free(s), free(carry), free(hm), free(cm);
    }
    for (int64_t d = 0; d < dim; ++d) {
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t b = 0; b < batch; ++b)
                acc += pA[(b * dim + d) * N + n], mag += qA[(b * dim + d) * N + n];
            dA[d * N + n] = acc;
            if (mA)
                mA[d * N + n] = mag;
        }
        double accD = 0.0, accb = 0.0, magD = 0.0, magb = 0.0;
        for (int64_t b = 0; b < batch; ++b) {
            accD += pD[b * dim + d], accb += pbias[b * dim + d];
            magD += qD[b * dim + d], magb += qbias[b * dim + d];
        }
        if (D)
            dD[d] = accD;
        if (delta_bias)
            ddelta_bias[d] = accb;
        if (D && mD)
            mD[d] = magD;
        if (delta_bias && mbias)
            mbias[d] = magb;
    }
    free(pA), free(pD), free(pbias), free(qA), free(qD), free(qbias);
    return bad ? -1 : 0;
}

/* With sequence starts, from a zero state, no |terms| sums. */
int ss_oracle_bwd_reset(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                        const double *u, const double *delta, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *z, const double *delta_bias, int delta_softplus,
                        const uint8_t *reset, const double *dy, double *du, double *ddelta,
                        double *dA, double *dB, double *dC, double *dD, double *dz,
                        double *ddelta_bias, int nthreads)
{
    return ss_oracle_bwd_full(batch, dim, seqlen, dstate, u, delta, A, B, C, D, z, delta_bias,
                              delta_softplus, reset, NULL, NULL, dy, du, ddelta, dA, dB, dC, dD, dz,
                              ddelta_bias, NULL, NULL, NULL, NULL, NULL, NULL, nthreads);
}

/* The walkthrough's form: no sequence starts. */
int ss_oracle_bwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                  const double *u, const double *delta, const double *A,
                  const double *B, const double *C, const double *D,
                  const double *z, const double *delta_bias, int delta_softplus,
                  const double *dy, double *du, double *ddelta, double *dA,
                  double *dB, double *dC, double *dD, double *dz,
                  double *ddelta_bias, int nthreads)
{
    return ss_oracle_bwd_reset(batch, dim, seqlen, dstate, u, delta, A, B, C, D, z, delta_bias,
                               delta_softplus, NULL, dy, du, ddelta, dA, dB, dC, dD, dz,
                               ddelta_bias, nthreads);
}

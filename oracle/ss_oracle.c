/*
 * Selective-scan forward: plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  The product path never calls this code; only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no source, header or helper with the CUDA library.
 *
 * What it computes follows the selective_scan_ref walkthrough
 * ("Mamba代码实战：手把手教你用PyTorch复现选择性扫描核心逻辑（附避坑指南）"):
 *   - §2.2 (delta的预处理): delta' = softplus(delta + bias) or exp(delta + bias),
 *     softplus taken as torch's default (beta 1, linear above 20);
 *   - §3.1 (参数离散化): dA = exp(delta' * A[d,n]), dB = delta' * B[b,n,l];
 *   - §3.2 (状态更新计算): the sequential loop over l with the state starting
 *     at zero, state = dA * state + dB * u, and y = sum over n of state * C;
 *     C is indexed C[b,n,l], the reading that agrees with the mamba-minimal
 *     page ("Mamba-minimal项目解析", 关键技术点 §1 选择性扫描算法);
 *   - §3.3 (加入跳跃连接): y += D[d] * u, then y *= silu(z) when z is given;
 *   - §6 (完整实现与测试): the optional last state is the state after step L.
 * Extension (no counterpart in the walkthrough, whose state always starts at
 * zero): an optional initial state replaces that zero, so that a sequence can
 * be run in pieces, each piece starting from the last state of the one before
 * (the streaming and single-step use of the recurrence that "告别‘炼丹’：从
 * Mamba-minimal入手..." describes in §2.1).
 * Extension: an optional (batch, seqlen) byte mask of sequence starts.  A
 * nonzero reset[b][l] sets the state of every row of batch entry b to zero
 * before step l, so that sequences laid end to end in one row do not leak
 * into one another: the boundary reset that "Mamba实战：如何用选择性状态空间
 * 模型提升你的长序列处理效率（附代码）" lists in §2 (and its periodic reset of
 * very long sequences in §5).  The pages give no interface for it; a reset at
 * step 0 overrides the initial state.
 * The "parallel" body printed in §4.2 / §6 (cumprod then cumsum) is NOT what
 * this follows: it disagrees with the §3.2 loop, which is the definition.
 *
 * Layouts (row-major, last index contiguous):
 *   u, delta, z, y : (batch, dim, seqlen)
 *   A              : (dim, dstate)
 *   B, C           : (batch, dstate, seqlen)
 *   D, delta_bias  : (dim)
 *   last_state, initial_state : (batch, dim, dstate)
 * D, z, delta_bias, last_state and initial_state may be NULL (absent).
 *
 * Rows (b, d) are independent; the only parallelism here is an OpenMP loop
 * over rows, each row running the plain sequential loop above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* torch.nn.functional.softplus with its defaults: beta = 1, threshold = 20. */
static double softplus_default(double x)
{
    if (x > 20.0)
        return x;
    return log1p(exp(x));
}

/* silu(z) = z * sigmoid(z) = z / (1 + exp(-z)). */
static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

int ss_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Returns 0 on success, -1 on a bad argument. nthreads <= 0 means "all". */
int ss_oracle_fwd_reset(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                        const double *u, const double *delta, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *z, const double *delta_bias, int delta_softplus,
                        const uint8_t *reset, const double *initial_state, double *y,
                        double *last_state, int nthreads)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1)
        return -1;
    if (batch * dim > 0 && (!u || !delta || !A || !B || !C || !y))
        return -1;
    const int64_t rows = batch * dim;
    int ok = 0;

#ifdef _OPENMP
    if (nthreads <= 0)
        nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : ok)
#endif
    for (int64_t row = 0; row < rows; ++row) {
        const int64_t b = row / dim;
        const int64_t d = row % dim;
        double *h = (double *)malloc((size_t)dstate * sizeof(double));
        if (!h) {
            ok |= 1;
            continue;
        }
        for (int64_t n = 0; n < dstate; ++n) /* zero (§3.2) unless an initial state is given */
            h[n] = initial_state ? initial_state[row * dstate + n] : 0.0;

        for (int64_t l = 0; l < seqlen; ++l) {
            const int64_t idx = row * seqlen + l;
            if (reset && reset[b * seqlen + l]) /* a sequence starts at l: no carried state */
                for (int64_t n = 0; n < dstate; ++n)
                    h[n] = 0.0;
            /* §2.2: add the per-channel bias, then make delta positive. */
            double x = delta[idx];
            if (delta_bias)
                x += delta_bias[d];
            const double dl = delta_softplus ? softplus_default(x) : exp(x);
            const double ul = u[idx];

            double yv = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                const int64_t bn = (b * dstate + n) * seqlen + l;
                const double dA = exp(dl * A[d * dstate + n]); /* §3.1 */
                const double dB = dl * B[bn];                    /* §3.1 */
                h[n] = dA * h[n] + dB * ul;                      /* §3.2 */
                yv += h[n] * C[bn];                              /* §3.2 */
            }
            if (D)
                yv += ul * D[d]; /* §3.3 skip connection */
            if (z)
                yv *= silu(z[idx]); /* §3.3 gate */
            y[idx] = yv;
        }
        if (last_state)
            for (int64_t n = 0; n < dstate; ++n)
                last_state[row * dstate + n] = h[n]; /* §6 */
        free(h);
    }
    return ok ? -1 : 0;
}

int ss_oracle_fwd_init(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                       const double *u, const double *delta, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *z, const double *delta_bias, int delta_softplus,
                       const double *initial_state, double *y, double *last_state,
                       int nthreads)
{
    return ss_oracle_fwd_reset(batch, dim, seqlen, dstate, u, delta, A, B, C, D, z, delta_bias,
                               delta_softplus, NULL, initial_state, y, last_state, nthreads);
}

/* The walkthrough's form: the state starts at zero. */
int ss_oracle_fwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                  const double *u, const double *delta, const double *A,
                  const double *B, const double *C, const double *D,
                  const double *z, const double *delta_bias, int delta_softplus,
                  double *y, double *last_state, int nthreads)
{
    return ss_oracle_fwd_init(batch, dim, seqlen, dstate, u, delta, A, B, C, D, z, delta_bias,
                              delta_softplus, NULL, y, last_state, nthreads);
}

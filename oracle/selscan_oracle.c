/*
 * selscan_oracle.c -- fp64 CPU oracle for the selective scan (S6) and its
 * scalar-A (Mamba-2 / SSD) form.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only tests/, the smoke() entry of
 * __graft_entry__.py and the CPU-baseline leg of bench.py load this library.
 * It shares no code, header, table or helper with the CUDA path
 * (selective_state_space_selscan_b200/csrc); neither side includes the other.
 *
 * Every routine is a plain, single-threaded loop in double precision that
 * follows the equations in the order the pages state them:
 *
 *   "03 -- Modelos de espacio de estados: RWKV, S4, Mamba y el selective scan"
 *     section "El mecanismo selectivo de Mamba": B, C and the step size Delta
 *       depend on the input token; A stays a fixed (diagonal) matrix.
 *     section "Discretizacion": the continuous system h' = A h + B x is
 *       discretised by zero-order hold; with diagonal A, exp(Delta A) is an
 *       elementwise exponential.
 *     section "Parallel scan": the discrete recurrence
 *       h_t = Abar_t h_{t-1} + Bbar_t x_t is associative (O(log T) depth).
 *     section "Coste de inferencia": one decode step costs O(N d) and keeps
 *       a state of fixed size.
 *   "P20 -- Mamba", section 5 "Matematica minima": selective SSM
 *       h_t = A(x_t) h_{t-1} + B(x_t) x_t, y_t = C(x_t) h_t.
 *   "Mamba-2 y state-space models", section 4.2: Mamba-2 (SSD) computes the
 *       same selective SSM with matrix products; "Mamba-3: un modelo de
 *       espacio de estados centrado en la inferencia", first section: in
 *       Mamba-2 the diagonal transition became a scalar times the identity.
 *
 * Readings taken where the pages are silent (the formulas of the
 * "Discretizacion" section did not survive extraction):
 *   - Abar = exp(delta * A[d,n]); the input term is Bbar x = delta * B * x
 *     (the ZOH rule for A with the simple Euler input term used by Mamba).
 *   - delta = softplus(Delta + delta_bias) when the softplus flag is set,
 *     otherwise Delta + delta_bias; the bias is added before the softplus.
 *   - y = C . h + D * x, and the optional gate multiplies the whole of y by
 *     silu(z) = z / (1 + exp(-z)).
 *   - the initial state is zero unless h0 is given.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* softplus(x) = log(1 + exp(x)), written so that neither branch overflows. */
static double oracle_softplus(double x)
{
    if (x > 0.0)
        return x + log1p(exp(-x));
    return log1p(exp(x));
}

static double oracle_silu(double v)
{
    return v / (1.0 + exp(-v));
}

/*
 * Diagonal-A selective scan.
 *
 * Shapes (C-contiguous, all double):
 *   u, delta, z, y   [batch][dim][L]
 *   A                [dim][N]
 *   B, C             [batch][ngroups][N][L]; channel d reads group
 *                    d / (dim / ngroups)
 *   delta_bias, D    [dim]            (may be NULL)
 *   z                                 (may be NULL: no gate)
 *   h0, last_state   [batch][dim][N]  (may be NULL)
 * Only channels d_begin <= d < d_end are computed; other rows of y and
 * last_state are left untouched, so that a caller can check a sample.
 */
int oracle_selscan(int64_t batch, int64_t dim, int64_t N, int64_t L,
                   int64_t ngroups,
                   const double *u, const double *delta,
                   const double *delta_bias, int softplus_flag,
                   const double *A, const double *B, const double *C,
                   const double *D, const double *z, const double *h0,
                   double *y, double *last_state,
                   int64_t d_begin, int64_t d_end)
{
    if (batch < 0 || dim < 0 || N <= 0 || L < 0 || ngroups <= 0)
        return ORACLE_ERR_ARG;
    if (dim % ngroups != 0 || d_begin < 0 || d_end > dim || d_begin > d_end)
        return ORACLE_ERR_ARG;
    const int64_t per_group = dim / ngroups;
    double *h = (double *)malloc(sizeof(double) * (size_t)N);
    if (!h)
        return ORACLE_ERR_NOMEM;

    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = d_begin; d < d_end; ++d) {
            const int64_t g = d / per_group;
            const double *Bg = B + (b * ngroups + g) * N * L;
            const double *Cg = C + (b * ngroups + g) * N * L;
            const int64_t row = (b * dim + d) * L;
            for (int64_t n = 0; n < N; ++n)
                h[n] = h0 ? h0[(b * dim + d) * N + n] : 0.0;

            for (int64_t t = 0; t < L; ++t) {
                /* step size for this token */
                double dt = delta[row + t] + (delta_bias ? delta_bias[d] : 0.0);
                if (softplus_flag)
                    dt = oracle_softplus(dt);
                const double x = u[row + t];
                /* discretise and advance every state of the channel */
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double abar = exp(dt * A[d * N + n]);
                    const double bbar_x = dt * Bg[n * L + t] * x;
                    h[n] = abar * h[n] + bbar_x;
                    acc += Cg[n * L + t] * h[n];
                }
                /* output: C . h plus the skip term, then the optional gate */
                double out = acc + (D ? D[d] * x : 0.0);
                if (z)
                    out *= oracle_silu(z[row + t]);
                y[row + t] = out;
            }
            if (last_state)
                for (int64_t n = 0; n < N; ++n)
                    last_state[(b * dim + d) * N + n] = h[n];
        }
    }
    free(h);
    return ORACLE_OK;
}

/*
 * One decode step of the same recurrence ("Coste de inferencia": constant
 * work and memory per token).  state [batch][dim][N] is read and updated in
 * place; u, delta, z, y are [batch][dim]; B, C are [batch][ngroups][N].
 */
int oracle_selscan_step(int64_t batch, int64_t dim, int64_t N, int64_t ngroups,
                        const double *u, const double *delta,
                        const double *delta_bias, int softplus_flag,
                        const double *A, const double *B, const double *C,
                        const double *D, const double *z,
                        double *state, double *y)
{
    if (batch < 0 || dim < 0 || N <= 0 || ngroups <= 0 || dim % ngroups != 0)
        return ORACLE_ERR_ARG;
    const int64_t per_group = dim / ngroups;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t g = d / per_group;
            double dt = delta[b * dim + d] + (delta_bias ? delta_bias[d] : 0.0);
            if (softplus_flag)
                dt = oracle_softplus(dt);
            const double x = u[b * dim + d];
            double *h = state + (b * dim + d) * N;
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                h[n] = exp(dt * A[d * N + n]) * h[n]
                     + dt * B[(b * ngroups + g) * N + n] * x;
                acc += C[(b * ngroups + g) * N + n] * h[n];
            }
            double out = acc + (D ? D[d] * x : 0.0);
            if (z)
                out *= oracle_silu(z[b * dim + d]);
            y[b * dim + d] = out;
        }
    }
    return ORACLE_OK;
}

/*
 * Scalar-A selective scan, recurrent form (Mamba-2: the transition is one
 * scalar per head times the identity).
 *
 *   x, z, y          [batch][nheads*headdim][L]   channel d = h*headdim + p
 *   dt               [batch][nheads][L]           step size per head
 *   dt_bias, A, D    [nheads]                     (dt_bias, D may be NULL)
 *   B, C             [batch][ngroups][N][L]; head h reads group
 *                    h / (nheads / ngroups)
 *   h0, last_state   [batch][nheads][headdim][N]  (may be NULL)
 * Heads h_begin <= h < h_end are computed.
 */
int oracle_selscan_scalarA(int64_t batch, int64_t nheads, int64_t headdim,
                           int64_t N, int64_t L, int64_t ngroups,
                           const double *x, const double *dt,
                           const double *dt_bias, int softplus_flag,
                           const double *A, const double *B, const double *C,
                           const double *D, const double *z, const double *h0,
                           double *y, double *last_state,
                           int64_t h_begin, int64_t h_end)
{
    if (batch < 0 || nheads <= 0 || headdim <= 0 || N <= 0 || L < 0 ||
        ngroups <= 0 || nheads % ngroups != 0 || h_begin < 0 ||
        h_end > nheads || h_begin > h_end)
        return ORACLE_ERR_ARG;
    const int64_t heads_per_group = nheads / ngroups;
    const int64_t dim = nheads * headdim;
    double *h = (double *)malloc(sizeof(double) * (size_t)N);
    if (!h)
        return ORACLE_ERR_NOMEM;

    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t hh = h_begin; hh < h_end; ++hh) {
            const int64_t g = hh / heads_per_group;
            const double *Bg = B + (b * ngroups + g) * N * L;
            const double *Cg = C + (b * ngroups + g) * N * L;
            const double *dth = dt + (b * nheads + hh) * L;
            for (int64_t p = 0; p < headdim; ++p) {
                const int64_t d = hh * headdim + p;
                const int64_t row = (b * dim + d) * L;
                for (int64_t n = 0; n < N; ++n)
                    h[n] = h0 ? h0[((b * nheads + hh) * headdim + p) * N + n] : 0.0;
                for (int64_t t = 0; t < L; ++t) {
                    double step = dth[t] + (dt_bias ? dt_bias[hh] : 0.0);
                    if (softplus_flag)
                        step = oracle_softplus(step);
                    const double abar = exp(step * A[hh]);
                    const double xv = x[row + t];
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        h[n] = abar * h[n] + step * Bg[n * L + t] * xv;
                        acc += Cg[n * L + t] * h[n];
                    }
                    double out = acc + (D ? D[hh] * xv : 0.0);
                    if (z)
                        out *= oracle_silu(z[row + t]);
                    y[row + t] = out;
                }
                if (last_state)
                    for (int64_t n = 0; n < N; ++n)
                        last_state[((b * nheads + hh) * headdim + p) * N + n] = h[n];
            }
        }
    }
    free(h);
    return ORACLE_OK;
}

/*
 * Scalar-A scan in the chunked matrix form of structured state-space
 * duality ("Mamba-2 y state-space models", section 4.2): within a chunk of
 * Q tokens the output is a masked, attention-like product, and chunks are
 * linked by passing the state.  Same argument meaning as
 * oracle_selscan_scalarA, plus the chunk length Q.  For every (batch, head)
 * and every chunk with tokens t0 <= t < t0+Q:
 *
 *   S_t        = sum_{r=t0..t} step_r                  (inclusive cumsum)
 *   y_t[p]     = sum_{s=t0..t} (sum_n C_t[n] B_s[n]) exp(A (S_t - S_s))
 *                                step_s x_s[p]                (intra-chunk)
 *              + exp(A S_t) sum_n C_t[n] hprev[n][p]           (carried in)
 *              + D x_t[p]                     then the optional silu gate
 *   hnext[n][p]= exp(A S_end) hprev[n][p]
 *              + sum_s B_s[n] exp(A (S_end - S_s)) step_s x_s[p]
 *
 * exp(A (S_t - S_s)) is the product of the per-token decays exp(step_r A)
 * for s < r <= t, so this equals the recurrence in exact arithmetic.
 */
int oracle_ssd_chunked(int64_t batch, int64_t nheads, int64_t headdim,
                       int64_t N, int64_t L, int64_t ngroups,
                       const double *x, const double *dt,
                       const double *dt_bias, int softplus_flag,
                       const double *A, const double *B, const double *C,
                       const double *D, const double *z, const double *h0,
                       double *y, double *last_state, int64_t Q)
{
    if (batch < 0 || nheads <= 0 || headdim <= 0 || N <= 0 || L < 0 ||
        ngroups <= 0 || nheads % ngroups != 0 || Q <= 0)
        return ORACLE_ERR_ARG;
    const int64_t heads_per_group = nheads / ngroups;
    const int64_t dim = nheads * headdim;
    double *S = (double *)malloc(sizeof(double) * (size_t)Q);
    double *step = (double *)malloc(sizeof(double) * (size_t)Q);
    double *hprev = (double *)malloc(sizeof(double) * (size_t)(N * headdim));
    double *hnext = (double *)malloc(sizeof(double) * (size_t)(N * headdim));
    if (!S || !step || !hprev || !hnext) {
        free(S); free(step); free(hprev); free(hnext);
        return ORACLE_ERR_NOMEM;
    }

    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t hh = 0; hh < nheads; ++hh) {
            const int64_t g = hh / heads_per_group;
            const double *Bg = B + (b * ngroups + g) * N * L;
            const double *Cg = C + (b * ngroups + g) * N * L;
            const double *dth = dt + (b * nheads + hh) * L;
            const double a = A[hh];
            for (int64_t p = 0; p < headdim; ++p)
                for (int64_t n = 0; n < N; ++n)
                    hprev[n * headdim + p] =
                        h0 ? h0[((b * nheads + hh) * headdim + p) * N + n] : 0.0;

            for (int64_t t0 = 0; t0 < L; t0 += Q) {
                const int64_t q = (L - t0 < Q) ? (L - t0) : Q;
                double run = 0.0;
                for (int64_t i = 0; i < q; ++i) {
                    double s = dth[t0 + i] + (dt_bias ? dt_bias[hh] : 0.0);
                    if (softplus_flag)
                        s = oracle_softplus(s);
                    step[i] = s;
                    run += s;
                    S[i] = run;
                }
                const double S_end = S[q - 1];

                for (int64_t i = 0; i < q; ++i) {          /* token t0+i */
                    const int64_t t = t0 + i;
                    for (int64_t p = 0; p < headdim; ++p) {
                        const int64_t row = (b * dim + hh * headdim + p) * L;
                        double intra = 0.0;
                        for (int64_t j = 0; j <= i; ++j) {  /* token t0+j */
                            double cb = 0.0;
                            for (int64_t n = 0; n < N; ++n)
                                cb += Cg[n * L + t] * Bg[n * L + t0 + j];
                            intra += cb * exp(a * (S[i] - S[j])) * step[j]
                                   * x[row + t0 + j];
                        }
                        double carried = 0.0;
                        for (int64_t n = 0; n < N; ++n)
                            carried += Cg[n * L + t] * hprev[n * headdim + p];
                        carried *= exp(a * S[i]);
                        double out = intra + carried + (D ? D[hh] * x[row + t] : 0.0);
                        if (z)
                            out *= oracle_silu(z[row + t]);
                        y[row + t] = out;
                    }
                }

                for (int64_t n = 0; n < N; ++n) {
                    for (int64_t p = 0; p < headdim; ++p) {
                        const int64_t row = (b * dim + hh * headdim + p) * L;
                        double acc = exp(a * S_end) * hprev[n * headdim + p];
                        for (int64_t j = 0; j < q; ++j)
                            acc += Bg[n * L + t0 + j] * exp(a * (S_end - S[j]))
                                 * step[j] * x[row + t0 + j];
                        hnext[n * headdim + p] = acc;
                    }
                }
                memcpy(hprev, hnext, sizeof(double) * (size_t)(N * headdim));
            }
            if (last_state)
                for (int64_t p = 0; p < headdim; ++p)
                    for (int64_t n = 0; n < N; ++n)
                        last_state[((b * nheads + hh) * headdim + p) * N + n] =
                            hprev[n * headdim + p];
        }
    }
    free(S); free(step); free(hprev); free(hnext);
    return ORACLE_OK;
}

/*
 * Gradients of the diagonal-A selective scan (reverse-mode differentiation
 * of oracle_selscan, step by step, in fp64).  The loss is
 *     sum_{b,d,t} dy[b,d,t] y[b,d,t] + sum_{b,d,n} dlast[b,d,n] h_L[b,d,n]
 * (dlast may be NULL: the final state is not an output of the loss).
 *
 * With delta_t the step size, abar_t[n] = exp(delta_t A[d,n]),
 * h_t = abar_t h_{t-1} + delta_t B_t u_t, out_t = C_t . h_t + D u_t and
 * y_t = out_t silu(z_t), walking t from L-1 down to 0 with
 * g = dLoss/dh_t (starting from dlast):
 *     dout   = dy_t silu(z_t)             dz_t += dy_t out_t silu'(z_t)
 *     g     += dout C_t                   dC_t += dout h_t
 *     du_t   = dout D + sum_n g delta_t B_t
 *     dB_t  += g delta_t u_t              dD   += dout u_t
 *     ddelta = sum_n g (A abar_t h_{t-1} + B_t u_t)
 *     dA    += g delta_t abar_t h_{t-1}
 *     g      = abar_t g                   (now dLoss/dh_{t-1})
 *     dDelta_t = ddelta * sigmoid(Delta_t + bias) with the softplus (its
 *     derivative), ddelta otherwise;  dbias += dDelta_t
 * and after t = 0, dh0 = g.
 *
 * Shapes as in oracle_selscan; dy [batch][dim][L]; dlast, dh0
 * [batch][dim][N].  Outputs du, ddelta, dz [batch][dim][L] are written;
 * dA [dim][N], dB, dC [batch][ngroups][N][L], dD, dbias [dim] are
 * ACCUMULATED (the caller zeroes them); dz, dD, dbias, dh0 may be NULL.
 */
int oracle_selscan_bwd(int64_t batch, int64_t dim, int64_t N, int64_t L,
                       int64_t ngroups,
                       const double *u, const double *delta,
                       const double *delta_bias, int softplus_flag,
                       const double *A, const double *B, const double *C,
                       const double *D, const double *z, const double *h0,
                       const double *dy, const double *dlast,
                       double *du, double *ddelta, double *dA, double *dB,
                       double *dC, double *dD, double *dz, double *dbias,
                       double *dh0)
{
    if (batch < 0 || dim < 0 || N <= 0 || L < 0 || ngroups <= 0 || dim % ngroups != 0)
        return ORACLE_ERR_ARG;
    const int64_t per_group = dim / ngroups;
    /* forward states h_t for t = -1 .. L-1 of one channel, and step sizes */
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *dts = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    double *g = (double *)malloc(sizeof(double) * (size_t)N);
    if (!hs || !dts || !g) {
        free(hs);
        free(dts);
        free(g);
        return ORACLE_ERR_NOMEM;
    }
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t grp = d / per_group;
            const double *Bg = B + (b * ngroups + grp) * N * L;
            const double *Cg = C + (b * ngroups + grp) * N * L;
            double *dBg = dB + (b * ngroups + grp) * N * L;
            double *dCg = dC + (b * ngroups + grp) * N * L;
            const int64_t row = (b * dim + d) * L;
            const double bias = delta_bias ? delta_bias[d] : 0.0;
            /* forward, keeping every state (hs[t+1] = h_t, hs[0] = h_{-1}) */
            for (int64_t n = 0; n < N; ++n)
                hs[n] = h0 ? h0[(b * dim + d) * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                double dt = delta[row + t] + bias;
                if (softplus_flag)
                    dt = oracle_softplus(dt);
                dts[t] = dt;
                for (int64_t n = 0; n < N; ++n)
                    hs[(t + 1) * N + n] = exp(dt * A[d * N + n]) * hs[t * N + n]
                                        + dt * Bg[n * L + t] * u[row + t];
            }
            /* backward */
            for (int64_t n = 0; n < N; ++n)
                g[n] = dlast ? dlast[(b * dim + d) * N + n] : 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const double dt = dts[t];
                const double x = u[row + t];
                const double *h_t = hs + (t + 1) * N;
                const double *h_prev = hs + t * N;
                double out = (D ? D[d] * x : 0.0);
                for (int64_t n = 0; n < N; ++n)
                    out += Cg[n * L + t] * h_t[n];
                double dout = dy[row + t];
                if (z) {
                    const double zv = z[row + t];
                    const double sg = 1.0 / (1.0 + exp(-zv));
                    const double dsilu = sg * (1.0 + zv * (1.0 - sg));
                    if (dz)
                        dz[row + t] = dy[row + t] * out * dsilu;
                    dout = dy[row + t] * zv * sg;
                }
                double dx = D ? dout * D[d] : 0.0;
                if (dD)
                    dD[d] += dout * x;
                double ddt = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = A[d * N + n];
                    const double abar = exp(dt * a);
                    g[n] += dout * Cg[n * L + t];
                    dCg[n * L + t] += dout * h_t[n];
                    dx += g[n] * dt * Bg[n * L + t];
                    dBg[n * L + t] += g[n] * dt * x;
                    ddt += g[n] * (a * abar * h_prev[n] + Bg[n * L + t] * x);
                    dA[d * N + n] += g[n] * dt * abar * h_prev[n];
                    g[n] *= abar;
                }
                du[row + t] = dx;
                double dDelta = ddt;
                if (softplus_flag)
                    dDelta = ddt / (1.0 + exp(-(delta[row + t] + bias)));
                ddelta[row + t] = dDelta;
                if (dbias)
                    dbias[d] += dDelta;
            }
            if (dh0)
                for (int64_t n = 0; n < N; ++n)
                    dh0[(b * dim + d) * N + n] = g[n];
        }
    }
    free(hs);
    free(dts);
    free(g);
    return ORACLE_OK;
}

/*
 * mm_oracle.c -- plain, slow, fp64 CPU oracle for the Momentum Mamba
 * selective scan (forward and backward) and its Mamba-2 scalar-A chunked
 * (SSD) form.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * Every input arrives as the fp32 values the GPU path reads (bf16 inputs are
 * passed already rounded, as fp32 numbers); every operation below is done in
 * double precision.  There is no blocking, fusion or reordering beyond what
 * the cited definition or algorithm states.  Loops over independent channels
 * may run on several OpenMP threads; that does not change any arithmetic.
 *
 * Sources (cited by page title and section):
 *  [MM]  "Momentum Mamba: Enhanced State Space Models with Momentum"
 *        (t-khanusa/Momentum_Mamba README), sections "Momentum Mamba
 *        Recurrence", "Discretization Note", "selective_scan_fn",
 *        "Mamba Module" (step / velocity_state), "Gradient Flow" and
 *        "Backward Pass: Reconstructed Forward + Reverse Scans".
 *  [SEL] "Mamba: Choosing What to Remember Based on the Input", section
 *        "Expressing the update and read as equations" (read-out of the
 *        post-update state).
 *  [SSD] "Mamba-2 -- SSM = structured matrix multiply", sections "4-Step
 *        Algorithm" and "Multi-Head Expansion", and the L_ij matrix form in
 *        its "why it works" section.
 *
 * Parity status: every function here is pinned by the CPU tests against
 * values and identities fixed outside this file (worked examples, closed
 * forms, an FFT convolution, brute-force matrices); none is "parity unpinned".
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_ALLOC 2

/* ------------------------------------------------------------------------ */
/* Mamba-1 momentum scan: the definition, one time step after another.      */
/* ------------------------------------------------------------------------ */

/*
 * [MM] "Momentum Mamba Recurrence" with the first-order discretization of
 * [MM] "Discretization Note" (A_bar = exp(delta*A), B_bar = delta*B):
 *
 *     v_t = beta * v_{t-1} + alpha * (delta_t * B_t[n] * x_t)
 *     h_t = exp(delta_t * A[d,n]) * h_{t-1} + v_t
 *     y_t = sum_n C_t[n] * h_t[n]          (read-out of the updated state)
 *
 * Layouts follow [MM] "selective_scan_fn": x, delta, y are (batch, dim, L),
 * A is (dim, dstate), B and C are (batch, dstate, L) and are shared by every
 * channel d; states h0, v0, hT, vT are (batch, dim, dstate).  h0/v0 may be
 * NULL, meaning zero ([MM]: the velocity starts at zero).
 *
 * `chan` lists the channels to compute as flat indices b*dim + d (NULL means
 * all batch*dim channels, in order); output row r of y/hT/vT belongs to
 * chan[r].  y is (nchan, L); hT, vT are (nchan, dstate) and may be NULL.
 */
int oracle_scan_seq(const float *x, const float *delta, const float *A,
                    const float *Bm, const float *Cm,
                    const double *h0, const double *v0,
                    double beta, double alpha,
                    int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                    const int64_t *chan, int64_t nchan,
                    double *y, double *hT, double *vT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1) return ORACLE_ERR_ARG;
    if (!chan) nchan = batch * dim;
    if (nchan < 0) return ORACLE_ERR_ARG;

    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nchan; ++r) {
        const int64_t c = chan ? chan[r] : r;
        const int64_t b = c / dim;
        const int64_t d = c % dim;
        const float *xr = x + c * seqlen;
        const float *dr = delta + c * seqlen;
        double *yr = y + r * seqlen;
        for (int64_t t = 0; t < seqlen; ++t) yr[t] = 0.0;

        for (int64_t n = 0; n < dstate; ++n) {
            double h = h0 ? h0[c * dstate + n] : 0.0;
            double v = v0 ? v0[c * dstate + n] : 0.0;
            const double a_dn = (double)A[d * dstate + n];
            const float *Bn = Bm + (b * dstate + n) * seqlen;
            const float *Cn = Cm + (b * dstate + n) * seqlen;
            for (int64_t t = 0; t < seqlen; ++t) {
                const double dt = (double)dr[t];
                const double abar = exp(dt * a_dn);
                v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);
                h = abar * h + v;
                yr[t] += (double)Cn[t] * h;
            }
            if (hT) hT[r * dstate + n] = h;
            if (vT) vT[r * dstate + n] = v;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* The full selective_scan_fn forward: delta bias and softplus, D skip, z gate */
/* ------------------------------------------------------------------------ */

/*
 * [MM] "selective_scan_fn" lists, besides u (= x), delta, A, B, C and the
 * momentum pair, a skip weight D (dim), a gate z (batch, dim, L), a delta
 * bias (dim) and a softplus switch; [SEL] "Where the state computation sits
 * in a Mamba block" places the gate after the scan: SiLU of the gate branch
 * multiplies the scan's output elementwise.  Readings (the pages give the
 * arguments but no formulas):
 *
 *     delta'_t = delta_t + delta_bias[d]                   (bias NULL: + 0)
 *     delta'_t = ln(1 + e^{delta'_t})                      (if softplus)
 *     y_t      = sum_n C_t[n] h_t[n]   (recurrence above, with delta')
 *     out_t    = y_t + D[d] * x_t                          (D NULL: + 0)
 *     out_t    = out_t * z_t / (1 + e^{-z_t})              (z NULL: no gate)
 *
 * The states hT, vT are those of the recurrence.  Same layouts, channel
 * selection and outputs as oracle_scan_seq (y holds out).
 */
static double softplus_f64(double u)
{
    /* ln(1 + e^u) without overflow: max(u, 0) + ln(1 + e^{-|u|}) */
    return (u > 0.0 ? u : 0.0) + log1p(exp(-fabs(u)));
}

int oracle_scan_gated(const float *x, const float *delta, const float *A,
                      const float *Bm, const float *Cm,
                      const float *Dv, const float *z, const float *dbias, int softplus,
                      const double *h0, const double *v0,
                      double beta, double alpha,
                      int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                      const int64_t *chan, int64_t nchan,
                      double *y, double *hT, double *vT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1) return ORACLE_ERR_ARG;
    if (!chan) nchan = batch * dim;
    if (nchan < 0) return ORACLE_ERR_ARG;

    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nchan; ++r) {
        const int64_t c = chan ? chan[r] : r;
        const int64_t b = c / dim;
        const int64_t d = c % dim;
        const float *xr = x + c * seqlen;
        const float *dr = delta + c * seqlen;
        double *yr = y + r * seqlen;
        for (int64_t t = 0; t < seqlen; ++t) yr[t] = 0.0;

        for (int64_t n = 0; n < dstate; ++n) {
            double h = h0 ? h0[c * dstate + n] : 0.0;
            double v = v0 ? v0[c * dstate + n] : 0.0;
            const double a_dn = (double)A[d * dstate + n];
            const float *Bn = Bm + (b * dstate + n) * seqlen;
            const float *Cn = Cm + (b * dstate + n) * seqlen;
            for (int64_t t = 0; t < seqlen; ++t) {
                double dt = (double)dr[t] + (dbias ? (double)dbias[d] : 0.0);
                if (softplus) dt = softplus_f64(dt);
                const double abar = exp(dt * a_dn);
                v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);
                h = abar * h + v;
                yr[t] += (double)Cn[t] * h;
            }
            if (hT) hT[r * dstate + n] = h;
            if (vT) vT[r * dstate + n] = v;
        }
        for (int64_t t = 0; t < seqlen; ++t) {
            double o = yr[t] + (Dv ? (double)Dv[d] * (double)xr[t] : 0.0);
            if (z) {
                const double zt = (double)z[c * seqlen + t];
                o *= zt / (1.0 + exp(-zt));
            }
            yr[t] = o;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Backward of the full selective_scan_fn forward                           */
/* ------------------------------------------------------------------------ */

/*
 * [MM] "Gradient Flow" and "Backward Pass: Reconstructed Forward + Reverse
 * Scans": the forward states are rebuilt, then the gradients with respect to
 * the hidden state and the velocity run backwards in time.  The printed
 * formulas use one symbol for both of those gradients and leave a term out
 * of the velocity's, so the recursions are derived here from the forward
 * recurrence itself.  With G_t = dL/dh_t and P_t = dL/dv_t (total
 * derivatives: everything that depends on the state later is included),
 *
 *     G_t = dy_t C_t[n] + a_{t+1} G_{t+1}      (for t = L-1: + dhT instead)
 *     P_t = G_t + beta P_{t+1}                 (for t = L-1: + dvT instead)
 *
 * because h_t feeds y_t and h_{t+1} (factor a_{t+1}), and v_t feeds h_t
 * (factor 1) and v_{t+1} (factor beta).  The local terms are the ones the
 * pages list, with dL/dh_t and dL/dv_t read as G_t and P_t:
 *
 *     dx_t       += alpha delta'_t B_t[n] P_t
 *     ddelta'_t  += alpha B_t[n] x_t P_t + A[d,n] a_t h_{t-1} G_t
 *     dA[d,n]    += delta'_t a_t h_{t-1} G_t           (all t and b)
 *     dB_t[n]    += alpha delta'_t x_t P_t             (all d of the batch row)
 *     dC_t[n]    += dy_t h_t                           (all d of the batch row)
 *     dh0 = a_0 G_0,   dv0 = beta P_0
 *
 * with a_t = exp(delta'_t A[d,n]).  dy is the gradient that reaches the
 * read-out.  Around it, following the readings of oracle_scan_gated, with
 * o_t = y_t + D x_t and s_t = 1 / (1 + e^{-z_t}):
 *
 *     dy_t = dout_t z_t s_t         (no gate: dy_t = dout_t)
 *     dz_t = dout_t o_t s_t (1 + z_t (1 - s_t))
 *     dx_t += D dy_t,   dD += dy_t x_t
 *     ddelta_t = ddelta'_t / (1 + e^{-(delta_t + bias)})   (softplus; else ddelta'_t)
 *     dbias += ddelta_t
 */

/* delta' of channel c and the gradient dy reaching its read-out; dz_r and
 * the gate-side terms are written when asked for.  The forward over all
 * states is run once when the gate needs y. */
static void bwd_channel_prep(int64_t c, const float *x, const float *delta, const float *A,
                             const float *Bm, const float *Cm, const float *Dv, const float *z,
                             const float *dbias, int softplus, const double *h0, const double *v0,
                             double beta, double alpha, const float *dout,
                             int64_t seqlen, int64_t dim, int64_t dstate,
                             double *dp, double *dy, double *dz_r)
{
    const int64_t b = c / dim;
    const int64_t d = c % dim;
    const float *xr = x + c * seqlen;
    const float *dr = delta + c * seqlen;
    for (int64_t t = 0; t < seqlen; ++t) {
        double u = (double)dr[t] + (dbias ? (double)dbias[d] : 0.0);
        dp[t] = softplus ? softplus_f64(u) : u;
        dy[t] = (double)dout[c * seqlen + t];
    }
    if (!z) return;
    /* the gate needs o_t = y_t + D x_t */
    double *o = (double *)calloc((size_t)seqlen, sizeof(double));
    for (int64_t n = 0; n < dstate; ++n) {
        double h = h0 ? h0[c * dstate + n] : 0.0;
        double v = v0 ? v0[c * dstate + n] : 0.0;
        const double a_dn = (double)A[d * dstate + n];
        const float *Bn = Bm + (b * dstate + n) * seqlen;
        const float *Cn = Cm + (b * dstate + n) * seqlen;
        for (int64_t t = 0; t < seqlen; ++t) {
            v = beta * v + alpha * (dp[t] * (double)Bn[t] * (double)xr[t]);
            h = exp(dp[t] * a_dn) * h + v;
            o[t] += (double)Cn[t] * h;
        }
    }
    for (int64_t t = 0; t < seqlen; ++t) {
        const double ot = o[t] + (Dv ? (double)Dv[d] * (double)xr[t] : 0.0);
        const double zt = (double)z[c * seqlen + t];
        const double st = 1.0 / (1.0 + exp(-zt));
        if (dz_r) dz_r[t] = dy[t] * ot * st * (1.0 + zt * (1.0 - st));
        dy[t] = dy[t] * zt * st;
    }
    free(o);
}

/* One (b, d, n) chain: the forward states of every step, then the reverse
 * sweep giving G_t and P_t.  Returns a_0 G_0 and beta P_0 in *gh0, *gv0. */
static void bwd_chain(const double *dp, const float *xr, double a_dn, const float *Bn,
                      const float *Cn, const double *dy, double h_init, double v_init,
                      double beta, double alpha, double gT, double pT, int64_t seqlen,
                      double *hs, double *vs, double *as, double *G, double *P,
                      double *gh0, double *gv0)
{
    double h = h_init, v = v_init;
    for (int64_t t = 0; t < seqlen; ++t) {
        const double abar = exp(dp[t] * a_dn);
        v = beta * v + alpha * (dp[t] * (double)Bn[t] * (double)xr[t]);
        h = abar * h + v;
        hs[t] = h;
        vs[t] = v;
        as[t] = abar;
    }
    double cg = gT, cp = pT;          /* a_{t+1} G_{t+1} and beta P_{t+1} */
    for (int64_t t = seqlen - 1; t >= 0; --t) {
        const double g = dy[t] * (double)Cn[t] + cg;
        const double p = g + cp;
        G[t] = g;
        P[t] = p;
        cg = as[t] * g;
        cp = beta * p;
    }
    *gh0 = cg;
    *gv0 = cp;
}

/*
 * Arguments as oracle_scan_gated, plus dout (batch, dim, L) and dhT, dvT
 * (batch, dim, dstate; NULL = 0), the gradients arriving at the outputs.
 * Per-channel results are computed for the channels `chan` lists (NULL: all,
 * in order) and written as rows r: dx, ddelta, dz (nchan, L); dh0, dv0
 * (nchan, dstate).  dA (dim, dstate), dD and dbias (dim) sum the listed
 * channels' terms (all channels: the full gradients).  dB and dC rows are
 * computed for the (b, n) pairs `bn` lists as flat indices b*dstate + n
 * (NULL: all, in order), each summed over every d: (nbn, L).  Any output
 * may be NULL.
 */
int oracle_scan_bwd(const float *x, const float *delta, const float *A,
                    const float *Bm, const float *Cm,
                    const float *Dv, const float *z, const float *dbias, int softplus,
                    const double *h0, const double *v0, double beta, double alpha,
                    const float *dout, const double *dhT, const double *dvT,
                    int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                    const int64_t *chan, int64_t nchan, const int64_t *bn, int64_t nbn,
                    double *dx, double *ddelta, double *dz, double *dh0, double *dv0,
                    double *dA, double *dD, double *ddbias, double *dB, double *dC)
{
    if (!x || !delta || !A || !Bm || !Cm || !dout) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1) return ORACLE_ERR_ARG;
    if (!chan) nchan = batch * dim;
    if (!bn) nbn = batch * dstate;
    if (nchan < 0 || nbn < 0) return ORACLE_ERR_ARG;
    const size_t L = (size_t)seqlen;

    /* per-channel terms of dA, dD, dbias, summed in channel order afterwards */
    double *dA_r = (double *)calloc((size_t)nchan * (size_t)dstate, sizeof(double));
    double *dD_r = (double *)calloc((size_t)nchan, sizeof(double));
    double *db_r = (double *)calloc((size_t)nchan, sizeof(double));

    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nchan; ++r) {
        const int64_t c = chan ? chan[r] : r;
        const int64_t b = c / dim;
        const int64_t d = c % dim;
        const float *xr = x + c * seqlen;
        double *buf = (double *)malloc(9 * L * sizeof(double));
        double *dp = buf, *dy = buf + L, *hs = buf + 2 * L, *vs = buf + 3 * L, *as = buf + 4 * L;
        double *G = buf + 5 * L, *P = buf + 6 * L, *gx = buf + 7 * L, *gd = buf + 8 * L;
        bwd_channel_prep(c, x, delta, A, Bm, Cm, Dv, z, dbias, softplus, h0, v0, beta, alpha,
                         dout, seqlen, dim, dstate, dp, dy, dz ? dz + r * seqlen : NULL);
        for (size_t t = 0; t < L; ++t) gx[t] = gd[t] = 0.0;
        for (int64_t n = 0; n < dstate; ++n) {
            const double a_dn = (double)A[d * dstate + n];
            const float *Bn = Bm + (b * dstate + n) * seqlen;
            const float *Cn = Cm + (b * dstate + n) * seqlen;
            const double hi = h0 ? h0[c * dstate + n] : 0.0;
            const double vi = v0 ? v0[c * dstate + n] : 0.0;
            double gh0, gv0;
            bwd_chain(dp, xr, a_dn, Bn, Cn, dy, hi, vi, beta, alpha,
                      dhT ? dhT[c * dstate + n] : 0.0, dvT ? dvT[c * dstate + n] : 0.0,
                      seqlen, hs, vs, as, G, P, &gh0, &gv0);
            double acc_a = 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                const double hprev = t > 0 ? hs[t - 1] : hi;
                const double decay_term = as[t] * hprev * G[t];      /* a_t h_{t-1} G_t */
                gx[t] += alpha * dp[t] * (double)Bn[t] * P[t];
                gd[t] += alpha * (double)Bn[t] * (double)xr[t] * P[t] + a_dn * decay_term;
                acc_a += dp[t] * decay_term;
            }
            dA_r[r * dstate + n] = acc_a;
            if (dh0) dh0[r * dstate + n] = gh0;
            if (dv0) dv0[r * dstate + n] = gv0;
        }
        double accD = 0.0, accb = 0.0;
        for (int64_t t = 0; t < seqlen; ++t) {
            double g_delta = gd[t];
            if (softplus) {
                const double u = (double)delta[c * seqlen + t] + (dbias ? (double)dbias[d] : 0.0);
                g_delta *= 1.0 / (1.0 + exp(-u));
            }
            const double g_x = gx[t] + (Dv ? (double)Dv[d] * dy[t] : 0.0);
            if (dx) dx[r * seqlen + t] = g_x;
            if (ddelta) ddelta[r * seqlen + t] = g_delta;
            accD += dy[t] * (double)xr[t];
            accb += g_delta;
        }
        dD_r[r] = accD;
        db_r[r] = accb;
        free(buf);
    }
    if (dA) {
        for (int64_t i = 0; i < dim * dstate; ++i) dA[i] = 0.0;
        for (r = 0; r < nchan; ++r) {
            const int64_t d = (chan ? chan[r] : r) % dim;
            for (int64_t n = 0; n < dstate; ++n) dA[d * dstate + n] += dA_r[r * dstate + n];
        }
    }
    if (dD || ddbias) {
        for (int64_t i = 0; i < dim; ++i) {
            if (dD) dD[i] = 0.0;
            if (ddbias) ddbias[i] = 0.0;
        }
        for (r = 0; r < nchan; ++r) {
            const int64_t d = (chan ? chan[r] : r) % dim;
            if (dD) dD[d] += dD_r[r];
            if (ddbias) ddbias[d] += db_r[r];
        }
    }
    free(dA_r);
    free(dD_r);
    free(db_r);

    if (dB || dC) {
        int64_t k;
#pragma omp parallel for schedule(dynamic, 1)
        for (k = 0; k < nbn; ++k) {
            const int64_t f = bn ? bn[k] : k;
            const int64_t b = f / dstate;
            const int64_t n = f % dstate;
            const float *Bn = Bm + (b * dstate + n) * seqlen;
            const float *Cn = Cm + (b * dstate + n) * seqlen;
            double *buf = (double *)malloc(7 * L * sizeof(double));
            double *dp = buf, *dy = buf + L, *hs = buf + 2 * L, *vs = buf + 3 * L, *as = buf + 4 * L;
            double *G = buf + 5 * L, *P = buf + 6 * L;
            if (dB) for (int64_t t = 0; t < seqlen; ++t) dB[k * seqlen + t] = 0.0;
            if (dC) for (int64_t t = 0; t < seqlen; ++t) dC[k * seqlen + t] = 0.0;
            for (int64_t d = 0; d < dim; ++d) {
                const int64_t c = b * dim + d;
                const float *xr = x + c * seqlen;
                bwd_channel_prep(c, x, delta, A, Bm, Cm, Dv, z, dbias, softplus, h0, v0, beta,
                                 alpha, dout, seqlen, dim, dstate, dp, dy, NULL);
                double gh0, gv0;
                bwd_chain(dp, xr, (double)A[d * dstate + n], Bn, Cn, dy,
                          h0 ? h0[c * dstate + n] : 0.0, v0 ? v0[c * dstate + n] : 0.0,
                          beta, alpha, dhT ? dhT[c * dstate + n] : 0.0,
                          dvT ? dvT[c * dstate + n] : 0.0, seqlen, hs, vs, as, G, P, &gh0, &gv0);
                for (int64_t t = 0; t < seqlen; ++t) {
                    if (dB) dB[k * seqlen + t] += alpha * dp[t] * (double)xr[t] * P[t];
                    if (dC) dC[k * seqlen + t] += dy[t] * hs[t];
                }
            }
            free(buf);
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* The same scan in chunked form: per-chunk affine maps, then a carry fold.  */
/* ------------------------------------------------------------------------ */

/*
 * [MM] "Forward Pass: Two-Stage Parallel Scan": both recurrences are affine
 * maps of the previous state, so a run of steps composes into one map and a
 * long sequence can be cut into chunks whose maps are chained by a running
 * prefix.  Over one chunk of k steps, starting from (v_in, h_in):
 *
 *     v_out = beta^k * v_in + V
 *     h_out = P * h_in + Q * v_in + H
 *
 * where, stepping t through the chunk from P=1, Q=0, V=H=0,
 *     P <- abar_t * P,   Q <- abar_t * Q + beta^(steps so far),
 *     V <- beta * V + w_t,   H <- abar_t * H + V        (w_t = alpha*delta*B*x)
 *
 * i.e. the joint carry [[beta^k, 0], [Q, P]] acting on (v, h) plus (V, H).
 * This routine builds every chunk's map from the chunk's own data alone,
 * folds the maps onto the incoming state chunk after chunk, and then replays
 * each chunk from its true incoming state to produce y.  Same arguments as
 * oracle_scan_seq plus the chunk length (the last chunk may be shorter).
 */
int oracle_scan_chunked(const float *x, const float *delta, const float *A,
                        const float *Bm, const float *Cm,
                        const double *h0, const double *v0,
                        double beta, double alpha,
                        int64_t batch, int64_t seqlen, int64_t dim, int64_t dstate,
                        int64_t chunk,
                        const int64_t *chan, int64_t nchan,
                        double *y, double *hT, double *vT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || dim < 1 || dstate < 1 || chunk < 1)
        return ORACLE_ERR_ARG;
    if (!chan) nchan = batch * dim;
    if (nchan < 0) return ORACLE_ERR_ARG;
    const int64_t nchunks = (seqlen + chunk - 1) / chunk;

    int err = ORACLE_OK;
    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nchan; ++r) {
        const int64_t c = chan ? chan[r] : r;
        const int64_t b = c / dim;
        const int64_t d = c % dim;
        const float *xr = x + c * seqlen;
        const float *dr = delta + c * seqlen;
        double *yr = y + r * seqlen;
        /* incoming state of every chunk, per state n */
        double *vin = (double *)malloc(sizeof(double) * (size_t)(nchunks + 1));
        double *hin = (double *)malloc(sizeof(double) * (size_t)(nchunks + 1));
        if (!vin || !hin) {
            free(vin); free(hin);
#pragma omp atomic write
            err = ORACLE_ERR_ALLOC;
            continue;
        }
        for (int64_t t = 0; t < seqlen; ++t) yr[t] = 0.0;

        for (int64_t n = 0; n < dstate; ++n) {
            const double a_dn = (double)A[d * dstate + n];
            const float *Bn = Bm + (b * dstate + n) * seqlen;
            const float *Cn = Cm + (b * dstate + n) * seqlen;
            vin[0] = v0 ? v0[c * dstate + n] : 0.0;
            hin[0] = h0 ? h0[c * dstate + n] : 0.0;

            /* 1) each chunk's map from its own data, 2) fold onto the state */
            for (int64_t k = 0; k < nchunks; ++k) {
                const int64_t t0 = k * chunk;
                const int64_t t1 = (t0 + chunk < seqlen) ? t0 + chunk : seqlen;
                double P = 1.0, Q = 0.0, V = 0.0, H = 0.0, bk = 1.0;
                for (int64_t t = t0; t < t1; ++t) {
                    const double dt = (double)dr[t];
                    const double abar = exp(dt * a_dn);
                    const double w = alpha * (dt * (double)Bn[t] * (double)xr[t]);
                    bk *= beta;              /* beta^(t - t0 + 1) */
                    P = abar * P;
                    Q = abar * Q + bk;
                    V = beta * V + w;
                    H = abar * H + V;
                }
                vin[k + 1] = bk * vin[k] + V;
                hin[k + 1] = P * hin[k] + Q * vin[k] + H;
            }
            /* 3) replay every chunk from its true incoming state for y */
            for (int64_t k = 0; k < nchunks; ++k) {
                const int64_t t0 = k * chunk;
                const int64_t t1 = (t0 + chunk < seqlen) ? t0 + chunk : seqlen;
                double v = vin[k], h = hin[k];
                for (int64_t t = t0; t < t1; ++t) {
                    const double dt = (double)dr[t];
                    const double abar = exp(dt * a_dn);
                    v = beta * v + alpha * (dt * (double)Bn[t] * (double)xr[t]);
                    h = abar * h + v;
                    yr[t] += (double)Cn[t] * h;
                }
            }
            if (hT) hT[r * dstate + n] = hin[nchunks];
            if (vT) vT[r * dstate + n] = vin[nchunks];
        }
        free(vin);
        free(hin);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 scalar-A multi-head form, sequential definition.                 */
/* ------------------------------------------------------------------------ */

/*
 * [SSD] "Multi-Head Expansion": H heads of dimension P, one scalar A per
 * head.  With the same first-order discretization as [MM], every (head h,
 * head-channel p, state n) lane follows the momentum recurrence of
 * oracle_scan_seq with delta_{b,t,h}, A_h, input x[b,t,h,p] and the group's
 * B/C rows (head h reads group h / (H/G)):
 *
 *     v = beta*v + alpha*delta*B[n]*x[p];  h[p,n] = exp(delta*A_h)*h[p,n] + v
 *     y[b,t,h,p] = sum_n C[n] * h[p,n]
 *
 * Layouts: x, y (batch, L, H, P); delta (batch, L, H); A (H);
 * B, C (batch, L, G, N); states h0, v0 (batch, H, P, N), may be NULL.
 *
 * `lane` lists the (b, h, p) lanes to compute as flat indices
 * (b*H + h)*P + p (NULL means all, in order).  Output row r belongs to
 * lane[r]: y is (nlane, L), hT and vT are (nlane, N) and may be NULL.
 */
int oracle_ssd_seq(const float *x, const float *delta, const float *A,
                   const float *Bm, const float *Cm,
                   const double *h0, const double *v0,
                   double beta, double alpha,
                   int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                   int64_t dstate, int64_t ngroups,
                   const int64_t *lane, int64_t nlane,
                   double *y, double *hT, double *vT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || nheads < 1 || headdim < 1 || dstate < 1 ||
        ngroups < 1 || nheads % ngroups != 0)
        return ORACLE_ERR_ARG;
    const int64_t heads_per_group = nheads / ngroups;
    if (!lane) nlane = batch * nheads * headdim;
    if (nlane < 0) return ORACLE_ERR_ARG;

    int64_t r;
#pragma omp parallel for schedule(dynamic, 1)
    for (r = 0; r < nlane; ++r) {
        const int64_t l = lane ? lane[r] : r;
        const int64_t b = l / (nheads * headdim);
        const int64_t hh = (l / headdim) % nheads;
        const int64_t p = l % headdim;
        const int64_t g = hh / heads_per_group;
        const double a_h = (double)A[hh];
        double *yr = y + r * seqlen;
        for (int64_t t = 0; t < seqlen; ++t) yr[t] = 0.0;
        for (int64_t n = 0; n < dstate; ++n) {
            const int64_t sidx = l * dstate + n;
            double h = h0 ? h0[sidx] : 0.0;
            double v = v0 ? v0[sidx] : 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                const double dt = (double)delta[(b * seqlen + t) * nheads + hh];
                const double xv = (double)x[((b * seqlen + t) * nheads + hh) * headdim + p];
                const int64_t bc = ((b * seqlen + t) * ngroups + g) * dstate + n;
                const double abar = exp(dt * a_h);
                v = beta * v + alpha * (dt * (double)Bm[bc] * xv);
                h = abar * h + v;
                yr[t] += (double)Cm[bc] * h;
            }
            if (hT) hT[r * dstate + n] = h;
            if (vT) vT[r * dstate + n] = v;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 SSD: the 4-step chunked algorithm (beta = 0).                    */
/* ------------------------------------------------------------------------ */

/*
 * [SSD] "4-Step Algorithm", with the matrix form L_ij = C_i . (A_i...A_{j+1})
 * . B_j of its "why it works" section, for scalar A per head and B_bar =
 * alpha*delta*B (first-order discretization as in [MM]).  For every (batch,
 * head) and every chunk of `chunk` steps (the last may be shorter), with the
 * in-chunk cumulative log-decay cs_i = sum_{t <= i, t in chunk} delta_t*A_h:
 *
 *  1. intra-chunk output  Y_diag[i,p] = sum_{j<=i} (C_i . B_j)
 *                                        * exp(cs_i - cs_j) * alpha*delta_j * x_j[p]
 *  2. chunk final state   s[p,n] = sum_j exp(cs_last - cs_j) * alpha*delta_j
 *                                        * B_j[n] * x_j[p]
 *  3. inter-chunk scan    S_c = exp(cs_last) * S_{c-1} + s_c,   S_{-1} = h0
 *  4. combine             y_i = Y_diag[i] + exp(cs_i) * sum_n C_i[n] * S_{c-1}[.,n]
 *
 * hT = S after the last chunk.  This is the plain (beta = 0) recurrence only;
 * beta must be 0.  Same layouts as oracle_ssd_seq.
 */
int oracle_ssd_chunked(const float *x, const float *delta, const float *A,
                       const float *Bm, const float *Cm, const double *h0,
                       double beta, double alpha,
                       int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                       int64_t dstate, int64_t ngroups, int64_t chunk,
                       double *y, double *hT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (beta != 0.0) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || nheads < 1 || headdim < 1 || dstate < 1 ||
        ngroups < 1 || nheads % ngroups != 0 || chunk < 1)
        return ORACLE_ERR_ARG;
    const int64_t heads_per_group = nheads / ngroups;
    const int64_t nchunks = (seqlen + chunk - 1) / chunk;
    const int64_t PN = headdim * dstate;

    int err = ORACLE_OK;
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < batch * nheads; ++bh) {
        const int64_t b = bh / nheads;
        const int64_t hh = bh % nheads;
        const int64_t g = hh / heads_per_group;
        const double a_h = (double)A[hh];
        double *S = (double *)malloc(sizeof(double) * (size_t)PN);     /* S_{c-1} */
        double *s = (double *)malloc(sizeof(double) * (size_t)PN);     /* s_c     */
        double *cs = (double *)malloc(sizeof(double) * (size_t)chunk);
        if (!S || !s || !cs) {
            free(S); free(s); free(cs);
#pragma omp atomic write
            err = ORACLE_ERR_ALLOC;
            continue;
        }
        for (int64_t k = 0; k < PN; ++k)
            S[k] = h0 ? h0[(b * nheads + hh) * PN + k] : 0.0;

        for (int64_t c = 0; c < nchunks; ++c) {
            const int64_t t0 = c * chunk;
            const int64_t q = (t0 + chunk < seqlen) ? chunk : seqlen - t0;
#define X_AT(t, p) ((double)x[((b * seqlen + (t)) * nheads + hh) * headdim + (p)])
#define D_AT(t) ((double)delta[(b * seqlen + (t)) * nheads + hh])
#define B_AT(t, n) ((double)Bm[((b * seqlen + (t)) * ngroups + g) * dstate + (n)])
#define C_AT(t, n) ((double)Cm[((b * seqlen + (t)) * ngroups + g) * dstate + (n)])
#define Y_AT(t, p) y[((b * seqlen + (t)) * nheads + hh) * headdim + (p)]
            /* in-chunk cumulative log-decay */
            double acc = 0.0;
            for (int64_t i = 0; i < q; ++i) {
                acc += D_AT(t0 + i) * a_h;
                cs[i] = acc;
            }
            const double cs_last = cs[q - 1];

            /* step 1 + step 4: intra-chunk output plus the carried state */
            for (int64_t i = 0; i < q; ++i) {
                for (int64_t p = 0; p < headdim; ++p) Y_AT(t0 + i, p) = 0.0;
                for (int64_t j = 0; j <= i; ++j) {
                    double cb = 0.0;                      /* C_i . B_j */
                    for (int64_t n = 0; n < dstate; ++n)
                        cb += C_AT(t0 + i, n) * B_AT(t0 + j, n);
                    const double lij = cb * exp(cs[i] - cs[j]) * alpha * D_AT(t0 + j);
                    for (int64_t p = 0; p < headdim; ++p)
                        Y_AT(t0 + i, p) += lij * X_AT(t0 + j, p);
                }
                const double ei = exp(cs[i]);
                for (int64_t p = 0; p < headdim; ++p) {
                    double yo = 0.0;
                    for (int64_t n = 0; n < dstate; ++n)
                        yo += C_AT(t0 + i, n) * S[p * dstate + n];
                    Y_AT(t0 + i, p) += ei * yo;
                }
            }
            /* step 2: this chunk's own final state from a zero start */
            for (int64_t p = 0; p < headdim; ++p)
                for (int64_t n = 0; n < dstate; ++n) {
                    double acc2 = 0.0;
                    for (int64_t j = 0; j < q; ++j)
                        acc2 += exp(cs_last - cs[j]) * alpha * D_AT(t0 + j) *
                                B_AT(t0 + j, n) * X_AT(t0 + j, p);
                    s[p * dstate + n] = acc2;
                }
            /* step 3: inter-chunk recurrence on the states */
            const double decay = exp(cs_last);
            for (int64_t k = 0; k < PN; ++k) S[k] = decay * S[k] + s[k];
#undef X_AT
#undef D_AT
#undef B_AT
#undef C_AT
#undef Y_AT
        }
        if (hT)
            for (int64_t k = 0; k < PN; ++k) hT[(b * nheads + hh) * PN + k] = S[k];
        free(S);
        free(s);
        free(cs);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Mamba-2 SSD with momentum: the chunked algorithm for beta != 0.          */
/* ------------------------------------------------------------------------ */

/*
 * The [MM] momentum recurrence in the [SSD] chunked form.  Within a chunk of
 * q steps that starts from the states (H0, V0) (P x N per head), with
 * cs_i = sum_{t <= i} delta_t A_h and w_j[p, n] = alpha delta_j B_j[n] x_j[p],
 * unrolling v_i = beta v_{i-1} + w_i and h_i = exp(delta_i A_h) h_{i-1} + v_i
 * gives
 *
 *     v_i = beta^{i+1} V0 + sum_{j <= i} beta^{i-j} w_j
 *     h_i = exp(cs_i) H0 + m_i V0 + sum_{j <= i} M_ij w_j
 *     M_ij = sum_{k=j}^{i} exp(cs_i - cs_k) beta^{k-j}          (j <= i)
 *     m_i  = sum_{k=0}^{i} exp(cs_i - cs_k) beta^{k+1}
 *
 * so the chunk's output and carried states are
 *
 *  1. intra-chunk   Y_diag[i, p] = sum_{j <= i} M_ij (C_i . B_j) alpha delta_j x_j[p]
 *  2. carried in    Y_off[i, p]  = exp(cs_i) C_i . H0[p, :] + m_i C_i . V0[p, :]
 *  3. carried out   H_end = h_{q-1},  V_end = beta^q V0 + sum_j beta^{q-1-j} w_j
 *
 * With beta = 0, M_ij reduces to exp(cs_i - cs_j) and m_i to 0: the 4-step
 * algorithm of oracle_ssd_chunked.  M and m are written as their sums, not a
 * closed form.  Same layouts as oracle_ssd_seq; v0 and vT as h0 and hT.
 */
int oracle_ssd_chunked_momentum(const float *x, const float *delta, const float *A,
                                const float *Bm, const float *Cm, const double *h0,
                                const double *v0, double beta, double alpha,
                                int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                                int64_t dstate, int64_t ngroups, int64_t chunk,
                                double *y, double *hT, double *vT)
{
    if (!x || !delta || !A || !Bm || !Cm || !y) return ORACLE_ERR_ARG;
    if (batch < 1 || seqlen < 1 || nheads < 1 || headdim < 1 || dstate < 1 ||
        ngroups < 1 || nheads % ngroups != 0 || chunk < 1)
        return ORACLE_ERR_ARG;
    const int64_t heads_per_group = nheads / ngroups;
    const int64_t nchunks = (seqlen + chunk - 1) / chunk;
    const int64_t PN = headdim * dstate;

    int err = ORACLE_OK;
    int64_t bh;
#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < batch * nheads; ++bh) {
        const int64_t b = bh / nheads;
        const int64_t hh = bh % nheads;
        const int64_t g = hh / heads_per_group;
        const double a_h = (double)A[hh];
        double *H = (double *)malloc(sizeof(double) * (size_t)PN);
        double *V = (double *)malloc(sizeof(double) * (size_t)PN);
        double *Hn = (double *)malloc(sizeof(double) * (size_t)PN);
        double *Vn = (double *)malloc(sizeof(double) * (size_t)PN);
        double *cs = (double *)malloc(sizeof(double) * (size_t)chunk);
        double *M = (double *)malloc(sizeof(double) * (size_t)chunk * (size_t)chunk);
        double *mv = (double *)malloc(sizeof(double) * (size_t)chunk);
        if (!H || !V || !Hn || !Vn || !cs || !M || !mv) {
            free(H); free(V); free(Hn); free(Vn); free(cs); free(M); free(mv);
#pragma omp atomic write
            err = ORACLE_ERR_ALLOC;
            continue;
        }
        for (int64_t k = 0; k < PN; ++k) {
            H[k] = h0 ? h0[(b * nheads + hh) * PN + k] : 0.0;
            V[k] = v0 ? v0[(b * nheads + hh) * PN + k] : 0.0;
        }
        for (int64_t c = 0; c < nchunks; ++c) {
            const int64_t t0 = c * chunk;
            const int64_t q = (t0 + chunk < seqlen) ? chunk : seqlen - t0;
#define X_AT(t, p) ((double)x[((b * seqlen + (t)) * nheads + hh) * headdim + (p)])
#define D_AT(t) ((double)delta[(b * seqlen + (t)) * nheads + hh])
#define B_AT(t, n) ((double)Bm[((b * seqlen + (t)) * ngroups + g) * dstate + (n)])
#define C_AT(t, n) ((double)Cm[((b * seqlen + (t)) * ngroups + g) * dstate + (n)])
#define Y_AT(t, p) y[((b * seqlen + (t)) * nheads + hh) * headdim + (p)]
            double acc = 0.0;
            for (int64_t i = 0; i < q; ++i) {
                acc += D_AT(t0 + i) * a_h;
                cs[i] = acc;
            }
            /* the chunk's mask and carry weights, as their defining sums */
            for (int64_t i = 0; i < q; ++i) {
                for (int64_t j = 0; j <= i; ++j) {
                    double sum = 0.0;
                    for (int64_t k = j; k <= i; ++k) sum += exp(cs[i] - cs[k]) * pow(beta, (double)(k - j));
                    M[i * chunk + j] = sum;
                }
                double sm = 0.0;
                for (int64_t k = 0; k <= i; ++k) sm += exp(cs[i] - cs[k]) * pow(beta, (double)(k + 1));
                mv[i] = sm;
            }
            /* steps 1 and 2: the chunk's outputs */
            for (int64_t i = 0; i < q; ++i) {
                for (int64_t p = 0; p < headdim; ++p) Y_AT(t0 + i, p) = 0.0;
                for (int64_t j = 0; j <= i; ++j) {
                    double cb = 0.0;
                    for (int64_t n = 0; n < dstate; ++n) cb += C_AT(t0 + i, n) * B_AT(t0 + j, n);
                    const double lij = M[i * chunk + j] * cb * alpha * D_AT(t0 + j);
                    for (int64_t p = 0; p < headdim; ++p) Y_AT(t0 + i, p) += lij * X_AT(t0 + j, p);
                }
                const double ei = exp(cs[i]);
                for (int64_t p = 0; p < headdim; ++p) {
                    double ch = 0.0, cv = 0.0;
                    for (int64_t n = 0; n < dstate; ++n) {
                        ch += C_AT(t0 + i, n) * H[p * dstate + n];
                        cv += C_AT(t0 + i, n) * V[p * dstate + n];
                    }
                    Y_AT(t0 + i, p) += ei * ch + mv[i] * cv;
                }
            }
            /* step 3: the states carried out of the chunk */
            const int64_t last = q - 1;
            const double elast = exp(cs[last]);
            const double bq = pow(beta, (double)q);
            for (int64_t p = 0; p < headdim; ++p)
                for (int64_t n = 0; n < dstate; ++n) {
                    double hs = 0.0, vs = 0.0;
                    for (int64_t j = 0; j < q; ++j) {
                        const double wj = alpha * D_AT(t0 + j) * B_AT(t0 + j, n) * X_AT(t0 + j, p);
                        hs += M[last * chunk + j] * wj;
                        vs += pow(beta, (double)(last - j)) * wj;
                    }
                    const int64_t k = p * dstate + n;
                    Hn[k] = elast * H[k] + mv[last] * V[k] + hs;
                    Vn[k] = bq * V[k] + vs;
                }
            for (int64_t k = 0; k < PN; ++k) {
                H[k] = Hn[k];
                V[k] = Vn[k];
            }
#undef X_AT
#undef D_AT
#undef B_AT
#undef C_AT
#undef Y_AT
        }
        for (int64_t k = 0; k < PN; ++k) {
            if (hT) hT[(b * nheads + hh) * PN + k] = H[k];
            if (vT) vT[(b * nheads + hh) * PN + k] = V[k];
        }
        free(H); free(V); free(Hn); free(Vn); free(cs); free(M); free(mv);
    }
    return err;
}

/* Number of OpenMP threads the oracle's parallel loops use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

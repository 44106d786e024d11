/*
 * mm_oracle.c -- plain, slow, fp64 CPU oracle for the Momentum Mamba forward
 * selective scan and its Mamba-2 scalar-A chunked (SSD) form.
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
 *        "Mamba Module" (step / velocity_state).
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

/*
 * ssm_oracle.c -- plain fp64 CPU oracle for the selective state-space scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only the
 * test suite, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header or constant with the CUDA library and must never be
 * linked into it.
 *
 * What it computes, written out as the definition with no blocking, fusion or
 * reordering (every index is spelled out so it can be checked by eye):
 *
 *   for every sequence b and channel d, starting from h = h0[b,d,:] (zero if absent):
 *     for t = 0 .. L-1:
 *       v      = delta[b,d,t] + bias[d]                      (bias optional)
 *       Delta  = softplus(v) if the flag is set, else v
 *       for n = 0 .. N-1:
 *         Abar = exp(Delta * A[d,n])                         zero-order hold, decay factor
 *         Bbar = Delta * B[b,t,n]                            Euler input gain (default)
 *              = expm1(Delta*A[d,n]) / A[d,n] * B[b,t,n]     exact zero-order hold (mode 1)
 *         h[n] = Abar * h[n] + Bbar * x[b,d,t]               the linear recurrence
 *       y      = sum_n C[b,t,n] * h[n]  +  D[d] * x[b,d,t]   readout plus skip (D optional)
 *       y     *= z * sigmoid(z)                              SiLU gate (z optional)
 *     final_state[b,d,:] = h
 *
 * Sources (page title, section / equation):
 *  - "Module 19: State-Space Models (Mamba)" (learnllm), "The Math: The State-Space
 *    Recurrence": Abar = exp(Delta A), exact ZOH Bbar = A^-1 (exp(Delta A) - I) B,
 *    its small-step (Euler) limit Bbar ~ Delta B, which the lesson names as the form
 *    Mamba's own kernel uses, and the recurrence h_t = Abar h_{t-1} + Bbar x_t,
 *    y_t = C h_t.
 *  - "Beyond attention with Mamba..." (xmarva lesson 10), section 3 "Selectivity":
 *    h_t = exp(Delta_t a) h_{t-1} + Delta_t b_t x_t, y_t = c_t^T h_t; section 4 "The
 *    Mamba block": Delta = softplus(dt_proj(seed) + bias), the skip y + u*D, then the
 *    gate y * SiLU(z), in that order; section 7: the same recurrence for one token.
 *  - "State-space models (Mamba, S4, hybrids)" (askaiml), section 1: y_t = C h_t + D x_t.
 *
 * Readings where the pages are silent: h0 = 0 unless given (the learnllm lesson unrolls
 * the recurrence starting at a zero state); softplus(v) is written in the overflow-free
 * form max(v,0) + log1p(exp(-|v|)), which is the same function; the exact-ZOH gain at
 * A = 0 takes its limit Delta * B.
 *
 * Build:  gcc -O2 -fopenmp -shared -fPIC ssm_oracle.c -o libssm_oracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double oracle_softplus(double v)
{
    /* softplus(v) = log(1 + e^v); the identity softplus(v) = v + softplus(-v) keeps
     * exp() from overflowing for large v. */
    return (v > 0.0 ? v : 0.0) + log1p(exp(-fabs(v)));
}

static double oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* One token of the recurrence for one (sequence, channel): updates h[0..N) in place and
 * returns the gated output.  delta_t is the step after any bias / softplus. */
static double oracle_token(double *h, int64_t N, double delta_t, double x_t,
                           const double *A_d,  /* A[d, 0..N)        */
                           const double *B_t,  /* B[b, t, 0..N)     */
                           const double *C_t,  /* C[b, t, 0..N)     */
                           int has_D, double D_d, int has_z, double z_t, int zoh_exact)
{
    double y = 0.0;
    for (int64_t n = 0; n < N; ++n) {
        double a = A_d[n];
        double Abar = exp(delta_t * a);
        double Bbar;
        if (zoh_exact)
            Bbar = (a == 0.0 ? delta_t : expm1(delta_t * a) / a) * B_t[n];
        else
            Bbar = delta_t * B_t[n];
        h[n] = Abar * h[n] + Bbar * x_t;
        y += C_t[n] * h[n];
    }
    if (has_D)
        y += D_d * x_t;
    if (has_z)
        y *= oracle_silu(z_t);
    return y;
}

/*
 * Full-sequence scan.
 *   x, delta, z, y : [batch][dim][seqlen]
 *   B, C           : [batch][seqlen][dstate]
 *   A              : [dim][dstate]
 *   D, delta_bias  : [dim]                 (NULL = absent)
 *   h0, final_state: [batch][dim][dstate]  (NULL = zero start / not wanted)
 *   z              : NULL = no gate
 * nthreads <= 0 uses the OpenMP default.  Returns the number of threads used, or -1
 * for a size it cannot handle (dstate above 256, negative sizes).
 */
int oracle_scan(const double *x, const double *delta, const double *delta_bias,
                int delta_softplus, const double *A, const double *B, const double *C,
                const double *D, const double *z, const double *h0, int zoh_exact,
                double *y, double *final_state,
                int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, int nthreads)
{
    int used = 1;
    if (dstate < 0 || dstate > 256 || batch < 0 || dim < 0 || seqlen < 0)
        return -1;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    const int64_t channels = batch * dim;
#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        used = omp_get_num_threads();
#endif
        double h[256];
#pragma omp for schedule(dynamic, 1)
        for (int64_t ch = 0; ch < channels; ++ch) {
            const int64_t b = ch / dim;
            const int64_t d = ch % dim;
            for (int64_t n = 0; n < dstate; ++n)
                h[n] = h0 ? h0[(b * dim + d) * dstate + n] : 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                const int64_t i = (b * dim + d) * seqlen + t;
                double v = delta[i] + (delta_bias ? delta_bias[d] : 0.0);
                double dt = delta_softplus ? oracle_softplus(v) : v;
                y[i] = oracle_token(h, dstate, dt, x[i], A + d * dstate,
                                    B + (b * seqlen + t) * dstate,
                                    C + (b * seqlen + t) * dstate,
                                    D != NULL, D ? D[d] : 0.0,
                                    z != NULL, z ? z[i] : 0.0, zoh_exact);
            }
            if (final_state)
                for (int64_t n = 0; n < dstate; ++n)
                    final_state[(b * dim + d) * dstate + n] = h[n];
        }
    }
    return used;
}

/*
 * One decode step (one token per sequence), state updated in place.
 *   state          : [batch][dim][dstate]   in/out
 *   x, delta, z, y : [batch][dim]           delta is the final step (already activated)
 *   B, C           : [batch][dstate]
 *   A              : [dim][dstate];  D: [dim] or NULL;  z: NULL = no gate
 */
void oracle_step(double *state, const double *x, const double *delta, const double *A,
                 const double *B, const double *C, const double *D, const double *z,
                 double *y, int64_t batch, int64_t dim, int64_t dstate)
{
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t i = b * dim + d;
            y[i] = oracle_token(state + i * dstate, dstate, delta[i], x[i], A + d * dstate,
                                B + b * dstate, C + b * dstate, D != NULL, D ? D[d] : 0.0,
                                z != NULL, z ? z[i] : 0.0, 0);
        }
}

/*
 * Causal depthwise convolution of width K, optional bias and SiLU, per (sequence, channel):
 *   u[b,d,t] = act( bias[d] + sum_{i=0..K-1} w[d,i] * xe[b,d,t-(K-1)+i] )
 * where xe is the input preceded by K-1 history values (hist[b,d,0..K-2], oldest first;
 * zeros when hist is NULL -- the left padding by K-1 of the learnllm lesson, section "The
 * Causal Convolution", and of the xmarva lesson's conv1d(padding=k-1)[..., :L], section 4).
 * act is SiLU when silu != 0 (both pages apply SiLU to the convolution output).
 * hist_out[b,d,0..K-2] (optional) receives the last K-1 values of xe: the window a decode
 * step continues from (xmarva lesson, section 7).
 *   x, u: [batch][dim][seqlen]; w: [dim][K]; bias: [dim] or NULL; hist, hist_out: [batch][dim][K-1]
 */
void oracle_causal_conv1d(const double *x, const double *w, const double *bias, const double *hist,
                          int silu, double *u, double *hist_out,
                          int64_t batch, int64_t dim, int64_t seqlen, int64_t K)
{
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            for (int64_t t = 0; t < seqlen; ++t) {
                double acc = bias ? bias[d] : 0.0;
                for (int64_t i = 0; i < K; ++i) {
                    const int64_t src = t - (K - 1) + i;       /* index into x; < 0 means history */
                    double v;
                    if (src >= 0)
                        v = x[row * seqlen + src];
                    else
                        v = hist ? hist[row * (K - 1) + (K - 1) + src] : 0.0;
                    acc += w[d * K + i] * v;
                }
                u[row * seqlen + t] = silu ? oracle_silu(acc) : acc;
            }
            if (hist_out)
                for (int64_t j = 0; j < K - 1; ++j) {
                    const int64_t src = seqlen - (K - 1) + j;
                    hist_out[row * (K - 1) + j] =
                        src >= 0 ? x[row * seqlen + src]
                                 : (hist ? hist[row * (K - 1) + (K - 1) + src] : 0.0);
                }
        }
}

/*
 * One decode token of the convolution: window[b,d,0..K-2] holds the previous K-1 inputs
 * (oldest first); u = act(bias + sum_{i<K-1} w[i] window[i] + w[K-1] x); the window then
 * drops its oldest value and appends x.   window: [batch][dim][K-1] in/out; x, u: [batch][dim].
 */
void oracle_conv1d_step(double *window, const double *x, const double *w, const double *bias,
                        int silu, double *u, int64_t batch, int64_t dim, int64_t K)
{
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            double *win = window + row * (K - 1);
            double acc = bias ? bias[d] : 0.0;
            for (int64_t i = 0; i < K - 1; ++i)
                acc += w[d * K + i] * win[i];
            acc += w[d * K + K - 1] * x[row];
            u[row] = silu ? oracle_silu(acc) : acc;
            for (int64_t i = 0; i + 1 < K - 1; ++i)
                win[i] = win[i + 1];
            if (K > 1)
                win[K - 2] = x[row];
        }
}

/*
 * Backward of the scan (Euler gain): the gradients of a scalar loss
 *     loss = sum_{b,d,t} dy[b,d,t] * y[b,d,t]  +  sum_{b,d,n} dfinal[b,d,n] * h_{L-1}[b,d,n]
 * with respect to every input, by reverse-mode differentiation of the recurrence written
 * above -- the training half that the xmarva lesson (section 6, the paragraph on Mamba's
 * own kernel) describes as recomputing the states in the backward pass instead of
 * storing them.  Here the states of one channel are stored (the oracle has memory to
 * spare); the kernel recomputes them.
 *
 * With h_{-1} = h0, Delta_t, Abar_t[n] = exp(Delta_t A[n]) and y_t as in oracle_scan,
 * going t = L-1 .. 0 with mu[n] = dfinal[n] (the adjoint flowing into h_{L-1} from later
 * tokens):
 *     g_t       = SiLU(z_t)                     (1 without a gate)
 *     dypre_t   = dy_t * g_t                    (adjoint of the pre-gate output)
 *     dz_t      = dy_t * ypre_t * SiLU'(z_t),   SiLU'(z) = s (1 + z (1 - s)), s = sigmoid(z)
 *     lambda[n] = dypre_t C_t[n] + mu[n]        (adjoint of h_t)
 *     dC_t[n]  += dypre_t h_t[n]                dB_t[n] += lambda[n] Delta_t x_t
 *     dx_t      = dypre_t D + sum_n lambda[n] Delta_t B_t[n]
 *     dDelta_t  = sum_n lambda[n] (B_t[n] x_t + h_{t-1}[n] Abar_t[n] A[n])
 *     dA[n]    += lambda[n] h_{t-1}[n] Abar_t[n] Delta_t
 *     mu[n]     = Abar_t[n] lambda[n]           (adjoint of h_{t-1})
 *     ddelta_t  = dDelta_t * sigmoid(delta_t + bias)   (the softplus' slope; 1 without it)
 *     dbias    += ddelta_t,  dD += dypre_t x_t
 * and dh0 = mu after t = 0.  dB, dC sum over channels; dA, dD, dbias over sequences and
 * positions.  Accumulated outputs are zeroed here first.
 *   dy, dx, ddelta, dz : [batch][dim][seqlen];  dB, dC: [batch][seqlen][dstate]
 *   dA: [dim][dstate];  dD, ddelta_bias: [dim];  dfinal, h0, dh0: [batch][dim][dstate]
 * Optional (NULL): dfinal (zero), h0 (zero), D and dD, z and dz, delta_bias and
 * ddelta_bias, dh0.  Returns 0, or -1 for sizes it cannot handle or a failed allocation.
 */
int oracle_scan_bwd(const double *x, const double *delta, const double *delta_bias,
                    int delta_softplus, const double *A, const double *B, const double *C,
                    const double *D, const double *z, const double *h0,
                    const double *dy, const double *dfinal,
                    double *dx, double *ddelta, double *dA, double *dB, double *dC,
                    double *dD, double *dz, double *ddelta_bias, double *dh0,
                    int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate)
{
    if (dstate < 1 || dstate > 256 || batch < 0 || dim < 0 || seqlen < 0)
        return -1;
    const int64_t N = dstate;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((seqlen + 1) * N + 2 * seqlen + 1));
    if (!hs)
        return -1;
    double *step = hs + (seqlen + 1) * N;   /* Delta_t      */
    double *ypre = step + seqlen;           /* y_t before the gate */
    for (int64_t i = 0; i < dim * N; ++i) dA[i] = 0.0;
    for (int64_t i = 0; i < batch * seqlen * N; ++i) { dB[i] = 0.0; dC[i] = 0.0; }
    if (dD) for (int64_t i = 0; i < dim; ++i) dD[i] = 0.0;
    if (ddelta_bias) for (int64_t i = 0; i < dim; ++i) ddelta_bias[i] = 0.0;

    for (int64_t b = 0; b < batch; ++b)
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            const double *x_r = x + row * seqlen;
            const double *A_d = A + d * N;
            /* forward: keep every state, h_{t} at hs[(t+1)*N] and h_{-1} at hs[0] */
            for (int64_t n = 0; n < N; ++n)
                hs[n] = h0 ? h0[row * N + n] : 0.0;
            for (int64_t t = 0; t < seqlen; ++t) {
                double v = delta[row * seqlen + t] + (delta_bias ? delta_bias[d] : 0.0);
                step[t] = delta_softplus ? oracle_softplus(v) : v;
                const double *B_t = B + (b * seqlen + t) * N;
                const double *C_t = C + (b * seqlen + t) * N;
                double yp = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    double h = exp(step[t] * A_d[n]) * hs[t * N + n] + step[t] * B_t[n] * x_r[t];
                    hs[(t + 1) * N + n] = h;
                    yp += C_t[n] * h;
                }
                if (D)
                    yp += D[d] * x_r[t];
                ypre[t] = yp;
            }
            /* reverse */
            double mu[256];
            for (int64_t n = 0; n < N; ++n)
                mu[n] = dfinal ? dfinal[row * N + n] : 0.0;
            for (int64_t t = seqlen - 1; t >= 0; --t) {
                const double dy_t = dy[row * seqlen + t];
                double g = 1.0;
                if (z) {
                    const double zt = z[row * seqlen + t];
                    const double s = 1.0 / (1.0 + exp(-zt));
                    g = zt * s;
                    dz[row * seqlen + t] = dy_t * ypre[t] * s * (1.0 + zt * (1.0 - s));
                }
                const double dypre = dy_t * g;
                const double *B_t = B + (b * seqlen + t) * N;
                const double *C_t = C + (b * seqlen + t) * N;
                double *dB_t = dB + (b * seqlen + t) * N;
                double *dC_t = dC + (b * seqlen + t) * N;
                double dxt = D ? dypre * D[d] : 0.0;
                double dstep = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double lam = dypre * C_t[n] + mu[n];
                    const double abar = exp(step[t] * A_d[n]);
                    const double hprev = hs[t * N + n];
                    dC_t[n] += dypre * hs[(t + 1) * N + n];
                    dB_t[n] += lam * step[t] * x_r[t];
                    dxt += lam * step[t] * B_t[n];
                    dstep += lam * (B_t[n] * x_r[t] + hprev * abar * A_d[n]);
                    dA[d * N + n] += lam * hprev * abar * step[t];
                    mu[n] = abar * lam;
                }
                double dd = dstep;
                if (delta_softplus) {
                    const double v = delta[row * seqlen + t] + (delta_bias ? delta_bias[d] : 0.0);
                    dd *= 1.0 / (1.0 + exp(-v));
                }
                ddelta[row * seqlen + t] = dd;
                if (ddelta_bias)
                    ddelta_bias[d] += dd;
                if (dD)
                    dD[d] += dypre * x_r[t];
                dx[row * seqlen + t] = dxt;
            }
            if (dh0)
                for (int64_t n = 0; n < N; ++n)
                    dh0[row * N + n] = mu[n];
        }
    free(hs);
    return 0;
}

/*
 * Mamba-2 state-space dual (SSD) recurrence, written out as the step-by-step loop of the
 * xmarva lesson 10, section 8 "Mamba-2: the same model as attention": one scalar decay per
 * head, the state of a head a P x N matrix.  Per sequence b and head h, from S = h0 (zero
 * if absent):
 *     for t:  S[p][n] = exp(a[b,t,h]) * S[p][n] + x[b,t,h,p] * B[b,t,h,n]
 *             y[b,t,h,p] = sum_n S[p][n] * C[b,t,h,n]
 * x already carries the step (x = Delta * input) and a = Delta * A, as in that section.
 *   x, y: [batch][L][heads][P];  a: [batch][L][heads];  B, C: [batch][L][heads][N]
 *   h0, hN: [batch][heads][P][N] (NULL: zero start / not wanted)
 * Returns 0, or -1 on a failed allocation or bad sizes.
 */
int oracle_ssd_loop(const double *x, const double *a, const double *B, const double *C,
                    const double *h0, double *y, double *hN,
                    int64_t batch, int64_t L, int64_t heads, int64_t P, int64_t N)
{
    if (batch < 0 || L < 0 || heads < 0 || P < 1 || N < 1)
        return -1;
    double *S = (double *)malloc(sizeof(double) * (size_t)(P * N));
    if (!S)
        return -1;
    for (int64_t b = 0; b < batch; ++b)
        for (int64_t h = 0; h < heads; ++h) {
            for (int64_t i = 0; i < P * N; ++i)
                S[i] = h0 ? h0[((b * heads + h) * P) * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const double e = exp(a[(b * L + t) * heads + h]);
                const double *x_t = x + ((b * L + t) * heads + h) * P;
                const double *B_t = B + ((b * L + t) * heads + h) * N;
                const double *C_t = C + ((b * L + t) * heads + h) * N;
                double *y_t = y + ((b * L + t) * heads + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
                        S[p * N + n] = e * S[p * N + n] + x_t[p] * B_t[n];
                        acc += S[p * N + n] * C_t[n];
                    }
                    y_t[p] = acc;
                }
            }
            if (hN)
                for (int64_t i = 0; i < P * N; ++i)
                    hN[((b * heads + h) * P) * N + i] = S[i];
        }
    free(S);
    return 0;
}

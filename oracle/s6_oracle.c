/*
 * s6_oracle.c -- plain, sequential fp64 CPU oracle for the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (Mamba: Linear-Time Sequence Modeling with Selective State
 * Spaces, page "xyznot.com/ar/paper/2312.00752", sections "Method" and
 * "Selection mechanism (S6)"; plus the serial "MambaMini" scan and the Q&A on
 * page "yongjin360.com/news/29389"):
 *
 *   for every independent (batch, channel) lane, with h[0..N) = h0 (0 if absent):
 *     for t = 0 .. L-1:
 *       x      = delta_raw[t] + delta_bias                 (bias added before tau)
 *       Delta  = softplus(x)  if softplus else x           (tau_Delta = softplus)
 *       for n:  Abar_n = exp(Delta * A[n])                 (ZOH: Abar = exp(Delta A))
 *               h[n]   = Abar_n * h[n] + w_n * B[n,t] * u[t]
 *               w_n    = Delta                             (Bbar = Delta * B, the
 *                                                           element-wise product the
 *                                                           page-2 Q&A describes), or
 *               w_n    = expm1(Delta A[n]) / A[n]          (zoh != 0: the exact ZOH
 *                                                           Bbar = (Delta A)^-1 (exp(Delta A)
 *                                                           - I) Delta B of page 4
 *                                                           "Method"; Delta when A[n] = 0)
 *       y[t]  = (sum_n C[n,t] * h[n] + D * u[t]) * silu(z[t])
 *     last_state = h
 *
 * The output at step t reads the state AFTER the update at step t (h_t = Abar h_{t-1}
 * + Bbar x_t, y_t = C h_t, page 4 "Method").  Absent D / z / delta_bias act as
 * 0 / no gate / 0.  Arithmetic is IEEE double with libm exp/log1p, no fast-math,
 * strictly sequential in t; OpenMP only spreads independent lanes over cores.
 *
 * Every function here is pinned by tests that do not reuse its code: hand-worked
 * examples, the LTI convolution form, the associative-combine prefix, closed
 * forms and limiting cases (see tests/test_oracle_pins.py).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

#define S6O_OK 0
#define S6O_ERR_ARG (-1)
#define S6O_MAX_N 256 /* largest state width the scan accepts */

/* softplus(x) = log(1 + e^x), written so neither branch overflows.
 * Page 4, "Selection mechanism": Delta = tau_Delta(Parameter + s_Delta(x)) with
 * tau_Delta = softplus. */
double s6o_softplus(double x) {
    if (x > 0.0) return x + log1p(exp(-x));
    return log1p(exp(x));
}

/* Step size for one (lane, t): bias first, then the optional softplus. */
static double step_size(double delta_raw, double bias, int softplus) {
    double x = delta_raw + bias;
    return softplus ? s6o_softplus(x) : x;
}

/* Weight of the input in one state's update: Bbar = w * B.  The page-2 Q&A forms Bbar as
 * Delta * B; page 4 "Method" gives the exact zero-order hold Bbar = (Delta A)^-1
 * (exp(Delta A) - I) Delta B, which for a diagonal A is expm1(Delta A_n) / A_n per state
 * (its limit Delta as A_n -> 0).  expm1 keeps the small-(Delta A) case exact. */
static double input_weight(double dt, double a, int zoh) {
    if (!zoh || a == 0.0) return dt;
    return expm1(dt * a) / a;
}

/* SiLU gate: z * sigmoid(z) = z / (1 + e^{-z}) (page 2 Q&A on the gate). */
static double silu(double z) {
    if (z >= 0.0) return z / (1.0 + exp(-z));
    double e = exp(z);
    return z * e / (1.0 + e);
}

/*
 * Discretisation only: Delta[lane, t] and Abar[lane, t, n] = exp(Delta * A[lane, n]).
 * Page 4 "Method" (ZOH: Abar = exp(Delta A)); Delta as in the selection mechanism.
 * Shapes: delta_raw (nlanes, L); A (nlanes, N); delta_bias (nlanes) or NULL.
 */
int s6o_discretize(long nlanes, long N, long L, const double* delta_raw,
                   const double* A, const double* delta_bias, int softplus,
                   double* delta_out, double* abar_out) {
    if (nlanes < 0 || N < 1 || L < 0 || !delta_raw || !A) return S6O_ERR_ARG;
    for (long i = 0; i < nlanes; ++i) {
        double bias = delta_bias ? delta_bias[i] : 0.0;
        for (long t = 0; t < L; ++t) {
            double dt = step_size(delta_raw[i * L + t], bias, softplus);
            if (delta_out) delta_out[i * L + t] = dt;
            if (abar_out)
                for (long n = 0; n < N; ++n)
                    abar_out[(i * L + t) * N + n] = exp(dt * A[i * N + n]);
        }
    }
    return S6O_OK;
}

/*
 * The sequential selective scan over independent lanes.
 *
 *   u, delta_raw, z : (nlanes, L)          z may be NULL (no gate)
 *   A               : (nlanes, N)
 *   D, delta_bias   : (nlanes) or NULL
 *   Bm, Cm          : (nbatch, N, L); lane i reads batch lane_batch[i]
 *   h0              : (nlanes, N) or NULL (zero initial state, h_{-1} = 0)
 *   y               : (nlanes, L)          required
 *   h_last          : (nlanes, N) or NULL
 *   h_all           : (nlanes, L, N) or NULL  every state h_t (small inputs only)
 *   zoh             : 0 for Bbar = Delta B, nonzero for the exact ZOH Bbar
 */
int s6o_scan(long nlanes, long N, long L, long nbatch,
             const double* u, const double* delta_raw, const double* z,
             const double* A, const double* D, const double* delta_bias,
             const double* Bm, const double* Cm, const long* lane_batch,
             int softplus, int zoh, const double* h0,
             double* y, double* h_last, double* h_all) {
    if (nlanes < 0 || N < 1 || N > S6O_MAX_N || L < 0 || nbatch < 1) return S6O_ERR_ARG;
    if (!u || !delta_raw || !A || !Bm || !Cm || !lane_batch || !y) return S6O_ERR_ARG;
    for (long i = 0; i < nlanes; ++i)
        if (lane_batch[i] < 0 || lane_batch[i] >= nbatch) return S6O_ERR_ARG;

#pragma omp parallel for schedule(dynamic, 1)
    for (long i = 0; i < nlanes; ++i) {
        double hv[S6O_MAX_N];
        for (long n = 0; n < N; ++n) hv[n] = h0 ? h0[i * N + n] : 0.0;
        const double* Bb = Bm + lane_batch[i] * N * L;
        const double* Cb = Cm + lane_batch[i] * N * L;
        double bias = delta_bias ? delta_bias[i] : 0.0;
        double dskip = D ? D[i] : 0.0;
        for (long t = 0; t < L; ++t) {
            double ut = u[i * L + t];
            double dt = step_size(delta_raw[i * L + t], bias, softplus);
            double acc = 0.0;
            for (long n = 0; n < N; ++n) {
                double abar = exp(dt * A[i * N + n]);
                double wt = input_weight(dt, A[i * N + n], zoh);
                hv[n] = abar * hv[n] + wt * Bb[n * L + t] * ut;
                acc += Cb[n * L + t] * hv[n];
                if (h_all) h_all[(i * L + t) * N + n] = hv[n];
            }
            acc += dskip * ut;
            if (z) acc *= silu(z[i * L + t]);
            y[i * L + t] = acc;
        }
        if (h_last)
            for (long n = 0; n < N; ++n) h_last[i * N + n] = hv[n];
    }
    return S6O_OK;
}

/*
 * One decode step (selective_state_update): the scan body for a single token,
 * applied in place to the carried state (page 4 FAQ: generation keeps only a
 * fixed D x N state per layer and costs O(1) per token).
 *
 *   state : (nlanes, N) in/out;   u, delta_raw, z : (nlanes)   z may be NULL
 *   A     : (nlanes, N);          D, delta_bias   : (nlanes) or NULL
 *   Bv, Cv: (nbatch, N); lane i reads row lane_batch[i]
 *   y     : (nlanes);                 zoh: as in s6o_scan
 */
int s6o_state_update(long nlanes, long N, long nbatch, double* state,
                     const double* u, const double* delta_raw, const double* z,
                     const double* A, const double* D, const double* delta_bias,
                     const double* Bv, const double* Cv, const long* lane_batch,
                     int softplus, int zoh, double* y) {
    if (nlanes < 0 || N < 1 || nbatch < 1) return S6O_ERR_ARG;
    if (!state || !u || !delta_raw || !A || !Bv || !Cv || !lane_batch || !y)
        return S6O_ERR_ARG;
    for (long i = 0; i < nlanes; ++i)
        if (lane_batch[i] < 0 || lane_batch[i] >= nbatch) return S6O_ERR_ARG;

#pragma omp parallel for schedule(static)
    for (long i = 0; i < nlanes; ++i) {
        const double* Bb = Bv + lane_batch[i] * N;
        const double* Cb = Cv + lane_batch[i] * N;
        double dt = step_size(delta_raw[i], delta_bias ? delta_bias[i] : 0.0, softplus);
        double acc = 0.0;
        for (long n = 0; n < N; ++n) {
            double abar = exp(dt * A[i * N + n]);
            double hn = abar * state[i * N + n] + input_weight(dt, A[i * N + n], zoh) * Bb[n] * u[i];
            state[i * N + n] = hn;
            acc += Cb[n] * hn;
        }
        acc += (D ? D[i] : 0.0) * u[i];
        if (z) acc *= silu(z[i]);
        y[i] = acc;
    }
    return S6O_OK;
}

/*
 * Backward of the scan (gradients of a scalar loss through y), for lanes.
 *
 * Forward recap per lane: x_t = delta_raw_t + bias; Delta_t = softplus(x_t) (or x_t);
 * Abar_tn = exp(Delta_t A_n); q_t = Delta_t u_t; h_tn = Abar_tn h_{t-1,n} + q_t B_tn
 * (h_{-1} = 0); yt_t = sum_n C_tn h_tn + D u_t (pre-gate); y_t = yt_t silu(z_t).
 *
 * Reverse sweep (chain rule, adjoint state g_n = dL/dh_tn accumulated backwards):
 *   dyt_t = dy_t silu(z_t);   dz_t = dy_t yt_t silu'(z_t)
 *   g_n  += dyt_t C_tn                        (g also holds Abar_{t+1} g_{t+1})
 *   dC_tn += dyt_t h_tn;  dB_tn += g_n q_t;   dq_t = sum_n g_n B_tn
 *   dDelta_t = dq_t u_t + sum_n g_n h_{t-1,n} Abar_tn A_n
 *   dA_n += g_n h_{t-1,n} Abar_tn Delta_t;    dD += dyt_t u_t
 *   du_t = dyt_t D + dq_t Delta_t;  dx_t = dDelta_t softplus'(x_t) (= sigmoid(x_t))
 *   dbias += dx_t;  then g_n *= Abar_tn  (carried to step t-1)
 *
 * With zoh nonzero the input weight q_t B_tn becomes w_tn u_t B_tn with the exact ZOH
 * w_tn = expm1(Delta_t A_n) / A_n (Delta_t when A_n = 0), and the terms through it change
 * to the derivatives of w: dB_tn += g_n w_tn u_t; du_t = dyt_t D + sum_n g_n w_tn B_tn;
 * dDelta_t gains sum_n g_n B_tn u_t dw/dDelta with dw/dDelta = Abar_tn (instead of
 * dq_t u_t); dA_n gains g_n B_tn u_t dw/dA with dw/dA = Delta_t^2 psi(Delta_t A_n),
 * psi(y) = (y e^y - expm1(y)) / y^2 = 1/2 + y/3 + y^2/8 + y^3/30 + ... (the series for
 * |y| < 1e-3, where the closed form cancels).
 *
 * Shapes as in s6o_scan; dy (nlanes, L); outputs du, ddelta, dz (nlanes, L);
 * dA (nlanes, N); dD, dbias (nlanes); dB, dC (nbatch, N, L) accumulated over lanes
 * (zeroed here first).  Any output pointer may be NULL except du and ddelta.
 * Sequential over lanes (dB / dC are shared by the lanes of a batch).
 */
static double sigmoid(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    double e = exp(x);
    return e / (1.0 + e);
}

/* psi(y) = (y e^y - expm1(y)) / y^2, the factor of Delta^2 in d(expm1(Delta A) / A) / dA */
static double zoh_psi(double y) {
    if (fabs(y) < 1e-3)
        return 0.5 + y * (1.0 / 3.0 + y * (1.0 / 8.0 + y * (1.0 / 30.0 + y * (1.0 / 144.0))));
    return (y * exp(y) - expm1(y)) / (y * y);
}

int s6o_scan_backward(long nlanes, long N, long L, long nbatch,
                      const double* u, const double* delta_raw, const double* z,
                      const double* A, const double* D, const double* delta_bias,
                      const double* Bm, const double* Cm, const long* lane_batch,
                      int softplus, int zoh, const double* dy,
                      double* du, double* ddelta, double* dz, double* dA, double* dD,
                      double* dbias, double* dB, double* dC) {
    if (nlanes < 0 || N < 1 || N > S6O_MAX_N || L < 0 || nbatch < 1) return S6O_ERR_ARG;
    if (!u || !delta_raw || !A || !Bm || !Cm || !lane_batch || !dy || !du || !ddelta)
        return S6O_ERR_ARG;
    for (long i = 0; i < nlanes; ++i)
        if (lane_batch[i] < 0 || lane_batch[i] >= nbatch) return S6O_ERR_ARG;
    if (dB) for (long k = 0; k < nbatch * N * L; ++k) dB[k] = 0.0;
    if (dC) for (long k = 0; k < nbatch * N * L; ++k) dC[k] = 0.0;
    double* hs = (double*)malloc(sizeof(double) * (size_t)(L + 1) * (size_t)N);
    if (!hs) return S6O_ERR_ARG;
    for (long i = 0; i < nlanes; ++i) {
        const double* Bb = Bm + lane_batch[i] * N * L;
        const double* Cb = Cm + lane_batch[i] * N * L;
        const double bias = delta_bias ? delta_bias[i] : 0.0;
        const double dskip = D ? D[i] : 0.0;
        /* forward, keeping every state: hs[(t+1)*N + n] = h_tn, hs[n] = h_{-1} = 0 */
        for (long n = 0; n < N; ++n) hs[n] = 0.0;
        for (long t = 0; t < L; ++t) {
            const double dt = step_size(delta_raw[i * L + t], bias, softplus);
            for (long n = 0; n < N; ++n)
                hs[(t + 1) * N + n] = exp(dt * A[i * N + n]) * hs[t * N + n] +
                                      input_weight(dt, A[i * N + n], zoh) * u[i * L + t] *
                                          Bb[n * L + t];
        }
        double g[S6O_MAX_N], dAn[S6O_MAX_N];
        for (long n = 0; n < N; ++n) g[n] = 0.0, dAn[n] = 0.0;
        double dDi = 0.0, dbi = 0.0;
        for (long t = L - 1; t >= 0; --t) {
            const double x = delta_raw[i * L + t] + bias;
            const double dt = softplus ? s6o_softplus(x) : x;
            const double ut = u[i * L + t];
            double yt = dskip * ut;
            for (long n = 0; n < N; ++n) yt += Cb[n * L + t] * hs[(t + 1) * N + n];
            double dyt = dy[i * L + t];
            if (z) {
                const double zz = z[i * L + t], sg = sigmoid(zz);
                if (dz) dz[i * L + t] = dy[i * L + t] * yt * sg * (1.0 + zz * (1.0 - sg));
                dyt = dy[i * L + t] * zz * sg;
            } else if (dz) {
                dz[i * L + t] = 0.0;
            }
            double dq = 0.0, ddt = 0.0, duw = 0.0;
            for (long n = 0; n < N; ++n) {
                const double an = A[i * N + n];
                const double abar = exp(dt * an);
                const double w = input_weight(dt, an, zoh);
                g[n] += dyt * Cb[n * L + t];
                if (dC) dC[(lane_batch[i] * N + n) * L + t] += dyt * hs[(t + 1) * N + n];
                if (dB) dB[(lane_batch[i] * N + n) * L + t] += g[n] * w * ut;
                if (zoh) {
                    const double gb = g[n] * Bb[n * L + t];
                    duw += gb * w;                        /* du through the weight */
                    ddt += gb * ut * abar;                /* dw/dDelta = Abar */
                    dAn[n] += gb * ut * dt * dt * zoh_psi(dt * an);  /* dw/dA */
                } else {
                    dq += g[n] * Bb[n * L + t];
                }
                const double gh = g[n] * hs[t * N + n] * abar;
                ddt += gh * an;
                dAn[n] += gh * dt;
                g[n] *= abar;
            }
            ddt += dq * ut;
            dDi += dyt * ut;
            du[i * L + t] = dyt * dskip + (zoh ? duw : dq * dt);
            const double dx = softplus ? ddt * sigmoid(x) : ddt;
            ddelta[i * L + t] = dx;
            dbi += dx;
        }
        if (dA) for (long n = 0; n < N; ++n) dA[i * N + n] = dAn[n];
        if (dD) dD[i] = dDi;
        if (dbias) dbias[i] = dbi;
    }
    free(hs);
    return S6O_OK;
}

/*
 * Causal depthwise 1-D convolution with an optional SiLU, per independent row (one
 * (batch, channel) pair): the step the Mamba block applies to the projected input
 * before the SSM (page 2 Q&A: a convolution first aggregates local context, an
 * activation after it adds the non-linearity; page 4 "Mamba Block": input projections,
 * a 1-D convolution, the selective SSM and multiplicative gating).
 *
 *   out[t] = act(bias + sum_{k=0}^{K-1} w[k] * x[t - (K-1) + k])
 *
 * Inputs before the sequence (t - (K-1) + k < 0) come from init, the K-1 inputs that
 * precede it, oldest first (zero when init is NULL).  act is SiLU when silu != 0, the
 * identity otherwise.  final, when not NULL, receives the last K-1 inputs of the
 * extended sequence init ++ x, oldest first (the state decode continues from).
 *
 *   x, out : (nrows, L);  w : (nrows, K);  bias : (nrows) or NULL
 *   init, final : (nrows, K-1) or NULL;  1 <= K <= 64
 */
int s6o_causal_conv1d(long nrows, long L, long K, const double* x, const double* w,
                      const double* bias, const double* init, int silu_on, double* out,
                      double* final_state) {
    if (nrows < 0 || L < 0 || K < 1 || K > 64 || !w || (L > 0 && (!x || !out)))
        return S6O_ERR_ARG;
    for (long i = 0; i < nrows; ++i) {
        const double* xi = x ? x + i * L : NULL;
        for (long t = 0; t < L; ++t) {
            double acc = bias ? bias[i] : 0.0;
            for (long k = 0; k < K; ++k) {
                long s = t - (K - 1) + k;  /* position in x; negative: before the sequence */
                double v;
                if (s >= 0)
                    v = xi[s];
                else
                    v = init ? init[i * (K - 1) + (K - 1) + s] : 0.0;
                acc += w[i * K + k] * v;
            }
            out[i * L + t] = silu_on ? silu(acc) : acc;
        }
        if (final_state) {
            for (long k = 0; k < K - 1; ++k) {
                long s = L - (K - 1) + k;
                double v;
                if (s >= 0)
                    v = xi[s];
                else
                    v = init ? init[i * (K - 1) + (K - 1) + s] : 0.0;
                final_state[i * (K - 1) + k] = v;
            }
        }
    }
    return S6O_OK;
}

/*
 * One decode token of the same convolution: state (nrows, K-1) holds the previous K-1
 * inputs, oldest first.  out = act(bias + sum_{k<K-1} w[k] state[k] + w[K-1] x); then
 * the state drops its oldest input and appends x.
 */
int s6o_causal_conv1d_update(long nrows, long K, double* state, const double* x,
                             const double* w, const double* bias, int silu_on, double* out) {
    if (nrows < 0 || K < 1 || K > 64 || !x || !w || !out || (K > 1 && !state))
        return S6O_ERR_ARG;
    for (long i = 0; i < nrows; ++i) {
        double acc = bias ? bias[i] : 0.0;
        for (long k = 0; k < K - 1; ++k) acc += w[i * K + k] * state[i * (K - 1) + k];
        acc += w[i * K + K - 1] * x[i];
        out[i] = silu_on ? silu(acc) : acc;
        for (long k = 0; k + 1 < K - 1; ++k) state[i * (K - 1) + k] = state[i * (K - 1) + k + 1];
        if (K > 1) state[i * (K - 1) + K - 2] = x[i];
    }
    return S6O_OK;
}

/*
 * Gradients of sum_t out[t] * dout[t] for the convolution above (the chain rule of its
 * definition; the block trains end to end through it).  With pre[t] the value before
 * the activation and g[t] = dout[t] * act'(pre[t]) (act' = 1 without SiLU, else
 * sigmoid(p) * (1 + p * (1 - sigmoid(p)))):
 *   dx[s]    = sum_k w[k] * g[s + (K-1) - k]        over the t = s + (K-1) - k in [0, L)
 *   dw[k]    = sum_t g[t] * xe[t - (K-1) + k]       (xe = init ++ x, zero before init)
 *   dbias    = sum_t g[t]
 *   dinit[j] = dx at position j - (K-1) of xe, for the K-1 inputs before the sequence
 *              (written only when init and dinit are given)
 * Per row i: dx (nrows, L), dw (nrows, K), dbias (nrows).  dbias may be NULL.
 */
int s6o_causal_conv1d_backward(long nrows, long L, long K, const double* x, const double* w,
                               const double* bias, const double* init, int silu_on,
                               const double* dout, double* dx, double* dw, double* dbias,
                               double* dinit) {
    if (nrows < 0 || L < 0 || K < 1 || K > 64 || !w || !dw || (L > 0 && (!x || !dout || !dx)))
        return S6O_ERR_ARG;
    double* g = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
    if (!g) return S6O_ERR_ARG;
    for (long i = 0; i < nrows; ++i) {
        const double* xi = x ? x + i * L : NULL;
        const double* wi = w + i * K;
        double sb = 0.0;
        for (long t = 0; t < L; ++t) {
            double pre = bias ? bias[i] : 0.0;
            for (long k = 0; k < K; ++k) {
                long s = t - (K - 1) + k;
                double v;
                if (s >= 0)
                    v = xi[s];
                else
                    v = init ? init[i * (K - 1) + (K - 1) + s] : 0.0;
                pre += wi[k] * v;
            }
            double d = 1.0;
            if (silu_on) {
                double sg = 1.0 / (1.0 + exp(-pre));
                d = sg * (1.0 + pre * (1.0 - sg));
            }
            g[t] = dout[i * L + t] * d;
            sb += g[t];
        }
        if (dbias) dbias[i] = sb;
        for (long k = 0; k < K; ++k) {
            double acc = 0.0;
            for (long t = 0; t < L; ++t) {
                long s = t - (K - 1) + k;
                double v;
                if (s >= 0)
                    v = xi[s];
                else
                    v = init ? init[i * (K - 1) + (K - 1) + s] : 0.0;
                acc += g[t] * v;
            }
            dw[i * K + k] = acc;
        }
        /* positions s of xe from -(K-1) to L-1: the outputs t = s + (K-1) - k that read it */
        for (long s = -(K - 1); s < L; ++s) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k) {
                long t = s + (K - 1) - k;
                if (t >= 0 && t < L) acc += wi[k] * g[t];
            }
            if (s >= 0)
                dx[i * L + s] = acc;
            else if (init && dinit)
                dinit[i * (K - 1) + (K - 1) + s] = acc;
        }
    }
    free(g);
    return S6O_OK;
}

/* Threads the OpenMP runtime would use for the parallel loops above. */
#ifdef _OPENMP
#include <omp.h>
int s6o_num_threads(void) { return omp_get_max_threads(); }
/* Threads for the following parallel loops (n >= 1); returns the previous setting. */
int s6o_set_num_threads(int n) {
    int old = omp_get_max_threads();
    if (n >= 1) omp_set_num_threads(n);
    return old;
}
#else
int s6o_num_threads(void) { return 1; }
int s6o_set_num_threads(int n) { (void)n; return 1; }
#endif

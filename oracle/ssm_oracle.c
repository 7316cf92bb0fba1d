/*
 * Float64 CPU oracle for the Mamba selective-SSM scan, the single-token
 * state update, the short convolution, the backward pass and the Mamba-2 layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the package's smoke check and the benchmark's
 * CPU-baseline / reference arm use it.  It shares no code, header, table or
 * constant with the CUDA library.
 *
 * It is the plain definition, written out one step at a time in float64:
 *
 *   Delta_t   = softplus(delta_t + bias_d)   (or delta_t + bias_d, softplus off)
 *   Abar_t,n  = exp(Delta_t * A_d,n)
 *   h_t,n     = Abar_t,n * h_{t-1},n + Delta_t * B_t,n * u_t,   h_{-1} = 0
 *   y_t       = sum_n C_t,n * h_t,n + D_d * u_t
 *   out_t     = y_t * silu(z_t)              (when z is given, else y_t)
 *
 * Two options (the *_ex entry points; the plain ones are Euler, zero start):
 *  - zero-order hold: the input term uses the exact discretisation
 *    Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B, which for the diagonal A
 *    is expm1(Delta A_d,n) / A_d,n * B_t,n (Delta * B_t,n when A_d,n = 0);
 *  - an initial state h_{-1} given per (b, d, n) instead of zero.
 *
 * Sources (page title, section):
 *  - "超越注意力：探索Mamba与状态空间模型" (ai-lab.club), section
 *    "状态空间模型基础": the discretised recurrence h_t = Abar h_{t-1} + Bbar x_t,
 *    y_t = C h_t + D x_t with Abar = exp(Delta A).
 *  - same page, section "选择性状态空间模型": Delta_t = softplus(W x_t + b),
 *    B_t and C_t depend on the token.  Here the projection outputs are inputs
 *    (delta, B, C); the bias b is delta_bias.
 *  - same page, section "代码实现概览": the simplified forward uses the Euler
 *    input matrix Bbar = Delta * B and starts from a zero state.  That is the
 *    default here; the section "状态空间模型基础" zero-order-hold Bbar and a
 *    given start state are the options above.
 *  - "Mamba 与状态空间模型" (world.lapla.si), section "由词元决定": the amount
 *    of old state kept is exp(Delta * A).
 *  - The output gate y * silu(z) is the Mamba block's multiplicative gate; no
 *    page prints it.  silu(z) = z / (1 + exp(-z)).
 *
 * The short causal convolution of the Mamba block ("Mamba 与状态空间模型",
 * section 固定大小的状态: besides its 16 state numbers each channel keeps a
 * short convolution over the 4 most recent inputs) is here too, as the plain
 * weighted sum over a depthwise window of W taps:
 *   out_t = act(bias_d + sum_{k<W} w_d,k x_{t-W+1+k}),  act = silu or identity,
 * where x at negative times comes from a conv state holding the W most recent
 * inputs, oldest first (zero when none is given).  The decode step shifts that
 * state by one, appends x_t and applies the same sum.
 *
 * The backward pass (gradients of the scan) is the adjoint of the same
 * recurrence, taken in reverse time ("Mamba 与状态空间模型", section
 * 在芯片上扫过去: the intermediate states the backward pass needs are not kept
 * but computed again).  With lambda_t = dLoss/dh_t (all paths through later
 * steps included):
 *   lambda_t,n = C_t,n dy_t + Abar_t+1,n lambda_t+1,n   (lambda_L-1 from dlast_state)
 *   dC_t,n = dy_t h_t,n,  dB_t,n = lambda_t,n Delta_t u_t,
 *   dDelta_t = sum_n lambda_t,n (B_t,n u_t + A_n Abar_t,n h_t-1,n),
 *   dA_n = sum_t lambda_t,n Delta_t Abar_t,n h_t-1,n,
 *   du_t = D dy_t + sum_n lambda_t,n Delta_t B_t,n,   dh_-1 = Abar_0 lambda_0,
 * with dy = dout silu(z) and dz = dout y silu'(z) when gated, and the softplus
 * derivative sigmoid(delta + bias) applied to dDelta.
 *
 * The Mamba-2 layer (scalar A per head, a (headdim x dstate) state per head,
 * B and C shared by a group of heads) is the last function, as its plain
 * recurrence; the tests pin it to the lower-triangular matrix the same layer
 * applies ("Mamba 与状态空间模型", section "Mamba-2：两种算法").
 *
 * Loops: chains (b, d) are independent; OpenMP splits them across threads
 * (the backward runs them in order, since its gradients of A, B, C, D and the
 * bias sum over chains).
 * Within a chain, t runs forward one step at a time and n ascends; nothing is
 * blocked, fused or reordered.
 *
 * Layouts (all row-major, contiguous):
 *   scan:   u, delta, z, out (batch, dim, seqlen); B, C (batch, dstate, seqlen);
 *           A (dim, dstate); D, delta_bias (dim); initial_state and
 *           last_state (batch, dim, dstate)
 *   update: state (batch, dim, dstate) read and returned in new_state;
 *           x, dt, z, out (batch, dim); B, C (batch, dstate); A (dim, dstate);
 *           D, dt_bias (dim)
 * Optional pointers (D, z, bias, initial_state, last_state) may be NULL.
 * Return value: 0 on success, -1 on a bad size.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_MAX_DSTATE 256

/* softplus(s) = log(1 + e^s).  For s > 30 the same value is taken as
 * s + log1p(e^-s), which avoids overflowing exp. */
static double oracle_softplus(double s)
{
    if (s > 30.0)
        return s + log1p(exp(-s));
    return log1p(exp(s));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^-z). */
static double oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* Zero-order-hold input gain of one diagonal entry a of A:
 * (Delta a)^-1 (exp(Delta a) - 1) Delta = expm1(Delta a) / a, and Delta in the
 * limit a = 0.  expm1 keeps the digits that exp(Delta a) - 1 would cancel. */
static double oracle_zoh_gain(double dt, double a)
{
    if (a == 0.0)
        return dt;
    return expm1(dt * a) / a;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of later parallel loops (n >= 1), for timing the oracle on one core
 * and on all of them.  The results do not depend on it: every parallel loop
 * runs independent chains (the backward pass runs sequentially). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n >= 1)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_selective_scan_ex_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                 const double *u, const double *delta, const double *A,
                                 const double *B, const double *C, const double *D,
                                 const double *z, const double *delta_bias, int softplus,
                                 int zoh, const double *initial_state, double *out,
                                 double *last_state)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1 || dstate > ORACLE_MAX_DSTATE)
        return -1;

    int64_t chains = batch * dim;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t chain = 0; chain < chains; ++chain) {
        int64_t b = chain / dim;
        int64_t d = chain % dim;
        double h[ORACLE_MAX_DSTATE];
        for (int64_t n = 0; n < dstate; ++n)
            h[n] = initial_state ? initial_state[(b * dim + d) * dstate + n] : 0.0;

        const double *u_row = u + (b * dim + d) * seqlen;
        const double *delta_row = delta + (b * dim + d) * seqlen;
        const double *z_row = z ? z + (b * dim + d) * seqlen : NULL;
        double *out_row = out + (b * dim + d) * seqlen;

        for (int64_t t = 0; t < seqlen; ++t) {
            double dt = delta_row[t];
            if (delta_bias)
                dt += delta_bias[d];
            if (softplus)
                dt = oracle_softplus(dt);
            double x = u_row[t];

            double y = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                double a_dn = A[d * dstate + n];
                double a_bar = exp(dt * a_dn);
                double gain = zoh ? oracle_zoh_gain(dt, a_dn) : dt;
                double b_tn = B[(b * dstate + n) * seqlen + t];
                double c_tn = C[(b * dstate + n) * seqlen + t];
                h[n] = a_bar * h[n] + gain * b_tn * x;
                y += c_tn * h[n];
            }
            if (D)
                y += D[d] * x;
            if (z_row)
                y *= oracle_silu(z_row[t]);
            out_row[t] = y;
        }
        if (last_state)
            for (int64_t n = 0; n < dstate; ++n)
                last_state[(b * dim + d) * dstate + n] = h[n];
    }
    return 0;
}

int oracle_selective_scan_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                              const double *u, const double *delta, const double *A,
                              const double *B, const double *C, const double *D,
                              const double *z, const double *delta_bias, int softplus,
                              double *out, double *last_state)
{
    return oracle_selective_scan_ex_f64(batch, dim, dstate, seqlen, u, delta, A, B, C, D, z,
                                        delta_bias, softplus, 0, NULL, out, last_state);
}

int oracle_selective_state_update_ex_f64(int64_t batch, int64_t dim, int64_t dstate,
                                         const double *state, const double *x, const double *dt,
                                         const double *A, const double *B, const double *C,
                                         const double *D, const double *z, const double *dt_bias,
                                         int dt_softplus, int zoh, double *new_state, double *out)
{
    if (batch < 0 || dim < 0 || dstate < 1 || dstate > ORACLE_MAX_DSTATE)
        return -1;

    int64_t chains = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t chain = 0; chain < chains; ++chain) {
        int64_t b = chain / dim;
        int64_t d = chain % dim;
        double delta = dt[chain];
        if (dt_bias)
            delta += dt_bias[d];
        if (dt_softplus)
            delta = oracle_softplus(delta);
        double xv = x[chain];

        double y = 0.0;
        for (int64_t n = 0; n < dstate; ++n) {
            double a_dn = A[d * dstate + n];
            double a_bar = exp(delta * a_dn);
            double gain = zoh ? oracle_zoh_gain(delta, a_dn) : delta;
            double h = a_bar * state[chain * dstate + n] + gain * B[b * dstate + n] * xv;
            new_state[chain * dstate + n] = h;
            y += C[b * dstate + n] * h;
        }
        if (D)
            y += D[d] * xv;
        if (z)
            y *= oracle_silu(z[chain]);
        out[chain] = y;
    }
    return 0;
}

int oracle_selective_state_update_f64(int64_t batch, int64_t dim, int64_t dstate,
                                      const double *state, const double *x, const double *dt,
                                      const double *A, const double *B, const double *C,
                                      const double *D, const double *z, const double *dt_bias,
                                      int dt_softplus, double *new_state, double *out)
{
    return oracle_selective_state_update_ex_f64(batch, dim, dstate, state, x, dt, A, B, C, D, z,
                                                dt_bias, dt_softplus, 0, new_state, out);
}

/* Input x_s of the conv window for chain `chain`: s >= 0 reads the sequence,
 * s in [-W, -1] the initial conv state (index W + s), zero without one. */
static double oracle_conv_input(const double *x_row, const double *state, int64_t chain,
                                int64_t width, int64_t s)
{
    if (s >= 0)
        return x_row[s];
    return state ? state[chain * width + (width + s)] : 0.0;
}

int oracle_causal_conv1d_f64(int64_t batch, int64_t dim, int64_t seqlen, int64_t width,
                             const double *x, const double *weight, const double *bias,
                             const double *initial_conv_state, int silu, double *out,
                             double *final_conv_state)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || width < 1)
        return -1;

    int64_t chains = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t chain = 0; chain < chains; ++chain) {
        int64_t d = chain % dim;
        const double *x_row = x + chain * seqlen;
        double *out_row = out + chain * seqlen;
        for (int64_t t = 0; t < seqlen; ++t) {
            double acc = bias ? bias[d] : 0.0;
            for (int64_t k = 0; k < width; ++k) {
                int64_t s = t - (width - 1) + k;
                acc += weight[d * width + k] *
                       oracle_conv_input(x_row, initial_conv_state, chain, width, s);
            }
            out_row[t] = silu ? oracle_silu(acc) : acc;
        }
        if (final_conv_state)
            for (int64_t j = 0; j < width; ++j)
                final_conv_state[chain * width + j] =
                    oracle_conv_input(x_row, initial_conv_state, chain, width, seqlen - width + j);
    }
    return 0;
}

int oracle_causal_conv1d_update_f64(int64_t batch, int64_t dim, int64_t width,
                                    const double *conv_state, const double *x,
                                    const double *weight, const double *bias, int silu,
                                    double *new_conv_state, double *out)
{
    if (batch < 0 || dim < 0 || width < 1)
        return -1;

    int64_t chains = batch * dim;
#pragma omp parallel for schedule(static)
    for (int64_t chain = 0; chain < chains; ++chain) {
        int64_t d = chain % dim;
        const double *old = conv_state + chain * width;
        double *cur = new_conv_state + chain * width;
        for (int64_t j = 0; j + 1 < width; ++j)
            cur[j] = old[j + 1];
        cur[width - 1] = x[chain];
        double acc = bias ? bias[d] : 0.0;
        for (int64_t k = 0; k < width; ++k)
            acc += weight[d * width + k] * cur[k];
        out[chain] = silu ? oracle_silu(acc) : acc;
    }
    return 0;
}

/* d silu / dz = sigmoid(z) (1 + z (1 - sigmoid(z))). */
static double oracle_silu_grad(double z)
{
    double sg = 1.0 / (1.0 + exp(-z));
    return sg * (1.0 + z * (1.0 - sg));
}

/* d softplus / ds = sigmoid(s). */
static double oracle_softplus_grad(double s)
{
    return 1.0 / (1.0 + exp(-s));
}

/* Derivative of the zero-order-hold gain g(dt, a) = expm1(dt a) / a with
 * respect to a: (x e^x - expm1(x)) / a^2 with x = dt a, i.e.
 * dt^2 (x e^x - expm1(x)) / x^2.  Near x = 0 the difference cancels, so there
 * the series dt^2 (1/2 + x/3 + x^2/8 + x^3/30 + x^4/144) (coefficients
 * (k + 1) / (k + 2)!) is used; its limit at a = 0 is dt^2 / 2.  (With respect
 * to dt the gain's derivative is exp(dt a) = Abar.) */
static double oracle_zoh_gain_da(double dt, double a)
{
    double x = dt * a;
    if (fabs(x) < 1e-3)
        return dt * dt * (0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0 + x / 144.0))));
    return (x * exp(x) - expm1(x)) / (a * a);
}

/* Gradients of sum_t dout_t out_t + sum_n dlast_n last_state_n with respect to
 * every input of oracle_selective_scan_ex_f64, with the Euler input term
 * (zoh = 0) or the zero-order-hold one (zoh = 1).  With the input gain
 * g = Delta (Euler) or expm1(Delta a) / a (zero-order hold), one step is
 * h_t = Abar h_t-1 + g B_t u_t, and its adjoint, with lambda = dLoss/dh_t:
 *   dB += lambda g u,   du += lambda g B,
 *   dDelta += lambda (dg/dDelta B u + a Abar h_t-1),   dg/dDelta = 1 or Abar,
 *   dA += lambda (Delta Abar h_t-1 + dg/da B u),       dg/da = 0 or
 *         oracle_zoh_gain_da,
 *   lambda_t-1 = Abar lambda.
 * Gradient outputs for NULL inputs may be NULL; all others are overwritten.
 * Returns -1 on a bad size, -2 if the scratch cannot be allocated. */
int oracle_selective_scan_bwd_ex_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                     const double *u, const double *delta, const double *A,
                                     const double *B, const double *C, const double *D,
                                     const double *z, const double *delta_bias, int softplus,
                                     int zoh, const double *initial_state, const double *dout,
                                     const double *dlast_state, double *du, double *ddelta,
                                     double *dA, double *dB, double *dC, double *dD, double *dz,
                                     double *ddelta_bias, double *dinitial_state)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1 || dstate > ORACLE_MAX_DSTATE)
        return -1;
    for (int64_t i = 0; i < dim * dstate; ++i)
        dA[i] = 0.0;
    for (int64_t i = 0; i < batch * dstate * seqlen; ++i) {
        dB[i] = 0.0;
        dC[i] = 0.0;
    }
    if (dD)
        for (int64_t d = 0; d < dim; ++d)
            dD[d] = 0.0;
    if (ddelta_bias)
        for (int64_t d = 0; d < dim; ++d)
            ddelta_bias[d] = 0.0;
    /* states h_t of one chain, t = -1 .. L-1 */
    double *hs = malloc(sizeof(double) * (size_t)(seqlen + 1) * (size_t)dstate);
    double *dts = malloc(sizeof(double) * (size_t)(seqlen > 0 ? seqlen : 1));
    double *ys = malloc(sizeof(double) * (size_t)(seqlen > 0 ? seqlen : 1));
    if (!hs || !dts || !ys) {
        free(hs);
        free(dts);
        free(ys);
        return -2;
    }
    for (int64_t chain = 0; chain < batch * dim; ++chain) {
        int64_t b = chain / dim;
        int64_t d = chain % dim;
        const double *u_row = u + chain * seqlen;
        const double *delta_row = delta + chain * seqlen;
        /* forward, keeping every state */
        for (int64_t n = 0; n < dstate; ++n)
            hs[n] = initial_state ? initial_state[chain * dstate + n] : 0.0;
        for (int64_t t = 0; t < seqlen; ++t) {
            double s = delta_row[t] + (delta_bias ? delta_bias[d] : 0.0);
            double dt = softplus ? oracle_softplus(s) : s;
            dts[t] = dt;
            double y = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                double a_bar = exp(dt * A[d * dstate + n]);
                double gain_f = zoh ? oracle_zoh_gain(dt, A[d * dstate + n]) : dt;
                double h = a_bar * hs[t * dstate + n] + gain_f * B[(b * dstate + n) * seqlen + t] * u_row[t];
                hs[(t + 1) * dstate + n] = h;
                y += C[(b * dstate + n) * seqlen + t] * h;
            }
            ys[t] = y + (D ? D[d] * u_row[t] : 0.0);
        }
        /* reverse */
        double lam[ORACLE_MAX_DSTATE];
        for (int64_t n = 0; n < dstate; ++n)
            lam[n] = dlast_state ? dlast_state[chain * dstate + n] : 0.0;
        for (int64_t t = seqlen - 1; t >= 0; --t) {
            double g = dout[chain * seqlen + t];
            double dy = g;
            if (z) {
                double zt = z[chain * seqlen + t];
                dy = g * oracle_silu(zt);
                if (dz)
                    dz[chain * seqlen + t] = g * ys[t] * oracle_silu_grad(zt);
            }
            double x = u_row[t];
            double dt = dts[t];
            double dut = D ? dy * D[d] : 0.0;
            if (dD)
                dD[d] += dy * x;
            double ddt = 0.0;
            for (int64_t n = 0; n < dstate; ++n) {
                double b_tn = B[(b * dstate + n) * seqlen + t];
                double c_tn = C[(b * dstate + n) * seqlen + t];
                double a_dn = A[d * dstate + n];
                double a_bar = exp(dt * a_dn);
                double h_prev = hs[t * dstate + n];
                double gain = zoh ? oracle_zoh_gain(dt, a_dn) : dt;
                double gain_dt = zoh ? a_bar : 1.0;
                double gain_da = zoh ? oracle_zoh_gain_da(dt, a_dn) : 0.0;
                lam[n] += c_tn * dy;
                dC[(b * dstate + n) * seqlen + t] += dy * hs[(t + 1) * dstate + n];
                dB[(b * dstate + n) * seqlen + t] += lam[n] * gain * x;
                ddt += lam[n] * (gain_dt * b_tn * x + a_dn * a_bar * h_prev);
                dA[d * dstate + n] += lam[n] * (dt * a_bar * h_prev + gain_da * b_tn * x);
                dut += lam[n] * gain * b_tn;
                lam[n] *= a_bar;
            }
            du[chain * seqlen + t] = dut;
            double s = delta_row[t] + (delta_bias ? delta_bias[d] : 0.0);
            double ds = softplus ? ddt * oracle_softplus_grad(s) : ddt;
            ddelta[chain * seqlen + t] = ds;
            if (ddelta_bias)
                ddelta_bias[d] += ds;
        }
        if (dinitial_state)
            for (int64_t n = 0; n < dstate; ++n)
                dinitial_state[chain * dstate + n] = lam[n];
    }
    free(hs);
    free(dts);
    free(ys);
    return 0;
}

/* The Euler-term backward (oracle_selective_scan_bwd_ex_f64 with zoh = 0). */
int oracle_selective_scan_bwd_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                                  const double *u, const double *delta, const double *A,
                                  const double *B, const double *C, const double *D,
                                  const double *z, const double *delta_bias, int softplus,
                                  const double *initial_state, const double *dout,
                                  const double *dlast_state, double *du, double *ddelta,
                                  double *dA, double *dB, double *dC, double *dD, double *dz,
                                  double *ddelta_bias, double *dinitial_state)
{
    return oracle_selective_scan_bwd_ex_f64(batch, dim, dstate, seqlen, u, delta, A, B, C, D, z,
                                            delta_bias, softplus, 0, initial_state, dout,
                                            dlast_state, du, ddelta, dA, dB, dC, dD, dz,
                                            ddelta_bias, dinitial_state);
}

/*
 * Mamba-2 state-space layer with a scalar A per head ("Mamba 与状态空间模型",
 * section "Mamba-2：两种算法": A is one number times the identity, and the layer
 * is one lower-triangular matrix applied to the whole input).  This is the
 * recurrence form of that matrix, step by step in float64.  For every
 * (b, head h) the state S is a (headdim x dstate) matrix:
 *
 *   Delta_t  = softplus(dt_t,h + dt_bias_h)          (or dt + bias, softplus off)
 *   S_t      = exp(Delta_t A_h) S_{t-1} + Delta_t x_t,h B_t,g^T   (S_{-1} = S0 or 0)
 *   y_t,h,p  = sum_n C_t,g,n S_t[p][n] + D_h x_t,h,p
 *   out      = y * silu(z)                            (when z is given)
 *
 * where the head's group is g = h / (nheads / ngroups): B and C are shared by
 * the heads of one group.  The input term is Delta_t x_t B_t (Euler), the same
 * discretisation as the diagonal scan above.
 *
 * Layouts (row-major, contiguous): x, z, out (batch, seqlen, nheads, headdim);
 * dt (batch, seqlen, nheads); A, D, dt_bias (nheads); B, C (batch, seqlen,
 * ngroups, dstate); initial_state, final_state (batch, nheads, headdim,
 * dstate).  D, z, dt_bias, initial_state and final_state may be NULL.
 * Returns 0, or -1 on a bad size (ngroups must divide nheads).
 */
int oracle_ssd_scan_f64(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim,
                        int64_t ngroups, int64_t dstate, const double *x, const double *dt,
                        const double *A, const double *B, const double *C, const double *D,
                        const double *z, const double *dt_bias, int dt_softplus,
                        const double *initial_state, double *out, double *final_state)
{
    if (batch < 0 || seqlen < 0 || nheads < 1 || headdim < 1 || dstate < 1 || ngroups < 1 ||
        nheads % ngroups != 0)
        return -1;
    int64_t heads_per_group = nheads / ngroups;
    int64_t chains = batch * nheads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t chain = 0; chain < chains; ++chain) {
        int64_t b = chain / nheads;
        int64_t h = chain % nheads;
        int64_t g = h / heads_per_group;
        double *S = (double *)malloc(sizeof(double) * headdim * dstate);
        if (!S) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        for (int64_t i = 0; i < headdim * dstate; ++i)
            S[i] = initial_state ? initial_state[chain * headdim * dstate + i] : 0.0;

        for (int64_t t = 0; t < seqlen; ++t) {
            double delta = dt[(b * seqlen + t) * nheads + h];
            if (dt_bias)
                delta += dt_bias[h];
            if (dt_softplus)
                delta = oracle_softplus(delta);
            double decay = exp(delta * A[h]);
            const double *x_t = x + ((b * seqlen + t) * nheads + h) * headdim;
            const double *B_t = B + ((b * seqlen + t) * ngroups + g) * dstate;
            const double *C_t = C + ((b * seqlen + t) * ngroups + g) * dstate;
            double *out_t = out + ((b * seqlen + t) * nheads + h) * headdim;
            const double *z_t = z ? z + ((b * seqlen + t) * nheads + h) * headdim : NULL;
            for (int64_t p = 0; p < headdim; ++p) {
                double *S_p = S + p * dstate;
                double y = 0.0;
                for (int64_t n = 0; n < dstate; ++n) {
                    S_p[n] = decay * S_p[n] + delta * x_t[p] * B_t[n];
                    y += C_t[n] * S_p[n];
                }
                if (D)
                    y += D[h] * x_t[p];
                if (z_t)
                    y *= oracle_silu(z_t[p]);
                out_t[p] = y;
            }
        }
        if (final_state)
            for (int64_t i = 0; i < headdim * dstate; ++i)
                final_state[chain * headdim * dstate + i] = S[i];
        free(S);
    }
    return failed ? -1 : 0;
}

/*
 * mamba_oracle.c -- fp64 CPU oracle of the Mamba selective scan and of the
 * single-token selective state update.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg use it. It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (sources are the web pages on Mamba this project follows):
 *  - "Mamba (deep learning)" wiki page, paragraph on state space models: the
 *    discretised transition is A_bar = exp(Delta*A), applied per state.
 *  - "Mamba-1/2/3 Markdown図解" blog, section 1 (数式で見ると): the recurrence
 *    h_t = A_bar_t h_{t-1} + B_bar_t x_t and the readout y_t = C_t h_t.
 *  - Same blog, section 2 (Mamba-1): Delta_t, B_t, C_t are per-token inputs
 *    (selectivity); the block gates the SSM output with a second branch.
 *  - The input term B_bar_t x_t is taken as Delta_t * B_t * u_t (Euler form of
 *    the input; the pages lost that equation), Delta_t = softplus(delta_t +
 *    bias_d) when the softplus flag is set, the D skip sits inside the gate,
 *    and the gate is silu(z) = z * sigmoid(z). These are the readings this
 *    project fixes for steps the pages leave open.
 *  - Generation is the same recurrence taken one token at a time from a stored
 *    state (blog, section 2, "1トークン生成 → recurrent update").
 *  - The block's input path (blog, section 2, block diagram): the projected
 *    input passes a short causal convolution along the tokens, one filter per
 *    channel, then silu, and the result is the SSM's input u. Read here as
 *    u_t = silu(bias_d + sum_{k<W} w[d][k] * x_{t-(W-1)+k}), with the W-1
 *    tokens before t = 0 taken from a given history or zero.
 *
 * Layouts (all arrays dense, row-major, fp64):
 *   u, delta, z, y      [batch][dim][seqlen]
 *   A                   [dim][dstate]
 *   B, C                [batch][dstate][seqlen]   (one group shared by all dim)
 *   D, delta_bias       [dim]
 *   h0, last_state      [batch][dim][dstate]
 *   decode: x, delta, z, y [batch][dim]; B, C [batch][dstate]; state [batch][dim][dstate]
 * Nullable: D, z, delta_bias, h0 (zero initial state), last_state.
 *   conv: x, u [batch][dim][seqlen]; w [dim][W]; bias [dim]; x0 [batch][dim][W-1]
 *   (x0[b][d][j] is x_{-(W-1)+j}); bias and x0 nullable.
 *
 * Built with -O2 and no fast-math; exp/log1p are the C library's.
 * ORACLE_MUTANT (compile-time, tests only) plants one known mistake so that a
 * test can show the pins catch it; the default build plants none.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <pthread.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* softplus(x) = log(1 + e^x), written so that neither branch overflows. */
double oracle_softplus(double x)
{
    double ax = fabs(x);
    return (x > 0.0 ? x : 0.0) + log1p(exp(-ax));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^-z). */
double oracle_silu(double z)
{
#if ORACLE_MUTANT == 8
    return 1.0 / (1.0 + exp(-z)); /* mutant: sigmoid gate instead of silu */
#else
    return z / (1.0 + exp(-z));
#endif
}

/* Delta_t from the raw per-token value: bias added first, then softplus. */
static double step_size(double raw, double bias, int softplus_flag)
{
#if ORACLE_MUTANT == 7
    (void)bias;
    double v = raw; /* mutant: bias dropped */
#else
    double v = raw + bias;
#endif
#if ORACLE_MUTANT == 6
    (void)softplus_flag;
    return v; /* mutant: softplus never applied */
#else
    return softplus_flag ? oracle_softplus(v) : v;
#endif
}

/*
 * One channel (b, d) over tokens [0, L): the recurrence of the blog's
 * section 1 with A_bar = exp(Delta*A) (wiki page) per state n, readout C.h,
 * D skip, then the silu(z) gate. h (length N) is the running state: on entry
 * the initial state, on exit the state after token L-1.
 * Strides: u/delta/z/y step 1 per token; B/C: element (n, t) at n*bc_sn + t.
 */
static void scan_channel(int64_t N, int64_t L,
                         const double *u, const double *delta, const double *A_d,
                         const double *B, const double *C, int64_t bc_sn,
                         const double *D_d, const double *z, const double *bias_d,
                         int softplus_flag, double *h, double *y)
{
    for (int64_t t = 0; t < L; ++t) {
        double dt = step_size(delta[t], bias_d ? *bias_d : 0.0, softplus_flag);
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 10
            double A_n = A_d[N - 1 - n]; /* mutant: state index reversed in A */
#else
            double A_n = A_d[n];
#endif
#if ORACLE_MUTANT == 2
            double abar = exp(-dt * A_n); /* mutant: wrong sign in the exponent */
#else
            double abar = exp(dt * A_n);
#endif
#if ORACLE_MUTANT == 3
            double bx = u[t] * B[n * bc_sn + t]; /* mutant: Delta dropped from the input term */
#elif ORACLE_MUTANT == 5
            double bx = dt * u[t] * C[n * bc_sn + t]; /* mutant: B and C swapped */
#elif ORACLE_MUTANT == 9
            double bx = dt * u[t] * (t > 0 ? B[n * bc_sn + t - 1] : 0.0); /* mutant: B one token late */
#else
            double bx = dt * u[t] * B[n * bc_sn + t];
#endif
#if ORACLE_MUTANT == 4
            acc += (ORACLE_MUTANT == 5 ? B : C)[n * bc_sn + t] * h[n]; /* mutant: readout before update */
            h[n] = abar * h[n] + bx;
#else
            h[n] = abar * h[n] + bx;
#if ORACLE_MUTANT == 5
            acc += B[n * bc_sn + t] * h[n];
#else
            acc += C[n * bc_sn + t] * h[n];
#endif
#endif
        }
#if ORACLE_MUTANT == 1
        double yv = acc; /* mutant: D skip dropped */
#else
        double yv = acc + (D_d ? *D_d : 0.0) * u[t];
#endif
        if (z) yv *= oracle_silu(z[t]);
        y[t] = yv;
    }
}

/* Scan over channels [c0, c1) of the flattened (batch, dim) range. */
static void scan_range(int64_t c0, int64_t c1, int64_t batch, int64_t dim, int64_t N, int64_t L,
                       const double *u, const double *delta, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *z, const double *delta_bias, int softplus_flag,
                       const double *h0, double *y, double *last_state)
{
    (void)batch;
    double *h = (double *)malloc((size_t)N * sizeof(double));
    if (!h) return;
    for (int64_t c = c0; c < c1; ++c) {
        int64_t b = c / dim, d = c % dim;
        for (int64_t n = 0; n < N; ++n) h[n] = h0 ? h0[c * N + n] : 0.0;
        const int64_t row = c * L;
        scan_channel(N, L, u + row, delta + row, A + d * N,
                     B + b * N * L, C + b * N * L, L,
                     D ? D + d : NULL, z ? z + row : NULL,
                     delta_bias ? delta_bias + d : NULL, softplus_flag, h, y + row);
#if ORACLE_MUTANT == 12
        (void)last_state; /* mutant: final state never written */
#else
        if (last_state)
            for (int64_t n = 0; n < N; ++n) last_state[c * N + n] = h[n];
#endif
    }
    free(h);
}

/*
 * Selective scan over a whole batch. Returns 0, or -1 on a bad size or a
 * missing required array.
 */
int oracle_scan_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                    const double *u, const double *delta, const double *A,
                    const double *B, const double *C, const double *D,
                    const double *z, const double *delta_bias, int softplus_flag,
                    const double *h0, double *y, double *last_state)
{
    if (batch < 0 || dim < 0 || dstate < 1 || seqlen < 0) return -1;
    if (batch * dim * seqlen > 0 && (!u || !delta || !A || !B || !C || !y)) return -1;
    scan_range(0, batch * dim, batch, dim, dstate, seqlen, u, delta, A, B, C, D, z,
               delta_bias, softplus_flag, h0, y, last_state);
    return 0;
}

struct mt_job {
    int64_t c0, c1, batch, dim, N, L;
    const double *u, *delta, *A, *B, *C, *D, *z, *bias, *h0;
    int flag;
    double *y, *last;
};

static void *mt_worker(void *p)
{
    struct mt_job *j = (struct mt_job *)p;
    scan_range(j->c0, j->c1, j->batch, j->dim, j->N, j->L, j->u, j->delta, j->A, j->B,
               j->C, j->D, j->z, j->bias, j->flag, j->h0, j->y, j->last);
    return NULL;
}

/*
 * Same result as oracle_scan_f64; the independent (batch, dim) channels are
 * split over nthreads POSIX threads. The per-channel arithmetic is unchanged.
 */
int oracle_scan_f64_mt(int nthreads, int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                       const double *u, const double *delta, const double *A,
                       const double *B, const double *C, const double *D,
                       const double *z, const double *delta_bias, int softplus_flag,
                       const double *h0, double *y, double *last_state)
{
    if (nthreads <= 1)
        return oracle_scan_f64(batch, dim, dstate, seqlen, u, delta, A, B, C, D, z,
                               delta_bias, softplus_flag, h0, y, last_state);
    if (batch < 0 || dim < 0 || dstate < 1 || seqlen < 0) return -1;
    int64_t nch = batch * dim;
    if (nch * seqlen > 0 && (!u || !delta || !A || !B || !C || !y)) return -1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    struct mt_job jobs[256];
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        struct mt_job j = {nch * i / nthreads, nch * (i + 1) / nthreads, batch, dim, dstate, seqlen,
                           u, delta, A, B, C, D, z, delta_bias, h0, softplus_flag, y, last_state};
        jobs[i] = j;
        if (pthread_create(&th[i], NULL, mt_worker, &jobs[i]) == 0) {
            ++started;
        } else {
            mt_worker(&jobs[i]); /* could not start a thread: do this share here */
            th[i] = 0;
        }
    }
    for (int i = 0; i < nthreads; ++i)
        if (th[i]) pthread_join(th[i], NULL);
    (void)started;
    return 0;
}

/*
 * Single-token selective state update for a batch: for every (b, d) one step
 * of the recurrence from the stored state, which is read and overwritten.
 * x is the token input (u in the scan's notation).
 */
int oracle_state_update_f64(int64_t batch, int64_t dim, int64_t dstate,
                            double *state, const double *x, const double *delta,
                            const double *A, const double *B, const double *C,
                            const double *D, const double *z, const double *delta_bias,
                            int softplus_flag, double *y)
{
    if (batch < 0 || dim < 0 || dstate < 1) return -1;
    if (batch * dim > 0 && (!state || !x || !delta || !A || !B || !C || !y)) return -1;
    const int64_t N = dstate;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            int64_t c = b * dim + d;
#if ORACLE_MUTANT == 11
            for (int64_t n = 0; n < N; ++n) state[c * N + n] = 0.0; /* mutant: stored state ignored */
#endif
            /* One token: the same per-channel step as the scan with L = 1; B/C
               for this batch row hold one value per state (stride 1 in n). */
            scan_channel(N, 1, x + c, delta + c, A + d * N, B + b * N, C + b * N, 1,
                         D ? D + d : NULL, z ? z + c : NULL,
                         delta_bias ? delta_bias + d : NULL, softplus_flag,
                         state + c * N, y + c);
        }
    }
    return 0;
}

/*
 * Causal depthwise convolution of the block's input path, then silu (when
 * silu_flag): for every (b, d) and token t,
 *   u_t = act(bias_d + sum_{k=0}^{W-1} w[d][k] * x_{t-(W-1)+k}),
 * where x_s for s < 0 is x0[b][d][s + W - 1] (zero when x0 is NULL). The
 * filter's last tap w[d][W-1] weights the current token. Returns 0, or -1 on
 * a bad size or a missing required array.
 */
int oracle_causal_conv_f64(int64_t batch, int64_t dim, int64_t seqlen, int64_t width,
                           const double *x, const double *w, const double *bias,
                           const double *x0, int silu_flag, double *u)
{
    if (batch < 0 || dim < 0 || seqlen < 0 || width < 1) return -1;
    if (batch * dim * seqlen > 0 && (!x || !w || !u)) return -1;
    const int64_t W = width;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t c = b * dim + d;
            const double *xr = x + c * seqlen;
            for (int64_t t = 0; t < seqlen; ++t) {
                double acc = bias ? bias[d] : 0.0;
                for (int64_t k = 0; k < W; ++k) {
                    const int64_t s = t - (W - 1) + k; /* token under tap k */
                    double xs;
                    if (s >= 0) {
                        xs = xr[s];
                    } else {
#if ORACLE_MUTANT == 15
                        xs = 0.0; /* mutant: history before token 0 ignored */
#else
                        xs = x0 ? x0[c * (W - 1) + (s + W - 1)] : 0.0;
#endif
                    }
#if ORACLE_MUTANT == 13
                    acc += w[d * W + (W - 1 - k)] * xs; /* mutant: filter taps reversed */
#else
                    acc += w[d * W + k] * xs;
#endif
                }
#if ORACLE_MUTANT == 14
                (void)silu_flag;
                u[c * seqlen + t] = acc; /* mutant: activation dropped */
#else
                u[c * seqlen + t] = silu_flag ? oracle_silu(acc) : acc;
#endif
            }
        }
    }
    return 0;
}

/*
 * Gradients of the selective scan (reverse mode of the recurrence above; the
 * blog's section 2 notes the same model is trained through the scan). For a
 * scalar loss with dL/dy = dout [batch][dim][seqlen] on the gated output and
 * dL/dlast_state = dlast [batch][dim][dstate] (nullable = 0), per channel:
 *   forward, kept per token: Delta_t, A_bar_t[n], h_t[n], the pre-gate output
 *     q_t = sum_n C_t[n] h_t[n] + D u_t, and the gate g_t = silu(z_t) (1 without z);
 *   backward over t = L-1 .. 0, with lam the adjoint of h_t:
 *     dq_t = dout_t g_t;  dz_t = dout_t q_t silu'(z_t);  dD += dq_t u_t;  du_t = D dq_t
 *     lam[n] = C_t[n] dq_t + carry[n]           (carry = dlast at t = L-1)
 *     dC_t[n] += dq_t h_t[n]
 *     dh_{t-1}[n] through A_bar: dAbar = lam[n] h_{t-1}[n]
 *     dA[n] += dAbar A_bar_t[n] Delta_t;  dDelta_t += dAbar A_bar_t[n] A[n]
 *     input term Delta_t u_t B_t[n]: dDelta_t += lam u_t B_t[n]; du_t += lam Delta_t B_t[n];
 *                                    dB_t[n] += lam Delta_t u_t
 *     carry[n] = A_bar_t[n] lam[n]
 *   ddelta_t = dDelta_t * sigmoid(delta_t + bias) (softplus' ; 1 without the flag),
 *   dbias += ddelta_t, dh0 = carry after t = 0.
 * dB, dC, dA, dD, dbias are sums over channels/tokens/batch and are
 * ACCUMULATED into (callers zero them); du, ddelta, dz, dh0 are written.
 * Nullable outputs: dz (needs z), dD, dbias, dh0; nullable inputs as the scan.
 */
static double silu_grad(double z)
{
    double s = 1.0 / (1.0 + exp(-z));
#if ORACLE_MUTANT == 16
    return s; /* mutant: derivative of silu missing the z*s*(1-s) term */
#else
    return s * (1.0 + z * (1.0 - s));
#endif
}

int oracle_scan_bwd_f64(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                        const double *u, const double *delta, const double *A,
                        const double *B, const double *C, const double *D,
                        const double *z, const double *delta_bias, int softplus_flag,
                        const double *h0, const double *dout, const double *dlast,
                        double *du, double *ddelta, double *dA, double *dB, double *dC,
                        double *dD, double *dz, double *dbias, double *dh0)
{
    if (batch < 0 || dim < 0 || dstate < 1 || seqlen < 0) return -1;
    if (batch * dim * seqlen > 0 &&
        (!u || !delta || !A || !B || !C || !dout || !du || !ddelta || !dA || !dB || !dC)) return -1;
    const int64_t N = dstate, L = seqlen;
    double *hs = (double *)malloc((size_t)((L + 1) * N) * sizeof(double)); /* h_{-1..L-1} */
    double *ab = (double *)malloc((size_t)((L > 0 ? L : 1) * N) * sizeof(double));
    double *dts = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    double *q = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    double *lam = (double *)malloc((size_t)N * sizeof(double));
    double *carry = (double *)malloc((size_t)N * sizeof(double));
    if (!hs || !ab || !dts || !q || !lam || !carry) {
        free(hs); free(ab); free(dts); free(q); free(lam); free(carry);
        return -1;
    }
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t c = b * dim + d, row = c * L;
            const double *Bb = B + b * N * L, *Cb = C + b * N * L;
            const double Dd = D ? D[d] : 0.0, bias = delta_bias ? delta_bias[d] : 0.0;
            /* forward, keeping what the backward needs */
            for (int64_t n = 0; n < N; ++n) hs[n] = h0 ? h0[c * N + n] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const double dt = step_size(delta[row + t], bias, softplus_flag);
                dts[t] = dt;
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = exp(dt * A[d * N + n]);
                    ab[t * N + n] = a;
                    const double h = a * hs[t * N + n] + dt * u[row + t] * Bb[n * L + t];
                    hs[(t + 1) * N + n] = h;
                    acc += Cb[n * L + t] * h;
                }
                q[t] = acc + Dd * u[row + t];
            }
            /* backward */
            for (int64_t n = 0; n < N; ++n) carry[n] = dlast ? dlast[c * N + n] : 0.0;
            double dDacc = 0.0, dbacc = 0.0;
            for (int64_t t = L - 1; t >= 0; --t) {
                const double ut = u[row + t], dt = dts[t];
                const double g = z ? oracle_silu(z[row + t]) : 1.0;
                const double dq = dout[row + t] * g;
                if (z && dz) dz[row + t] = dout[row + t] * q[t] * silu_grad(z[row + t]);
                dDacc += dq * ut;
                double dut = Dd * dq, ddt = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double Bt = Bb[n * L + t], Ct = Cb[n * L + t];
                    const double ht = hs[(t + 1) * N + n], hprev = hs[t * N + n];
                    const double a = ab[t * N + n];
#if ORACLE_MUTANT == 17
                    lam[n] = Ct * dq + a * carry[n]; /* mutant: adjoint decayed by this token's A_bar */
#else
                    lam[n] = Ct * dq + carry[n];
#endif
                    dC[b * N * L + n * L + t] += dq * ht;
                    const double dab = lam[n] * hprev;
                    dA[d * N + n] += dab * a * dt;
#if ORACLE_MUTANT == 18
                    (void)0; /* mutant: Delta's path through A_bar dropped */
#else
                    ddt += dab * a * A[d * N + n];
#endif
                    ddt += lam[n] * ut * Bt;
                    dut += lam[n] * dt * Bt;
                    dB[b * N * L + n * L + t] += lam[n] * dt * ut;
                    carry[n] = a * lam[n];
                }
                const double v = delta[row + t] + bias;
                const double dv = softplus_flag ? ddt / (1.0 + exp(-v)) : ddt;
                du[row + t] = dut;
                ddelta[row + t] = dv;
                dbacc += dv;
            }
            if (dD) dD[d] += dDacc;
            if (dbias) dbias[d] += dbacc;
            if (dh0)
                for (int64_t n = 0; n < N; ++n) dh0[c * N + n] = carry[n];
        }
    }
    free(hs); free(ab); free(dts); free(q); free(lam); free(carry);
    return 0;
}

/*
 * Mamba-2 state space duality layer ('Mamba-1/2/3 Markdown図解' blog,
 * section 3: one model with a recurrent view, used for decoding, and a
 * matrix view computed chunk by chunk for training and prefill; the
 * transition is a scalar times the identity within a head). This oracle is
 * the recurrent view. For batch b, head h (head dim P, state N, group
 * g = h / (H / G) sharing B and C):
 *   Delta_t = softplus(dt[b,t,h] + dt_bias[h])  (plain sum without the flag)
 *   S_t[p][n] = exp(Delta_t A[h]) S_{t-1}[p][n] + Delta_t B[b,t,g,n] x[b,t,h,p]
 *   y[b,t,h,p] = sum_n C[b,t,g,n] S_t[p][n] + D[h] x[b,t,h,p]
 * Layouts (dense, fp64): x, y [b][L][H][P]; dt [b][L][H]; B, C [b][L][G][N];
 * A, D, dt_bias [H]; s0, s_last [b][H][P][N]. Nullable: D, dt_bias, s0 (zero),
 * s_last.
 */
int oracle_ssd_f64(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                   int64_t ngroups, const double *x, const double *dt, const double *A,
                   const double *B, const double *C, const double *D, const double *dt_bias,
                   int softplus_flag, const double *s0, double *y, double *s_last)
{
    const int64_t H = nheads, P = headdim, N = dstate, G = ngroups, L = seqlen;
    if (batch < 0 || L < 0 || H < 1 || P < 1 || N < 1 || G < 1 || H % G != 0) return -1;
    if (batch * L > 0 && (!x || !dt || !A || !B || !C || !y)) return -1;
    double *S = (double *)malloc((size_t)(P * N) * sizeof(double));
    if (!S) return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t h = 0; h < H; ++h) {
#if ORACLE_MUTANT == 19
            const int64_t g = h % G; /* mutant: heads assigned to groups round-robin */
#else
            const int64_t g = h / (H / G);
#endif
            for (int64_t i = 0; i < P * N; ++i) S[i] = s0 ? s0[(b * H + h) * P * N + i] : 0.0;
            for (int64_t t = 0; t < L; ++t) {
                const double dlt = step_size(dt[(b * L + t) * H + h], dt_bias ? dt_bias[h] : 0.0, softplus_flag);
                const double a = exp(dlt * A[h]);
                const double *Bt = B + ((b * L + t) * G + g) * N;
                const double *Ct = C + ((b * L + t) * G + g) * N;
                const double *xt = x + ((b * L + t) * H + h) * P;
                double *yt = y + ((b * L + t) * H + h) * P;
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t n = 0; n < N; ++n) {
#if ORACLE_MUTANT == 20
                        S[p * N + n] = a * (S[p * N + n] + dlt * Bt[n] * xt[p]); /* mutant: input decayed too */
#elif ORACLE_MUTANT == 21
                        S[p * N + n] = a * S[p * N + n] + Bt[n] * xt[p]; /* mutant: Delta dropped from the input */
#else
                        S[p * N + n] = a * S[p * N + n] + dlt * Bt[n] * xt[p];
#endif
                        acc += Ct[n] * S[p * N + n];
                    }
                    yt[p] = acc + (D ? D[h] : 0.0) * xt[p];
                }
            }
            if (s_last)
                for (int64_t i = 0; i < P * N; ++i) s_last[(b * H + h) * P * N + i] = S[i];
        }
    }
    free(S);
    return 0;
}

/*
 * s6_oracle.c -- plain fp64 CPU reference of the selective scan (S6) forward
 * pass and of its one-token state update.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test-suite, the smoke check and the benchmark's CPU
 * baseline use it.  It shares no code, header, table or constant with the CUDA
 * library.
 *
 * What it computes (one independent recurrence per (batch b, channel d)).
 * Sources are sections of the page "Mamba SSM concept and implementation in
 * Keras and TensorFlow":
 *
 *   delta_t = delta_raw[b,d,t] + bias[d]              the bias belongs to the dt
 *                                                     projection and is applied
 *                                                     before softplus (MambaBlock.ssm)
 *   delta_t = softplus(delta_t)   if the flag is set  (MambaBlock.ssm)
 *   Abar    = exp(delta_t * A[d,n])                   zero-order hold of A ("Going from
 *                                                     continuous to discrete spaces";
 *                                                     the selective_scan listing forms
 *                                                     delta*A and exponentiates it)
 *   Bbar u  = delta_t * B[b,n,t] * u[b,d,t]           the simplified B discretisation of
 *                                                     the selective_scan listing
 *   h_t[n]  = Abar * h_{t-1}[n] + Bbar u              recurrent form; h_{-1} = h0, zero
 *                                                     by default (the page unrolls the
 *                                                     recurrence from a zero state)
 *   y_t     = sum_n C[b,n,t] * h_t[n] + D[d] * u[b,d,t]   readout plus the D skip
 *                                                     connection (selective_scan)
 *   out_t   = y_t * silu(z[b,d,t])    if z is given   the gate of MambaBlock.call (swish of
 *                                                     the residual half of the input
 *                                                     projection)
 *   last_state[b,d,n] = h_{L-1}[n]
 *
 * and, for the step before the scan in the same block, the causal depthwise
 * convolution with bias and silu that produces u (s6_oracle_conv1d, and its
 * one-token form s6_oracle_conv1d_update; equations beside them).
 *
 * Layouts (row-major, contiguous):
 *   u, delta_raw, z, out : (batch, dim, seqlen)
 *   B, C                 : (batch, dstate, seqlen)
 *   A                    : (dim, dstate)
 *   D, bias              : (dim)
 *   h0, last_state, state: (batch, dim, dstate)
 *
 * Inputs arrive as fp32 arrays holding the exact values the device sees
 * (bf16 values widen to fp32 exactly); every operation below is done in fp64,
 * in the order written above, with no blocking, fusion or reordering.
 * Time is strictly sequential; independent (b, d) rows are spread over
 * POSIX threads, which does not change any result.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <unistd.h>

/* softplus(x) = ln(1 + e^x), written in the overflow-free split form
 * max(x, 0) + ln(1 + e^{-|x|}); the Keras/TensorFlow page applies
 * tf.nn.softplus to the dt projection. */
double s6_oracle_softplus(double x)
{
    if (x > 0.0)
        return x + log1p(exp(-x));
    return log1p(exp(x));
}

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z}) (the page's tf.nn.swish). */
double s6_oracle_silu(double z)
{
    return z / (1.0 + exp(-z));
}

typedef struct {
    const float *u, *delta, *A, *B, *C, *D, *z, *bias;
    const double *h0;
    int softplus;
    double *out, *last_state;
    int64_t dim, seqlen, dstate;
    int64_t row_begin, row_end; /* rows are flattened (b * dim + d) */
} scan_job_t;

/* One (b, d) recurrence over the whole sequence. */
static void scan_row(const scan_job_t *j, int64_t row, double *h)
{
    const int64_t L = j->seqlen, N = j->dstate;
    const int64_t b = row / j->dim, d = row % j->dim;
    const float *u = j->u + row * L;
    const float *dr = j->delta + row * L;
    const float *z = j->z ? j->z + row * L : NULL;
    const float *Bb = j->B + b * N * L;
    const float *Cb = j->C + b * N * L;
    const float *Ad = j->A + d * N;
    const double Dd = j->D ? (double)j->D[d] : 0.0;
    const double bias = j->bias ? (double)j->bias[d] : 0.0;
    double *out = j->out + row * L;

    for (int64_t n = 0; n < N; ++n)
        h[n] = j->h0 ? j->h0[row * N + n] : 0.0;

    for (int64_t t = 0; t < L; ++t) {
        double delta = (double)dr[t] + bias;
        if (j->softplus)
            delta = s6_oracle_softplus(delta);
        const double ut = (double)u[t];
        double y = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            const double Abar = exp(delta * (double)Ad[n]);
            const double Bbar_u = delta * (double)Bb[n * L + t] * ut;
            h[n] = Abar * h[n] + Bbar_u;
            y += (double)Cb[n * L + t] * h[n];
        }
        y += Dd * ut;
        if (z)
            y *= s6_oracle_silu((double)z[t]);
        out[t] = y;
    }
    if (j->last_state)
        for (int64_t n = 0; n < N; ++n)
            j->last_state[row * N + n] = h[n];
}

static void *scan_worker(void *arg)
{
    const scan_job_t *j = (const scan_job_t *)arg;
    double *h = (double *)malloc(sizeof(double) * (size_t)j->dstate);
    if (!h)
        return (void *)1;
    for (int64_t row = j->row_begin; row < j->row_end; ++row)
        scan_row(j, row, h);
    free(h);
    return NULL;
}

/* Full scan over all (b, d) rows.  nthreads <= 0 uses every online core.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation failure. */
int s6_oracle_scan(const float *u, const float *delta, const float *A,
                   const float *B, const float *C, const float *D,
                   const float *z, const float *delta_bias, int softplus,
                   const double *h0, double *out, double *last_state,
                   int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                   int nthreads)
{
    if (!u || !delta || !A || !B || !C || !out)
        return -1;
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0)
        return -1;
    const int64_t rows = batch * dim;
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > rows)
        nthreads = (int)rows;

    scan_job_t base = {u, delta, A, B, C, D, z, delta_bias, h0, softplus,
                       out, last_state, dim, seqlen, dstate, 0, rows};
    if (nthreads == 1) {
        return scan_worker(&base) ? -2 : 0;
    }
    scan_job_t *jobs = (scan_job_t *)malloc(sizeof(scan_job_t) * (size_t)nthreads);
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return -2;
    }
    int rc = 0;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].row_begin = rows * i / nthreads;
        jobs[i].row_end = rows * (i + 1) / nthreads;
        if (pthread_create(&tids[i], NULL, scan_worker, &jobs[i]) != 0) {
            /* run the remainder on this thread */
            jobs[i].row_end = rows;
            if (scan_worker(&jobs[i]))
                rc = -2;
            break;
        }
        ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(tids[i], &ret);
        if (ret)
            rc = -2;
    }
    free(jobs);
    free(tids);
    return rc;
}

/* Causal depthwise convolution over time with bias and optional silu: the
 * step before the scan in the block of the page "Mamba SSM concept and
 * implementation in Keras and TensorFlow" (MambaBlock: a Conv1D with one
 * group per channel, channels-first, causal padding, bias, cut to the input
 * length, then swish):
 *   v[b,d,t]   = bias[d] + sum_{k=0}^{K-1} w[d,k] * x[b,d,t-(K-1)+k],
 *                x[b,d,t] = 0 for t < 0 (the causal padding)
 *   out[b,d,t] = silu(v[b,d,t]) if the flag is set, else v[b,d,t]
 * x rows of batch row b start at b * x_batch_stride (dim * seqlen for a
 * contiguous tensor; larger when x is the first part of a wider tensor, as
 * the x half of the input projection's output is); w is (dim, K) row-major;
 * out is contiguous (batch, dim, seqlen).  The sum starts from the bias and
 * adds k = 0 .. K-1 in order. */
int s6_oracle_conv1d(const float *x, const float *w, const float *bias, int silu,
                     double *out, int64_t batch, int64_t dim, int64_t seqlen,
                     int64_t width, int64_t x_batch_stride)
{
    if (!x || !w || !out || batch <= 0 || dim <= 0 || seqlen <= 0 || width <= 0)
        return -1;
    if (x_batch_stride < dim * seqlen)
        return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const float *xr = x + b * x_batch_stride + d * seqlen;
            const float *wr = w + d * width;
            double *o = out + (b * dim + d) * seqlen;
            for (int64_t t = 0; t < seqlen; ++t) {
                double v = bias ? (double)bias[d] : 0.0;
                for (int64_t k = 0; k < width; ++k) {
                    const int64_t s = t - (width - 1) + k;
                    if (s >= 0)
                        v += (double)wr[k] * (double)xr[s];
                }
                o[t] = silu ? s6_oracle_silu(v) : v;
            }
        }
    }
    return 0;
}

/* One token of the same convolution, for decoding.  state (batch, dim, K-1)
 * holds each row's last K-1 inputs, oldest first (zeros before the sequence
 * starts); the token's input x[b,d] is the newest.  The output is formed as
 * in s6_oracle_conv1d (bias, then k = 0 .. K-1 over the K inputs oldest
 * first), then the state drops its oldest input and appends x[b,d]. */
int s6_oracle_conv1d_update(double *state, const float *x, const float *w,
                            const float *bias, int silu, double *out,
                            int64_t batch, int64_t dim, int64_t width)
{
    if (!state || !x || !w || !out || batch <= 0 || dim <= 0 || width <= 0)
        return -1;
    const int64_t S = width - 1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            double *st = state + (b * dim + d) * S;
            const float *wr = w + d * width;
            const double xt = (double)x[b * dim + d];
            double v = bias ? (double)bias[d] : 0.0;
            for (int64_t k = 0; k < width; ++k)
                v += (double)wr[k] * (k < S ? st[k] : xt);
            out[b * dim + d] = silu ? s6_oracle_silu(v) : v;
            for (int64_t k = 0; k + 1 < S; ++k)
                st[k] = st[k + 1];
            if (S > 0)
                st[S - 1] = xt;
        }
    }
    return 0;
}

/* One recurrent step for every (b, d): the same update as one iteration of
 * the scan's time loop, applied to a state held by the caller (the decoding
 * form that generation uses one token at a time).
 *   state       : (batch, dim, dstate), read and overwritten
 *   u, delta, z : (batch, dim);  B, C : (batch, dstate);  out : (batch, dim) */
int s6_oracle_state_update(double *state, const float *u, const float *delta,
                           const float *A, const float *B, const float *C,
                           const float *D, const float *z,
                           const float *delta_bias, int softplus, double *out,
                           int64_t batch, int64_t dim, int64_t dstate)
{
    if (!state || !u || !delta || !A || !B || !C || !out)
        return -1;
    if (batch <= 0 || dim <= 0 || dstate <= 0)
        return -1;
    const int64_t N = dstate;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const int64_t row = b * dim + d;
            double delta_t = (double)delta[row] + (delta_bias ? (double)delta_bias[d] : 0.0);
            if (softplus)
                delta_t = s6_oracle_softplus(delta_t);
            const double ut = (double)u[row];
            double *h = state + row * N;
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double Abar = exp(delta_t * (double)A[d * N + n]);
                const double Bbar_u = delta_t * (double)B[b * N + n] * ut;
                h[n] = Abar * h[n] + Bbar_u;
                y += (double)C[b * N + n] * h[n];
            }
            y += (D ? (double)D[d] : 0.0) * ut;
            if (z)
                y *= s6_oracle_silu((double)z[row]);
            out[row] = y;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ backward
 * Gradients of the forward scan above for a loss L with dL/dout = dout and
 * (optionally) dL/dlast_state = dlast: reverse-mode differentiation of the
 * recurrence written out (the scan is differentiated as a whole sequence;
 * the training path the pages describe back-propagates through it, and the
 * Mamba paper's hardware-aware algorithm recomputes the states in the
 * backward pass instead of storing them -- this plain loop stores them).
 *
 * Per (b, d), with g[n] = dL/dh_t[n] carried backwards from g = dlast:
 *   y_t  = sum_n C[n,t] h_t[n] + D u_t            (recomputed from stored h)
 *   dz_t = dout_t * y_t * silu'(z_t),  silu'(z) = s (1 + z (1 - s)), s = 1/(1+e^-z)
 *   dy_t = dout_t * silu(z_t)  (dout_t without a gate)
 *   dD  += dy_t u_t;  du_t = dy_t D;  dC[b,n,t] += dy_t h_t[n];  g[n] += dy_t C[n,t]
 *   with hp = h_{t-1}[n] (h0 or 0 at t = 0) and Abar = exp(delta_t A[n]):
 *   ddelta_t += g[n] (hp Abar A[n] + B[n,t] u_t)
 *   dA[d,n]  += g[n] hp Abar delta_t
 *   dB[b,n,t]+= g[n] delta_t u_t
 *   du_t     += g[n] delta_t B[n,t]
 *   g[n]      = g[n] Abar                        (dL/dh_{t-1}[n])
 *   ddelta_raw_t = ddelta_t * sigmoid(delta_raw_t + bias[d]) with softplus,
 *   ddelta_t itself without;  dbias[d] += ddelta_raw_t
 *   dh0 = g after t = 0.
 * Outputs: du, ddelta, dz (batch, dim, L); dA (dim, N); dB, dC (batch, N, L);
 * dD, ddelta_bias (dim); dh0 (batch, dim, N) -- all fp64; dz, dD,
 * ddelta_bias, dh0 may be NULL when not wanted (dz must be NULL without z).
 * Channel rows are spread over POSIX threads; the sums over channels (dA,
 * dB, dC, dD, dbias) are accumulated per thread and added in thread order,
 * so results do not depend on timing. */
typedef struct {
    const float *u, *delta, *A, *B, *C, *D, *z, *bias;
    const double *h0, *dout, *dlast;
    int softplus;
    double *du, *ddelta, *dz, *dh0;
    double *dA, *dB, *dC, *dD, *dbias; /* this thread's partial sums */
    int64_t batch, dim, seqlen, dstate;
    int64_t row_begin, row_end;
    int status;
} bwd_job_t;

static double s6_oracle_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static void *bwd_worker(void *arg)
{
    bwd_job_t *j = (bwd_job_t *)arg;
    const int64_t L = j->seqlen, N = j->dstate;
    double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
    double *g = (double *)malloc(sizeof(double) * (size_t)N);
    if (!hs || !g) {
        free(hs);
        free(g);
        j->status = -2;
        return NULL;
    }
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / j->dim, d = row % j->dim;
        const float *u = j->u + row * L;
        const float *dr = j->delta + row * L;
        const float *z = j->z ? j->z + row * L : NULL;
        const float *Bw = j->B + b * N * L;
        const float *Cw = j->C + b * N * L;
        const float *Aw = j->A + d * N;
        const double Dd = j->D ? (double)j->D[d] : 0.0;
        const double bias = j->bias ? (double)j->bias[d] : 0.0;
        const double *dout = j->dout + row * L;
        /* forward, keeping every state: hs[(t + 1) N + n] = h_t[n], hs[n] = h_{-1} */
        for (int64_t n = 0; n < N; ++n)
            hs[n] = j->h0 ? j->h0[row * N + n] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double delta = (double)dr[t] + bias;
            if (j->softplus)
                delta = s6_oracle_softplus(delta);
            for (int64_t n = 0; n < N; ++n)
                hs[(t + 1) * N + n] = exp((double)Aw[n] * delta) * hs[t * N + n] +
                                      delta * (double)Bw[n * L + t] * (double)u[t];
        }
        for (int64_t n = 0; n < N; ++n)
            g[n] = j->dlast ? j->dlast[row * N + n] : 0.0;
        for (int64_t t = L - 1; t >= 0; --t) {
            const double draw = (double)dr[t] + bias;
            const double delta = j->softplus ? s6_oracle_softplus(draw) : draw;
            const double ut = (double)u[t];
            const double *h = hs + (t + 1) * N, *hp = hs + t * N;
            double y = Dd * ut;
            for (int64_t n = 0; n < N; ++n)
                y += (double)Cw[n * L + t] * h[n];
            double dy = dout[t];
            if (z) {
                const double zt = (double)z[t], s = s6_oracle_sigmoid(zt);
                if (j->dz)
                    j->dz[row * L + t] = dout[t] * y * s * (1.0 + zt * (1.0 - s));
                dy = dout[t] * s6_oracle_silu(zt);
            }
            j->dD[d] += dy * ut;
            double du = dy * Dd, ddelta = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                j->dC[b * N * L + n * L + t] += dy * h[n];
                g[n] += dy * (double)Cw[n * L + t];
                const double Abar = exp((double)Aw[n] * delta);
                ddelta += g[n] * (hp[n] * Abar * (double)Aw[n] + (double)Bw[n * L + t] * ut);
                j->dA[d * N + n] += g[n] * hp[n] * Abar * delta;
                j->dB[b * N * L + n * L + t] += g[n] * delta * ut;
                du += g[n] * delta * (double)Bw[n * L + t];
                g[n] *= Abar;
            }
            const double ddraw = j->softplus ? ddelta * s6_oracle_sigmoid(draw) : ddelta;
            j->du[row * L + t] = du;
            j->ddelta[row * L + t] = ddraw;
            j->dbias[d] += ddraw;
        }
        if (j->dh0)
            for (int64_t n = 0; n < N; ++n)
                j->dh0[row * N + n] = g[n];
    }
    free(hs);
    free(g);
    return NULL;
}

int s6_oracle_scan_bwd(const float *u, const float *delta, const float *A,
                       const float *B, const float *C, const float *D,
                       const float *z, const float *delta_bias, int softplus,
                       const double *h0, const double *dout, const double *dlast,
                       double *du, double *ddelta, double *dA, double *dB,
                       double *dC, double *dD, double *dz, double *ddelta_bias,
                       double *dh0, int64_t batch, int64_t dim, int64_t seqlen,
                       int64_t dstate, int nthreads)
{
    if (!u || !delta || !A || !B || !C || !dout || !du || !ddelta || !dA || !dB || !dC)
        return -1;
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0 || (dz && !z))
        return -1;
    const int64_t rows = batch * dim, N = dstate, L = seqlen;
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > rows)
        nthreads = (int)rows;
    const size_t nA = (size_t)(dim * N), nBC = (size_t)(batch * N * L), nd = (size_t)dim;
    const size_t per = 2 * nBC + nA + 2 * nd; /* dB, dC, dA, dD, dbias */
    double *acc = (double *)calloc((size_t)nthreads * per, sizeof(double));
    bwd_job_t *jobs = (bwd_job_t *)malloc(sizeof(bwd_job_t) * (size_t)nthreads);
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!acc || !jobs || !tids) {
        free(acc);
        free(jobs);
        free(tids);
        return -2;
    }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        double *a = acc + (size_t)i * per;
        bwd_job_t jb = {u, delta, A, B, C, D, z, delta_bias, h0, dout, dlast, softplus,
                        du, ddelta, dz, dh0, a + 2 * nBC, a, a + nBC, a + 2 * nBC + nA,
                        a + 2 * nBC + nA + nd, batch, dim, seqlen, dstate,
                        rows * i / nthreads, rows * (i + 1) / nthreads, 0};
        jobs[i] = jb;
    }
    for (int i = 0; i < nthreads; ++i) {
        if (nthreads == 1 || pthread_create(&tids[i], NULL, bwd_worker, &jobs[i]) != 0) {
            for (int k = i; k < nthreads; ++k) /* run the rest on this thread */
                bwd_worker(&jobs[k]);
            break;
        }
        ++started;
    }
    for (int i = 0; i < started; ++i)
        pthread_join(tids[i], NULL);
    int rc = 0;
    for (size_t k = 0; k < nBC; ++k) {
        dB[k] = 0.0;
        dC[k] = 0.0;
    }
    for (size_t k = 0; k < nA; ++k)
        dA[k] = 0.0;
    for (size_t k = 0; k < nd; ++k) {
        if (dD)
            dD[k] = 0.0;
        if (ddelta_bias)
            ddelta_bias[k] = 0.0;
    }
    for (int i = 0; i < nthreads; ++i) {
        if (jobs[i].status)
            rc = jobs[i].status;
        const double *a = acc + (size_t)i * per;
        for (size_t k = 0; k < nBC; ++k) {
            dB[k] += a[k];
            dC[k] += a[nBC + k];
        }
        for (size_t k = 0; k < nA; ++k)
            dA[k] += a[2 * nBC + k];
        for (size_t k = 0; k < nd; ++k) {
            if (dD)
                dD[k] += a[2 * nBC + nA + k];
            if (ddelta_bias)
                ddelta_bias[k] += a[2 * nBC + nA + nd + k];
        }
    }
    free(acc);
    free(jobs);
    free(tids);
    return rc;
}

/*
 * Complex-valued mode: the same recurrence with a complex diagonal A and
 * complex, input-dependent B and C (the complex SSM the Mamba paper compares
 * with the real one on audio, Appendix E.4.1, and the "complex number mode"
 * on the roadmap of the "Mamba x JAX" page).  The pages give no formulas for
 * it; this is the real recurrence above read over the complex numbers, with
 * the output taken as the real part of the readout:
 *
 *   delta_t = softplus(delta_raw + bias)          (real, as above)
 *   Abar    = exp(delta_t * A[d,n])                complex exponential
 *   Bbar u  = delta_t * B[b,n,t] * u[b,d,t]        complex
 *   h_t[n]  = Abar * h_{t-1}[n] + Bbar u           complex state
 *   y_t     = Re(sum_n C[b,n,t] * h_t[n]) + D[d] * u[b,d,t]
 *   out_t   = y_t * silu(z[b,d,t])    if z is given
 *
 * Complex arrays are interleaved (real, imaginary) pairs of the real layouts:
 *   A (dim, dstate, 2); B, C (batch, dstate, seqlen, 2);
 *   h0, last_state (batch, dim, dstate, 2).
 */
#include <complex.h>

typedef struct {
    const float *u, *delta, *A, *B, *C, *D, *z, *bias;
    const double *h0;
    int softplus;
    double *out, *last_state;
    int64_t dim, seqlen, dstate;
    int64_t row_begin, row_end;
} cscan_job_t;

static void *cscan_worker(void *arg)
{
    const cscan_job_t *j = (const cscan_job_t *)arg;
    const int64_t L = j->seqlen, N = j->dstate;
    double complex *h = (double complex *)malloc(sizeof(double complex) * (size_t)N);
    if (!h)
        return (void *)1;
    for (int64_t row = j->row_begin; row < j->row_end; ++row) {
        const int64_t b = row / j->dim, d = row % j->dim;
        const float *u = j->u + row * L;
        const float *dr = j->delta + row * L;
        const float *z = j->z ? j->z + row * L : NULL;
        const float *Bb = j->B + b * N * L * 2;
        const float *Cb = j->C + b * N * L * 2;
        const float *Ad = j->A + d * N * 2;
        const double Dd = j->D ? (double)j->D[d] : 0.0;
        const double bias = j->bias ? (double)j->bias[d] : 0.0;
        double *out = j->out + row * L;

        for (int64_t n = 0; n < N; ++n)
            h[n] = j->h0 ? j->h0[(row * N + n) * 2] + I * j->h0[(row * N + n) * 2 + 1] : 0.0;
        for (int64_t t = 0; t < L; ++t) {
            double delta = (double)dr[t] + bias;
            if (j->softplus)
                delta = s6_oracle_softplus(delta);
            const double ut = (double)u[t];
            double y = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                const double complex An = (double)Ad[2 * n] + I * (double)Ad[2 * n + 1];
                const double complex Bn = (double)Bb[(n * L + t) * 2] + I * (double)Bb[(n * L + t) * 2 + 1];
                const double complex Cn = (double)Cb[(n * L + t) * 2] + I * (double)Cb[(n * L + t) * 2 + 1];
                const double complex Abar = cexp(delta * An);
                const double complex Bbar_u = delta * Bn * ut;
                h[n] = Abar * h[n] + Bbar_u;
                y += creal(Cn * h[n]);
            }
            y += Dd * (double)u[t];
            if (z)
                y = y * s6_oracle_silu((double)z[t]);
            out[t] = y;
        }
        if (j->last_state)
            for (int64_t n = 0; n < N; ++n) {
                j->last_state[(row * N + n) * 2] = creal(h[n]);
                j->last_state[(row * N + n) * 2 + 1] = cimag(h[n]);
            }
    }
    free(h);
    return NULL;
}

/* Complex-mode scan over all (b, d) rows; threads and return codes as
 * s6_oracle_scan. */
int s6_oracle_scan_complex(const float *u, const float *delta, const float *A,
                           const float *B, const float *C, const float *D,
                           const float *z, const float *delta_bias, int softplus,
                           const double *h0, double *out, double *last_state,
                           int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
                           int nthreads)
{
    if (!u || !delta || !A || !B || !C || !out)
        return -1;
    if (batch <= 0 || dim <= 0 || seqlen <= 0 || dstate <= 0)
        return -1;
    const int64_t rows = batch * dim;
    if (nthreads <= 0) {
        long nc = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = nc > 0 ? (int)nc : 1;
    }
    if (nthreads > rows)
        nthreads = (int)rows;
    cscan_job_t base = {u, delta, A, B, C, D, z, delta_bias, h0, softplus,
                        out, last_state, dim, seqlen, dstate, 0, rows};
    cscan_job_t *jobs = (cscan_job_t *)malloc(sizeof(cscan_job_t) * (size_t)nthreads);
    pthread_t *tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !tids) {
        free(jobs);
        free(tids);
        return -2;
    }
    int rc = 0, started = 0;
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = base;
        jobs[i].row_begin = rows * i / nthreads;
        jobs[i].row_end = rows * (i + 1) / nthreads;
        if (pthread_create(&tids[i], NULL, cscan_worker, &jobs[i]) != 0) {
            jobs[i].row_end = rows;
            if (cscan_worker(&jobs[i]))
                rc = -2;
            break;
        }
        ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(tids[i], &ret);
        if (ret)
            rc = -2;
    }
    free(jobs);
    free(tids);
    return rc;
}

/*
 * fp64 oracle for the Mamba selective-SSM (S6) forward scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the bench's CPU
 * baseline do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes, per batch b and channel d, exactly as the pages define
 * the method and in the same order, in fp64:
 *
 *   Mamba "architecture-details" page, "How S6 Works" (selective SSM):
 *     h(t) = discretize(A, delta(t)) * h(t-1) + delta(t) * B(t) * x(t)
 *     y(t) = C(t) * h(t)
 *   "Agent 229: SSM optimization patterns" page, section 7 "Selective
 *   Attention Mechanism" (mathematical formulation):  A_bar_t = exp(delta_t * A)
 *   "architecture-details" page, "Parallel Algorithm", sequential mode: the
 *     RNN-style loop over time with a constant-size state.
 *
 * plus the forward-scan interface around it: the step size is
 * dt = softplus(delta + delta_bias) (or delta + delta_bias when softplus is off),
 * the skip term D*u is added to y, the output is gated by silu(z) = z/(1+e^-z),
 * and the state after the last step is returned.
 *
 * The loop is plain: for each state n, h_n <- exp(dt*A_n) h_n + dt*B_n*u, and
 * y <- y + C_n h_n; no blocking, no reassociation.  Independent (b, d)
 * sequences are spread over threads, which changes no arithmetic.
 *
 * Extra outputs for the tolerance check: mag[t] = |silu(z)| * (sum_n |C_n h_n| + |D u|),
 * the size of the terms that are summed into out[t] (the fp32 GPU sum has an
 * error proportional to it).
 *
 * Shapes (row-major):
 *   full mode (channels == NULL):
 *     u, z (batch, dim, L); delta (batch, nheads, L); out, mag (batch, dim, L)
 *   row mode (channels != NULL, nch entries, each c = b*dim + d):
 *     u, z, delta (nch, L): the rows for those channels (delta: the row of
 *     the channel's head); out, mag (nch, L)
 *   both:  B, C (batch, ngroups, N, L);  A (dim, N), or (nheads) when
 *     nheads < dim (one scalar A per head); D (dim); delta_bias (nheads);
 *     h0 (batch, dim, N) in full mode or (nch, N) in row mode;
 *     last_state like h0.
 * Channel d belongs to head d / (dim/nheads) and group d / (dim/ngroups).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>

typedef struct {
    int64_t batch, dim, seqlen, dstate, nheads, ngroups;
} oracle_dims_t;

typedef struct {
    const oracle_dims_t* dm;
    const double *u, *delta, *A, *B, *C, *D, *z, *bias, *h0;
    const int64_t* channels;
    int64_t nch;
    int softplus;
    double *out, *last, *mag;
    int64_t begin, end;
} job_t;

/* log(1 + e^x), written so that neither branch overflows */
static double softplus_f64(double x) {
    if (x > 0.0) return x + log1p(exp(-x));
    return log1p(exp(x));
}

static double silu_f64(double z) { return z / (1.0 + exp(-z)); }

static void scan_one(const job_t* j, int64_t k) {
    const oracle_dims_t* dm = j->dm;
    const int64_t L = dm->seqlen, N = dm->dstate, Dm = dm->dim;
    const int64_t H = dm->nheads, G = dm->ngroups;
    const int64_t c = j->channels ? j->channels[k] : k; /* flat channel b*dim + d */
    const int64_t b = c / Dm, d = c % Dm;
    const int64_t hd = d / (Dm / H), g = d / (Dm / G);
    const int head_mode = H != Dm;
    const int64_t row = j->channels ? k : c;                 /* row of u, z, out */
    const int64_t drow = j->channels ? k : b * H + hd;       /* row of delta */
    const double* u = j->u + row * L;
    const double* z = j->z ? j->z + row * L : NULL;
    const double* dl = j->delta + drow * L;
    const double* Bg = j->B + (b * G + g) * N * L;
    const double* Cg = j->C + (b * G + g) * N * L;
    double* out = j->out + row * L;
    double* mag = j->mag ? j->mag + row * L : NULL;
    const double bias = j->bias ? j->bias[hd] : 0.0;
    const double Dd = j->D ? j->D[d] : 0.0;

    double* h = (double*)malloc((size_t)N * sizeof(double));
    for (int64_t n = 0; n < N; ++n) h[n] = j->h0 ? j->h0[row * N + n] : 0.0;

    for (int64_t t = 0; t < L; ++t) {
        double x = dl[t] + bias;
        double dt = j->softplus ? softplus_f64(x) : x;
        double y = 0.0, s = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double a = head_mode ? j->A[hd] : j->A[d * N + n];
            double dA = exp(dt * a);
            h[n] = dA * h[n] + dt * Bg[n * L + t] * u[t];
            y += Cg[n * L + t] * h[n];
            s += fabs(Cg[n * L + t] * h[n]);
        }
        y += Dd * u[t];
        s += fabs(Dd * u[t]);
        double gate = z ? silu_f64(z[t]) : 1.0;
        out[t] = y * gate;
        if (mag) mag[t] = fabs(gate) * s;
    }
    if (j->last)
        for (int64_t n = 0; n < N; ++n) j->last[row * N + n] = h[n];
    free(h);
}

static void* run_job(void* arg) {
    job_t* j = (job_t*)arg;
    for (int64_t k = j->begin; k < j->end; ++k) scan_one(j, k);
    return NULL;
}

/*
 * Returns 0 on success, -1 on inconsistent sizes or a missing required pointer.
 */
int oracle_selective_scan_f64(const oracle_dims_t* dm, const double* u, const double* delta,
                              const double* A, const double* B, const double* C, const double* D,
                              const double* z, const double* delta_bias, int softplus,
                              const double* h0, const int64_t* channels, int64_t nch,
                              double* out, double* last_state, double* mag, int nthreads) {
    if (!dm || dm->batch < 0 || dm->dim <= 0 || dm->seqlen < 0 || dm->dstate <= 0) return -1;
    if (dm->nheads <= 0 || dm->ngroups <= 0) return -1;
    if (dm->dim % dm->nheads || dm->dim % dm->ngroups) return -1;
    if (!u || !delta || !A || !B || !C || !out) return -1;
    int64_t total = channels ? nch : dm->batch * dm->dim;
    if (channels)
        for (int64_t k = 0; k < nch; ++k)
            if (channels[k] < 0 || channels[k] >= dm->batch * dm->dim) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (total < nthreads) nthreads = total > 0 ? (int)total : 1;
    job_t jobs[256];
    pthread_t th[256];
    int live[256] = {0};
    int64_t per = (total + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        job_t* j = &jobs[t];
        j->dm = dm; j->u = u; j->delta = delta; j->A = A; j->B = B; j->C = C; j->D = D;
        j->z = z; j->bias = delta_bias; j->h0 = h0; j->channels = channels; j->nch = nch;
        j->softplus = softplus; j->out = out; j->last = last_state; j->mag = mag;
        j->begin = t * per < total ? t * per : total;
        j->end = (t + 1) * per < total ? (t + 1) * per : total;
    }
    for (int t = 1; t < nthreads; ++t) {
        live[t] = pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0;
        if (!live[t]) run_job(&jobs[t]);
    }
    run_job(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (live[t]) pthread_join(th[t], NULL);
    return 0;
}

/*
 * Causal depthwise convolution over time: the local convolution in front of
 * the SSM ("architecture-details" page, "Model Configuration": d_conv, the
 * convolution width, and conv_bias; "Parameter Impact": d_conv is the local
 * context window before the SSM).  Each channel has its own `width` taps; the
 * input is zero before t = 0, so output t sees steps t-width+1 .. t only.
 * Per batch b, channel d, step t, in fp64:
 *
 *   v = bias[d] + sum_{k=0}^{width-1} w[d][k] * x[b][d][t - (width-1) + k]
 *   out[b][d][t] = silu ? v / (1 + exp(-v)) : v
 *
 * (the activation after the convolution is a flag: the pages name the
 * convolution, not what follows it).  bias may be NULL (zero).
 * Layouts: x, out (batch, dim, seqlen); w (dim, width); bias (dim).
 * Returns 0, or -1 on a bad size or a missing required pointer.
 */
int oracle_causal_conv1d_f64(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, const double* x,
                             const double* w, const double* bias, int silu, double* out) {
    if (batch < 0 || dim <= 0 || seqlen < 0 || width <= 0) return -1;
    if (!x || !w || !out) return -1;
    for (int64_t b = 0; b < batch; ++b) {
        for (int64_t d = 0; d < dim; ++d) {
            const double* xr = x + (b * dim + d) * seqlen;
            double* orow = out + (b * dim + d) * seqlen;
            const double* wr = w + d * width;
            for (int64_t t = 0; t < seqlen; ++t) {
                double v = bias ? bias[d] : 0.0;
                for (int64_t k = 0; k < width; ++k) {
                    const int64_t s = t - (width - 1) + k;
                    if (s >= 0) v += wr[k] * xr[s];
                }
                orow[t] = silu ? v / (1.0 + exp(-v)) : v;
            }
        }
    }
    return 0;
}

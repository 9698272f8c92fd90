/*
 * fp64 oracle for the Mamba selective-SSM (S6) forward scan, its gradient
 * (oracle_selective_scan_bwd_f64, further down) and the causal convolution.
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

/*
 * Gradient of the forward scan above (reverse-mode chain rule through the
 * recurrence), in fp64: given dout = dLoss/dout and, optionally, dlast =
 * dLoss/dlast_state, the gradients of every input.  The pages ask for the
 * backward pass to recompute the activations it needs instead of storing them
 * ("Agent 229: SSM optimization patterns" page, section 4 "Activation
 * Recomputation"; "architecture-details" page, "Memory Efficiency", training);
 * here the whole state history of one channel is simply recomputed first.
 *
 * With x_t = delta_t + bias, dt_t = softplus(x_t) (or x_t), dA_tn = exp(dt_t a_n),
 * h_tn = dA_tn h_(t-1)n + dt_t B_tn u_t, y_t = sum_n C_tn h_tn + D u_t and
 * out_t = y_t silu(z_t), walking t from L-1 down to 0 with the carried
 * gradient g_n of the state (g_n = dlast_n before the last step):
 *
 *   dy_t    = dout_t silu(z_t)                  dz_t = dout_t y_t silu'(z_t)
 *   g_n    += dy_t C_tn                          (now dLoss/dh_tn)
 *   dC_tn  += dy_t h_tn                          dB_tn += g_n dt_t u_t
 *   du_t    = dy_t D + sum_n g_n dt_t B_tn       dD    += dy_t u_t
 *   ddt_t   = sum_n (g_n B_tn u_t + g_n h_(t-1)n a_n dA_tn)
 *   da_n   += g_n h_(t-1)n dt_t dA_tn            g_n   <- dA_tn g_n
 *   ddelta_t = ddt_t sigmoid(x_t) (ddt_t without softplus); dbias += ddelta_t
 *   dh0_n   = g_n after step 0
 *
 * silu'(z) = s (1 + z (1 - s)), s = sigmoid(z).  Per-head layout: ddelta,
 * da and dbias of a head sum over its channels (and da over n); dB and dC of a
 * group sum over its channels.  Accumulation order: dB, dC, ddelta over the
 * channels of a batch row in increasing d; dA, dD, dbias over b in increasing
 * order of b after the per-row sums.
 *
 * Tolerance magnitudes (mags, same shapes, optional): the same sums with every
 * term replaced by its absolute value and the state and its gradient by their
 * magnitude recurrences  mh_t = dA mh_(t-1) + |dt B u|,
 * mg = dA mg + |dy C| (mg = |dlast| at the start); an fp32 evaluation of a
 * gradient errs by a small multiple of its magnitude.
 *
 * Layouts as in the forward; grads: du, dz (batch, dim, L); ddelta (batch,
 * nheads, L); dA like A; dB, dC (batch, ngroups, N, L); dD (dim); ddelta_bias
 * (nheads); dh0 (batch, dim, N).  dz, dD, ddelta_bias and dh0 may be NULL
 * (not wanted); mags may be NULL, or any of its pointers.
 * Returns 0, or -1 on a bad size or a missing required pointer.
 */
typedef struct {
    double *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias, *dh0;
} oracle_grads_t;

typedef struct {
    const oracle_dims_t* dm;
    const double *u, *delta, *A, *B, *C, *D, *z, *bias, *h0, *dout, *dlast;
    int softplus;
    oracle_grads_t g, m;      /* outputs; for dA, dD, ddelta_bias: this job's partial sums */
    int64_t b0, b1;           /* batch rows of this job */
} bjob_t;

static double sigmoid_f64(double x) {
    if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
    const double e = exp(x);
    return e / (1.0 + e);
}

#define ADD(ptr, i, v) do { if (ptr) (ptr)[i] += (v); } while (0)

static void bwd_rows(bjob_t* j) {
    const oracle_dims_t* dm = j->dm;
    const int64_t L = dm->seqlen, N = dm->dstate, Dm = dm->dim;
    const int64_t H = dm->nheads, G = dm->ngroups;
    const int head_mode = H != Dm;
    double* hs = (double*)malloc((size_t)(L + 1) * N * sizeof(double));   /* h_(t-1) at row t */
    double* mhs = (double*)malloc((size_t)(L + 1) * N * sizeof(double));
    double* dts = (double*)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
    double* gs = (double*)malloc((size_t)N * sizeof(double));
    double* mgs = (double*)malloc((size_t)N * sizeof(double));
    for (int64_t b = j->b0; b < j->b1; ++b) {
        for (int64_t d = 0; d < Dm; ++d) {
            const int64_t hd = d / (Dm / H), g = d / (Dm / G);
            const int64_t row = b * Dm + d, drow = b * H + hd;
            const double* u = j->u + row * L;
            const double* z = j->z ? j->z + row * L : NULL;
            const double* dl = j->delta + drow * L;
            const double* go = j->dout + row * L;
            const double* Bg = j->B + (b * G + g) * N * L;
            const double* Cg = j->C + (b * G + g) * N * L;
            const double bias = j->bias ? j->bias[hd] : 0.0;
            const double Dd = j->D ? j->D[d] : 0.0;
            /* recompute the states: hs row t holds h_(t-1) */
            for (int64_t n = 0; n < N; ++n) {
                hs[n] = j->h0 ? j->h0[row * N + n] : 0.0;
                mhs[n] = fabs(hs[n]);
            }
            for (int64_t t = 0; t < L; ++t) {
                const double x = dl[t] + bias;
                const double dt = j->softplus ? softplus_f64(x) : x;
                dts[t] = dt;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = head_mode ? j->A[hd] : j->A[d * N + n];
                    const double dA = exp(dt * a);
                    hs[(t + 1) * N + n] = dA * hs[t * N + n] + dt * Bg[n * L + t] * u[t];
                    mhs[(t + 1) * N + n] = dA * mhs[t * N + n] + fabs(dt * Bg[n * L + t] * u[t]);
                }
            }
            for (int64_t n = 0; n < N; ++n) {
                gs[n] = j->dlast ? j->dlast[row * N + n] : 0.0;
                mgs[n] = fabs(gs[n]);
            }
            for (int64_t t = L - 1; t >= 0; --t) {
                const double dt = dts[t];
                const double x = dl[t] + bias;
                const double* hp = hs + t * N;         /* h_(t-1) */
                const double* hc = hs + (t + 1) * N;   /* h_t */
                const double* mhp = mhs + t * N;
                const double* mhc = mhs + (t + 1) * N;
                const double gate = z ? silu_f64(z[t]) : 1.0;
                const double dy = go[t] * gate;
                if (z) {
                    double y = Dd * u[t], ym = fabs(Dd * u[t]);
                    for (int64_t n = 0; n < N; ++n) {
                        y += Cg[n * L + t] * hc[n];
                        ym += fabs(Cg[n * L + t]) * mhc[n];
                    }
                    const double s = sigmoid_f64(z[t]);
                    const double dsilu = s * (1.0 + z[t] * (1.0 - s));
                    j->g.dz[row * L + t] = go[t] * y * dsilu;
                    /* silu'(z) = s + z s (1 - s) is a sum of two terms: its magnitude is s (1 + |z| (1 - s)) */
                    if (j->m.dz) j->m.dz[row * L + t] = fabs(go[t]) * s * (1.0 + fabs(z[t]) * (1.0 - s)) * ym;
                }
                ADD(j->g.dD, d, dy * u[t]);
                ADD(j->m.dD, d, fabs(dy * u[t]));
                double du = dy * Dd, mdu = fabs(dy * Dd), ddt = 0.0, mddt = 0.0;
                for (int64_t n = 0; n < N; ++n) {
                    const double a = head_mode ? j->A[hd] : j->A[d * N + n];
                    const double dA = exp(dt * a);
                    const int64_t bc = (b * G + g) * N * L + n * L + t;
                    const int64_t ai = head_mode ? hd : d * N + n;
                    gs[n] += dy * Cg[n * L + t];
                    mgs[n] += fabs(dy * Cg[n * L + t]);
                    j->g.dC[bc] += dy * hc[n];
                    if (j->m.dC) j->m.dC[bc] += fabs(dy) * mhc[n];
                    j->g.dB[bc] += gs[n] * dt * u[t];
                    if (j->m.dB) j->m.dB[bc] += mgs[n] * dt * fabs(u[t]);
                    du += gs[n] * dt * Bg[n * L + t];
                    mdu += mgs[n] * dt * fabs(Bg[n * L + t]);
                    const double gdA = gs[n] * hp[n];      /* dLoss/d(dA_tn) */
                    const double mgdA = mgs[n] * mhp[n];
                    ddt += gs[n] * Bg[n * L + t] * u[t] + gdA * a * dA;
                    mddt += mgs[n] * fabs(Bg[n * L + t] * u[t]) + mgdA * fabs(a) * dA;
                    j->g.dA[ai] += gdA * dt * dA;
                    ADD(j->m.dA, ai, mgdA * dt * dA);
                    gs[n] = dA * gs[n];
                    mgs[n] = dA * mgs[n];
                }
                const double sp = j->softplus ? sigmoid_f64(x) : 1.0;
                j->g.du[row * L + t] = du;
                if (j->m.du) j->m.du[row * L + t] = mdu;
                j->g.ddelta[drow * L + t] += ddt * sp;
                if (j->m.ddelta) j->m.ddelta[drow * L + t] += mddt * sp;
                ADD(j->g.ddelta_bias, hd, ddt * sp);
                ADD(j->m.ddelta_bias, hd, mddt * sp);
            }
            if (j->g.dh0)
                for (int64_t n = 0; n < N; ++n) {
                    j->g.dh0[row * N + n] = gs[n];
                    if (j->m.dh0) j->m.dh0[row * N + n] = mgs[n];
                }
        }
    }
    free(hs); free(mhs); free(dts); free(gs); free(mgs);
}

static void* run_bjob(void* arg) {
    bwd_rows((bjob_t*)arg);
    return NULL;
}

static void zero(double* p, int64_t n) {
    if (p)
        for (int64_t i = 0; i < n; ++i) p[i] = 0.0;
}

int oracle_selective_scan_bwd_f64(const oracle_dims_t* dm, const double* u, const double* delta,
                                  const double* A, const double* B, const double* C, const double* D,
                                  const double* z, const double* delta_bias, int softplus, const double* h0,
                                  const double* dout, const double* dlast, const oracle_grads_t* grads,
                                  const oracle_grads_t* mags, int nthreads) {
    if (!dm || dm->batch < 0 || dm->dim <= 0 || dm->seqlen < 0 || dm->dstate <= 0) return -1;
    if (dm->nheads <= 0 || dm->ngroups <= 0) return -1;
    if (dm->dim % dm->nheads || dm->dim % dm->ngroups) return -1;
    if (!u || !delta || !A || !B || !C || !dout || !grads) return -1;
    if (!grads->du || !grads->ddelta || !grads->dA || !grads->dB || !grads->dC) return -1;
    if (z && !grads->dz) return -1;
    const int64_t Bt = dm->batch, Dm = dm->dim, L = dm->seqlen, N = dm->dstate;
    const int64_t H = dm->nheads, G = dm->ngroups;
    const int64_t nA = H != Dm ? H : Dm * N;
    oracle_grads_t none = {0};
    const oracle_grads_t* m = mags ? mags : &none;
    /* zero what is accumulated */
    zero(grads->ddelta, Bt * H * L); zero(grads->dB, Bt * G * N * L); zero(grads->dC, Bt * G * N * L);
    zero(m->ddelta, Bt * H * L); zero(m->dB, Bt * G * N * L); zero(m->dC, Bt * G * N * L);
    zero(grads->dA, nA); zero(grads->dD, Dm); zero(grads->ddelta_bias, H);
    zero(m->dA, nA); zero(m->dD, Dm); zero(m->ddelta_bias, H);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 64) nthreads = 64;
    if (Bt < nthreads) nthreads = Bt > 0 ? (int)Bt : 1;
    bjob_t jobs[64];
    pthread_t th[64];
    int live[64] = {0};
    /* per-job partial sums of the parameter gradients, added in job (= batch) order */
    const int64_t np = 2 * (nA + Dm + H);
    double* part = (double*)calloc((size_t)(np * nthreads > 0 ? np * nthreads : 1), sizeof(double));
    if (!part) return -1;
    const int64_t per = (Bt + nthreads - 1) / nthreads;
    for (int t = 0; t < nthreads; ++t) {
        bjob_t* j = &jobs[t];
        double* pp = part + t * np;
        j->dm = dm; j->u = u; j->delta = delta; j->A = A; j->B = B; j->C = C; j->D = D; j->z = z;
        j->bias = delta_bias; j->h0 = h0; j->dout = dout; j->dlast = dlast; j->softplus = softplus;
        j->g = *grads;
        j->m = *m;
        j->g.dA = pp; j->g.dD = grads->dD ? pp + nA : NULL; j->g.ddelta_bias = grads->ddelta_bias ? pp + nA + Dm : NULL;
        pp += nA + Dm + H;
        j->m.dA = m->dA ? pp : NULL; j->m.dD = m->dD ? pp + nA : NULL; j->m.ddelta_bias = m->ddelta_bias ? pp + nA + Dm : NULL;
        j->b0 = t * per < Bt ? t * per : Bt;
        j->b1 = (t + 1) * per < Bt ? (t + 1) * per : Bt;
    }
    for (int t = 1; t < nthreads; ++t) {
        live[t] = pthread_create(&th[t], NULL, run_bjob, &jobs[t]) == 0;
        if (!live[t]) run_bjob(&jobs[t]);
    }
    run_bjob(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        if (live[t]) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads; ++t) {
        const double* pp = part + t * np;
        for (int64_t i = 0; i < nA; ++i) {
            grads->dA[i] += pp[i];
            ADD(m->dA, i, pp[nA + Dm + H + i]);
        }
        for (int64_t i = 0; i < Dm; ++i) {
            ADD(grads->dD, i, pp[nA + i]);
            ADD(m->dD, i, pp[2 * nA + Dm + H + i]);
        }
        for (int64_t i = 0; i < H; ++i) {
            ADD(grads->ddelta_bias, i, pp[nA + Dm + i]);
            ADD(m->ddelta_bias, i, pp[2 * nA + 2 * Dm + H + i]);
        }
    }
    free(part);
    return 0;
}

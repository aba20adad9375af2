/*
 * CPU oracle for the Mamba-1 selective-SSM layer core — TEST INFRASTRUCTURE.
 *
 * Plain, slow, obviously-correct fp64 C. Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product library never
 * does, and this file shares no code, header or table with the CUDA path.
 *
 * What is computed, and where the pages define it:
 *   conv   "hung-phan ml-skills mamba", section "Mamba: Selective State
 *          Spaces (S6)" (the SelectiveSSM sketch: depthwise Conv1d with
 *          padding d_conv-1, output cut to the first L steps, then SiLU) and
 *          section "Mamba Block Architecture" (Conv1d(k=4) -> SiLU).
 *   delta  same sketch: delta = softplus(dt) "to keep the step positive";
 *          the per-channel bias is the dt_bias of "Key Training Tips" 1.
 *   scan   same page, "Architecture Diagram" (S6 block): A_bar = exp(delta*A),
 *          B_bar = delta*B, h_t = A_bar*h_{t-1} + B_bar*x_t, y_t = C_t*h_t;
 *          section "Core Concept" adds the D*x feed-through; the sketch gates
 *          y * silu(z).
 *   resets "FLA Mamba and Mamba2" (Axolotl), packing paragraph: convolution
 *          and recurrent state start independently for every document.
 *   complex A  "S4: Structured State Spaces for Sequences" (S4D), see below.
 *   SSD    "Mamba-2: Structured State Space Duality (SSD)": scalar A per
 *          head, heads, groups of shared B / C (see below).
 *
 * Readings taken where the pages are silent:
 *   - A is passed directly (negative for the S4D-real init), not A_log.exp().
 *   - conv taps are cross-correlation: w[d][W-1] multiplies x_t and w[d][0]
 *     multiplies x_{t-W+1} (PyTorch Conv1d with left padding W-1).
 *   - a document boundary is any t with seq_idx[t] != seq_idx[t-1]; a conv tap
 *     counts only when its token is in the same segment as the output token.
 *   - u (the conv+SiLU output) feeds both B_bar*x and D*x.
 *   - the backward is hand-derived reverse mode of the definitions above.
 *
 * Threading: every core routine works on one (batch, channel) row; the *_mt
 * drivers only hand rows to pthreads and add per-thread partial sums in a
 * fixed order. Nothing is blocked, fused or reordered inside a row.
 */
#include <complex.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "ssm_oracle.h"

/* ---------------------------------------------------------------- helpers */
static double sigm(double v) { return 1.0 / (1.0 + exp(-v)); }

/* softplus(v) = log(1 + exp(v)), written so that neither branch overflows. */
static double softplus(double v) {
    if (v > 0.0) return v + log1p(exp(-v));
    return log1p(exp(v));
}

static int seg_of(const int32_t* seq, int L, int b, int t) {
    return seq ? seq[(size_t)b * L + t] : 0;
}

/* Round one double to the nearest bfloat16 value (8 significant bits,
 * ties to even). Used only to mirror where the GPU path stores bf16. */
static double round_bf16_one(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    double m = frexp(v, &e);               /* v = m * 2^e, 0.5 <= |m| < 1 */
    if (e < -125) {                        /* below the bf16 normal range */
        double q = ldexp(1.0, -133);       /* bf16 subnormal spacing */
        return nearbyint(v / q) * q;
    }
    double r = ldexp(nearbyint(ldexp(m, 8)), e - 8);
    return r;
}

void oracle_round_bf16(const double* in, double* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = round_bf16_one(in[i]);
}

/* ------------------------------------------------------------- conv1d fwd */
/* One row (b, d): c_t = bias + sum_k w[k] x_{t-W+1+k} over taps inside the
 * sequence and the output token's segment; u_t = silu(c_t) or c_t. */
static void conv_fwd_row(const double* x, const double* w, double bias,
                         const int32_t* seq, int b, int L, int W, int silu,
                         double* c, double* u) {
    for (int t = 0; t < L; ++t) {
        int st = seg_of(seq, L, b, t);
        double acc = bias;
        for (int k = 0; k < W; ++k) {
            int s = t - (W - 1) + k;
            if (s < 0) continue;
            if (seg_of(seq, L, b, s) != st) continue;
            acc += w[k] * x[s];
        }
        if (c) c[t] = acc;
        u[t] = silu ? acc * sigm(acc) : acc;
    }
}

void oracle_conv1d_fwd(const double* x, const double* w, const double* bias,
                       const int32_t* seq, double* c, double* u,
                       int B, int D, int L, int W, int silu) {
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            size_t row = ((size_t)b * D + d) * L;
            conv_fwd_row(x + row, w + (size_t)d * W, bias ? bias[d] : 0.0, seq,
                         b, L, W, silu, c ? c + row : NULL, u + row);
        }
}

/* ------------------------------------------------------------- conv1d bwd */
/* Transpose of conv_fwd_row under the same masks. dw/dbias accumulate. */
static void conv_bwd_row(const double* x, const double* w, double bias,
                         const int32_t* seq, int b, int L, int W, int silu,
                         const double* du, double* dx, double* dw, double* dbias) {
    for (int s = 0; s < L; ++s) dx[s] = 0.0;
    for (int t = 0; t < L; ++t) {
        int st = seg_of(seq, L, b, t);
        double c = bias;
        for (int k = 0; k < W; ++k) {
            int s = t - (W - 1) + k;
            if (s < 0 || seg_of(seq, L, b, s) != st) continue;
            c += w[k] * x[s];
        }
        double dc = du[t];
        if (silu) {
            double sg = sigm(c);
            dc *= sg * (1.0 + c * (1.0 - sg));
        }
        *dbias += dc;
        for (int k = 0; k < W; ++k) {
            int s = t - (W - 1) + k;
            if (s < 0 || seg_of(seq, L, b, s) != st) continue;
            dx[s] += w[k] * dc;
            dw[k] += x[s] * dc;
        }
    }
}

void oracle_conv1d_bwd(const double* x, const double* w, const double* bias,
                       const int32_t* seq, const double* du, double* dx,
                       double* dw, double* dbias, int B, int D, int L, int W,
                       int silu) {
    memset(dw, 0, sizeof(double) * (size_t)D * W);
    memset(dbias, 0, sizeof(double) * (size_t)D);
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            size_t row = ((size_t)b * D + d) * L;
            conv_bwd_row(x + row, w + (size_t)d * W, bias ? bias[d] : 0.0, seq, b,
                         L, W, silu, du + row, dx + row, dw + (size_t)d * W,
                         dbias + d);
        }
}

/* --------------------------------------------------------------- scan fwd */
typedef struct {
    const double *u, *delta, *z, *A, *Dskip, *delta_bias, *Bm, *Cm;
    const int32_t* seq;
    int B, D, L, N, softplus_on;
    const double* h0;   /* [B][D][N] state before token 0, NULL = zero */
    int zoh;            /* 0: B_bar = dt B; 1: zero-order hold B_bar = (exp(dt A) - 1) / A B */
} scan_in_t;

/* The factor multiplying B_t u_t in the state update: dt (the S6 block of
 * "Architecture Diagram") or, with zero-order hold ("Discretization"),
 * A^{-1} (exp(dt A) - 1), whose A -> 0 limit is dt. */
static double bbar_factor(const scan_in_t* p, double dt, double A) {
    if (!p->zoh) return dt;
    return A == 0.0 ? dt : expm1(dt * A) / A;
}

/* d(bbar_factor)/dA for zero-order hold: (dt e^{dt A} A - (e^{dt A} - 1)) / A^2,
 * by its Taylor series dt^2 (1/2 + x/3 + x^2/8 + x^3/30 + x^4/144) near
 * x = dt A = 0 (where the closed form cancels). */
static double bbar_factor_dA(double dt, double A) {
    double x = dt * A;
    if (fabs(x) < 1e-3)
        return dt * dt * (0.5 + x * (1.0 / 3.0 + x * (1.0 / 8.0 + x * (1.0 / 30.0 + x / 144.0))));
    return (dt * exp(x) * A - expm1(x)) / (A * A);
}

/* State before token 0 of row (b, d), state n. */
static double h0_at(const scan_in_t* p, int b, int d, int n) {
    return p->h0 ? p->h0[((size_t)b * p->D + d) * p->N + n] : 0.0;
}

/* delta_t for row (b, d), token t (softplus of raw + bias, or raw + bias). */
static double delta_at(const scan_in_t* p, int d, size_t row, int t) {
    double v = p->delta[row + t] + (p->delta_bias ? p->delta_bias[d] : 0.0);
    return p->softplus_on ? softplus(v) : v;
}

/* One row: sequential recurrence over t, all N states. Writes out (gated),
 * y (before the gate, optional) and the state after the last token. */
static void scan_fwd_row(const scan_in_t* p, int b, int d, double* out,
                         double* y_out, double* final_state) {
    const int L = p->L, N = p->N;
    size_t row = ((size_t)b * p->D + d) * L;
    double* h = (double*)calloc((size_t)N, sizeof(double));
    for (int n = 0; n < N; ++n) h[n] = h0_at(p, b, d, n);
    for (int t = 0; t < L; ++t) {
        double dt = delta_at(p, d, row, t);
        double ut = p->u[row + t];
        int reset = (t > 0) && seg_of(p->seq, L, b, t) != seg_of(p->seq, L, b, t - 1);
        double y = 0.0;
        for (int n = 0; n < N; ++n) {
            double abar = exp(dt * p->A[(size_t)d * N + n]);
            double bt = p->Bm[((size_t)b * N + n) * L + t];
            double ct = p->Cm[((size_t)b * N + n) * L + t];
            double hprev = reset ? 0.0 : h[n];
            h[n] = abar * hprev + bbar_factor(p, dt, p->A[(size_t)d * N + n]) * bt * ut;
            y += ct * h[n];
        }
        if (p->Dskip) y += p->Dskip[d] * ut;
        if (y_out) y_out[row + t] = y;
        if (p->z) {
            double zt = p->z[row + t];
            out[row + t] = y * zt * sigm(zt);
        } else {
            out[row + t] = y;
        }
    }
    if (final_state)
        for (int n = 0; n < N; ++n) final_state[((size_t)b * p->D + d) * N + n] = h[n];
    free(h);
}

void oracle_scan_fwd(const double* u, const double* delta, const double* z,
                     const double* A, const double* Dskip, const double* delta_bias,
                     const double* Bm, const double* Cm, int softplus_on, int zoh,
                     const int32_t* seq, const double* h0, double* out, double* y_out,
                     double* final_state, int B, int D, int L, int N) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, zoh};
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) scan_fwd_row(&p, b, d, out, y_out, final_state);
}

/* --------------------------------------------------------------- scan bwd */
typedef struct {
    const double* dout;
    double *du, *ddelta, *dz;          /* per row, overwritten */
    double *dA, *dB, *dC, *dD, *ddb;   /* accumulated */
    double* dh0;                       /* [B][D][N] per row, overwritten; may be NULL */
    const double* dhL;                 /* [B][D][N] dL/dh_{L-1} from outside; may be NULL */
} scan_grad_t;

/* One row. Re-runs the forward keeping every h_t and A_bar_t, then walks t
 * backwards with g_t = dL/dh_t:
 *   g_t = dy_t C_t + r_{t+1} A_bar_{t+1} g_{t+1}
 * and collects every input / parameter gradient from it. */
static void scan_bwd_row(const scan_in_t* p, const scan_grad_t* g, int b, int d) {
    const int L = p->L, N = p->N;
    size_t row = ((size_t)b * p->D + d) * L;
    double* hs = (double*)malloc(sizeof(double) * (size_t)L * N);
    double* ab = (double*)malloc(sizeof(double) * (size_t)L * N);
    double* dts = (double*)malloc(sizeof(double) * (size_t)L);
    double* ys = (double*)malloc(sizeof(double) * (size_t)L);
    int* rs = (int*)malloc(sizeof(int) * (size_t)L);
    double* carry = (double*)calloc((size_t)N, sizeof(double));
    double Dd = p->Dskip ? p->Dskip[d] : 0.0;
    /* a gradient reaching h_{L-1} from outside enters g_{L-1} like the carry */
    if (g->dhL)
        for (int n = 0; n < N; ++n) carry[n] = g->dhL[((size_t)b * p->D + d) * N + n];

    for (int t = 0; t < L; ++t) {
        double dt = delta_at(p, d, row, t);
        double ut = p->u[row + t];
        int reset = (t > 0) && seg_of(p->seq, L, b, t) != seg_of(p->seq, L, b, t - 1);
        double y = 0.0;
        dts[t] = dt;
        rs[t] = reset ? 0 : 1;
        for (int n = 0; n < N; ++n) {
            double abar = exp(dt * p->A[(size_t)d * N + n]);
            double bt = p->Bm[((size_t)b * N + n) * L + t];
            double ct = p->Cm[((size_t)b * N + n) * L + t];
            double hprev = reset ? 0.0 : (t == 0 ? h0_at(p, b, d, n) : hs[(size_t)(t - 1) * N + n]);
            double h = abar * hprev + bbar_factor(p, dt, p->A[(size_t)d * N + n]) * bt * ut;
            hs[(size_t)t * N + n] = h;
            ab[(size_t)t * N + n] = abar;
            y += ct * h;
        }
        ys[t] = y + Dd * ut;
    }

    for (int t = L - 1; t >= 0; --t) {
        double ut = p->u[row + t];
        double dt = dts[t];
        double go = g->dout[row + t];
        double dy;
        if (p->z) {
            double zt = p->z[row + t];
            double sg = sigm(zt);
            dy = go * zt * sg;
            g->dz[row + t] = go * ys[t] * sg * (1.0 + zt * (1.0 - sg));
        } else {
            dy = go;
            if (g->dz) g->dz[row + t] = 0.0;
        }
        if (g->dD) g->dD[d] += dy * ut;
        double sgB = 0.0, sAq = 0.0;
        for (int n = 0; n < N; ++n) {
            size_t bn = ((size_t)b * N + n) * L + t;
            double An = p->A[(size_t)d * N + n];
            double gt = dy * p->Cm[bn] + carry[n];
            double hprev = (t == 0) ? h0_at(p, b, d, n) : hs[(size_t)(t - 1) * N + n];
            double q = gt * rs[t] * ab[(size_t)t * N + n] * hprev; /* g * dh/d(A_bar) * A_bar */
            g->dC[bn] += dy * hs[(size_t)t * N + n];
            if (p->zoh) {
                /* h_t = A_bar h_{t-1} + phi B u with phi = (e^{dt A} - 1) / A:
                 * dphi/d(dt) = A_bar, dphi/dA from bbar_factor_dA */
                double phi = bbar_factor(p, dt, An);
                g->dB[bn] += gt * phi * ut;
                g->dA[(size_t)d * N + n] += q * dt + gt * p->Bm[bn] * ut * bbar_factor_dA(dt, An);
                sgB += gt * phi * p->Bm[bn];                       /* -> du */
                sAq += An * q + gt * p->Bm[bn] * ut * ab[(size_t)t * N + n];  /* -> d(dt) */
            } else {
                g->dB[bn] += gt * dt * ut;
                g->dA[(size_t)d * N + n] += q * dt;
                sgB += gt * p->Bm[bn];
                sAq += An * q;
            }
            carry[n] = rs[t] * ab[(size_t)t * N + n] * gt;
        }
        g->du[row + t] = dy * Dd + (p->zoh ? sgB : dt * sgB);
        double ddt = p->zoh ? sAq : ut * sgB + sAq;
        double dv = ddt;
        if (p->softplus_on) {
            double v = p->delta[row + t] + (p->delta_bias ? p->delta_bias[d] : 0.0);
            dv = ddt * sigm(v);
        }
        g->ddelta[row + t] = dv;
        if (g->ddb) g->ddb[d] += dv;
    }
    /* h_{-1} enters token 0 only through A_bar_0 h_{-1}: its gradient is the
     * carry left after token 0 */
    if (g->dh0)
        for (int n = 0; n < N; ++n) g->dh0[((size_t)b * p->D + d) * N + n] = carry[n];
    free(hs); free(ab); free(dts); free(ys); free(rs); free(carry);
}

void oracle_scan_bwd(const double* u, const double* delta, const double* z,
                     const double* A, const double* Dskip, const double* delta_bias,
                     const double* Bm, const double* Cm, int softplus_on, int zoh,
                     const int32_t* seq, const double* h0, const double* dout, double* du,
                     double* ddelta, double* dz, double* dA, double* dB,
                     double* dC, double* dD, double* ddelta_bias, double* dh0,
                     const double* dhL, int B, int D, int L, int N) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, zoh};
    memset(dA, 0, sizeof(double) * (size_t)D * N);
    memset(dB, 0, sizeof(double) * (size_t)B * N * L);
    memset(dC, 0, sizeof(double) * (size_t)B * N * L);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)D);
    if (ddelta_bias) memset(ddelta_bias, 0, sizeof(double) * (size_t)D);
    scan_grad_t g = {dout, du, ddelta, dz, dA, dB, dC, dD, ddelta_bias, dh0, dhL};
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) scan_bwd_row(&p, &g, b, d);
}

/* ------------------------------------------------- threaded row drivers */
/* Rows are independent; only the reductions over rows (dA, dB, dC, dD,
 * ddelta_bias) need per-thread partials, added afterwards in thread order. */
typedef struct {
    const scan_in_t* p;
    scan_grad_t g;      /* per-thread accumulators for the reductions */
    double *out, *y_out, *final_state;
    int row_begin, row_end, bwd;
} job_t;

static void* run_job(void* arg) {
    job_t* j = (job_t*)arg;
    for (int r = j->row_begin; r < j->row_end; ++r) {
        int b = r / j->p->D, d = r % j->p->D;
        if (j->bwd) scan_bwd_row(j->p, &j->g, b, d);
        else scan_fwd_row(j->p, b, d, j->out, j->y_out, j->final_state);
    }
    return NULL;
}

void oracle_scan_fwd_mt(const double* u, const double* delta, const double* z,
                        const double* A, const double* Dskip, const double* delta_bias,
                        const double* Bm, const double* Cm, int softplus_on, int zoh,
                        const int32_t* seq, const double* h0, double* out, double* y_out,
                        double* final_state, int B, int D, int L, int N, int nthreads) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, zoh};
    int rows = B * D;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = rows;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].p = &p;
        jobs[i].out = out; jobs[i].y_out = y_out; jobs[i].final_state = final_state;
        jobs[i].row_begin = (int)((long)rows * i / nthreads);
        jobs[i].row_end = (int)((long)rows * (i + 1) / nthreads);
        pthread_create(&th[i], NULL, run_job, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th); free(jobs);
}

void oracle_scan_bwd_mt(const double* u, const double* delta, const double* z,
                        const double* A, const double* Dskip, const double* delta_bias,
                        const double* Bm, const double* Cm, int softplus_on, int zoh,
                        const int32_t* seq, const double* h0, const double* dout, double* du,
                        double* ddelta, double* dz, double* dA, double* dB,
                        double* dC, double* dD, double* ddelta_bias, double* dh0,
                        const double* dhL, int B, int D, int L, int N, int nthreads) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, zoh};
    int rows = B * D;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > rows) nthreads = rows;
    size_t nA = (size_t)D * N, nBC = (size_t)B * N * L;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    job_t* jobs = (job_t*)calloc((size_t)nthreads, sizeof(job_t));
    for (int i = 0; i < nthreads; ++i) {
        jobs[i].p = &p;
        jobs[i].bwd = 1;
        jobs[i].g.dout = dout;
        jobs[i].g.du = du; jobs[i].g.ddelta = ddelta; jobs[i].g.dz = dz;
        jobs[i].g.dh0 = dh0;
        jobs[i].g.dhL = dhL;
        jobs[i].g.dA = (double*)calloc(nA, sizeof(double));
        jobs[i].g.dB = (double*)calloc(nBC, sizeof(double));
        jobs[i].g.dC = (double*)calloc(nBC, sizeof(double));
        jobs[i].g.dD = (double*)calloc((size_t)D, sizeof(double));
        jobs[i].g.ddb = (double*)calloc((size_t)D, sizeof(double));
        jobs[i].row_begin = (int)((long)rows * i / nthreads);
        jobs[i].row_end = (int)((long)rows * (i + 1) / nthreads);
        pthread_create(&th[i], NULL, run_job, &jobs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    memset(dA, 0, sizeof(double) * nA);
    memset(dB, 0, sizeof(double) * nBC);
    memset(dC, 0, sizeof(double) * nBC);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)D);
    if (ddelta_bias) memset(ddelta_bias, 0, sizeof(double) * (size_t)D);
    for (int i = 0; i < nthreads; ++i) {
        for (size_t k = 0; k < nA; ++k) dA[k] += jobs[i].g.dA[k];
        for (size_t k = 0; k < nBC; ++k) { dB[k] += jobs[i].g.dB[k]; dC[k] += jobs[i].g.dC[k]; }
        for (int k = 0; k < D; ++k) {
            if (dD) dD[k] += jobs[i].g.dD[k];
            if (ddelta_bias) ddelta_bias[k] += jobs[i].g.ddb[k];
        }
        free(jobs[i].g.dA); free(jobs[i].g.dB); free(jobs[i].g.dC);
        free(jobs[i].g.dD); free(jobs[i].g.ddb);
    }
    free(th); free(jobs);
}

/* ------------------------------------------------------- recurrent step */
/* One token for every (b, d): the recurrent (decode) form of the layer.
 * conv_state[b][d][0..W-2] holds the W-1 previous inputs x_{t-W+1} .. x_{t-1}
 * (oldest first); the causal conv reads them and x_t, then the window shifts
 * by one. The state h[b][d][n] (h_{t-1} on entry) becomes h_t. Follows the
 * same definitions as the sequence form: conv taps w[d][k] on x_{t-W+1+k},
 * u = SiLU(c), delta = softplus(raw + bias), h_t = exp(delta A) h_{t-1} +
 * delta B_t u, y = C_t . h_t + D u, out = y SiLU(z). u_out may be NULL. */
void oracle_decode_step(const double* x, double* conv_state, const double* w,
                        const double* conv_bias, const double* delta, const double* z,
                        const double* Bt, const double* Ct, const double* A,
                        const double* Dskip, const double* delta_bias, int softplus_on,
                        double* h, double* out, double* u_out, int B, int D, int N, int W) {
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            size_t bd = (size_t)b * D + d;
            double* cs = conv_state + bd * (size_t)(W - 1);
            double c = conv_bias ? conv_bias[d] : 0.0;
            for (int k = 0; k < W - 1; ++k) c += w[(size_t)d * W + k] * cs[k];
            c += w[(size_t)d * W + W - 1] * x[bd];
            for (int k = 0; k + 1 < W - 1; ++k) cs[k] = cs[k + 1];
            if (W > 1) cs[W - 2] = x[bd];
            double u = c * sigm(c);
            if (u_out) u_out[bd] = u;
            double v = delta[bd] + (delta_bias ? delta_bias[d] : 0.0);
            double dt = softplus_on ? softplus(v) : v;
            double y = 0.0;
            for (int n = 0; n < N; ++n) {
                double* hn = h + bd * (size_t)N + n;
                *hn = exp(dt * A[(size_t)d * N + n]) * *hn + dt * Bt[(size_t)b * N + n] * u;
                y += Ct[(size_t)b * N + n] * *hn;
            }
            if (Dskip) y += Dskip[d] * u;
            out[bd] = z ? y * z[bd] * sigm(z[bd]) : y;
        }
}

/* ------------------------------------------------- complex diagonal A */
/* Diagonal A with complex entries ("hung-phan ml-skills mamba", section
 * "S4: Structured State Spaces for Sequences", the S4D simplification; the
 * same page's Mamba-3 list names a complex-valued state update), made
 * selective like the real scan:
 *   a_t = exp(dt_t A_n),  h_t = a_t h_{t-1} + dt_t u_t B_t   (complex h, B)
 *   y_t = 2 Re(sum_n C_t h_t) + D u_t,  out = y silu(z)
 * The pages do not say how a complex state yields a real output; this takes
 * S4D's convention that each state stands for itself and its conjugate,
 * hence 2 Re. Layouts: A [D][N][2] (re, im); Bm, Cm [B][N][2][L] (real
 * plane then imaginary plane per state); h0 / final state [B][D][N][2].
 * Document resets as in the real scan. */
typedef double complex cplx;

static cplx cld(const double* p) { return p[0] + I * p[1]; }

/* One row. out_row / y_row point at the row's L outputs (y_row nullable);
 * with hs / as (L x N each) the states and decays are kept for the
 * backward. */
static void cscan_fwd_row(const scan_in_t* p, int b, int d, double* out_row, double* y_row,
                          double* final_state, cplx* hs, cplx* as) {
    const int L = p->L, N = p->N;
    size_t row = ((size_t)b * p->D + d) * L;
    size_t bd = (size_t)b * p->D + d;
    cplx* h = (cplx*)calloc((size_t)N, sizeof(cplx));
    for (int n = 0; n < N; ++n)
        if (p->h0) h[n] = cld(p->h0 + (bd * N + n) * 2);
    for (int t = 0; t < L; ++t) {
        double dt = delta_at(p, d, row, t);
        double ut = p->u[row + t];
        int reset = (t > 0) && seg_of(p->seq, L, b, t) != seg_of(p->seq, L, b, t - 1);
        double y = 0.0;
        for (int n = 0; n < N; ++n) {
            cplx An = cld(p->A + ((size_t)d * N + n) * 2);
            size_t bn = (((size_t)b * N + n) * 2) * L + t;   /* real plane; imag at + L */
            cplx Bt = p->Bm[bn] + I * p->Bm[bn + L];
            cplx Ct = p->Cm[bn] + I * p->Cm[bn + L];
            cplx a = cexp(dt * An);
            cplx hp = reset ? 0.0 : h[n];
            h[n] = a * hp + dt * ut * Bt;
            if (hs) {
                hs[(size_t)t * N + n] = h[n];
                as[(size_t)t * N + n] = a;
            }
            y += 2.0 * creal(Ct * h[n]);
        }
        if (p->Dskip) y += p->Dskip[d] * ut;
        if (y_row) y_row[t] = y;
        out_row[t] = p->z ? y * p->z[row + t] * sigm(p->z[row + t]) : y;
    }
    if (final_state)
        for (int n = 0; n < N; ++n) {
            double* f = final_state + (bd * N + n) * 2;
            f[0] = creal(h[n]);
            f[1] = cimag(h[n]);
        }
    free(h);
}

void oracle_cscan_fwd(const double* u, const double* delta, const double* z, const double* A,
                      const double* Dskip, const double* delta_bias, const double* Bm,
                      const double* Cm, int softplus_on, const int32_t* seq, const double* h0,
                      double* out, double* y_out, double* final_state, int B, int D, int L, int N) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, 0};
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            size_t row = ((size_t)b * D + d) * L;
            cscan_fwd_row(&p, b, d, out + row, y_out ? y_out + row : NULL, final_state, NULL, NULL);
        }
}

/* Reverse mode, with g_t = dL/dRe(h_t) + i dL/dIm(h_t):
 *   g_t = 2 dy_t conj(C_t) + conj(a_{t+1}) g_{t+1}   (no carry into a document's end)
 * For a real parameter theta entering through a complex w(theta) the
 * gradient is Re(conj(dL/dw) dw/dtheta): dL/da_t = g_t conj(h_{t-1}) (0 at a
 * document start), da/d(dt) = A a, da/dRe A = dt a, da/dIm A = i dt a;
 * dL/d(dt u) = Re(conj(g) B); dL/dB = dt u g; dL/dC = 2 dy conj(h). */
void oracle_cscan_bwd(const double* u, const double* delta, const double* z, const double* A,
                      const double* Dskip, const double* delta_bias, const double* Bm,
                      const double* Cm, int softplus_on, const int32_t* seq, const double* h0,
                      const double* dout, double* du, double* ddelta, double* dz, double* dA,
                      double* dB, double* dC, double* dD, double* ddelta_bias, double* dh0,
                      const double* dhL, int B, int D, int L, int N) {
    scan_in_t p = {u, delta, z, A, Dskip, delta_bias, Bm, Cm, seq, B, D, L, N, softplus_on, h0, 0};
    memset(dA, 0, sizeof(double) * (size_t)D * N * 2);
    memset(dB, 0, sizeof(double) * (size_t)B * N * 2 * L);
    memset(dC, 0, sizeof(double) * (size_t)B * N * 2 * L);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)D);
    if (ddelta_bias) memset(ddelta_bias, 0, sizeof(double) * (size_t)D);
    cplx* hs = (cplx*)malloc(sizeof(cplx) * (size_t)L * N);
    cplx* as = (cplx*)malloc(sizeof(cplx) * (size_t)L * N);
    double* ys = (double*)malloc(sizeof(double) * (size_t)L);
    double* os = (double*)malloc(sizeof(double) * (size_t)L);
    cplx* carry = (cplx*)malloc(sizeof(cplx) * (size_t)N);
    for (int b = 0; b < B; ++b)
        for (int d = 0; d < D; ++d) {
            size_t row = ((size_t)b * D + d) * L;
            size_t bd = (size_t)b * D + d;
            cscan_fwd_row(&p, b, d, os, ys, NULL, hs, as);  /* h_t, a_t, y_t of this row */
            double Dd = Dskip ? Dskip[d] : 0.0;
            for (int n = 0; n < N; ++n)  /* dL/dh_{L-1} from outside, or 0 */
                carry[n] = dhL ? cld(dhL + (bd * N + n) * 2) : 0.0;
            for (int t = L - 1; t >= 0; --t) {
                double ut = u[row + t];
                double dt = delta_at(&p, d, row, t);
                double go = dout[row + t];
                int reset = (t > 0) && seg_of(seq, L, b, t) != seg_of(seq, L, b, t - 1);
                double dy;
                if (z) {
                    double zt = z[row + t], sg = sigm(zt);
                    dy = go * zt * sg;
                    dz[row + t] = go * ys[t] * sg * (1.0 + zt * (1.0 - sg));
                } else {
                    dy = go;
                    if (dz) dz[row + t] = 0.0;
                }
                if (dD) dD[d] += dy * ut;
                double sgB = 0.0, sA = 0.0;
                for (int n = 0; n < N; ++n) {
                    cplx An = cld(A + ((size_t)d * N + n) * 2);
                    size_t bn = (((size_t)b * N + n) * 2) * L + t;
                    cplx Bt = Bm[bn] + I * Bm[bn + L];
                    cplx Ct = Cm[bn] + I * Cm[bn + L];
                    cplx h = hs[(size_t)t * N + n], a = as[(size_t)t * N + n];
                    cplx g = 2.0 * dy * conj(Ct) + carry[n];
                    cplx hprev = t == 0 ? (h0 ? cld(h0 + (bd * N + n) * 2) : 0.0)
                                        : hs[(size_t)(t - 1) * N + n];
                    cplx Ga = reset ? 0.0 : g * conj(hprev);
                    double* dAn = dA + ((size_t)d * N + n) * 2;
                    dAn[0] += creal(conj(Ga) * dt * a);
                    dAn[1] += creal(conj(Ga) * I * dt * a);
                    sA += creal(conj(Ga) * An * a);
                    sgB += creal(conj(g) * Bt);
                    dB[bn] += creal(g) * dt * ut;
                    dB[bn + L] += cimag(g) * dt * ut;
                    dC[bn] += 2.0 * dy * creal(h);
                    dC[bn + L] += -2.0 * dy * cimag(h);
                    carry[n] = reset ? 0.0 : conj(a) * g;
                    if (t == 0 && dh0) {
                        double* o = dh0 + (bd * N + n) * 2;
                        o[0] = creal(carry[n]);
                        o[1] = cimag(carry[n]);
                    }
                }
                du[row + t] = dy * Dd + dt * sgB;
                double ddt = ut * sgB + sA;
                double dv = ddt;
                if (softplus_on) {
                    double v = delta[row + t] + (delta_bias ? delta_bias[d] : 0.0);
                    dv = ddt * sigm(v);
                }
                ddelta[row + t] = dv;
                if (ddelta_bias) ddelta_bias[d] += dv;
            }
        }
    free(hs); free(as); free(ys); free(os); free(carry);
}

/* ------------------------------------------------------ Mamba-2 SSD form */
/* "hung-phan ml-skills mamba", section "Mamba-2: Structured State Space
 * Duality (SSD)": A restricted to a scalar times the identity, per head;
 * multi-head (d split into H heads of width P); B and C shared by the heads
 * of a group (G groups, head h in group h / (H / G)). Per (batch, head), with
 * a_t = exp(dt_t A_h) and a state h of P x N:
 *   h_t[p][n] = a_t h_{t-1}[p][n] + dt_t x_t[p] B_t[n]
 *   y_t[p]    = sum_n C_t[n] h_t[p][n] + D_h x_t[p]
 * dt_t = softplus(dt_raw_t + dt_bias_h) (or without softplus); a document
 * start (seq_idx change) zeroes a_t as in the Mamba-1 scan. Layouts
 * (token-major): x, y, dx [B][L][H][P]; dt [B][L][H]; A, D, dt_bias [H];
 * Bm, Cm [B][L][G][N]; final state [B][H][P][N]. */
typedef struct {
    const double *x, *dt_raw, *A, *Bm, *Cm, *Dh, *dt_bias;
    const int32_t* seq;
    int B, L, H, P, G, N, softplus_on;
} ssd_in_t;

static double ssd_dt(const ssd_in_t* p, int b, int t, int h) {
    double v = p->dt_raw[((size_t)b * p->L + t) * p->H + h] + (p->dt_bias ? p->dt_bias[h] : 0.0);
    return p->softplus_on ? softplus(v) : v;
}

/* One (batch, head): runs the recurrence, keeping every state when hs is
 * non-NULL ([L][P][N]). */
static void ssd_fwd_head(const ssd_in_t* p, int b, int h, double* y, double* final_state,
                         double* hs) {
    const int L = p->L, H = p->H, P = p->P, G = p->G, N = p->N;
    const int g = h / (H / G);
    double* st = (double*)calloc((size_t)P * N, sizeof(double));
    for (int t = 0; t < L; ++t) {
        const double dt = ssd_dt(p, b, t, h);
        const int reset = (t > 0) && seg_of(p->seq, L, b, t) != seg_of(p->seq, L, b, t - 1);
        const double a = reset ? 0.0 : exp(dt * p->A[h]);
        const double* xt = p->x + (((size_t)b * L + t) * H + h) * P;
        const double* Bt = p->Bm + (((size_t)b * L + t) * G + g) * N;
        const double* Ct = p->Cm + (((size_t)b * L + t) * G + g) * N;
        for (int q = 0; q < P; ++q) {
            double acc = 0.0;
            for (int n = 0; n < N; ++n) {
                double* s = st + (size_t)q * N + n;
                *s = a * *s + dt * xt[q] * Bt[n];
                acc += Ct[n] * *s;
            }
            if (y) y[(((size_t)b * L + t) * H + h) * P + q] = acc + (p->Dh ? p->Dh[h] * xt[q] : 0.0);
        }
        if (hs) memcpy(hs + (size_t)t * P * N, st, sizeof(double) * (size_t)P * N);
    }
    if (final_state)
        memcpy(final_state + ((size_t)b * H + h) * P * N, st, sizeof(double) * (size_t)P * N);
    free(st);
}

void oracle_ssd_fwd(const double* x, const double* dt_raw, const double* A, const double* Bm,
                    const double* Cm, const double* Dh, const double* dt_bias, int softplus_on,
                    const int32_t* seq, double* y, double* final_state, int B, int L, int H, int P,
                    int G, int N) {
    ssd_in_t p = {x, dt_raw, A, Bm, Cm, Dh, dt_bias, seq, B, L, H, P, G, N, softplus_on};
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) ssd_fwd_head(&p, b, h, y, final_state, NULL);
}

/* Reverse mode, per (batch, head), with the adjoint of the state
 *   Gs_t[p][n] = dy_t[p] C_t[n] + a_{t+1} Gs_{t+1}[p][n]   (a_{t+1} = 0 at a start)
 * dx_t[p]   = D_h dy_t[p] + dt_t sum_n Gs_t[p][n] B_t[n]
 * d dt_t    = sum_{p,n} Gs_t[p][n] (x_t[p] B_t[n] + a_t A_h h_{t-1}[p][n])
 * dA_h     += sum_t dt_t sum_{p,n} Gs_t[p][n] a_t h_{t-1}[p][n]
 * dB_t[n]  += dt_t sum_p Gs_t[p][n] x_t[p]      (summed over the group's heads)
 * dC_t[n]  += sum_p dy_t[p] h_t[p][n]           (same)
 * dD_h     += sum_t sum_p dy_t[p] x_t[p]; d dt_raw = d dt * sigmoid(v) with softplus. */
void oracle_ssd_bwd(const double* x, const double* dt_raw, const double* A, const double* Bm,
                    const double* Cm, const double* Dh, const double* dt_bias, int softplus_on,
                    const int32_t* seq, const double* dy, double* dx, double* ddt_raw, double* dA,
                    double* dB, double* dC, double* dD, double* ddt_bias, int B, int L, int H,
                    int P, int G, int N) {
    ssd_in_t p = {x, dt_raw, A, Bm, Cm, Dh, dt_bias, seq, B, L, H, P, G, N, softplus_on};
    memset(dA, 0, sizeof(double) * (size_t)H);
    memset(dB, 0, sizeof(double) * (size_t)B * L * G * N);
    memset(dC, 0, sizeof(double) * (size_t)B * L * G * N);
    if (dD) memset(dD, 0, sizeof(double) * (size_t)H);
    if (ddt_bias) memset(ddt_bias, 0, sizeof(double) * (size_t)H);
    double* hs = (double*)malloc(sizeof(double) * (size_t)L * P * N);
    double* gs = (double*)calloc((size_t)P * N, sizeof(double));   /* a_{t+1} Gs_{t+1} */
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const int g = h / (H / G);
            ssd_fwd_head(&p, b, h, NULL, NULL, hs);
            memset(gs, 0, sizeof(double) * (size_t)P * N);
            for (int t = L - 1; t >= 0; --t) {
                const double dt = ssd_dt(&p, b, t, h);
                const int reset = (t > 0) && seg_of(seq, L, b, t) != seg_of(seq, L, b, t - 1);
                const double a = reset ? 0.0 : exp(dt * A[h]);
                const size_t xo = (((size_t)b * L + t) * H + h) * P;
                const size_t bo = (((size_t)b * L + t) * G + g) * N;
                double ddt = 0.0, dAh = 0.0;
                for (int q = 0; q < P; ++q) {
                    double sgb = 0.0;
                    const double dyq = dy[xo + q], xq = x[xo + q];
                    for (int n = 0; n < N; ++n) {
                        const double G_ = dyq * Cm[bo + n] + gs[(size_t)q * N + n];
                        const double hprev = t > 0 ? hs[(size_t)(t - 1) * P * N + (size_t)q * N + n] : 0.0;
                        sgb += G_ * Bm[bo + n];
                        ddt += G_ * (xq * Bm[bo + n] + a * A[h] * hprev);
                        dAh += G_ * a * dt * hprev;
                        dB[bo + n] += G_ * dt * xq;
                        dC[bo + n] += dyq * hs[(size_t)t * P * N + (size_t)q * N + n];
                        gs[(size_t)q * N + n] = a * G_;
                    }
                    dx[xo + q] = (Dh ? Dh[h] * dyq : 0.0) + dt * sgb;
                    if (dD) dD[h] += dyq * xq;
                }
                dA[h] += dAh;
                double dv = ddt;
                if (softplus_on) {
                    const double v = dt_raw[((size_t)b * L + t) * H + h] + (dt_bias ? dt_bias[h] : 0.0);
                    dv = ddt * sigm(v);
                }
                ddt_raw[((size_t)b * L + t) * H + h] = dv;
                if (ddt_bias) ddt_bias[h] += dv;
            }
        }
    free(hs);
    free(gs);
}

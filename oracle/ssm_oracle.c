/*
 * ssm_oracle.c -- plain, sequential, double-precision CPU oracle for the
 * selective scan (Mamba-1) and the scalar-decay scan (Mamba-2 / SSD).
 *
 * TEST INFRASTRUCTURE ONLY.  The test-suite, the smoke check and the CPU
 * baseline leg of the benchmark are the only users of this file.  The
 * library path never links, loads or calls it, and it shares no code,
 * header or constant with the CUDA kernels.
 *
 * Sources (page titles as printed on the pages):
 *  [P1] "Mamba ... 硬件感知 ... 并行扫描" (mhpq.cn), section 2.2: the LTI
 *       state space model x' = Ax + Bu, y = Cx + Du, discretised with
 *       A_d = exp(A*dt); section 2.3: the recurrence x_{k+1} = A x_k + B u_k.
 *       Section 3.1: A is diagonal, so exp(A*dt) is an elementwise exp.
 *  [P2] "从硬件感知到算法革命：Mamba如何重塑序列建模的计算效率"
 *       (tencentcloud), section 2: dt = softplus(Linear(x)), B and C are
 *       functions of the input; section 3: SiLU gate fused after the SSM.
 *  [P3] "Mamba与选择性SSM" (mlqm.cn), section 5.4: incremental decoding keeps
 *       only the fixed-size state between tokens.
 *  [P4] "Mamba状态空间模型的硬件感知推理优化" (ybb.press), section 1:
 *       h_t = A h_{t-1} + B x_t, y_t = C h_t; section 3.1: y = C h + D x;
 *       section 4: Mamba-2 scalar decay h_t = a_t h_{t-1} + b_t x_t.
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes of the repository):
 *  - the input term is dt' * B * u (the pages never spell out the
 *    discretisation of B; the Euler form is the plainest one that matches
 *    "B * x_t" in [P4] once the step size is applied);
 *  - dt' = softplus(dt + bias_d), softplus(s) = log1p(exp(s)), returned
 *    as s itself for s > 20;
 *  - with the softplus flag off, dt' = dt + bias_d;
 *  - the skip term D*u sits inside the gate: y = (C.h + D u) * silu(z);
 *  - A is passed already negative (no A_log exponentiation here);
 *  - Mamba-2: S <- a_t S + dt'_t x_t B_t^T with a_t = exp(dt'_t A_h),
 *    y_t = S C_t + D_h x_t, optional silu(z) gate.
 *
 * Parallelism: channels (b, d) -- or heads (b, h) -- are independent
 * problems; they are split across POSIX threads.  Within a channel the
 * arithmetic is strictly in time order and in state order n = 0..N-1.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>

/* softplus(s) = log(1 + e^s); for s > 20 the difference to s is < 3e-9. */
static double softplus_d(double s) { return s > 20.0 ? s : log1p(exp(s)); }

/* silu(z) = z * sigmoid(z) = z / (1 + e^{-z}). */
static double silu_d(double z) { return z / (1.0 + exp(-z)); }

static double step_size(double delta, const double* bias, int64_t d, int softplus) {
  double s = delta + (bias ? bias[d] : 0.0);
  return softplus ? softplus_d(s) : s;
}

/* ------------------------------------------------------------------ */
/* Mamba-1 selective scan.                                             */
/* u, delta, z, y : (batch, dim, seqlen)     B, C : (batch, dstate, seqlen)
 * A : (dim, dstate)   D, bias : (dim)   h0, h_last : (batch, dim, dstate) */
typedef struct {
  int64_t batch, dim, dstate, seqlen;
  const double *u, *delta, *A, *B, *C, *D, *z, *bias, *h0;
  int softplus;
  double *y, *h_last;
  int64_t row_begin, row_end; /* rows are flattened (b, d) pairs */
} scan_job;

static void* scan_rows(void* arg) {
  const scan_job* j = (const scan_job*)arg;
  const int64_t N = j->dstate, L = j->seqlen, Dm = j->dim;
  double* h = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  for (int64_t row = j->row_begin; row < j->row_end; ++row) {
    const int64_t b = row / Dm, d = row % Dm;
    for (int64_t n = 0; n < N; ++n) h[n] = j->h0 ? j->h0[row * N + n] : 0.0;
    const double* u = j->u + row * L;
    const double* dl = j->delta + row * L;
    const double* Bb = j->B + b * N * L;
    const double* Cb = j->C + b * N * L;
    const double* Ad = j->A + d * N;
    for (int64_t t = 0; t < L; ++t) {
      const double dt = step_size(dl[t], j->bias, d, j->softplus);
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double dA = exp(dt * Ad[n]);          /* A_d = exp(A dt), diagonal   */
        const double dBu = dt * Bb[n * L + t] * u[t]; /* input term dt' B u          */
        h[n] = dA * h[n] + dBu;                       /* h_t = A_d h_{t-1} + B_d u_t */
        acc += Cb[n * L + t] * h[n];                  /* y_t = C_t . h_t             */
      }
      double yv = acc + (j->D ? j->D[d] * u[t] : 0.0); /* skip term D u             */
      if (j->z) yv *= silu_d(j->z[row * L + t]);       /* gate y * silu(z)           */
      j->y[row * L + t] = yv;
    }
    if (j->h_last)
      for (int64_t n = 0; n < N; ++n) j->h_last[row * N + n] = h[n];
  }
  free(h);
  return NULL;
}

static int run_parallel(void* (*fn)(void*), void* jobs, size_t job_size, int64_t rows, int nthreads,
                        void (*set_range)(void*, int64_t, int64_t)) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > rows) nthreads = (int)(rows > 0 ? rows : 1);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
  int rc = 0;
  for (int i = 0; i < nthreads; ++i) {
    void* job = (char*)jobs + job_size * (size_t)i;
    set_range(job, rows * i / nthreads, rows * (i + 1) / nthreads);
    if (nthreads == 1) { fn(job); continue; }
    if (pthread_create(&th[i], NULL, fn, job) != 0) { fn(job); th[i] = 0; rc = 1; }
  }
  if (nthreads > 1)
    for (int i = 0; i < nthreads; ++i)
      if (th[i]) pthread_join(th[i], NULL);
  free(th);
  return rc;
}

static void scan_set_range(void* p, int64_t a, int64_t b) {
  ((scan_job*)p)->row_begin = a;
  ((scan_job*)p)->row_end = b;
}

int oracle_scan_fwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, const double* u,
                    const double* delta, const double* A, const double* B, const double* C,
                    const double* D, const double* z, const double* bias, int softplus,
                    const double* h0, double* y, double* h_last, int nthreads) {
  if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0) return -1;
  const int64_t rows = batch * dim;
  if (rows == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  scan_job* jobs = (scan_job*)calloc((size_t)nthreads, sizeof(scan_job));
  for (int i = 0; i < nthreads; ++i)
    jobs[i] = (scan_job){batch, dim, dstate, seqlen, u, delta, A, B, C, D, z, bias, h0, softplus,
                         y, h_last, 0, 0};
  run_parallel(scan_rows, jobs, sizeof(scan_job), rows, nthreads, scan_set_range);
  free(jobs);
  return 0;
}

/* ------------------------------------------------------------------ */
/* One decode step ([P3] section 5.4): the state (batch, dim, dstate) is
 * read and overwritten in place; u, delta, z, y : (batch, dim);
 * B, C : (batch, dstate). */
int oracle_scan_step(int64_t batch, int64_t dim, int64_t dstate, const double* u,
                     const double* delta, const double* A, const double* B, const double* C,
                     const double* D, const double* z, const double* bias, int softplus,
                     double* state, double* y) {
  if (batch < 0 || dim < 0 || dstate < 0) return -1;
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t d = 0; d < dim; ++d) {
      const int64_t row = b * dim + d;
      const double dt = step_size(delta[row], bias, d, softplus);
      double* h = state + row * dstate;
      double acc = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        h[n] = exp(dt * A[d * dstate + n]) * h[n] + dt * B[b * dstate + n] * u[row];
        acc += C[b * dstate + n] * h[n];
      }
      double yv = acc + (D ? D[d] * u[row] : 0.0);
      if (z) yv *= silu_d(z[row]);
      y[row] = yv;
    }
  return 0;
}

/* ------------------------------------------------------------------ */
/* Mamba-2 scalar-decay scan, sequential in time ([P4] section 4).
 * x, z, y : (batch, seqlen, nheads, headdim)   delta : (batch, seqlen, nheads)
 * B, C : (batch, seqlen, dstate)   A, D, bias : (nheads)
 * h0, h_last : (batch, nheads, headdim, dstate).  No chunking here: the
 * chunk length is an implementation parameter of the GPU path only. */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate;
  const double *x, *delta, *A, *B, *C, *D, *z, *bias, *h0;
  int softplus;
  double *y, *h_last;
  int64_t row_begin, row_end; /* rows are flattened (b, h) pairs */
} ssd_job;

static void* ssd_rows(void* arg) {
  const ssd_job* j = (const ssd_job*)arg;
  const int64_t L = j->seqlen, H = j->nheads, P = j->headdim, N = j->dstate;
  double* S = (double*)malloc(sizeof(double) * (size_t)(P * N > 0 ? P * N : 1));
  for (int64_t row = j->row_begin; row < j->row_end; ++row) {
    const int64_t b = row / H, hd = row % H;
    for (int64_t i = 0; i < P * N; ++i) S[i] = j->h0 ? j->h0[row * P * N + i] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double dt = step_size(j->delta[(b * L + t) * H + hd], j->bias, hd, j->softplus);
      const double a = exp(dt * j->A[hd]); /* scalar decay a_t */
      const double* Bt = j->B + (b * L + t) * N;
      const double* Ct = j->C + (b * L + t) * N;
      const int64_t xo = ((b * L + t) * H + hd) * P;
      for (int64_t p = 0; p < P; ++p) {
        const double xv = j->x[xo + p];
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) {
          S[p * N + n] = a * S[p * N + n] + dt * xv * Bt[n];
          acc += Ct[n] * S[p * N + n];
        }
        double yv = acc + (j->D ? j->D[hd] * xv : 0.0);
        if (j->z) yv *= silu_d(j->z[xo + p]);
        j->y[xo + p] = yv;
      }
    }
    if (j->h_last)
      for (int64_t i = 0; i < P * N; ++i) j->h_last[row * P * N + i] = S[i];
  }
  free(S);
  return NULL;
}

static void ssd_set_range(void* p, int64_t a, int64_t b) {
  ((ssd_job*)p)->row_begin = a;
  ((ssd_job*)p)->row_end = b;
}

int oracle_ssd_fwd(int64_t batch, int64_t seqlen, int64_t nheads, int64_t headdim, int64_t dstate,
                   const double* x, const double* delta, const double* A, const double* B,
                   const double* C, const double* D, const double* z, const double* bias,
                   int softplus, const double* h0, double* y, double* h_last, int nthreads) {
  if (batch < 0 || seqlen < 0 || nheads < 0 || headdim < 0 || dstate < 0) return -1;
  const int64_t rows = batch * nheads;
  if (rows == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  ssd_job* jobs = (ssd_job*)calloc((size_t)nthreads, sizeof(ssd_job));
  for (int i = 0; i < nthreads; ++i)
    jobs[i] = (ssd_job){batch, seqlen, nheads, headdim, dstate, x, delta, A, B, C, D, z, bias, h0,
                        softplus, y, h_last, 0, 0};
  run_parallel(ssd_rows, jobs, sizeof(ssd_job), rows, nthreads, ssd_set_range);
  free(jobs);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Causal depthwise convolution over time followed by SiLU, in front of the
 * scan.  [P2] section 3 (block flow: a local convolution captures
 * short-range patterns before the selective SSM; SiLU is the block's
 * activation; kernel size 4 among the block's hyperparameters).  Readings
 * (the page gives no formula): causal, one filter of `width` taps per
 * channel, the last tap on the current step, then the channel's bias:
 *   u[b,d,t] = silu(bias_d + sum_{k<width} w[d,k] x[b,d,t-(width-1)+k]);
 * inputs at negative times come from x_prev (batch, dim, width-1), whose
 * entry j is the input at time j-(width-1), or are zero without it.
 * x, u : (batch, dim, seqlen)   w : (dim, width)   bias : (dim) */
typedef struct {
  int64_t dim, seqlen, width;
  const double *x, *w, *bias, *x_prev;
  double* u;
  int64_t row_begin, row_end;
} conv_job;

static void* conv_rows(void* arg) {
  const conv_job* j = (const conv_job*)arg;
  const int64_t L = j->seqlen, K = j->width;
  for (int64_t row = j->row_begin; row < j->row_end; ++row) {
    const int64_t d = row % j->dim;
    for (int64_t t = 0; t < L; ++t) {
      double acc = j->bias ? j->bias[d] : 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const int64_t tt = t - (K - 1) + k; /* time of the input under tap k */
        double xv = 0.0;
        if (tt >= 0)
          xv = j->x[row * L + tt];
        else if (j->x_prev)
          xv = j->x_prev[row * (K - 1) + tt + (K - 1)];
        acc += j->w[d * K + k] * xv;
      }
      j->u[row * L + t] = silu_d(acc);
    }
  }
  return NULL;
}

static void conv_set_range(void* p, int64_t a, int64_t b) {
  ((conv_job*)p)->row_begin = a;
  ((conv_job*)p)->row_end = b;
}

int oracle_conv_silu(int64_t batch, int64_t dim, int64_t seqlen, int64_t width, const double* x,
                     const double* w, const double* bias, const double* x_prev, double* u,
                     int nthreads) {
  if (batch < 0 || dim < 0 || seqlen < 0 || width < 1) return -1;
  const int64_t rows = batch * dim;
  if (rows == 0 || seqlen == 0) return 0;
  if (nthreads < 1) nthreads = 1;
  conv_job* jobs = (conv_job*)calloc((size_t)nthreads, sizeof(conv_job));
  for (int i = 0; i < nthreads; ++i)
    jobs[i] = (conv_job){dim, seqlen, width, x, w, bias, x_prev, u, 0, 0};
  run_parallel(conv_rows, jobs, sizeof(conv_job), rows, nthreads, conv_set_range);
  free(jobs);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Gradients of the selective scan (reverse mode), for a loss whose gradient
 * with respect to y is dy.  [P2] section 1 ("recomputation": intermediate
 * states are rebuilt in the backward pass instead of stored) -- here the
 * states of one channel are simply recomputed in full, in order, before the
 * reverse sweep.  With s_t = sum_n C[t,n] h[t,n] + D u_t and y_t = s_t g_t,
 * g_t = silu(z_t) (1 without z), the adjoint of the recurrence is
 *   lambda[t,n] = ds_t C[t,n] + dA[t+1,n] lambda[t+1,n],  ds_t = dy_t g_t,
 * and every input receives the terms of the chain rule through dt'_t,
 * dA[t,n] = exp(dt'_t A[n]) and dt'_t B[t,n] u_t.  Single-threaded (B and C
 * gradients are sums over channels).  Outputs are overwritten; any of them
 * may be NULL.  Shapes as in oracle_scan_fwd; dA (dim, dstate), dD, dbias
 * (dim), dh0 (batch, dim, dstate). */
static double softplus_grad(double s) { return s > 20.0 ? 1.0 : 1.0 / (1.0 + exp(-s)); }

int oracle_scan_bwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen, const double* u,
                    const double* delta, const double* A, const double* B, const double* C,
                    const double* D, const double* z, const double* bias, int softplus,
                    const double* h0, const double* dy, double* du, double* ddelta, double* dA,
                    double* dB, double* dC, double* dD, double* dz, double* dbias, double* dh0) {
  if (batch < 0 || dim < 0 || dstate < 0 || seqlen < 0) return -1;
  const int64_t N = dstate, L = seqlen;
  if (dA) for (int64_t i = 0; i < dim * N; ++i) dA[i] = 0.0;
  if (dB) for (int64_t i = 0; i < batch * N * L; ++i) dB[i] = 0.0;
  if (dC) for (int64_t i = 0; i < batch * N * L; ++i) dC[i] = 0.0;
  if (dD) for (int64_t i = 0; i < dim; ++i) dD[i] = 0.0;
  if (dbias) for (int64_t i = 0; i < dim; ++i) dbias[i] = 0.0;
  double* hs = (double*)malloc(sizeof(double) * (size_t)((L + 1) * (N > 0 ? N : 1)));
  double* dts = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
  double* lam = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
  for (int64_t row = 0; row < batch * dim; ++row) {
    const int64_t b = row / dim, d = row % dim;
    const double* ur = u + row * L;
    const double* dl = delta + row * L;
    const double* Bb = B + b * N * L;
    const double* Cb = C + b * N * L;
    const double* Ad = A + d * N;
    /* forward: hs[(t + 1) N + n] = h[t, n], hs[n] = h0 */
    for (int64_t n = 0; n < N; ++n) hs[n] = h0 ? h0[row * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double dt = step_size(dl[t], bias, d, softplus);
      dts[t] = dt;
      for (int64_t n = 0; n < N; ++n)
        hs[(t + 1) * N + n] = exp(dt * Ad[n]) * hs[t * N + n] + dt * Bb[n * L + t] * ur[t];
    }
    /* reverse sweep */
    for (int64_t n = 0; n < N; ++n) lam[n] = 0.0;
    double dDd = 0.0, dbd = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
      const double dt = dts[t];
      double sv = D ? D[d] * ur[t] : 0.0;
      for (int64_t n = 0; n < N; ++n) sv += Cb[n * L + t] * hs[(t + 1) * N + n];
      double gate = 1.0, ds = dy[row * L + t];
      if (z) {
        const double zv = z[row * L + t], sg = 1.0 / (1.0 + exp(-zv));
        gate = zv * sg;
        if (dz) dz[row * L + t] = dy[row * L + t] * sv * (sg * (1.0 + zv * (1.0 - sg)));
      }
      ds *= gate;
      double du_t = D ? ds * D[d] : 0.0, ddt = 0.0;
      dDd += ds * ur[t];
      for (int64_t n = 0; n < N; ++n) {
        lam[n] += ds * Cb[n * L + t];                     /* lambda_t = ds C_t + dA_{t+1} lambda_{t+1} */
        const double a = exp(dt * Ad[n]), hp = hs[t * N + n];
        if (dC) dC[b * N * L + n * L + t] += ds * hs[(t + 1) * N + n];
        if (dB) dB[b * N * L + n * L + t] += lam[n] * dt * ur[t];
        du_t += lam[n] * dt * Bb[n * L + t];
        ddt += lam[n] * (Ad[n] * a * hp + Bb[n * L + t] * ur[t]);
        if (dA) dA[d * N + n] += lam[n] * dt * a * hp;
        lam[n] *= a;                                      /* carried to step t - 1 */
      }
      if (du) du[row * L + t] = du_t;
      const double sarg = dl[t] + (bias ? bias[d] : 0.0);
      const double dd = softplus ? ddt * softplus_grad(sarg) : ddt;
      if (ddelta) ddelta[row * L + t] = dd;
      dbd += dd;
    }
    if (dh0) for (int64_t n = 0; n < N; ++n) dh0[row * N + n] = lam[n];
    if (dD) dD[d] += dDd;
    if (dbias) dbias[d] += dbd;
  }
  free(hs);
  free(dts);
  free(lam);
  return 0;
}

int oracle_abi_version(void) { return 3; }

/*
 * ssm_oracle.c -- plain, slow, sequential fp64 reference for the Mamba selective scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file:
 * only the tests, the smoke check and the bench's CPU-baseline / reference arm use it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (sources are the pages collected on the "selective_state_space_15" subject):
 *   - "会议长序列建模状态空间模型加速" (ufo.work), §1.1: the discrete recurrence
 *       h_t = Abar h_{t-1} + Bbar x_t,  y_t = C h_t,  Abar = exp(Delta A),  Bbar = Delta B,
 *     with Delta, B, C input dependent (selective).
 *   - same page, §2.1 (the unfused loop): Delta_t = softplus(.) of a per-token quantity.
 *   - "企业官网建设流程全解析" (discosf.com), §1.1: the continuous model carries the skip term
 *     y = C h + D x;  §1.3: Delta_t = softplus(Linear(x_t)) -- here the linear map's output is
 *     the per-token input delta plus a per-channel bias.
 *   - ufo.work page §4.2 and discosf.com §2.1 (pitfall 4): packed sequences reset the state to
 *     zero at every sequence start (cu_seqlens boundaries).
 *   - ufo.work page §4.1 / its second article §4.1: a one-token state update over a persistent
 *     state pool indexed per request.
 *   - discosf.com §1.2 (and ufo.work §1.1, "or by a zero-order hold"): the zero-order-hold
 *     input matrix Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B, selected per call
 *     (zoh != 0) instead of Bbar = Delta B.
 * Readings where the pages are silent: the bias sits inside the softplus; the optional SiLU(z)
 * gate multiplies the whole output C h + D u and never feeds back into h; y uses h_t (not h_{t-1}).
 *
 * Everything is scalar fp64 with libm exp/log1p, evaluated in the order of the definition:
 * for each (batch, channel, state) and t = 0..L-1 in sequence.  There is no blocking, no
 * chunking and no reassociation.  Threads (optional) only split independent channels.
 *
 * Alongside each result the oracle runs an absolute-value recursion
 *   habs_t = Abar_t habs_{t-1} + |Bbar_t u_t|            (habs_{-1} = |h0|)
 *   ymag_t = |g(z_t)| (sum_n |C_t[n]| habs_t[n] + |D u_t|)
 * which bounds |h| and |y| from above; tests divide errors by these magnitudes.
 *
 * Layouts (row-major, time innermost):
 *   u, delta, z, y : [batch][dim][seqlen]      B, C : [batch][dstate][seqlen]
 *   A : [dim][dstate]   Dskip, bias : [dim]    h0, h_last : [batch][dim][dstate]
 * Varlen: u, delta, z, y : [dim][total]; B, C : [dstate][total]; cu_seqlens : [nseq+1];
 *   h_last : [nseq][dim][dstate].
 * Decode: pool : [num_slots][dim][dstate]; slot_ids : [R]; u, delta, z, y : [R][dim];
 *   B, C : [R][dstate].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

/* softplus(x) = log(1 + e^x), written in the overflow-free form max(x,0) + log1p(e^-|x|). */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* SiLU(z) = z * sigmoid(z) = z / (1 + e^-z). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Input coefficient of one step for one (channel, state): Bbar_t[n] = coef * B_t[n].
 * Euler (ufo.work §1.1): coef = Delta.  Zero-order hold (discosf.com §1.2): A is diagonal, so
 * (Delta A)^-1 (exp(Delta A) - 1) Delta is the scalar expm1(x) / x * Delta with x = Delta A;
 * at x = 0 (A = 0 or Delta = 0) the quotient is 1. */
static double input_coef(int zoh, double dt, double a) {
  if (!zoh) return dt;
  const double x = dt * a;
  return x == 0.0 ? dt : expm1(x) / x * dt;
}

/* One channel of one sequence.  u, delta, z, y point at the channel's row (stride 1 in time);
 * B and C point at the sequence's block, one row per state index, row stride bc_stride. */
typedef struct {
  int64_t dstate, len, bc_stride;
  int zoh;                                 /* nonzero: zero-order-hold Bbar */
  const double *u, *delta, *z, *B, *C, *A; /* A: this channel's dstate values */
  double dskip, bias;
  const double *h0;                        /* dstate values or NULL */
  double *y, *h_last, *y_mag, *h_mag;      /* y, y_mag: len values; h_*: dstate values */
} chan_job;

static void scan_channel(const chan_job *j) {
  const int64_t N = j->dstate;
  double *h = (double *)malloc(sizeof(double) * (size_t)N);
  double *ha = (double *)malloc(sizeof(double) * (size_t)N);
  for (int64_t n = 0; n < N; ++n) {
    h[n] = j->h0 ? j->h0[n] : 0.0;
    ha[n] = fabs(h[n]);
  }
  for (int64_t t = 0; t < j->len; ++t) {
    const double ut = j->u[t];
    const double dt = softplus(j->delta[t] + j->bias);         /* Delta_t */
    double acc = 0.0, acc_abs = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double abar = exp(dt * j->A[n]);                   /* Abar = exp(Delta A) */
      const double bx = input_coef(j->zoh, dt, j->A[n]) * j->B[n * j->bc_stride + t] * ut; /* Bbar x */
      h[n] = abar * h[n] + bx;                                 /* h_t = Abar h_{t-1} + Bbar x_t */
      ha[n] = abar * ha[n] + fabs(bx);
      const double c = j->C[n * j->bc_stride + t];
      acc += c * h[n];                                         /* C_t h_t */
      acc_abs += fabs(c) * ha[n];
    }
    double yt = acc + j->dskip * ut;                           /* + D u_t */
    double ym = acc_abs + fabs(j->dskip * ut);
    if (j->z) {
      const double g = silu(j->z[t]);                          /* gate multiplies all of y */
      yt *= g;
      ym *= fabs(g);
    }
    j->y[t] = yt;
    if (j->y_mag) j->y_mag[t] = ym;
  }
  for (int64_t n = 0; n < N; ++n) {
    if (j->h_last) j->h_last[n] = h[n];
    if (j->h_mag) j->h_mag[n] = ha[n];
  }
  free(h);
  free(ha);
}

typedef struct {
  const chan_job *jobs;
  int64_t njobs, first, step;
} worker_arg;

static void *worker(void *p) {
  const worker_arg *w = (const worker_arg *)p;
  for (int64_t i = w->first; i < w->njobs; i += w->step) scan_channel(&w->jobs[i]);
  return NULL;
}

static void run_jobs(const chan_job *jobs, int64_t njobs, int nthreads) {
  if (nthreads <= 1 || njobs <= 1) {
    for (int64_t i = 0; i < njobs; ++i) scan_channel(&jobs[i]);
    return;
  }
  if (nthreads > njobs) nthreads = (int)njobs;
  pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
  worker_arg *args = (worker_arg *)malloc(sizeof(worker_arg) * (size_t)nthreads);
  for (int i = 0; i < nthreads; ++i) {
    args[i].jobs = jobs; args[i].njobs = njobs; args[i].first = i; args[i].step = nthreads;
    pthread_create(&th[i], NULL, worker, &args[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(th);
  free(args);
}

/* Fixed-length batch.  Optional pointers: z, Dskip, bias, h0, h_last, y_mag, h_mag. */
int oracle_scan(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                const double *u, const double *delta, const double *z,
                const double *B, const double *C, const double *A,
                const double *Dskip, const double *bias, const double *h0,
                double *y, double *h_last, double *y_mag, double *h_mag, int zoh, int nthreads) {
  if (batch < 0 || dim < 0 || dstate <= 0 || seqlen < 0) return 1;
  const int64_t njobs = batch * dim;
  chan_job *jobs = (chan_job *)calloc((size_t)(njobs > 0 ? njobs : 1), sizeof(chan_job));
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t d = 0; d < dim; ++d) {
      chan_job *j = &jobs[b * dim + d];
      const int64_t xo = (b * dim + d) * seqlen, so = (b * dim + d) * dstate;
      j->dstate = dstate; j->len = seqlen; j->bc_stride = seqlen; j->zoh = zoh;
      j->u = u + xo; j->delta = delta + xo; j->z = z ? z + xo : NULL;
      j->B = B + b * dstate * seqlen; j->C = C + b * dstate * seqlen;
      j->A = A + d * dstate;
      j->dskip = Dskip ? Dskip[d] : 0.0; j->bias = bias ? bias[d] : 0.0;
      j->h0 = h0 ? h0 + so : NULL;
      j->y = y + xo; j->y_mag = y_mag ? y_mag + xo : NULL;
      j->h_last = h_last ? h_last + so : NULL; j->h_mag = h_mag ? h_mag + so : NULL;
    }
  run_jobs(jobs, njobs, nthreads);
  free(jobs);
  return 0;
}

/* Packed variable-length batch: every sequence starts from the zero state. */
int oracle_scan_varlen(int64_t dim, int64_t dstate, int64_t total,
                       const double *u, const double *delta, const double *z,
                       const double *B, const double *C, const double *A,
                       const double *Dskip, const double *bias,
                       const int64_t *cu_seqlens, int64_t nseq,
                       double *y, double *h_last, double *y_mag, double *h_mag, int zoh, int nthreads) {
  if (dim < 0 || dstate <= 0 || total < 0 || nseq < 0) return 1;
  if (cu_seqlens[0] != 0 || cu_seqlens[nseq] != total) return 2;
  for (int64_t s = 0; s < nseq; ++s)
    if (cu_seqlens[s + 1] < cu_seqlens[s]) return 3;
  const int64_t njobs = nseq * dim;
  chan_job *jobs = (chan_job *)calloc((size_t)(njobs > 0 ? njobs : 1), sizeof(chan_job));
  for (int64_t s = 0; s < nseq; ++s)
    for (int64_t d = 0; d < dim; ++d) {
      chan_job *j = &jobs[s * dim + d];
      const int64_t t0 = cu_seqlens[s], xo = d * total + t0, so = (s * dim + d) * dstate;
      j->dstate = dstate; j->len = cu_seqlens[s + 1] - t0; j->bc_stride = total; j->zoh = zoh;
      j->u = u + xo; j->delta = delta + xo; j->z = z ? z + xo : NULL;
      j->B = B + t0; j->C = C + t0;
      j->A = A + d * dstate;
      j->dskip = Dskip ? Dskip[d] : 0.0; j->bias = bias ? bias[d] : 0.0;
      j->h0 = NULL;
      j->y = y + xo; j->y_mag = y_mag ? y_mag + xo : NULL;
      j->h_last = h_last ? h_last + so : NULL; j->h_mag = h_mag ? h_mag + so : NULL;
    }
  run_jobs(jobs, njobs, nthreads);
  free(jobs);
  return 0;
}

/* One decode step: for each request r, pool[slot_ids[r]] advances by one token in place.
 * pool_mag (optional, same shape as pool) carries the magnitude recursion across steps. */
int oracle_state_update(int64_t num_slots, int64_t dim, int64_t dstate,
                        double *pool, double *pool_mag,
                        const int64_t *slot_ids, int64_t R,
                        const double *u, const double *delta, const double *z,
                        const double *B, const double *C, const double *A,
                        const double *Dskip, const double *bias,
                        double *y, double *y_mag, int zoh) {
  if (num_slots < 0 || dim < 0 || dstate <= 0 || R < 0) return 1;
  for (int64_t r = 0; r < R; ++r)
    if (slot_ids[r] < 0 || slot_ids[r] >= num_slots) return 4;
  for (int64_t r = 0; r < R; ++r) {
    const int64_t s = slot_ids[r];
    for (int64_t d = 0; d < dim; ++d) {
      double *h = pool + (s * dim + d) * dstate;
      double *ha = pool_mag ? pool_mag + (s * dim + d) * dstate : NULL;
      const double ut = u[r * dim + d];
      const double dt = softplus(delta[r * dim + d] + (bias ? bias[d] : 0.0));
      double acc = 0.0, acc_abs = 0.0;
      for (int64_t n = 0; n < dstate; ++n) {
        const double abar = exp(dt * A[d * dstate + n]);
        const double bx = input_coef(zoh, dt, A[d * dstate + n]) * B[r * dstate + n] * ut;
        h[n] = abar * h[n] + bx;
        const double hm = ha ? (ha[n] = abar * ha[n] + fabs(bx)) : fabs(h[n]);
        const double c = C[r * dstate + n];
        acc += c * h[n];
        acc_abs += fabs(c) * hm;
      }
      const double ds = Dskip ? Dskip[d] : 0.0;
      double yt = acc + ds * ut, ym = acc_abs + fabs(ds * ut);
      if (z) {
        const double g = silu(z[r * dim + d]);
        yt *= g;
        ym *= fabs(g);
      }
      y[r * dim + d] = yt;
      if (y_mag) y_mag[r * dim + d] = ym;
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------------------------
 * Backward (the adjoint of oracle_scan).  The ufo.work page, §2.2, discusses how a training
 * backward pass keeps or recomputes the states h_t; what it computes is fixed by the forward
 * definition: the gradients of a scalar loss L, given dL/dy (dy) and optionally dL/dh_last
 * (dh_last), with respect to every input.  This is the plain reverse-mode derivative of the
 * loop above: the forward states of a channel are recomputed and stored, then the loop runs
 * backwards over t.
 *
 *   y_t   = yraw_t g(z_t),  yraw_t = sum_n C_t[n] h_t[n] + D u_t,  g = SiLU (1 without z)
 *   h_t   = a_t h_{t-1} + c_t B_t u_t,  a_t = exp(Delta_t A),  c_t = input_coef(Delta_t, A)
 *   Delta = softplus(delta + bias)
 *
 * Outputs: du, ddelta, dz : [batch][dim][seqlen];  dB, dC : [batch][dstate][seqlen];
 * dA : [dim][dstate];  dDskip, dbias : [dim];  dh0 : [batch][dim][dstate] (optional).
 */

static double sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  const double e = exp(x);
  return e / (1.0 + e);
}

/* d/dz SiLU(z) = sigma(z) (1 + z (1 - sigma(z))). */
static double silu_grad(double z) {
  const double s = sigmoid(z);
  return s * (1.0 + z * (1.0 - s));
}

/* Partial derivatives of the input coefficient c(Delta, A).  Euler: c = Delta.  Zero-order
 * hold: c = expm1(x)/x * Delta with x = Delta A, so dc/dDelta = exp(x) and
 * dc/dA = Delta^2 phi'(x) with phi(x) = expm1(x)/x, phi'(x) = (x e^x - expm1(x)) / x^2; near
 * x = 0 the series phi'(x) = sum_{k>=1} k x^(k-1) / (k+1)! avoids the cancellation. */
static void input_coef_grad(int zoh, double dt, double a, double *dc_ddt, double *dc_da) {
  if (!zoh) {
    *dc_ddt = 1.0;
    *dc_da = 0.0;
    return;
  }
  const double x = dt * a;
  *dc_ddt = exp(x);
  double dphi;
  if (fabs(x) < 1e-2) {
    double term = 1.0, fact = 2.0;           /* x^(k-1), (k+1)! */
    dphi = 0.0;
    for (int k = 1; k <= 8; ++k) {
      dphi += k * term / fact;
      term *= x;
      fact *= (double)(k + 2);
    }
  } else {
    dphi = (x * exp(x) - expm1(x)) / (x * x);
  }
  *dc_da = dt * dt * dphi;
}

typedef struct {
  chan_job f;                 /* forward description of the channel (y fields unused)   */
  int64_t b, d;               /* batch row and channel                                 */
  const double *dy;           /* len values                                            */
  const double *dh_last;      /* dstate values or NULL                                 */
  double *du, *ddelta, *dz;   /* len values (dz only with a gate)                      */
  double *dh0;                /* dstate values or NULL                                 */
} bwd_job;

typedef struct {
  const bwd_job *jobs;
  int64_t njobs, first, step;
  int64_t dim, dstate, seqlen;
  /* this worker's accumulators */
  double *dB, *dC;            /* [batch][dstate][seqlen] */
  double *dA;                 /* [dim][dstate]           */
  double *dDskip, *dbias;     /* [dim]                   */
} bwd_worker;

static void scan_channel_bwd(const bwd_job *j, bwd_worker *w) {
  const chan_job *f = &j->f;
  const int64_t N = f->dstate, L = f->len;
  double *H = (double *)malloc(sizeof(double) * (size_t)(N * (L > 0 ? L : 1)));
  double *hprev0 = (double *)malloc(sizeof(double) * (size_t)N);
  double *dh = (double *)malloc(sizeof(double) * (size_t)N);
  /* forward: states h_t for every step */
  for (int64_t n = 0; n < N; ++n) hprev0[n] = f->h0 ? f->h0[n] : 0.0;
  for (int64_t t = 0; t < L; ++t) {
    const double dt = softplus(f->delta[t] + f->bias);
    for (int64_t n = 0; n < N; ++n) {
      const double hp = t > 0 ? H[(t - 1) * N + n] : hprev0[n];
      const double c = input_coef(f->zoh, dt, f->A[n]);
      H[t * N + n] = exp(dt * f->A[n]) * hp + c * f->B[n * f->bc_stride + t] * f->u[t];
    }
  }
  /* backward over t */
  for (int64_t n = 0; n < N; ++n) dh[n] = j->dh_last ? j->dh_last[n] : 0.0;
  double *dB = w->dB + j->b * N * w->seqlen, *dC = w->dC + j->b * N * w->seqlen;
  double *dA = w->dA + j->d * N;
  for (int64_t t = L - 1; t >= 0; --t) {
    const double ut = f->u[t];
    const double s = f->delta[t] + f->bias;
    const double dt = softplus(s);
    double yraw = f->dskip * ut;
    for (int64_t n = 0; n < N; ++n) yraw += f->C[n * f->bc_stride + t] * H[t * N + n];
    double dyraw = j->dy[t];
    if (f->z) {
      j->dz[t] = j->dy[t] * yraw * silu_grad(f->z[t]);
      dyraw *= silu(f->z[t]);
    }
    w->dDskip[j->d] += dyraw * ut;
    double du = dyraw * f->dskip;
    double ddt = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double Bt = f->B[n * f->bc_stride + t], Ct = f->C[n * f->bc_stride + t];
      const double hp = t > 0 ? H[(t - 1) * N + n] : hprev0[n];
      const double a = exp(dt * f->A[n]);
      const double c = input_coef(f->zoh, dt, f->A[n]);
      double dc_ddt, dc_da;
      input_coef_grad(f->zoh, dt, f->A[n], &dc_ddt, &dc_da);
      dh[n] += dyraw * Ct;                     /* y_t reads h_t */
      dC[n * w->seqlen + t] += dyraw * H[t * N + n];
      const double dcoef = dh[n] * Bt * ut;    /* h_t = a h_{t-1} + c B u */
      dB[n * w->seqlen + t] += dh[n] * c * ut;
      du += dh[n] * c * Bt;
      const double da = dh[n] * hp;
      ddt += da * a * f->A[n] + dcoef * dc_ddt;
      dA[n] += da * a * dt + dcoef * dc_da;
      dh[n] *= a;                              /* on to h_{t-1} */
    }
    j->du[t] = du;
    const double dd = ddt * sigmoid(s);        /* softplus' = sigmoid */
    j->ddelta[t] = dd;
    w->dbias[j->d] += dd;
  }
  if (j->dh0)
    for (int64_t n = 0; n < N; ++n) j->dh0[n] = dh[n];
  free(H);
  free(hprev0);
  free(dh);
}

static void *bwd_worker_run(void *p) {
  bwd_worker *w = (bwd_worker *)p;
  for (int64_t i = w->first; i < w->njobs; i += w->step) scan_channel_bwd(&w->jobs[i], w);
  return NULL;
}

/* Gradients of the fixed-length batch scan.  Optional: z (then dz is written), Dskip, bias,
 * h0, dh_last, dh0.  The per-channel outputs are written; the shared ones (dB, dC, dA,
 * dDskip, dbias) are summed over every (batch, channel, t) that uses them. */
int oracle_scan_bwd(int64_t batch, int64_t dim, int64_t dstate, int64_t seqlen,
                    const double *u, const double *delta, const double *z,
                    const double *B, const double *C, const double *A,
                    const double *Dskip, const double *bias, const double *h0,
                    const double *dy, const double *dh_last,
                    double *du, double *ddelta, double *dz, double *dB, double *dC, double *dA,
                    double *dDskip, double *dbias, double *dh0, int zoh, int nthreads) {
  if (batch < 0 || dim < 0 || dstate <= 0 || seqlen < 0) return 1;
  const int64_t njobs = batch * dim;
  bwd_job *jobs = (bwd_job *)calloc((size_t)(njobs > 0 ? njobs : 1), sizeof(bwd_job));
  for (int64_t b = 0; b < batch; ++b)
    for (int64_t d = 0; d < dim; ++d) {
      bwd_job *j = &jobs[b * dim + d];
      const int64_t xo = (b * dim + d) * seqlen, so = (b * dim + d) * dstate;
      chan_job *f = &j->f;
      f->dstate = dstate; f->len = seqlen; f->bc_stride = seqlen; f->zoh = zoh;
      f->u = u + xo; f->delta = delta + xo; f->z = z ? z + xo : NULL;
      f->B = B + b * dstate * seqlen; f->C = C + b * dstate * seqlen;
      f->A = A + d * dstate;
      f->dskip = Dskip ? Dskip[d] : 0.0; f->bias = bias ? bias[d] : 0.0;
      f->h0 = h0 ? h0 + so : NULL;
      j->b = b; j->d = d;
      j->dy = dy + xo; j->dh_last = dh_last ? dh_last + so : NULL;
      j->du = du + xo; j->ddelta = ddelta + xo; j->dz = z ? dz + xo : NULL;
      j->dh0 = dh0 ? dh0 + so : NULL;
    }
  if (nthreads < 1) nthreads = 1;
  if (nthreads > njobs) nthreads = njobs > 0 ? (int)njobs : 1;
  const size_t nbc = (size_t)(batch * dstate * seqlen), na = (size_t)(dim * dstate);
  bwd_worker *ws = (bwd_worker *)calloc((size_t)nthreads, sizeof(bwd_worker));
  for (int i = 0; i < nthreads; ++i) {
    bwd_worker *w = &ws[i];
    w->jobs = jobs; w->njobs = njobs; w->first = i; w->step = nthreads;
    w->dim = dim; w->dstate = dstate; w->seqlen = seqlen;
    w->dB = (double *)calloc(nbc ? nbc : 1, sizeof(double));
    w->dC = (double *)calloc(nbc ? nbc : 1, sizeof(double));
    w->dA = (double *)calloc(na ? na : 1, sizeof(double));
    w->dDskip = (double *)calloc((size_t)(dim ? dim : 1), sizeof(double));
    w->dbias = (double *)calloc((size_t)(dim ? dim : 1), sizeof(double));
  }
  if (nthreads == 1) {
    bwd_worker_run(&ws[0]);
  } else {
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker_run, &ws[i]);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
  }
  /* the workers' partial sums, in worker order */
  memset(dB, 0, sizeof(double) * nbc);
  memset(dC, 0, sizeof(double) * nbc);
  memset(dA, 0, sizeof(double) * na);
  memset(dDskip, 0, sizeof(double) * (size_t)dim);
  memset(dbias, 0, sizeof(double) * (size_t)dim);
  for (int i = 0; i < nthreads; ++i) {
    bwd_worker *w = &ws[i];
    for (size_t k = 0; k < nbc; ++k) { dB[k] += w->dB[k]; dC[k] += w->dC[k]; }
    for (size_t k = 0; k < na; ++k) dA[k] += w->dA[k];
    for (int64_t k = 0; k < dim; ++k) { dDskip[k] += w->dDskip[k]; dbias[k] += w->dbias[k]; }
    free(w->dB); free(w->dC); free(w->dA); free(w->dDskip); free(w->dbias);
  }
  free(ws);
  free(jobs);
  return 0;
}

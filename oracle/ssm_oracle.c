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

/*
 * fp64 CPU oracle for the selective scan (S6).
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the CPU
 * baseline / reference arm of bench.py may load this library.  It shares no
 * code, header, table or helper with the CUDA path; the only thing both sides
 * use is the seeded input generator in synth/.
 *
 * What it computes, and where the pages state it:
 *
 *  - Discretisation (zero-order hold) of a diagonal A with step Delta:
 *      Abar = exp(Delta * A)
 *    "Mamba: Linear-Time Sequence Modeling with Selective State Spaces"
 *    (xyznot.com reading guide), section "Metodo", ZOH equations.
 *    Input term, Euler form Bbar * u = Delta * B_t * u_t: "Как работает Mamba
 *    (State Space Model)..." (aivaro.ru), section 3 "Selective Scan", code
 *    example (B_bar = delta * B).  The exact ZOH form of the same section
 *    "Metodo", Bbar = (Delta A)^-1 (exp(Delta A) - I) Delta B, is available
 *    behind zoh_exact (diagonal A: (exp(Delta A_n) - 1) / A_n * B_n).
 *  - Selection: Delta_t = softplus(Parameter + s_Delta(x_t)), B_t, C_t input
 *    dependent; reading guide, section "O Mecanismo de Selecao (S6)".  Here
 *    Parameter is delta_bias[d] and s_Delta(x_t) is the raw delta input.
 *  - Recurrence h_t = Abar_t h_{t-1} + Bbar_t u_t and output y_t = C_t h_t:
 *    reading guide, section "Metodo"; skip term D u_t: "O que e um modelo
 *    Mamba?" (ibm.com), output equation y(t) = C h(t) + D x(t).
 *  - Gate: the SSM output is multiplied elementwise by the activated z branch
 *    ("O que e um modelo Mamba?", Mamba block walk-through); the activation
 *    is SiLU, out = y * z * sigmoid(z).
 *  - Initial state zero (aivaro.ru code example, h = zeros) unless h0 is
 *    given; last_state = h after the last step.
 *  - Backward: reverse-mode derivative of the above, one channel at a time,
 *    from the stored forward states (the pages recompute states instead of
 *    storing them: reading guide, "Expansao de Estado Ciente de Hardware";
 *    the oracle simply stores them, which is the same mathematics).
 *
 * Layouts (row-major, last index contiguous), all fp64:
 *   u, delta, z, y, dout, du, ddelta, dz : [batch][dim][seqlen]
 *   B, C, dB, dC                         : [batch][seqlen][dstate]
 *   A, dA                                : [dim][dstate]
 *   D, delta_bias, dD, ddelta_bias       : [dim]
 *   h0, last_state, dh0                  : [batch][dim][dstate]
 * Nullable: D, z, delta_bias, h0, last_state (fwd), dh0 (bwd).
 * Channels (b, d) are split over nthreads POSIX threads; each channel is a
 * plain sequential loop over t, the state loop over n inside it.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t batch, dim, seqlen, dstate;
  const double *u, *delta, *A, *B, *C, *D, *z, *delta_bias, *h0;
  int delta_softplus, zoh_exact;
  double *y, *last_state;
  /* backward */
  const double *dout;
  double *du, *ddelta, *dA, *dB, *dC, *dD, *dz, *ddelta_bias, *dh0;
  /* per-thread partial sums (backward) */
  double *pdA, *pdB, *pdC, *pdD, *pdbias;
  int64_t ch_lo, ch_hi;
  int status;
} job_t;

/* softplus(s) = log(1 + e^s), evaluated without overflow. */
static double softplus(double s) {
  return s > 0.0 ? s + log1p(exp(-s)) : log1p(exp(s));
}

static double sigmoid(double s) {
  return s >= 0.0 ? 1.0 / (1.0 + exp(-s)) : exp(s) / (1.0 + exp(s));
}

/* Bbar_n / B_n: Delta (Euler) or (exp(Delta A_n) - 1) / A_n (exact ZOH). */
static double bbar_scale(double dl, double a_n, int zoh_exact) {
  if (!zoh_exact) return dl;
  if (a_n == 0.0) return dl;
  return expm1(dl * a_n) / a_n;
}

/* Its derivative with respect to Delta: 1 (Euler) or exp(Delta A_n) (ZOH). */
static double bbar_scale_ddelta(double dl, double a_n, int zoh_exact) {
  return zoh_exact ? exp(dl * a_n) : 1.0;
}

/* Its derivative with respect to A_n: 0 (Euler); for ZOH
 *   d/dA [(e^{Delta A} - 1) / A] = (x e^x - (e^x - 1)) / A^2,  x = Delta A,
 * which is Delta^2 sum_{k>=2} x^(k-2) (k-1) / k!  (used for |x| < 0.1, where
 * the closed form cancels). */
static double bbar_scale_dA(double dl, double a_n, int zoh_exact) {
  if (!zoh_exact) return 0.0;
  const double x = dl * a_n;
  if (fabs(x) < 0.1) {
    double term = 1.0, sum = 0.0;  /* term = x^m, with m = k - 2 */
    double fact = 2.0;             /* (m + 2)! */
    for (int m = 0; m < 12; ++m) {
      sum += term * (double)(m + 1) / fact;
      term *= x;
      fact *= (double)(m + 3);
    }
    return dl * dl * sum;
  }
  return (x * exp(x) - expm1(x)) / (a_n * a_n);
}

static void *fwd_worker(void *arg) {
  job_t *j = (job_t *)arg;
  const int64_t L = j->seqlen, N = j->dstate, Dm = j->dim;
  double *h = (double *)malloc(sizeof(double) * (size_t)N);
  if (!h) { j->status = -1; return NULL; }
  for (int64_t ch = j->ch_lo; ch < j->ch_hi; ++ch) {
    const int64_t b = ch / Dm, d = ch % Dm;
    const double *u = j->u + ch * L, *dr = j->delta + ch * L;
    const double *z = j->z ? j->z + ch * L : NULL;
    const double *Bb = j->B + b * L * N, *Cb = j->C + b * L * N;
    const double *Ad = j->A + d * N;
    const double Dd = j->D ? j->D[d] : 0.0;
    const double bias = j->delta_bias ? j->delta_bias[d] : 0.0;
    double *y = j->y + ch * L;
    for (int64_t n = 0; n < N; ++n) h[n] = j->h0 ? j->h0[ch * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      const double s = dr[t] + bias;
      const double dl = j->delta_softplus ? softplus(s) : s;
      double yss = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double abar = exp(dl * Ad[n]);
        const double bbar = bbar_scale(dl, Ad[n], j->zoh_exact) * Bb[t * N + n];
        h[n] = abar * h[n] + bbar * u[t];
        yss += Cb[t * N + n] * h[n];
      }
      yss += Dd * u[t];
      y[t] = z ? yss * z[t] * sigmoid(z[t]) : yss;
    }
    if (j->last_state)
      for (int64_t n = 0; n < N; ++n) j->last_state[ch * N + n] = h[n];
  }
  free(h);
  return NULL;
}

static void *bwd_worker(void *arg) {
  job_t *j = (job_t *)arg;
  const int64_t L = j->seqlen, N = j->dstate, Dm = j->dim;
  /* hs[(t+1)*N + n] = h_t[n]; hs[0..N) = h_{-1} (the initial state) */
  double *hs = (double *)malloc(sizeof(double) * (size_t)((L + 1) * N));
  double *dl = (double *)malloc(sizeof(double) * (size_t)L);
  double *sv = (double *)malloc(sizeof(double) * (size_t)L);
  double *yss = (double *)malloc(sizeof(double) * (size_t)L);
  double *g = (double *)malloc(sizeof(double) * (size_t)N);
  if (!hs || !dl || !sv || !yss || !g) {
    j->status = -1;
    free(hs); free(dl); free(sv); free(yss); free(g);
    return NULL;
  }
  for (int64_t ch = j->ch_lo; ch < j->ch_hi; ++ch) {
    const int64_t b = ch / Dm, d = ch % Dm;
    const double *u = j->u + ch * L, *dr = j->delta + ch * L;
    const double *z = j->z ? j->z + ch * L : NULL;
    const double *Bb = j->B + b * L * N, *Cb = j->C + b * L * N;
    const double *Ad = j->A + d * N;
    const double Dd = j->D ? j->D[d] : 0.0;
    const double bias = j->delta_bias ? j->delta_bias[d] : 0.0;
    const double *dout = j->dout + ch * L;
    /* forward, keeping every state */
    for (int64_t n = 0; n < N; ++n) hs[n] = j->h0 ? j->h0[ch * N + n] : 0.0;
    for (int64_t t = 0; t < L; ++t) {
      sv[t] = dr[t] + bias;
      dl[t] = j->delta_softplus ? softplus(sv[t]) : sv[t];
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double abar = exp(dl[t] * Ad[n]);
        const double hn = abar * hs[t * N + n] + bbar_scale(dl[t], Ad[n], j->zoh_exact) * Bb[t * N + n] * u[t];
        hs[(t + 1) * N + n] = hn;
        acc += Cb[t * N + n] * hn;
      }
      yss[t] = acc + Dd * u[t];
    }
    /* reverse */
    for (int64_t n = 0; n < N; ++n) g[n] = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
      double dyy = dout[t];
      if (z) {
        const double sg = sigmoid(z[t]);
        j->dz[ch * L + t] = dout[t] * yss[t] * sg * (1.0 + z[t] * (1.0 - sg));
        dyy = dout[t] * z[t] * sg;
      }
      j->pdD[d] += dyy * u[t];
      double du = dyy * Dd;
      double ddl = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        const double ht = hs[(t + 1) * N + n], hp = hs[t * N + n];
        const double abar = exp(dl[t] * Ad[n]);
        const double Btn = Bb[t * N + n];
        const double beta = bbar_scale(dl[t], Ad[n], j->zoh_exact);
        g[n] += dyy * Cb[t * N + n];            /* dL/dh_t */
        j->pdC[(b * L + t) * N + n] += dyy * ht;
        /* h_t = abar h_{t-1} + beta B u, abar = exp(Delta A), beta = beta(Delta, A) */
        ddl += g[n] * (Ad[n] * abar * hp + bbar_scale_ddelta(dl[t], Ad[n], j->zoh_exact) * Btn * u[t]);
        j->pdA[d * N + n] += g[n] * (dl[t] * abar * hp +
                                     bbar_scale_dA(dl[t], Ad[n], j->zoh_exact) * Btn * u[t]);
        j->pdB[(b * L + t) * N + n] += g[n] * beta * u[t];
        du += g[n] * beta * Btn;
        g[n] *= abar;                            /* dL/dh_{t-1} via h_t */
      }
      const double ds = j->delta_softplus ? ddl * sigmoid(sv[t]) : ddl;
      j->ddelta[ch * L + t] = ds;
      j->pdbias[d] += ds;
      j->du[ch * L + t] = du;
    }
    if (j->dh0)
      for (int64_t n = 0; n < N; ++n) j->dh0[ch * N + n] = g[n];
  }
  free(hs); free(dl); free(sv); free(yss); free(g);
  return NULL;
}

/* Split the batch*dim channels into nthreads contiguous ranges. */
static int make_jobs(const job_t *base, int nthreads, job_t **jobs_out) {
  const int64_t nch = base->batch * base->dim;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > nch) nthreads = (int)(nch > 0 ? nch : 1);
  job_t *jobs = (job_t *)calloc((size_t)nthreads, sizeof(job_t));
  if (!jobs) return -1;
  for (int i = 0; i < nthreads; ++i) {
    jobs[i] = *base;
    jobs[i].ch_lo = nch * i / nthreads;
    jobs[i].ch_hi = nch * (i + 1) / nthreads;
  }
  *jobs_out = jobs;
  return nthreads;
}

int oracle_fwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
               const double *u, const double *delta, const double *A,
               const double *B, const double *C, const double *D,
               const double *z, const double *delta_bias, const double *h0,
               int delta_softplus, int zoh_exact,
               double *y, double *last_state, int nthreads) {
  if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1) return -2;
  if (!u || !delta || !A || !B || !C || !y) return -2;
  job_t base;
  memset(&base, 0, sizeof(base));
  base.batch = batch; base.dim = dim; base.seqlen = seqlen; base.dstate = dstate;
  base.u = u; base.delta = delta; base.A = A; base.B = B; base.C = C; base.D = D;
  base.z = z; base.delta_bias = delta_bias; base.h0 = h0;
  base.delta_softplus = delta_softplus; base.zoh_exact = zoh_exact;
  base.y = y; base.last_state = last_state;
  if (batch * dim == 0) return 0;
  job_t *jobs = NULL;
  int nt = make_jobs(&base, nthreads, &jobs);
  if (nt < 0) return -1;
  pthread_t *tid = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
  int status = 0;
  for (int i = 0; i < nt; ++i) pthread_create(&tid[i], NULL, fwd_worker, &jobs[i]);
  for (int i = 0; i < nt; ++i) {
    pthread_join(tid[i], NULL);
    if (jobs[i].status) status = jobs[i].status;
  }
  free(tid);
  free(jobs);
  return status;
}

int oracle_bwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate,
               const double *u, const double *delta, const double *A,
               const double *B, const double *C, const double *D,
               const double *z, const double *delta_bias, const double *h0,
               int delta_softplus, int zoh_exact, const double *dout,
               double *du, double *ddelta, double *dA, double *dB, double *dC,
               double *dD, double *dz, double *ddelta_bias, double *dh0,
               int nthreads) {
  if (batch < 0 || dim < 0 || seqlen < 0 || dstate < 1) return -2;
  if (!u || !delta || !A || !B || !C || !dout) return -2;
  if (!du || !ddelta || !dA || !dB || !dC || !dD || !ddelta_bias) return -2;
  if (z && !dz) return -2;
  const int64_t L = seqlen, N = dstate;
  memset(dA, 0, sizeof(double) * (size_t)(dim * N));
  memset(dB, 0, sizeof(double) * (size_t)(batch * L * N));
  memset(dC, 0, sizeof(double) * (size_t)(batch * L * N));
  memset(dD, 0, sizeof(double) * (size_t)dim);
  memset(ddelta_bias, 0, sizeof(double) * (size_t)dim);
  if (batch * dim == 0) return 0;
  job_t base;
  memset(&base, 0, sizeof(base));
  base.batch = batch; base.dim = dim; base.seqlen = seqlen; base.dstate = dstate;
  base.u = u; base.delta = delta; base.A = A; base.B = B; base.C = C; base.D = D;
  base.z = z; base.delta_bias = delta_bias; base.h0 = h0;
  base.delta_softplus = delta_softplus; base.zoh_exact = zoh_exact; base.dout = dout;
  base.du = du; base.ddelta = ddelta; base.dz = dz; base.dh0 = dh0;
  job_t *jobs = NULL;
  int nt = make_jobs(&base, nthreads, &jobs);
  if (nt < 0) return -1;
  int status = 0;
  for (int i = 0; i < nt; ++i) {
    jobs[i].pdA = (double *)calloc((size_t)(dim * N), sizeof(double));
    jobs[i].pdB = (double *)calloc((size_t)(batch * L * N), sizeof(double));
    jobs[i].pdC = (double *)calloc((size_t)(batch * L * N), sizeof(double));
    jobs[i].pdD = (double *)calloc((size_t)dim, sizeof(double));
    jobs[i].pdbias = (double *)calloc((size_t)dim, sizeof(double));
    if (!jobs[i].pdA || !jobs[i].pdB || !jobs[i].pdC || !jobs[i].pdD || !jobs[i].pdbias)
      status = -1;
  }
  pthread_t *tid = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
  if (!tid) status = -1;
  if (status == 0) {
    for (int i = 0; i < nt; ++i) pthread_create(&tid[i], NULL, bwd_worker, &jobs[i]);
    for (int i = 0; i < nt; ++i) {
      pthread_join(tid[i], NULL);
      if (jobs[i].status) status = jobs[i].status;
    }
    /* partial sums added in thread order: deterministic for a given nthreads */
    for (int i = 0; i < nt; ++i) {
      for (int64_t k = 0; k < dim * N; ++k) dA[k] += jobs[i].pdA[k];
      for (int64_t k = 0; k < batch * L * N; ++k) dB[k] += jobs[i].pdB[k];
      for (int64_t k = 0; k < batch * L * N; ++k) dC[k] += jobs[i].pdC[k];
      for (int64_t k = 0; k < dim; ++k) dD[k] += jobs[i].pdD[k];
      for (int64_t k = 0; k < dim; ++k) ddelta_bias[k] += jobs[i].pdbias[k];
    }
  }
  for (int i = 0; i < nt; ++i) {
    free(jobs[i].pdA); free(jobs[i].pdB); free(jobs[i].pdC);
    free(jobs[i].pdD); free(jobs[i].pdbias);
  }
  free(tid);
  free(jobs);
  return status;
}

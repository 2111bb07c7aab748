/* The fp64 oracle (oracle/ssm_oracle.c) built with AddressSanitizer and
 * UndefinedBehaviorSanitizer and run on small cases: every optional input on
 * and off, exact ZOH, an initial state, empty problems, one to three threads.
 * Any out-of-bounds access, use after free, leak or undefined operation in
 * the oracle's C code aborts with a report.  Test infrastructure only. */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

int oracle_fwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, const double *u,
               const double *delta, const double *A, const double *B, const double *C,
               const double *D, const double *z, const double *delta_bias, const double *h0,
               int delta_softplus, int zoh_exact, double *y, double *last_state, int nthreads);
int oracle_bwd(int64_t batch, int64_t dim, int64_t seqlen, int64_t dstate, const double *u,
               const double *delta, const double *A, const double *B, const double *C,
               const double *D, const double *z, const double *delta_bias, const double *h0,
               int delta_softplus, int zoh_exact, const double *dout, double *du, double *ddelta,
               double *dA, double *dB, double *dC, double *dD, double *dz, double *ddelta_bias,
               double *dh0, int nthreads);

static uint64_t rng = 0x2545F4914F6CDD1DULL;
static double uniform(void) {  /* xorshift64, mapped to (-1, 1) */
  rng ^= rng << 13;
  rng ^= rng >> 7;
  rng ^= rng << 17;
  return (double)(rng >> 11) / 4503599627370496.0 - 1.0;
}
static double *fill(size_t n, double scale, double offset) {
  double *p = (double *)malloc((n ? n : 1) * sizeof(double));
  if (!p) exit(2);
  for (size_t i = 0; i < n; ++i) p[i] = offset + scale * uniform();
  return p;
}

static int run(int64_t b, int64_t d, int64_t L, int64_t N, int opt, int zoh, int threads) {
  const size_t act = (size_t)(b * d * L), bc = (size_t)(b * L * N), an = (size_t)(d * N),
               st = (size_t)(b * d * N);
  double *u = fill(act, 1, 0), *delta = fill(act, 1, 0), *z = fill(act, 1, 0), *dout = fill(act, 1, 0);
  double *A = fill(an, 0.5, -1), *B = fill(bc, 1, 0), *C = fill(bc, 1, 0);
  double *D = fill((size_t)d, 1, 0), *bias = fill((size_t)d, 1, -3), *h0 = fill(st, 1, 0);
  double *y = fill(act, 0, 0), *ls = fill(st, 0, 0);
  double *du = fill(act, 0, 0), *ddelta = fill(act, 0, 0), *dz = fill(act, 0, 0);
  double *dA = fill(an, 0, 0), *dB = fill(bc, 0, 0), *dC = fill(bc, 0, 0);
  double *dD = fill((size_t)d, 0, 0), *dbias = fill((size_t)d, 0, 0), *dh0 = fill(st, 0, 0);
  const int with_z = opt & 1, with_D = opt & 2, with_bias = opt & 4, with_h0 = opt & 8;
  int rc = oracle_fwd(b, d, L, N, u, delta, A, B, C, with_D ? D : NULL, with_z ? z : NULL,
                      with_bias ? bias : NULL, with_h0 ? h0 : NULL, 1, zoh, y, ls, threads);
  if (rc == 0)
    rc = oracle_bwd(b, d, L, N, u, delta, A, B, C, with_D ? D : NULL, with_z ? z : NULL,
                    with_bias ? bias : NULL, with_h0 ? h0 : NULL, 1, zoh, dout, du, ddelta, dA, dB,
                    dC, dD, with_z ? dz : NULL, dbias, with_h0 ? dh0 : NULL, threads);
  free(u); free(delta); free(z); free(dout); free(A); free(B); free(C); free(D); free(bias);
  free(h0); free(y); free(ls); free(du); free(ddelta); free(dz); free(dA); free(dB); free(dC);
  free(dD); free(dbias); free(dh0);
  return rc;
}

int main(void) {
  const int64_t shapes[][4] = {{2, 3, 17, 4}, {1, 5, 1, 1}, {3, 2, 40, 16}, {1, 1, 64, 3},
                               {0, 4, 10, 4}, {2, 0, 10, 4}, {2, 3, 0, 4}};
  int failures = 0;
  for (size_t s = 0; s < sizeof(shapes) / sizeof(shapes[0]); ++s)
    for (int opt = 0; opt < 16; opt += 5)
      for (int zoh = 0; zoh < 2; ++zoh)
        for (int threads = 1; threads <= 3; threads += 2) {
          const int rc = run(shapes[s][0], shapes[s][1], shapes[s][2], shapes[s][3], opt, zoh, threads);
          if (rc != 0) {
            fprintf(stderr, "oracle rc %d at shape %zu opt %d zoh %d threads %d\n", rc, s, opt, zoh, threads);
            ++failures;
          }
        }
  if (failures) return 1;
  printf("oracle under sanitizers: ok\n");
  return 0;
}

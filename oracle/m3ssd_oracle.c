/*
 * m3ssd_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, sequential fp64 CPU statement of the Mamba-3 SISO selective
 * scan. It exists so that the CUDA library can be checked against something
 * that is obviously correct; no product code path may link, load or call it.
 * Only the test suite, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (sources, by page title and section):
 *   - "TorchMamba" README, table "Models", row Mamba-3 SISO, and "Math notes",
 *     paragraph "M3 SISO": the exponential-trapezoidal three-term recurrence
 *         h_t = alpha_t h_{t-1} + beta_t Bbar_{t-1} x_{t-1}^T + gamma_t Bbar_t x_t^T
 *     with complex state entering through accumulated, data-dependent pairwise
 *     rotations of B and C ("RoPE trick").
 *   - "TorchMamba" README, "Functional cores": the functional form
 *     trap_rope_loop(X, logdecay, B, C, theta_dt, lam) with X (B,L,H,P) and
 *     theta (B,L,H,N/2); "API reference": the decode cache
 *     Mamba3SisoCache(angle, ssm, x_prev, b_prev).
 *   - "VikramLex/mamba3-minimal", section "Two-SSD Decomposition": the beta
 *     term uses the previous step's B and x.
 *   - "TorchMamba" README, "Behavioral notes": lam = 1 is the exact two-term
 *     path (no previous-step contribution); theta absent is the real-only path;
 *     H % G == 0; N even.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - pairs are adjacent components (2i, 2i+1), rotated by the i-th angle;
 *   - the rotation is counter-clockwise, [[cos, -sin], [sin, cos]], applied to
 *     both B and C;
 *   - the angle is an inclusive running sum: Bbar_t and Cbar_t use
 *     phi_t = angle0 + sum_{s<=t} theta_s;
 *   - theta arrives already multiplied by the step size;
 *   - before the first token the previous-step term is bprev0 x xprev0 (zero
 *     when absent), with bprev0 rotated by angle0; h0 lives in the same
 *     (absolute) frame as Bbar;
 *   - y_t = Cbar_t^T h_t + D_h x_t, with D absent meaning 0;
 *   - head h uses B/C group g = h / (H / G).
 *
 * Precision: fp64 throughout; sin, cos and exp come from the host libm.
 * Parallelism: independent (b, h) sequences are spread over POSIX threads;
 * each sequence is computed strictly in time order, so threading does not
 * change a single rounding.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
} oracle_dims;

typedef struct {
  const oracle_dims* d;
  const double *X, *logdecay, *beta, *gamma, *B, *C, *theta, *D, *h0;
  const double *angle0, *xprev0, *bprev0;
  double *Y, *hT, *angleT, *xprevT, *bprevT;
  int64_t next_pair; /* work counter, guarded by mu */
  pthread_mutex_t mu;
  int status;
} fwd_job;

/* v rotated pairwise: out[2i], out[2i+1] = R(phi_i) (v[2i], v[2i+1]) */
static void rotate_pairs(const double* v, const double* phi, int64_t n, double* out) {
  for (int64_t i = 0; i < n / 2; ++i) {
    const double c = cos(phi[i]);
    const double s = sin(phi[i]);
    const double re = v[2 * i];
    const double im = v[2 * i + 1];
    out[2 * i] = c * re - s * im;
    out[2 * i + 1] = s * re + c * im;
  }
}

/* One (b, h) sequence, t = 0 .. L-1, exactly as the recurrence is written. */
static int fwd_one(fwd_job* j, int64_t b, int64_t h) {
  const oracle_dims* d = j->d;
  const int64_t L = d->seqlen, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
  const int64_t g = h / (H / G);
  const int64_t NH = N / 2;

  double* phi = calloc((size_t)NH, sizeof(double));     /* angle after token t */
  double* phi_prev = calloc((size_t)NH, sizeof(double));/* angle of the previous token */
  double* S = calloc((size_t)(N * P), sizeof(double));  /* state h, N x P, row-major */
  double* xp = calloc((size_t)P, sizeof(double));       /* x_{t-1} */
  double* Bp = calloc((size_t)N, sizeof(double));       /* B_{t-1}, unrotated */
  double* Bbar = malloc((size_t)N * sizeof(double));
  double* Cbar = malloc((size_t)N * sizeof(double));
  double* Bpbar = malloc((size_t)N * sizeof(double));
  if (!phi || !phi_prev || !S || !xp || !Bp || !Bbar || !Cbar || !Bpbar) {
    free(phi); free(phi_prev); free(S); free(xp); free(Bp); free(Bbar); free(Cbar); free(Bpbar);
    return 1;
  }

  for (int64_t i = 0; i < NH; ++i) phi[i] = j->angle0 ? j->angle0[(b * H + h) * NH + i] : 0.0;
  if (j->h0)
    for (int64_t e = 0; e < N * P; ++e) S[e] = j->h0[(b * H + h) * N * P + e];
  if (j->xprev0)
    for (int64_t p = 0; p < P; ++p) xp[p] = j->xprev0[(b * H + h) * P + p];
  if (j->bprev0)
    for (int64_t n = 0; n < N; ++n) Bp[n] = j->bprev0[(b * G + g) * N + n];
  memcpy(phi_prev, phi, (size_t)NH * sizeof(double));

  for (int64_t t = 0; t < L; ++t) {
    const int64_t th = (b * L + t) * H + h; /* index of (b, t, h) */
    const int64_t tg = (b * L + t) * G + g; /* index of (b, t, g) */
    const double* x = j->X + th * P;

    if (j->theta)
      for (int64_t i = 0; i < NH; ++i) phi[i] += j->theta[th * NH + i];

    rotate_pairs(j->B + tg * N, phi, N, Bbar);
    rotate_pairs(j->C + tg * N, phi, N, Cbar);
    rotate_pairs(Bp, phi_prev, N, Bpbar);

    const double alpha = exp(j->logdecay[th]);
    const double be = j->beta ? j->beta[th] : 0.0;
    const double ga = j->gamma[th];

    for (int64_t n = 0; n < N; ++n)
      for (int64_t p = 0; p < P; ++p)
        S[n * P + p] = alpha * S[n * P + p] + be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];

    const double dh = j->D ? j->D[h] : 0.0;
    for (int64_t p = 0; p < P; ++p) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) acc += Cbar[n] * S[n * P + p];
      j->Y[th * P + p] = acc + dh * x[p];
    }

    for (int64_t p = 0; p < P; ++p) xp[p] = x[p];
    for (int64_t n = 0; n < N; ++n) Bp[n] = j->B[tg * N + n];
    memcpy(phi_prev, phi, (size_t)NH * sizeof(double));
  }

  if (j->hT)
    for (int64_t e = 0; e < N * P; ++e) j->hT[(b * H + h) * N * P + e] = S[e];
  if (j->angleT)
    for (int64_t i = 0; i < NH; ++i) j->angleT[(b * H + h) * NH + i] = phi[i];
  if (j->xprevT)
    for (int64_t p = 0; p < P; ++p) j->xprevT[(b * H + h) * P + p] = xp[p];
  /* b_prev is per group; the first head of the group writes it. */
  if (j->bprevT && h % (H / G) == 0)
    for (int64_t n = 0; n < N; ++n) j->bprevT[(b * G + g) * N + n] = Bp[n];

  free(phi); free(phi_prev); free(S); free(xp); free(Bp); free(Bbar); free(Cbar); free(Bpbar);
  return 0;
}

static void* fwd_worker(void* arg) {
  fwd_job* j = (fwd_job*)arg;
  const int64_t npairs = j->d->batch * j->d->nheads;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    const int64_t k = j->next_pair++;
    pthread_mutex_unlock(&j->mu);
    if (k >= npairs) break;
    if (fwd_one(j, k / j->d->nheads, k % j->d->nheads) != 0) {
      pthread_mutex_lock(&j->mu);
      j->status = 1;
      pthread_mutex_unlock(&j->mu);
    }
  }
  return NULL;
}

static int dims_ok(const oracle_dims* d) {
  if (!d) return 0;
  if (d->batch < 0 || d->seqlen < 0 || d->nheads < 1 || d->headdim < 1) return 0;
  if (d->dstate < 2 || d->dstate % 2 != 0) return 0;
  if (d->ngroups < 1 || d->nheads % d->ngroups != 0) return 0;
  return 1;
}

/*
 * Forward over a whole sequence.  Layouts are row-major:
 *   X, Y (b,L,H,P); logdecay, beta, gamma (b,L,H); B, C (b,L,G,N);
 *   theta (b,L,H,N/2); D (H); h0, hT (b,H,N,P); angle0, angleT (b,H,N/2);
 *   xprev0, xprevT (b,H,P); bprev0, bprevT (b,G,N).
 * beta, theta, D, h0, angle0, xprev0, bprev0 may be NULL (read as zero);
 * hT, angleT, xprevT, bprevT may be NULL (not written).
 * Returns 0 on success, 1 on bad dimensions or pointers, 2 on allocation failure.
 */
int oracle_fwd(const oracle_dims* d, const double* X, const double* logdecay, const double* beta,
               const double* gamma, const double* B, const double* C, const double* theta,
               const double* D, const double* h0, const double* angle0, const double* xprev0,
               const double* bprev0, double* Y, double* hT, double* angleT, double* xprevT,
               double* bprevT, int nthreads) {
  if (!dims_ok(d)) return 1;
  if (d->batch * d->seqlen > 0 && (!X || !logdecay || !gamma || !B || !C || !Y)) return 1;
  fwd_job j = {d, X, logdecay, beta, gamma, B, C, theta, D, h0, angle0, xprev0, bprev0,
               Y, hT, angleT, xprevT, bprevT, 0, PTHREAD_MUTEX_INITIALIZER, 0};
  if (nthreads < 1) nthreads = 1;
  const int64_t npairs = d->batch * d->nheads;
  if (nthreads > npairs) nthreads = (int)(npairs > 0 ? npairs : 1);
  pthread_t* th = malloc((size_t)nthreads * sizeof(pthread_t));
  if (!th) return 2;
  int started = 0;
  for (int k = 0; k < nthreads; ++k) {
    if (pthread_create(&th[k], NULL, fwd_worker, &j) != 0) break;
    ++started;
  }
  if (started == 0) fwd_worker(&j);
  for (int k = 0; k < started; ++k) pthread_join(th[k], NULL);
  free(th);
  return j.status ? 2 : 0;
}

/*
 * One decode step on a cache, written as its own function (not a call into
 * the forward) so that "forward over L == L steps" compares two codings.
 * Cache layouts: angle (b,H,N/2), ssm (b,H,N,P), x_prev (b,H,P),
 * b_prev (b,G,N) unrotated; all updated in place.  Step tensors drop L:
 * x_t, y_t (b,H,P); logdecay_t, beta_t, gamma_t (b,H); B_t, C_t (b,G,N);
 * theta_t (b,H,N/2).  beta_t, theta_t, D may be NULL.
 */
int oracle_step(const oracle_dims* d, const double* x_t, const double* logdecay_t,
                const double* beta_t, const double* gamma_t, const double* B_t, const double* C_t,
                const double* theta_t, const double* D, double* angle, double* ssm,
                double* x_prev, double* b_prev, double* y_t) {
  if (!dims_ok(d)) return 1;
  const int64_t Bn = d->batch, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
  const int64_t NH = N / 2;
  double* phi_new = malloc((size_t)NH * sizeof(double));
  double* Bbar = malloc((size_t)N * sizeof(double));
  double* Cbar = malloc((size_t)N * sizeof(double));
  double* Bpbar = malloc((size_t)N * sizeof(double));
  if (!phi_new || !Bbar || !Cbar || !Bpbar) {
    free(phi_new); free(Bbar); free(Cbar); free(Bpbar);
    return 2;
  }
  for (int64_t b = 0; b < Bn; ++b) {
    for (int64_t h = 0; h < H; ++h) {
      const int64_t g = h / (H / G);
      const int64_t bh = b * H + h;
      double* ang = angle + bh * NH;
      for (int64_t i = 0; i < NH; ++i) phi_new[i] = ang[i] + (theta_t ? theta_t[bh * NH + i] : 0.0);
      rotate_pairs(b_prev + (b * G + g) * N, ang, N, Bpbar);
      rotate_pairs(B_t + (b * G + g) * N, phi_new, N, Bbar);
      rotate_pairs(C_t + (b * G + g) * N, phi_new, N, Cbar);
      const double alpha = exp(logdecay_t[bh]);
      const double be = beta_t ? beta_t[bh] : 0.0;
      const double ga = gamma_t[bh];
      double* S = ssm + bh * N * P;
      double* xp = x_prev + bh * P;
      const double* x = x_t + bh * P;
      for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < P; ++p)
          S[n * P + p] = alpha * S[n * P + p] + be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];
      const double dh = D ? D[h] : 0.0;
      for (int64_t p = 0; p < P; ++p) {
        double acc = 0.0;
        for (int64_t n = 0; n < N; ++n) acc += Cbar[n] * S[n * P + p];
        y_t[bh * P + p] = acc + dh * x[p];
      }
      for (int64_t p = 0; p < P; ++p) xp[p] = x[p];
      for (int64_t i = 0; i < NH; ++i) ang[i] = phi_new[i];
    }
    /* every head of a group has read b_prev; now it becomes this step's B */
    for (int64_t g = 0; g < G; ++g)
      for (int64_t n = 0; n < N; ++n) b_prev[(b * G + g) * N + n] = B_t[(b * G + g) * N + n];
  }
  free(phi_new); free(Bbar); free(Cbar); free(Bpbar);
  return 0;
}

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
 * Readings where the pages are silent (each one stated in full below):
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

/* ---------------------------------------------------------------------------
 * Backward (reverse-mode derivatives of the forward above).
 *
 * For one (b, h) the forward is recomputed with every state S_t kept, then the
 * adjoint of each step is taken in reverse time order.  With g = dL/dS_t (it
 * starts as dhT and collects every later step's contribution):
 *   y_t = Cbar_t^T S_t + D x_t      -> dCbar_t = S_t dy_t,  g += Cbar_t dy_t^T,
 *                                      dD += dy_t . x_t,    dx_t += D dy_t
 *   S_t = a_t S_{t-1} + beta_t Bpbar xp^T + gamma_t Bbar_t x_t^T, a_t = exp(logdecay_t)
 *                                   -> dlogdecay_t = a_t <g, S_{t-1}>,
 *                                      dbeta_t = Bpbar^T g xp,  dgamma_t = Bbar_t^T g x_t,
 *                                      dBbar_t = gamma_t g x_t, dx_t += gamma_t g^T Bbar_t,
 *                                      dBpbar = beta_t g xp,    dxp += beta_t g^T Bpbar,
 *                                      and g <- a_t g becomes dL/dS_{t-1}
 *   vbar = R(phi) v (each pair)     -> dv = R(phi)^T dvbar,
 *                                      dphi_i += dvbar_{2i} (-vbar_{2i+1}) + dvbar_{2i+1} vbar_{2i}
 *   phi_t = angle0 + sum_{s<=t} theta_s -> dtheta_s = sum_{t>=s} dphi_t,
 *                                      dangle0 = sum_{t>=-1} dphi_t
 * The previous-step inputs of token 0 are the cache entries xprev0 and bprev0
 * (rotated by angle0 = phi_{-1}); h0 = S_{-1} gets g after the last step.
 * --------------------------------------------------------------------------- */
typedef struct {
  const oracle_dims* d;
  const double *X, *logdecay, *beta, *gamma, *B, *C, *theta, *D, *h0;
  const double *angle0, *xprev0, *bprev0, *dY, *dhT;
  double *dX, *dlogdecay, *dbeta, *dgamma, *dtheta, *dh0, *dangle0, *dxprev0;
  double *dB_head;      /* (b,L,H,N): each head's share of dB, summed over the group later */
  double *dC_head;      /* (b,L,H,N) likewise for dC */
  double *dbprev_head;  /* (b,H,N) likewise for dbprev0 */
  double *dD_bh;        /* (b,H) partial sums of dD */
  int64_t next_pair;
  pthread_mutex_t mu;
  int status;
} bwd_job;

/* d(R(phi) v)/dphi_i . dvbar for each pair, and dv = R(phi)^T dvbar (accumulated). */
static void rotate_pairs_adjoint(const double* vbar, const double* dvbar, const double* phi,
                                 int64_t n, double* dv_acc, double* dphi_acc) {
  for (int64_t i = 0; i < n / 2; ++i) {
    const double c = cos(phi[i]);
    const double s = sin(phi[i]);
    const double d0 = dvbar[2 * i], d1 = dvbar[2 * i + 1];
    dv_acc[2 * i] += c * d0 + s * d1;
    dv_acc[2 * i + 1] += -s * d0 + c * d1;
    dphi_acc[i] += -d0 * vbar[2 * i + 1] + d1 * vbar[2 * i];
  }
}

static int bwd_one(bwd_job* j, int64_t b, int64_t h) {
  const oracle_dims* d = j->d;
  const int64_t L = d->seqlen, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
  const int64_t g = h / (H / G), NH = N / 2, NP = N * P, bh = b * H + h;
  /* phi_t and S_t for t = -1 .. L-1 live at index t + 1 */
  double* phi = calloc((size_t)((L + 1) * NH), sizeof(double));
  double* S = calloc((size_t)((L + 1) * NP), sizeof(double));
  double* dphi = calloc((size_t)((L + 1) * NH), sizeof(double));
  double* gS = calloc((size_t)NP, sizeof(double));
  double* zero = calloc((size_t)(N > P ? N : P), sizeof(double));
  double* vb = malloc((size_t)(6 * N) * sizeof(double));
  if (!phi || !S || !dphi || !gS || !zero || !vb) {
    free(phi); free(S); free(dphi); free(gS); free(zero); free(vb);
    return 1;
  }
  double *Bbar = vb, *Cbar = vb + N, *Bpbar = vb + 2 * N;
  double *dBbar = vb + 3 * N, *dCbar = vb + 4 * N, *dBpbar = vb + 5 * N;
  const double Dh = j->D ? j->D[h] : 0.0;
  const double* xprev0 = j->xprev0 ? j->xprev0 + bh * P : zero;
  const double* bprev0 = j->bprev0 ? j->bprev0 + (b * G + g) * N : zero;

  /* forward recompute, keeping every angle and state */
  for (int64_t i = 0; i < NH; ++i) phi[i] = j->angle0 ? j->angle0[bh * NH + i] : 0.0;
  if (j->h0)
    for (int64_t e = 0; e < NP; ++e) S[e] = j->h0[bh * NP + e];
  for (int64_t t = 0; t < L; ++t) {
    const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
    const double* x = j->X + th * P;
    const double* xp = t > 0 ? j->X + (th - H) * P : xprev0;
    const double* Bprev = t > 0 ? j->B + (tg - G) * N : bprev0;
    double* ph = phi + (t + 1) * NH;
    for (int64_t i = 0; i < NH; ++i) ph[i] = ph[i - NH] + (j->theta ? j->theta[th * NH + i] : 0.0);
    rotate_pairs(j->B + tg * N, ph, N, Bbar);
    rotate_pairs(Bprev, ph - NH, N, Bpbar);
    const double a = exp(j->logdecay[th]);
    const double be = j->beta ? j->beta[th] : 0.0, ga = j->gamma[th];
    const double* Sp = S + t * NP;
    double* St = S + (t + 1) * NP;
    for (int64_t n = 0; n < N; ++n)
      for (int64_t p = 0; p < P; ++p)
        St[n * P + p] = a * Sp[n * P + p] + be * Bpbar[n] * xp[p] + ga * Bbar[n] * x[p];
  }

  /* reverse sweep */
  for (int64_t t = 0; t < L; ++t)
    for (int64_t p = 0; p < P; ++p) j->dX[((b * L + t) * H + h) * P + p] = 0.0;
  if (j->dhT)
    for (int64_t e = 0; e < NP; ++e) gS[e] = j->dhT[bh * NP + e];
  double dD = 0.0;
  for (int64_t t = L - 1; t >= 0; --t) {
    const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
    const double* x = j->X + th * P;
    const double* xp = t > 0 ? j->X + (th - H) * P : xprev0;
    const double* Bprev = t > 0 ? j->B + (tg - G) * N : bprev0;
    const double* ph = phi + (t + 1) * NH;
    const double* St = S + (t + 1) * NP;
    const double* Sp = S + t * NP;
    const double* dy = j->dY + th * P;
    double* dx = j->dX + th * P;
    rotate_pairs(j->B + tg * N, ph, N, Bbar);
    rotate_pairs(j->C + tg * N, ph, N, Cbar);
    rotate_pairs(Bprev, ph - NH, N, Bpbar);

    /* y_t = Cbar_t^T S_t + D x_t */
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t p = 0; p < P; ++p) acc += St[n * P + p] * dy[p];
      dCbar[n] = acc;
    }
    for (int64_t n = 0; n < N; ++n)
      for (int64_t p = 0; p < P; ++p) gS[n * P + p] += Cbar[n] * dy[p];
    for (int64_t p = 0; p < P; ++p) {
      dD += dy[p] * x[p];
      dx[p] += Dh * dy[p];
    }

    /* S_t = a S_{t-1} + beta Bpbar xp^T + gamma Bbar x^T */
    const double a = exp(j->logdecay[th]);
    const double be = j->beta ? j->beta[th] : 0.0, ga = j->gamma[th];
    double da = 0.0, dbe = 0.0, dga = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      double gx = 0.0, gxp = 0.0;
      for (int64_t p = 0; p < P; ++p) {
        const double gv = gS[n * P + p];
        da += gv * Sp[n * P + p];
        gx += gv * x[p];
        gxp += gv * xp[p];
      }
      dga += Bbar[n] * gx;
      dbe += Bpbar[n] * gxp;
      dBbar[n] = ga * gx;
      dBpbar[n] = be * gxp;
    }
    for (int64_t p = 0; p < P; ++p) {
      double gb = 0.0, gbp = 0.0;
      for (int64_t n = 0; n < N; ++n) {
        gb += gS[n * P + p] * Bbar[n];
        gbp += gS[n * P + p] * Bpbar[n];
      }
      dx[p] += ga * gb;
      if (t > 0)
        j->dX[(th - H) * P + p] += be * gbp;
      else if (j->dxprev0)
        j->dxprev0[bh * P + p] = be * gbp;
    }
    j->dlogdecay[th] = a * da;
    j->dgamma[th] = dga;
    if (j->dbeta) j->dbeta[th] = dbe;
    for (int64_t e = 0; e < NP; ++e) gS[e] *= a;

    /* rotations: Bbar_t and Cbar_t by phi_t, the previous step's B by phi_{t-1} */
    double* dph = dphi + (t + 1) * NH;
    rotate_pairs_adjoint(Bbar, dBbar, ph, N, j->dB_head + th * N, dph);
    rotate_pairs_adjoint(Cbar, dCbar, ph, N, j->dC_head + th * N, dph);
    rotate_pairs_adjoint(Bpbar, dBpbar, ph - NH, N,
                         t > 0 ? j->dB_head + (th - H) * N : j->dbprev_head + bh * N, dph - NH);
  }
  if (j->dh0)
    for (int64_t e = 0; e < NP; ++e) j->dh0[bh * NP + e] = gS[e];
  /* phi_t = angle0 + sum_{s<=t} theta_s: suffix sums of dphi */
  for (int64_t i = 0; i < NH; ++i) {
    double run = 0.0;
    for (int64_t t = L - 1; t >= 0; --t) {
      run += dphi[(t + 1) * NH + i];
      if (j->dtheta) j->dtheta[((b * L + t) * H + h) * NH + i] = run;
    }
    if (j->dangle0) j->dangle0[bh * NH + i] = run + dphi[i];
  }
  j->dD_bh[bh] = dD;
  free(phi); free(S); free(dphi); free(gS); free(zero); free(vb);
  return 0;
}

static void* bwd_worker(void* arg) {
  bwd_job* j = (bwd_job*)arg;
  const int64_t npairs = j->d->batch * j->d->nheads;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    const int64_t k = j->next_pair++;
    pthread_mutex_unlock(&j->mu);
    if (k >= npairs) break;
    if (bwd_one(j, k / j->d->nheads, k % j->d->nheads) != 0) {
      pthread_mutex_lock(&j->mu);
      j->status = 1;
      pthread_mutex_unlock(&j->mu);
    }
  }
  return NULL;
}

/*
 * Backward of oracle_fwd for upstream gradients dY (b,L,H,P) and dhT
 * (b,H,N,P, NULL = 0).  Outputs use the layouts of the matching inputs:
 * dX, dlogdecay, dgamma, dB, dC are required; dbeta, dtheta, dD, dh0,
 * dangle0, dxprev0, dbprev0 may be NULL (not written).  The cache outputs
 * angleT, xprevT and bprevT get no upstream gradient.  An input passed as
 * NULL is read as zero and its gradient is the derivative there.  Group-shared
 * gradients (dB, dbprev0) and dD are summed in a fixed order after the
 * per-sequence work, so the result does not depend on the thread count.
 * Returns 0 on success, 1 on bad dimensions or pointers, 2 on allocation failure.
 */
int oracle_bwd(const oracle_dims* d, const double* X, const double* logdecay, const double* beta,
               const double* gamma, const double* B, const double* C, const double* theta,
               const double* D, const double* h0, const double* angle0, const double* xprev0,
               const double* bprev0, const double* dY, const double* dhT, double* dX,
               double* dlogdecay, double* dbeta, double* dgamma, double* dB, double* dC,
               double* dtheta, double* dD, double* dh0, double* dangle0, double* dxprev0,
               double* dbprev0, int nthreads) {
  if (!dims_ok(d)) return 1;
  const int64_t Bt = d->batch, L = d->seqlen, H = d->nheads, N = d->dstate, G = d->ngroups;
  if (Bt * L > 0 && (!X || !logdecay || !gamma || !B || !C || !dY || !dX || !dlogdecay ||
                     !dgamma || !dB || !dC))
    return 1;
  double* dB_head = calloc((size_t)(Bt * L * H * N + 1), sizeof(double));
  double* dC_head = calloc((size_t)(Bt * L * H * N + 1), sizeof(double));
  double* dbprev_head = calloc((size_t)(Bt * H * N + 1), sizeof(double));
  double* dD_bh = calloc((size_t)(Bt * H + 1), sizeof(double));
  if (!dB_head || !dC_head || !dbprev_head || !dD_bh) {
    free(dB_head); free(dC_head); free(dbprev_head); free(dD_bh);
    return 2;
  }
  bwd_job j = {d, X, logdecay, beta, gamma, B, C, theta, D, h0, angle0, xprev0, bprev0, dY, dhT,
               dX, dlogdecay, dbeta, dgamma, dtheta, dh0, dangle0, dxprev0,
               dB_head, dC_head, dbprev_head, dD_bh, 0, PTHREAD_MUTEX_INITIALIZER, 0};
  if (nthreads < 1) nthreads = 1;
  const int64_t npairs = Bt * H;
  if (nthreads > npairs) nthreads = (int)(npairs > 0 ? npairs : 1);
  pthread_t* th = malloc((size_t)nthreads * sizeof(pthread_t));
  int started = 0;
  if (th)
    for (int k = 0; k < nthreads; ++k) {
      if (pthread_create(&th[k], NULL, bwd_worker, &j) != 0) break;
      ++started;
    }
  if (started == 0) bwd_worker(&j);
  for (int k = 0; k < started; ++k) pthread_join(th[k], NULL);
  free(th);
  /* group sums over the heads h = g (H/G) .. (g+1) (H/G) - 1, in head order */
  const int64_t hpg = H / G;
  for (int64_t bt = 0; bt < Bt * L; ++bt)
    for (int64_t gg = 0; gg < G; ++gg)
      for (int64_t n = 0; n < N; ++n) {
        double sb = 0.0, sc = 0.0;
        for (int64_t k = 0; k < hpg; ++k) {
          sb += dB_head[(bt * H + gg * hpg + k) * N + n];
          sc += dC_head[(bt * H + gg * hpg + k) * N + n];
        }
        dB[(bt * G + gg) * N + n] = sb;
        dC[(bt * G + gg) * N + n] = sc;
      }
  if (dbprev0)
    for (int64_t b = 0; b < Bt; ++b)
      for (int64_t gg = 0; gg < G; ++gg)
        for (int64_t n = 0; n < N; ++n) {
          double sb = 0.0;
          for (int64_t k = 0; k < hpg; ++k) sb += dbprev_head[(b * H + gg * hpg + k) * N + n];
          dbprev0[(b * G + gg) * N + n] = sb;
        }
  if (dD)
    for (int64_t hh = 0; hh < H; ++hh) {
      double s = 0.0;
      for (int64_t b = 0; b < Bt; ++b) s += dD_bh[b * H + hh];
      dD[hh] = s;
    }
  free(dB_head); free(dC_head); free(dbprev_head); free(dD_bh);
  return j.status ? 2 : 0;
}

/* ---------------------------------------------------------------------------
 * MIMO rank R ("TorchMamba" README, table "Models", row Mamba-3 MIMO: a rank-R
 * matmul update on a shared (N, P) state; "Functional cores": mimo_loop with
 * X (B,L,H,P,R) -> Y (B,L,H,P,R), h (B,H,N,P); "Math notes", MIMO: the B x^T
 * outer product becomes a matmul).  Reading: B and C carry the rank axis as
 * (b,L,G,N,R); every rank column is rotated by the same angle; the update is
 *     h_t = a_t h_{t-1} + beta_t sum_r Bbar_{t-1,r} x_{t-1,r}^T + gamma_t sum_r Bbar_{t,r} x_{t,r}^T
 *     y_{t,r} = Cbar_{t,r}^T h_t + D_h x_{t,r}
 * and the cache holds x_prev (b,H,P,R) and b_prev (b,G,N,R).  At R = 1 this is
 * the SISO recurrence above.
 * --------------------------------------------------------------------------- */
typedef struct {
  int64_t batch, seqlen, nheads, headdim, dstate, ngroups, rank;
} oracle_mimo_dims;

/* column r of an (N, R) matrix rotated pairwise: out[(2i) R + r], out[(2i+1) R + r] */
static void rotate_pairs_col(const double* v, const double* phi, int64_t n, int64_t R,
                             double* out) {
  for (int64_t i = 0; i < n / 2; ++i) {
    const double c = cos(phi[i]);
    const double s = sin(phi[i]);
    for (int64_t r = 0; r < R; ++r) {
      const double re = v[(2 * i) * R + r];
      const double im = v[(2 * i + 1) * R + r];
      out[(2 * i) * R + r] = c * re - s * im;
      out[(2 * i + 1) * R + r] = s * re + c * im;
    }
  }
}

typedef struct {
  const oracle_mimo_dims* d;
  const double *X, *logdecay, *beta, *gamma, *B, *C, *theta, *D, *h0;
  const double *angle0, *xprev0, *bprev0;
  double *Y, *hT, *angleT, *xprevT, *bprevT;
  int64_t next_pair;
  pthread_mutex_t mu;
  int status;
} mimo_job;

/* one MIMO token: S, phi and the previous-token buffers updated in place */
static void mimo_token(const oracle_mimo_dims* d, int64_t h, const double* x, const double* B,
                       const double* C, const double* theta_t, double logdecay, double be,
                       double ga, const double* D, double* phi, double* phi_prev, double* S,
                       double* xp, double* Bp, double* Bbar, double* Cbar, double* Bpbar,
                       double* y) {
  const int64_t P = d->headdim, N = d->dstate, R = d->rank, NH = N / 2;
  if (theta_t)
    for (int64_t i = 0; i < NH; ++i) phi[i] += theta_t[i];
  rotate_pairs_col(B, phi, N, R, Bbar);
  rotate_pairs_col(C, phi, N, R, Cbar);
  rotate_pairs_col(Bp, phi_prev, N, R, Bpbar);
  const double alpha = exp(logdecay);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t p = 0; p < P; ++p) {
      double ub = 0.0, ug = 0.0;
      for (int64_t r = 0; r < R; ++r) {
        ub += Bpbar[n * R + r] * xp[p * R + r];
        ug += Bbar[n * R + r] * x[p * R + r];
      }
      S[n * P + p] = alpha * S[n * P + p] + be * ub + ga * ug;
    }
  const double dh = D ? D[h] : 0.0;
  for (int64_t p = 0; p < P; ++p)
    for (int64_t r = 0; r < R; ++r) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) acc += Cbar[n * R + r] * S[n * P + p];
      y[p * R + r] = acc + dh * x[p * R + r];
    }
  memcpy(xp, x, (size_t)(P * R) * sizeof(double));
  memcpy(Bp, B, (size_t)(N * R) * sizeof(double));
  memcpy(phi_prev, phi, (size_t)NH * sizeof(double));
}

static int mimo_one(mimo_job* j, int64_t b, int64_t h) {
  const oracle_mimo_dims* d = j->d;
  const int64_t L = d->seqlen, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
  const int64_t R = d->rank, g = h / (H / G), NH = N / 2, bh = b * H + h;
  double* phi = calloc((size_t)NH, sizeof(double));
  double* phi_prev = calloc((size_t)NH, sizeof(double));
  double* S = calloc((size_t)(N * P), sizeof(double));
  double* xp = calloc((size_t)(P * R), sizeof(double));
  double* Bp = calloc((size_t)(N * R), sizeof(double));
  double* buf = malloc((size_t)(3 * N * R) * sizeof(double));
  if (!phi || !phi_prev || !S || !xp || !Bp || !buf) {
    free(phi); free(phi_prev); free(S); free(xp); free(Bp); free(buf);
    return 1;
  }
  for (int64_t i = 0; i < NH; ++i) phi[i] = j->angle0 ? j->angle0[bh * NH + i] : 0.0;
  memcpy(phi_prev, phi, (size_t)NH * sizeof(double));
  if (j->h0) memcpy(S, j->h0 + bh * N * P, (size_t)(N * P) * sizeof(double));
  if (j->xprev0) memcpy(xp, j->xprev0 + bh * P * R, (size_t)(P * R) * sizeof(double));
  if (j->bprev0) memcpy(Bp, j->bprev0 + (b * G + g) * N * R, (size_t)(N * R) * sizeof(double));
  for (int64_t t = 0; t < L; ++t) {
    const int64_t th = (b * L + t) * H + h, tg = (b * L + t) * G + g;
    mimo_token(d, h, j->X + th * P * R, j->B + tg * N * R, j->C + tg * N * R,
               j->theta ? j->theta + th * NH : NULL, j->logdecay[th],
               j->beta ? j->beta[th] : 0.0, j->gamma[th], j->D, phi, phi_prev, S, xp, Bp, buf,
               buf + N * R, buf + 2 * N * R, j->Y + th * P * R);
  }
  if (j->hT) memcpy(j->hT + bh * N * P, S, (size_t)(N * P) * sizeof(double));
  if (j->angleT) memcpy(j->angleT + bh * NH, phi, (size_t)NH * sizeof(double));
  if (j->xprevT) memcpy(j->xprevT + bh * P * R, xp, (size_t)(P * R) * sizeof(double));
  if (j->bprevT && h % (H / G) == 0)
    memcpy(j->bprevT + (b * G + g) * N * R, Bp, (size_t)(N * R) * sizeof(double));
  free(phi); free(phi_prev); free(S); free(xp); free(Bp); free(buf);
  return 0;
}

static void* mimo_worker(void* arg) {
  mimo_job* j = (mimo_job*)arg;
  const int64_t npairs = j->d->batch * j->d->nheads;
  for (;;) {
    pthread_mutex_lock(&j->mu);
    const int64_t k = j->next_pair++;
    pthread_mutex_unlock(&j->mu);
    if (k >= npairs) break;
    if (mimo_one(j, k / j->d->nheads, k % j->d->nheads) != 0) {
      pthread_mutex_lock(&j->mu);
      j->status = 1;
      pthread_mutex_unlock(&j->mu);
    }
  }
  return NULL;
}

static int mimo_dims_ok(const oracle_mimo_dims* d) {
  if (!d || d->rank < 1) return 0;
  const oracle_dims s = {d->batch, d->seqlen, d->nheads, d->headdim, d->dstate, d->ngroups};
  return dims_ok(&s);
}

/*
 * MIMO forward.  Layouts: X, Y (b,L,H,P,R); logdecay, beta, gamma (b,L,H);
 * B, C (b,L,G,N,R); theta (b,L,H,N/2); D (H); h0, hT (b,H,N,P);
 * angle0, angleT (b,H,N/2); xprev0, xprevT (b,H,P,R); bprev0, bprevT (b,G,N,R).
 * NULL conventions and return codes as oracle_fwd.
 */
int oracle_mimo_fwd(const oracle_mimo_dims* d, const double* X, const double* logdecay,
                    const double* beta, const double* gamma, const double* B, const double* C,
                    const double* theta, const double* D, const double* h0, const double* angle0,
                    const double* xprev0, const double* bprev0, double* Y, double* hT,
                    double* angleT, double* xprevT, double* bprevT, int nthreads) {
  if (!mimo_dims_ok(d)) return 1;
  if (d->batch * d->seqlen > 0 && (!X || !logdecay || !gamma || !B || !C || !Y)) return 1;
  mimo_job j = {d, X, logdecay, beta, gamma, B, C, theta, D, h0, angle0, xprev0, bprev0,
                Y, hT, angleT, xprevT, bprevT, 0, PTHREAD_MUTEX_INITIALIZER, 0};
  if (nthreads < 1) nthreads = 1;
  const int64_t npairs = d->batch * d->nheads;
  if (nthreads > npairs) nthreads = (int)(npairs > 0 ? npairs : 1);
  pthread_t* th = malloc((size_t)nthreads * sizeof(pthread_t));
  int started = 0;
  if (th)
    for (int k = 0; k < nthreads; ++k) {
      if (pthread_create(&th[k], NULL, mimo_worker, &j) != 0) break;
      ++started;
    }
  if (started == 0) mimo_worker(&j);
  for (int k = 0; k < started; ++k) pthread_join(th[k], NULL);
  free(th);
  return j.status ? 2 : 0;
}

/*
 * One MIMO decode step on a cache (angle (b,H,N/2), ssm (b,H,N,P),
 * x_prev (b,H,P,R), b_prev (b,G,N,R) unrotated), updated in place; x_t, y_t
 * (b,H,P,R), B_t, C_t (b,G,N,R), logdecay_t, beta_t, gamma_t (b,H),
 * theta_t (b,H,N/2).  b_prev is replaced after every head has used it.
 */
int oracle_mimo_step(const oracle_mimo_dims* d, const double* x_t, const double* logdecay_t,
                     const double* beta_t, const double* gamma_t, const double* B_t,
                     const double* C_t, const double* theta_t, const double* D, double* angle,
                     double* ssm, double* x_prev, double* b_prev, double* y_t) {
  if (!mimo_dims_ok(d)) return 1;
  const int64_t Bt = d->batch, H = d->nheads, P = d->headdim, N = d->dstate, G = d->ngroups;
  const int64_t R = d->rank, NH = N / 2;
  double* phi_prev = malloc((size_t)NH * sizeof(double));
  double* Bp = malloc((size_t)(N * R) * sizeof(double));
  double* buf = malloc((size_t)(3 * N * R) * sizeof(double));
  if (!phi_prev || !Bp || !buf) {
    free(phi_prev); free(Bp); free(buf);
    return 2;
  }
  for (int64_t b = 0; b < Bt; ++b)
    for (int64_t h = 0; h < H; ++h) {
      const int64_t bh = b * H + h, g = h / (H / G);
      memcpy(phi_prev, angle + bh * NH, (size_t)NH * sizeof(double));
      memcpy(Bp, b_prev + (b * G + g) * N * R, (size_t)(N * R) * sizeof(double));
      mimo_token(d, h, x_t + bh * P * R, B_t + (b * G + g) * N * R, C_t + (b * G + g) * N * R,
                 theta_t ? theta_t + bh * NH : NULL, logdecay_t[bh], beta_t ? beta_t[bh] : 0.0,
                 gamma_t[bh], D, angle + bh * NH, phi_prev, ssm + bh * N * P,
                 x_prev + bh * P * R, Bp, buf, buf + N * R, buf + 2 * N * R, y_t + bh * P * R);
    }
  memcpy(b_prev, B_t, (size_t)(Bt * G * N * R) * sizeof(double));
  free(phi_prev); free(Bp); free(buf);
  return 0;
}

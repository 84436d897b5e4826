/*
 * m3_oracle.c -- plain, slow fp64 CPU oracle for the Mamba-3 SSM layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file: only tests/, the smoke check in __graft_entry__.py and the
 * cpu_baseline / reference legs of bench.py use it.  It shares no code, header,
 * table or constant with the CUDA library.
 *
 * What it computes (paper: "Mamba-3: Improved Sequence Modeling using State
 * Space Principles"; PaperWeekly page sections 2.1-2.3, wmrh.cn blog sections
 * 2.1-2.3, arXiv 2603.15569 abstract):
 *
 *   per (batch b, head h) an explicit complex state z in C^{(N/2) x P},
 *   z_k = h_{2k} + i h_{2k+1}  (section 2.1: complex SSM; section 2.2: the
 *   transition is a block-diagonal matrix of 2x2 rotation blocks, so the real
 *   state pairs rows (2k, 2k+1)).
 *
 *   Exponential-trapezoidal step (section 2.2 "generalized trapezoidal rule";
 *   blog section 2.1 "weights both endpoints"):
 *     alpha_t = exp(dt_t A_t),  phi_{t,k} = dt_t theta_{t,k}
 *     z <- alpha_t e^{i phi_{t,k}} ( z + (1-lam_t) dt_t sum_r b_{t-1,k,r} x_{t-1,r}^T )
 *          + lam_t dt_t sum_r b_{t,k,r} x_{t,r}^T
 *   i.e. h_t = alpha_t h_{t-1} + beta_t B_{t-1}x_{t-1}^T + gamma_t B_t x_t^T with
 *   beta_t = (1-lam_t) dt_t alpha_t (carrying the rotation) and gamma_t = lam_t dt_t.
 *   MIMO (section 2.3): the outer product is the rank-R product B_t X_t^T.
 *   Output (section 2.1: the real part is taken):
 *     y_{t,r} = sum_k Re( conj(c_{t,k,r}) z_k ) = C_{t,r}^T h_t.
 *
 * The parity reference is m3o_scan (the token-by-token recurrence).  Two
 * further, independently written forms are used only to pin the recurrence:
 *   m3o_scan_mask   -- the materialised structured mask of section 2.2 /
 *                      Figure 2: a cumulative decay-and-rotation mask times a
 *                      width-2 (bidiagonal) convolution, multiplied out as
 *                      complex L x L matrices per pair.
 *   m3o_scan_rope   -- the data-dependent RoPE form of section 2.2 / abstract:
 *                      B and C rotated by the cumulative angles with real 2x2
 *                      rotations, then a real quadratic (attention-like) form.
 *
 * Readings where the pages are silent (not stated on the pages):
 *   - pairs are adjacent rows (2k, 2k+1); rotation e^{+i phi};
 *   - theta is an angle rate [b][L][Gt][N/2]; the step angle is dt * theta;
 *     Gt (tgroups) is the B/C group count G by default, or H for per-head
 *     angle rates (a layout variant: head h reads theta group h / (H / Gt));
 *   - B, C are shared by the H/G heads of a group; A is per token and head;
 *   - the left-endpoint term is carried through the rotation and decay;
 *   - initial conditions: z = h0 (else 0); B_{-1} x_{-1} = B_prev x_prev (else 0).
 *
 * Layouts (row-major, contiguous) are the library's:
 *   x, y: [b][L][H][R][P]   B, C: [b][L][G][R][N]   dt, A, lam: [b][L][H]
 *   theta: [b][L][Gt][N/2]  h0, hL: [b][H][N][P]   B_prev: [b][G][R][N]
 *   x_prev: [b][H][R][P]
 */
#include <complex.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int64_t batch, seqlen, nheads, ngroups, headdim, dstate, rank;
  int64_t tgroups; /* theta groups: 0 or ngroups (shared like B, C) or nheads */
} m3o_dims;

/* theta group of head h */
static int64_t tgroup(const m3o_dims* d, int64_t h) {
  int64_t Gt = d->tgroups > 0 ? d->tgroups : d->ngroups;
  return h / (d->nheads / Gt);
}
static int64_t tgroups(const m3o_dims* d) { return d->tgroups > 0 ? d->tgroups : d->ngroups; }

/* ---- test-only fault planting (0 = exact method) -------------------------
 * Tests set a mutation to prove that the pins catch plausible mistakes.
 *   1 drop the left-endpoint (beta) term        2 rotation sign flipped
 *   3 left term uses B_t instead of B_{t-1}       4 lam and 1-lam swapped
 *   5 output without conjugation                 6 left term not decayed
 *   7 step angle theta instead of dt*theta        8 decay uses A instead of dt*A
 */
static int g_mutation = 0;
void m3o_set_mutation(int m) { g_mutation = m; }
int m3o_get_mutation(void) { return g_mutation; }

static inline double ld(const void* p, int64_t i, int f64) {
  return f64 ? ((const double*)p)[i] : (double)((const float*)p)[i];
}

/* One exponential-trapezoidal step for one (b, h) chain.
 * Bp/xp may be NULL (zero left endpoint).  z: [N/2][P].  yt: [R][P]. */
static void gtr_step(int64_t N, int64_t P, int64_t R, double complex* z,
                     double dt, double a, double lam, const double* theta,
                     const double* Bp, const double* xp,
                     const double* Bt, const double* xt,
                     const double* Ct, double* yt) {
  const int m = g_mutation;
  double lam_r = (m == 4) ? (1.0 - lam) : lam;
  double alpha = exp((m == 8 ? 1.0 : dt) * a);
  double gamma = lam_r * dt;          /* right endpoint weight */
  double eps = (1.0 - lam_r) * dt;    /* left endpoint weight before decay */
  if (m == 1) eps = 0.0;
  const double* Bl = (m == 3) ? Bt : Bp;
  const double* xl = (m == 3) ? xt : xp;
  for (int64_t k = 0; k < N / 2; ++k) {
    double ang = (m == 7 ? 1.0 : dt) * theta[k];
    if (m == 2) ang = -ang;
    double complex trans = alpha * cexp(I * ang);
    for (int64_t p = 0; p < P; ++p) {
      double complex left = 0.0, right = 0.0;
      for (int64_t r = 0; r < R; ++r) {
        if (Bl && xl)
          left += (Bl[r * N + 2 * k] + I * Bl[r * N + 2 * k + 1]) * xl[r * P + p];
        right += (Bt[r * N + 2 * k] + I * Bt[r * N + 2 * k + 1]) * xt[r * P + p];
      }
      double complex zk = z[k * P + p];
      if (m == 6)
        zk = trans * zk + eps * left + gamma * right;
      else
        zk = trans * (zk + eps * left) + gamma * right;
      z[k * P + p] = zk;
    }
  }
  if (!yt) return;
  for (int64_t r = 0; r < R; ++r)
    for (int64_t p = 0; p < P; ++p) {
      double acc = 0.0;
      for (int64_t k = 0; k < N / 2; ++k) {
        double complex c = Ct[r * N + 2 * k] + I * Ct[r * N + 2 * k + 1];
        double complex w = (m == 5) ? c * z[k * P + p] : conj(c) * z[k * P + p];
        acc += creal(w);
      }
      yt[r * P + p] = acc;
    }
}

/* ---- per-chain gather into contiguous fp64 buffers ----------------------- */
typedef struct {
  double *x, *dt, *A, *lam, *theta, *B, *C, *h0, *Bp, *xp, *y, *hL;
  double complex* z;
} chain_buf;

static int chain_alloc(const m3o_dims* d, chain_buf* cb) {
  int64_t L = d->seqlen, N = d->dstate, P = d->headdim, R = d->rank;
  memset(cb, 0, sizeof(*cb));
  cb->x = malloc(sizeof(double) * (L * R * P + 1));
  cb->y = malloc(sizeof(double) * (L * R * P + 1));
  cb->dt = malloc(sizeof(double) * (L + 1));
  cb->A = malloc(sizeof(double) * (L + 1));
  cb->lam = malloc(sizeof(double) * (L + 1));
  cb->theta = malloc(sizeof(double) * (L * (N / 2) + 1));
  cb->B = malloc(sizeof(double) * (L * R * N + 1));
  cb->C = malloc(sizeof(double) * (L * R * N + 1));
  cb->h0 = malloc(sizeof(double) * N * P);
  cb->hL = malloc(sizeof(double) * N * P);
  cb->Bp = malloc(sizeof(double) * R * N);
  cb->xp = malloc(sizeof(double) * R * P);
  cb->z = malloc(sizeof(double complex) * (N / 2) * P);
  return cb->x && cb->y && cb->dt && cb->A && cb->lam && cb->theta && cb->B &&
         cb->C && cb->h0 && cb->hL && cb->Bp && cb->xp && cb->z;
}

static void chain_free(chain_buf* cb) {
  free(cb->x); free(cb->y); free(cb->dt); free(cb->A); free(cb->lam);
  free(cb->theta); free(cb->B); free(cb->C); free(cb->h0); free(cb->hL);
  free(cb->Bp); free(cb->xp); free(cb->z);
}

typedef struct {
  m3o_dims d;
  int f64;
  const void *x, *dt, *A, *lam, *theta, *B, *C, *h0, *Bp, *xp;
  double *y, *hL;
  const int64_t* chains; /* flat (b * H + h) indices */
  int64_t nchains;
  int64_t next;          /* work counter (guarded by mu) */
  pthread_mutex_t mu;
  int failed;
} scan_job;

static void gather_chain(const scan_job* j, int64_t b, int64_t h, chain_buf* cb) {
  const m3o_dims* d = &j->d;
  int64_t L = d->seqlen, H = d->nheads, G = d->ngroups, N = d->dstate,
          P = d->headdim, R = d->rank;
  int64_t g = h / (H / G);
  for (int64_t t = 0; t < L; ++t) {
    int64_t bt = b * L + t;
    cb->dt[t] = ld(j->dt, bt * H + h, j->f64);
    cb->A[t] = ld(j->A, bt * H + h, j->f64);
    cb->lam[t] = ld(j->lam, bt * H + h, j->f64);
    for (int64_t k = 0; k < N / 2; ++k)
      cb->theta[t * (N / 2) + k] =
          ld(j->theta, (bt * tgroups(d) + tgroup(d, h)) * (N / 2) + k, j->f64);
    for (int64_t i = 0; i < R * N; ++i) {
      cb->B[t * R * N + i] = ld(j->B, (bt * G + g) * R * N + i, j->f64);
      cb->C[t * R * N + i] = ld(j->C, (bt * G + g) * R * N + i, j->f64);
    }
    for (int64_t i = 0; i < R * P; ++i)
      cb->x[t * R * P + i] = ld(j->x, (bt * H + h) * R * P + i, j->f64);
  }
  for (int64_t i = 0; i < N * P; ++i)
    cb->h0[i] = j->h0 ? ld(j->h0, (b * H + h) * N * P + i, j->f64) : 0.0;
  for (int64_t i = 0; i < R * N; ++i)
    cb->Bp[i] = j->Bp ? ld(j->Bp, (b * G + g) * R * N + i, j->f64) : 0.0;
  for (int64_t i = 0; i < R * P; ++i)
    cb->xp[i] = j->xp ? ld(j->xp, (b * H + h) * R * P + i, j->f64) : 0.0;
}

/* The recurrence, token by token, for one chain. */
static void chain_scan(const m3o_dims* d, chain_buf* cb, int have_prev) {
  int64_t L = d->seqlen, N = d->dstate, P = d->headdim, R = d->rank;
  for (int64_t k = 0; k < N / 2; ++k)
    for (int64_t p = 0; p < P; ++p)
      cb->z[k * P + p] = cb->h0[(2 * k) * P + p] + I * cb->h0[(2 * k + 1) * P + p];
  for (int64_t t = 0; t < L; ++t) {
    const double* Bp = t ? cb->B + (t - 1) * R * N : (have_prev ? cb->Bp : NULL);
    const double* xp = t ? cb->x + (t - 1) * R * P : (have_prev ? cb->xp : NULL);
    gtr_step(N, P, R, cb->z, cb->dt[t], cb->A[t], cb->lam[t],
             cb->theta + t * (N / 2), Bp, xp, cb->B + t * R * N,
             cb->x + t * R * P, cb->C + t * R * N, cb->y + t * R * P);
  }
  for (int64_t k = 0; k < N / 2; ++k)
    for (int64_t p = 0; p < P; ++p) {
      cb->hL[(2 * k) * P + p] = creal(cb->z[k * P + p]);
      cb->hL[(2 * k + 1) * P + p] = cimag(cb->z[k * P + p]);
    }
}

static void scatter_chain(scan_job* j, int64_t b, int64_t h, const chain_buf* cb) {
  const m3o_dims* d = &j->d;
  int64_t L = d->seqlen, H = d->nheads, N = d->dstate, P = d->headdim, R = d->rank;
  if (j->y)
    for (int64_t t = 0; t < L; ++t)
      memcpy(j->y + ((b * L + t) * H + h) * R * P, cb->y + t * R * P,
             sizeof(double) * R * P);
  if (j->hL) memcpy(j->hL + (b * H + h) * N * P, cb->hL, sizeof(double) * N * P);
}

static void* scan_worker(void* arg) {
  scan_job* j = (scan_job*)arg;
  chain_buf cb;
  if (!chain_alloc(&j->d, &cb)) {
    pthread_mutex_lock(&j->mu);
    j->failed = 1;
    pthread_mutex_unlock(&j->mu);
    chain_free(&cb);
    return NULL;
  }
  for (;;) {
    pthread_mutex_lock(&j->mu);
    int64_t i = j->next++;
    pthread_mutex_unlock(&j->mu);
    if (i >= j->nchains) break;
    int64_t c = j->chains ? j->chains[i] : i;
    int64_t b = c / j->d.nheads, h = c % j->d.nheads;
    gather_chain(j, b, h, &cb);
    chain_scan(&j->d, &cb, j->Bp != NULL && j->xp != NULL);
    scatter_chain(j, b, h, &cb);
  }
  chain_free(&cb);
  return NULL;
}

static int check_dims(const m3o_dims* d) {
  if (d->batch < 1 || d->seqlen < 0 || d->nheads < 1 || d->ngroups < 1 ||
      d->headdim < 1 || d->dstate < 2 || d->rank < 1)
    return -1;
  if (d->dstate % 2 || d->nheads % d->ngroups) return -1;
  if (d->tgroups < 0 || (d->tgroups > 0 && d->nheads % d->tgroups)) return -1;
  return 0;
}

/* Full oracle scan.  Inputs are fp32 (in_f64 == 0) or fp64 (in_f64 == 1);
 * every value is widened to fp64 before any arithmetic.  chains == NULL means
 * all batch*nheads chains, else `nchains` flat indices b*H + h; outputs of
 * other chains are left untouched.  y and/or hL may be NULL.  Returns 0, or
 * -1 on bad dimensions, -2 on allocation failure.  */
int m3o_scan(const m3o_dims* d, int in_f64, const void* x, const void* dt,
             const void* A, const void* lam, const void* theta, const void* B,
             const void* C, const void* h0, const void* B_prev,
             const void* x_prev, double* y, double* hL, const int64_t* chains,
             int64_t nchains, int nthreads) {
  if (check_dims(d)) return -1;
  scan_job j;
  memset(&j, 0, sizeof(j));
  j.d = *d; j.f64 = in_f64;
  j.x = x; j.dt = dt; j.A = A; j.lam = lam; j.theta = theta; j.B = B; j.C = C;
  j.h0 = h0; j.Bp = B_prev; j.xp = x_prev; j.y = y; j.hL = hL;
  j.chains = chains;
  j.nchains = chains ? nchains : d->batch * d->nheads;
  pthread_mutex_init(&j.mu, NULL);
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  int started = 0;
  for (int i = 0; i < nthreads; ++i)
    if (pthread_create(&th[i], NULL, scan_worker, &j) == 0) ++started;
  if (started == 0) scan_worker(&j);
  for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
  pthread_mutex_destroy(&j.mu);
  return j.failed ? -2 : 0;
}

/* One decode step for all (b, h): the same exponential-trapezoidal step.
 * state: [b][H][N][P] fp64 in/out.  x_t, x_prev, y: [b][H][R][P];
 * dt, A, lam: [b][H]; theta: [b][G][N/2]; B_t, C_t, B_prev: [b][G][R][N].
 * B_prev/x_prev may be NULL (zero left endpoint).  Inputs fp32 or fp64. */
int m3o_decode_step(const m3o_dims* d, int in_f64, double* state,
                    const void* x_t, const void* dt, const void* A,
                    const void* lam, const void* theta, const void* B_t,
                    const void* C_t, const void* B_prev, const void* x_prev,
                    double* y) {
  if (check_dims(d)) return -1;
  int64_t Bn = d->batch, H = d->nheads, G = d->ngroups, N = d->dstate,
          P = d->headdim, R = d->rank;
  double* th = malloc(sizeof(double) * (N / 2));
  double* Bt = malloc(sizeof(double) * R * N);
  double* Ct = malloc(sizeof(double) * R * N);
  double* Bp = malloc(sizeof(double) * R * N);
  double* xt = malloc(sizeof(double) * R * P);
  double* xp = malloc(sizeof(double) * R * P);
  double complex* z = malloc(sizeof(double complex) * (N / 2) * P);
  if (!th || !Bt || !Ct || !Bp || !xt || !xp || !z) {
    free(th); free(Bt); free(Ct); free(Bp); free(xt); free(xp); free(z);
    return -2;
  }
  int have_prev = B_prev != NULL && x_prev != NULL;
  for (int64_t b = 0; b < Bn; ++b)
    for (int64_t h = 0; h < H; ++h) {
      int64_t g = h / (H / G), bh = b * H + h, bg = b * G + g;
      for (int64_t k = 0; k < N / 2; ++k)
        th[k] = ld(theta, (b * tgroups(d) + tgroup(d, h)) * (N / 2) + k, in_f64);
      for (int64_t i = 0; i < R * N; ++i) {
        Bt[i] = ld(B_t, bg * R * N + i, in_f64);
        Ct[i] = ld(C_t, bg * R * N + i, in_f64);
        Bp[i] = have_prev ? ld(B_prev, bg * R * N + i, in_f64) : 0.0;
      }
      for (int64_t i = 0; i < R * P; ++i) {
        xt[i] = ld(x_t, bh * R * P + i, in_f64);
        xp[i] = have_prev ? ld(x_prev, bh * R * P + i, in_f64) : 0.0;
      }
      double* s = state + bh * N * P;
      for (int64_t k = 0; k < N / 2; ++k)
        for (int64_t p = 0; p < P; ++p)
          z[k * P + p] = s[(2 * k) * P + p] + I * s[(2 * k + 1) * P + p];
      gtr_step(N, P, R, z, ld(dt, bh, in_f64), ld(A, bh, in_f64),
               ld(lam, bh, in_f64), th, have_prev ? Bp : NULL,
               have_prev ? xp : NULL, Bt, xt, Ct, y ? y + bh * R * P : NULL);
      for (int64_t k = 0; k < N / 2; ++k)
        for (int64_t p = 0; p < P; ++p) {
          s[(2 * k) * P + p] = creal(z[k * P + p]);
          s[(2 * k + 1) * P + p] = cimag(z[k * P + p]);
        }
    }
  free(th); free(Bt); free(Ct); free(Bp); free(xt); free(xp); free(z);
  return 0;
}


/* ---- pin form 1: the materialised structured mask (decay x width-2 conv) --
 * Paper section 2.2 / Figure 2: unrolling the trapezoidal recurrence gives a
 * structured mask that factors as a cumulative decay part times a width-2
 * convolution.  Here it is multiplied out literally, per pair k, as complex
 * matrices over an extended index (position 0 = the carried initial state,
 * position i >= 1 = token i-1):
 *   Lx[i][j] = exp( sum_{u=j}^{i-1} dt_u (A_u + i theta_{u,k}) )   for i >= j
 *   Wx[0][0] = 1,  Wx[i][i] = lam_{i-1} dt_{i-1},
 *   Wx[i][i-1] = (1-lam_{i-1}) dt_{i-1} exp(dt_{i-1}(A_{i-1} + i theta_{i-1,k}))  (i >= 2)
 *   state_i = sum_j (Lx Wx)[i][j] u_j
 * with u_0 = h0 + (1-lam_0) dt_0 B_prev x_prev^T and u_i = B_{i-1} x_{i-1}^T
 * (rank-R sums, pair k as a complex number).  The exponent sums are formed
 * term by term for every (i, j); nothing is reused across entries.
 * Inputs fp64; O(L^3) per pair: small problems only.  */
int m3o_scan_mask(const m3o_dims* d, const double* x, const double* dt,
                  const double* A, const double* lam, const double* theta,
                  const double* B, const double* C, const double* h0,
                  const double* B_prev, const double* x_prev, double* y,
                  double* hL) {
  if (check_dims(d)) return -1;
  int64_t Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups,
          N = d->dstate, P = d->headdim, R = d->rank;
  if (L < 1) return 0;
  int have_prev = B_prev && x_prev;
  int64_t E = L + 1;
  double complex* Lx = malloc(sizeof(double complex) * E * E);
  double complex* Wx = malloc(sizeof(double complex) * E * E);
  double complex* Mx = malloc(sizeof(double complex) * E * E);
  double complex* u = malloc(sizeof(double complex) * E * P);
  double complex* st = malloc(sizeof(double complex) * E * P);
  if (!Lx || !Wx || !Mx || !u || !st) {
    free(Lx); free(Wx); free(Mx); free(u); free(st);
    return -2;
  }
  for (int64_t b = 0; b < Bn; ++b)
    for (int64_t h = 0; h < H; ++h) {
      int64_t g = h / (H / G);
#define MU(tok) (dt[(b * L + (tok)) * H + h] * (A[(b * L + (tok)) * H + h] + \
                 I * theta[((b * L + (tok)) * tgroups(d) + tgroup(d, h)) * (N / 2) + k]))
      if (y)
        for (int64_t t = 0; t < L; ++t)
          for (int64_t i = 0; i < R * P; ++i) y[((b * L + t) * H + h) * R * P + i] = 0.0;
      for (int64_t k = 0; k < N / 2; ++k) {
        for (int64_t i = 0; i < E; ++i)
          for (int64_t j = 0; j < E; ++j) {
            Wx[i * E + j] = 0.0;
            if (j > i) { Lx[i * E + j] = 0.0; continue; }
            double complex s = 0.0;
            for (int64_t tok = j; tok <= i - 1; ++tok) s += MU(tok);
            Lx[i * E + j] = cexp(s);
          }
        Wx[0] = 1.0;
        for (int64_t i = 1; i < E; ++i) {
          int64_t tok = i - 1;
          double dtt = dt[(b * L + tok) * H + h], lt = lam[(b * L + tok) * H + h];
          Wx[i * E + i] = lt * dtt;
          if (i >= 2) Wx[i * E + i - 1] = (1.0 - lt) * dtt * cexp(MU(tok));
        }
        for (int64_t i = 0; i < E; ++i)
          for (int64_t j = 0; j < E; ++j) {
            double complex acc = 0.0;
            for (int64_t m = 0; m < E; ++m) acc += Lx[i * E + m] * Wx[m * E + j];
            Mx[i * E + j] = acc;
          }
        for (int64_t p = 0; p < P; ++p) {
          double complex u0 = 0.0;
          if (h0)
            u0 = h0[((b * H + h) * N + 2 * k) * P + p] +
                 I * h0[((b * H + h) * N + 2 * k + 1) * P + p];
          if (have_prev) {
            double eps0 = (1.0 - lam[(b * L) * H + h]) * dt[(b * L) * H + h];
            for (int64_t r = 0; r < R; ++r)
              u0 += eps0 *
                    (B_prev[((b * G + g) * R + r) * N + 2 * k] +
                     I * B_prev[((b * G + g) * R + r) * N + 2 * k + 1]) *
                    x_prev[((b * H + h) * R + r) * P + p];
          }
          u[p] = u0;
          for (int64_t tok = 0; tok < L; ++tok) {
            int64_t bt = b * L + tok;
            double complex us = 0.0;
            for (int64_t r = 0; r < R; ++r)
              us += (B[((bt * G + g) * R + r) * N + 2 * k] +
                     I * B[((bt * G + g) * R + r) * N + 2 * k + 1]) *
                    x[((bt * H + h) * R + r) * P + p];
            u[(tok + 1) * P + p] = us;
          }
          for (int64_t i = 0; i < E; ++i) {
            double complex acc = 0.0;
            for (int64_t j = 0; j < E; ++j) acc += Mx[i * E + j] * u[j * P + p];
            st[i * P + p] = acc;
          }
        }
        for (int64_t tok = 0; tok < L; ++tok) {
          int64_t bt = b * L + tok;
          if (y)
            for (int64_t r = 0; r < R; ++r)
              for (int64_t p = 0; p < P; ++p) {
                double complex c = C[((bt * G + g) * R + r) * N + 2 * k] +
                                   I * C[((bt * G + g) * R + r) * N + 2 * k + 1];
                y[((bt * H + h) * R + r) * P + p] += creal(conj(c) * st[(tok + 1) * P + p]);
              }
        }
        if (hL)
          for (int64_t p = 0; p < P; ++p) {
            hL[((b * H + h) * N + 2 * k) * P + p] = creal(st[L * P + p]);
            hL[((b * H + h) * N + 2 * k + 1) * P + p] = cimag(st[L * P + p]);
          }
      }
#undef MU
    }
  free(Lx); free(Wx); free(Mx); free(u); free(st);
  return 0;
}

/* ---- pin form 2: the data-dependent RoPE form, all real arithmetic --------
 * Paper section 2.2 and abstract: the complex transition is equivalent to
 * rotating B and C by the cumulative angles (data-dependent RoPE) and running
 * a real, scalar-decay recurrence.  With global inclusive sums
 *   Lam_t = sum_{u<=t} dt_u A_u,   Phi_{t,k} = sum_{u<=t} dt_u theta_{u,k},
 * and Rot(phi) = [[cos, -sin], [sin, cos]] on rows (2k, 2k+1):
 *   Bt_s = Rot(-Phi_s) B_s,  Ct_t = Rot(-Phi_t) C_t,
 *   y_t = sum_{s<=t} exp(Lam_t - Lam_s) w_{t,s} (Ct_t^T Bt_s) x_s
 *         + exp(Lam_t) Ct_t^T u0,
 *   w_{t,t} = lam_t dt_t,  w_{t,s<t} = lam_s dt_s + (1-lam_{s+1}) dt_{s+1},
 *   u0 = h0 + (1-lam_0) dt_0 B_prev x_prev^T,
 *   h_{L-1} = Rot(Phi_{L-1}) [ sum_s exp(Lam_{L-1}-Lam_s) w_{L-1,s} Bt_s x_s^T
 *                              + exp(Lam_{L-1}) u0 ].
 * Inputs fp64; O(L^2) per chain: small problems only.  */
int m3o_scan_rope(const m3o_dims* d, const double* x, const double* dt,
                  const double* A, const double* lam, const double* theta,
                  const double* B, const double* C, const double* h0,
                  const double* B_prev, const double* x_prev, double* y,
                  double* hL) {
  if (check_dims(d)) return -1;
  int64_t Bn = d->batch, L = d->seqlen, H = d->nheads, G = d->ngroups,
          N = d->dstate, P = d->headdim, R = d->rank;
  if (L < 1) return 0;
  int have_prev = B_prev && x_prev;
  double* Lam = malloc(sizeof(double) * L);
  double* Phi = malloc(sizeof(double) * L * (N / 2));
  double* Bt = malloc(sizeof(double) * L * R * N);
  double* Ct = malloc(sizeof(double) * L * R * N);
  double* u0 = malloc(sizeof(double) * N * P);
  double* hs = malloc(sizeof(double) * N * P);
  if (!Lam || !Phi || !Bt || !Ct || !u0 || !hs) {
    free(Lam); free(Phi); free(Bt); free(Ct); free(u0); free(hs);
    return -2;
  }
  for (int64_t b = 0; b < Bn; ++b)
    for (int64_t h = 0; h < H; ++h) {
      int64_t g = h / (H / G);
      double lsum = 0.0;
      for (int64_t t = 0; t < L; ++t) {
        int64_t bt = b * L + t;
        lsum += dt[bt * H + h] * A[bt * H + h];
        Lam[t] = lsum;
        for (int64_t k = 0; k < N / 2; ++k) {
          double prev = t ? Phi[(t - 1) * (N / 2) + k] : 0.0;
          Phi[t * (N / 2) + k] =
              prev + dt[bt * H + h] * theta[(bt * tgroups(d) + tgroup(d, h)) * (N / 2) + k];
        }
        for (int64_t r = 0; r < R; ++r)
          for (int64_t k = 0; k < N / 2; ++k) {
            double c = cos(Phi[t * (N / 2) + k]), s = sin(Phi[t * (N / 2) + k]);
            const double* Bi = B + ((bt * G + g) * R + r) * N;
            const double* Ci = C + ((bt * G + g) * R + r) * N;
            /* Rot(-phi) = [[c, s], [-s, c]] */
            Bt[(t * R + r) * N + 2 * k] = c * Bi[2 * k] + s * Bi[2 * k + 1];
            Bt[(t * R + r) * N + 2 * k + 1] = -s * Bi[2 * k] + c * Bi[2 * k + 1];
            Ct[(t * R + r) * N + 2 * k] = c * Ci[2 * k] + s * Ci[2 * k + 1];
            Ct[(t * R + r) * N + 2 * k + 1] = -s * Ci[2 * k] + c * Ci[2 * k + 1];
          }
      }
      for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < P; ++p) {
          double v = h0 ? h0[((b * H + h) * N + n) * P + p] : 0.0;
          if (have_prev) {
            double eps0 = (1.0 - lam[(b * L) * H + h]) * dt[(b * L) * H + h];
            for (int64_t r = 0; r < R; ++r)
              v += eps0 * B_prev[((b * G + g) * R + r) * N + n] *
                   x_prev[((b * H + h) * R + r) * P + p];
          }
          u0[n * P + p] = v;
        }
      for (int64_t t = 0; t < L; ++t) {
        int64_t bt = b * L + t;
        for (int64_t r = 0; r < R; ++r)
          for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
              acc += Ct[(t * R + r) * N + n] * u0[n * P + p];
            acc *= exp(Lam[t]);
            for (int64_t s = 0; s <= t; ++s) {
              int64_t bs = b * L + s;
              double w = lam[bs * H + h] * dt[bs * H + h];
              if (s < t) w += (1.0 - lam[(bs + 1) * H + h]) * dt[(bs + 1) * H + h];
              double dec = exp(Lam[t] - Lam[s]) * w;
              for (int64_t r2 = 0; r2 < R; ++r2) {
                double cb = 0.0;
                for (int64_t n = 0; n < N; ++n)
                  cb += Ct[(t * R + r) * N + n] * Bt[(s * R + r2) * N + n];
                acc += dec * cb * x[((bs * H + h) * R + r2) * P + p];
              }
            }
            if (y) y[((bt * H + h) * R + r) * P + p] = acc;
          }
      }
      if (hL) {
        int64_t t = L - 1;
        for (int64_t n = 0; n < N; ++n)
          for (int64_t p = 0; p < P; ++p) {
            double acc = exp(Lam[t]) * u0[n * P + p];
            for (int64_t s = 0; s <= t; ++s) {
              int64_t bs = b * L + s;
              double w = lam[bs * H + h] * dt[bs * H + h];
              if (s < t) w += (1.0 - lam[(bs + 1) * H + h]) * dt[(bs + 1) * H + h];
              double dec = exp(Lam[t] - Lam[s]) * w;
              for (int64_t r2 = 0; r2 < R; ++r2)
                acc += dec * Bt[(s * R + r2) * N + n] * x[((bs * H + h) * R + r2) * P + p];
            }
            hs[n * P + p] = acc;
          }
        for (int64_t k = 0; k < N / 2; ++k) {
          double c = cos(Phi[t * (N / 2) + k]), s = sin(Phi[t * (N / 2) + k]);
          for (int64_t p = 0; p < P; ++p) {
            double a0 = hs[(2 * k) * P + p], a1 = hs[(2 * k + 1) * P + p];
            hL[((b * H + h) * N + 2 * k) * P + p] = c * a0 - s * a1;
            hL[((b * H + h) * N + 2 * k + 1) * P + p] = s * a0 + c * a1;
          }
        }
      }
    }
  free(Lam); free(Phi); free(Bt); free(Ct); free(u0); free(hs);
  return 0;
}

/*
 * Mamba-3 selective recurrence -- plain fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  The CUDA
 * library never includes, links or calls anything in this directory, and this
 * file includes nothing from the CUDA side.
 *
 * What it computes (sources are the pages on the Mamba-3 paper):
 *
 *  - "Mamba-3: 2x smaller state ... MIMO decoding hardware efficiency"
 *    (MarkTechPost, Korean translation), section 1.1 Exponential-Trapezoidal
 *    Discretization: the three-term update
 *        h_t = e^{dt_t A} h_{t-1} + (1 - lam_t) dt_t e^{dt_t A} B_{t-1} x_{t-1}
 *              + lam_t dt_t B_t x_t .
 *  - same page, section 1.2 Complex SSM and the "RoPE trick": the state is
 *    complex; each adjacent pair (2k, 2k+1) of B and C is one complex number
 *    (real, imaginary) and the transition of pair k is exp(dt_t (A + i th_tk)).
 *    The equivalent real form rotates B and C by the angle accumulated over
 *    time, Phi_t = Phi_0 + sum_{s<=t} dt_s th_s.
 *  - same page, section 1.3 MIMO: B_t is N x R, x_t is P x R; the rank-R input
 *    term sum_r B_t[:,r] x_t[:,r]^T replaces the outer product.
 *  - readout y_t[:,r] = Re(sum_k conj(c_tk,r) H_t[k,:]) + D x_t[:,r]; the pages
 *    do not print the readout; this is the standard SSM readout C_t^T h_t with
 *    a per-head skip D (the plainest reading; one output per rank).
 *
 * Three independent formulations live here, all in fp64:
 *   m3o_scan_complex    -- the definition: explicit complex-diagonal state.
 *   m3o_scan_rope       -- real state, B and C rotated by -Phi_t (RoPE form).
 *   m3o_scan_quadratic  -- the L x L masked-kernel ("quadratic") form, brute
 *                          force, for tiny inputs.
 * plus m3o_decode_step, which is one token of m3o_scan_complex continued
 * from a state, and m3o_bc_norm, the RMS normalisation of raw B or C
 * projections over the state dimension with a per-(head, rank) weight and bias
 * (same page, section 2: "BC norm" and head-specific B/C bias), which the
 * recurrence then consumes.
 *
 * Layouts (row-major, contiguous; b = batch, L = seqlen, H = heads):
 *   x      [b, L, H, R, P]     B, C  [b, L, H, R, N]     theta [b, L, H, N/2]
 *   dt,lam [b, L, H]           A, D  [H]                 y     [b, L, H, R, P]
 * Optional: A_t [b, L, H] (a decay rate per token, replacing A), and grouped
 * B, C [b, L, G, R, N] with ngroups G dividing H, head h reading group
 * h / (H / G) (the Mamba line's shared B/C; not on the pages, whose heads each
 * have their own: a grouped input equals the per-head one with every group's
 * rows repeated over its heads).
 * State (the real frame rotated by -Phi, as the CUDA library stores it):
 *   h [b,H,N,P]  (row 2k = Re, row 2k+1 = Im of e^{-i Phi} H)
 *   b_prev [b,H,R,N] (B of the last token, rotated by -Phi of that token)
 *   x_prev [b,H,R,P] (x of the last token)      angle [b,H,N/2] (Phi)
 */
#include <complex.h>
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
  int batch, seqlen, nheads, headdim, dstate, rank;
  int ngroups; /* 0: B, C per head; else B, C [b, L, ngroups, R, N] shared by nheads / ngroups heads */
} m3o_dims;

typedef struct {
  const double *x, *B, *C, *theta, *dt, *lam, *A, *D;  /* D may be NULL */
  const double *h0, *bprev0, *xprev0, *angle0;          /* all NULL = zero state */
  double *y;                                            /* may be NULL */
  double *h_out, *bprev_out, *xprev_out, *angle_out;    /* all NULL = no export */
  const double* A_t; /* NULL, or a time-varying decay [b, L, H] that replaces A[h] token by token */
} m3o_io;

/* The decay rate of token t: A_t[b, t, h] when given (section 1.1 writes the
 * discretisation with a per-step A_t), else the per-head A[h]. */
static double decay_rate(const m3o_io* io, size_t it, int h) { return io->A_t ? io->A_t[it] : io->A[h]; }

/* ------------------------------------------------------------------------- */
/* index helpers                                                               */
/* ------------------------------------------------------------------------- */
static size_t ix_tok(const m3o_dims* d, int b, int t, int h) {
  return ((size_t)b * d->seqlen + t) * d->nheads + h;
}
/* row (b, t, group of head h) of B and C: heads h = g * (H / G) ... (g + 1) * (H / G) - 1
 * share group g (the Mamba line's grouped B/C; the pages use one per head) */
static size_t ix_bc(const m3o_dims* d, int b, int t, int h) {
  if (d->ngroups <= 0) return ix_tok(d, b, t, h);
  return ((size_t)b * d->seqlen + t) * d->ngroups + h / (d->nheads / d->ngroups);
}
static size_t ix_state(const m3o_dims* d, int b, int h) {
  return (size_t)b * d->nheads + h;
}

/* ------------------------------------------------------------------------- */
/* complex-state form (the definition)                                         */
/* ------------------------------------------------------------------------- */
static void unit_complex(const m3o_dims* d, const m3o_io* io, int b, int h) {
  const int L = d->seqlen, P = d->headdim, N = d->dstate, R = d->rank, K = N / 2;
  const double Dh = io->D ? io->D[h] : 0.0;
  double complex* Hs = calloc((size_t)K * P, sizeof(double complex));  /* state H */
  double complex* u_prev = calloc((size_t)K * P, sizeof(double complex));
  double complex* u_cur = calloc((size_t)K * P, sizeof(double complex));
  double complex* a = calloc((size_t)K, sizeof(double complex));
  double* Phi = calloc((size_t)K, sizeof(double));
  const size_t us = ix_state(d, b, h);

  /* initial state: rotate the stored frame back by +Phi_0 */
  if (io->angle0)
    for (int k = 0; k < K; ++k) Phi[k] = io->angle0[us * K + k];
  if (io->h0)
    for (int k = 0; k < K; ++k)
      for (int p = 0; p < P; ++p) {
        double complex g = io->h0[(us * N + 2 * k) * P + p] + I * io->h0[(us * N + 2 * k + 1) * P + p];
        Hs[k * P + p] = cexp(I * Phi[k]) * g;
      }
  if (io->bprev0 && io->xprev0)
    for (int k = 0; k < K; ++k)
      for (int p = 0; p < P; ++p) {
        double complex s = 0;
        for (int r = 0; r < R; ++r) {
          double complex bt = io->bprev0[(us * R + r) * N + 2 * k] + I * io->bprev0[(us * R + r) * N + 2 * k + 1];
          s += cexp(I * Phi[k]) * bt * io->xprev0[(us * R + r) * P + p];
        }
        u_prev[k * P + p] = s;
      }

  for (int t = 0; t < L; ++t) {
    const size_t it = ix_tok(d, b, t, h);
    const double dt = io->dt[it], lam = io->lam[it];
    const double* x = io->x + it * R * P;
    const double* Bt = io->B + ix_bc(d, b, t, h) * R * N;
    const double* Ct = io->C + ix_bc(d, b, t, h) * R * N;
    const double* th = io->theta + it * K;
    const double At = decay_rate(io, it, h);
    for (int k = 0; k < K; ++k) {
      a[k] = cexp(dt * (At + I * th[k]));
      Phi[k] += dt * th[k];
    }
    /* u_t = sum_r b_{t,r} x_{t,r}^T with b complexified by adjacent pairs */
    for (int k = 0; k < K; ++k)
      for (int p = 0; p < P; ++p) {
        double complex s = 0;
        for (int r = 0; r < R; ++r)
          s += (Bt[r * N + 2 * k] + I * Bt[r * N + 2 * k + 1]) * x[r * P + p];
        u_cur[k * P + p] = s;
      }
    /* three-term exponential-trapezoidal update */
    for (int k = 0; k < K; ++k)
      for (int p = 0; p < P; ++p)
        Hs[k * P + p] = a[k] * Hs[k * P + p] + (1.0 - lam) * dt * a[k] * u_prev[k * P + p] +
                        lam * dt * u_cur[k * P + p];
    /* readout, one output per rank */
    if (io->y)
      for (int r = 0; r < R; ++r)
        for (int p = 0; p < P; ++p) {
          double s = 0;
          for (int k = 0; k < K; ++k) {
            double complex c = Ct[r * N + 2 * k] + I * Ct[r * N + 2 * k + 1];
            s += creal(conj(c) * Hs[k * P + p]);
          }
          io->y[it * R * P + r * P + p] = s + Dh * x[r * P + p];
        }
    double complex* tmp = u_prev;
    u_prev = u_cur;
    u_cur = tmp;
  }

  /* export in the frame rotated by -Phi_L */
  if (io->h_out)
    for (int k = 0; k < K; ++k)
      for (int p = 0; p < P; ++p) {
        double complex g = cexp(-I * Phi[k]) * Hs[k * P + p];
        io->h_out[(us * N + 2 * k) * P + p] = creal(g);
        io->h_out[(us * N + 2 * k + 1) * P + p] = cimag(g);
      }
  if (io->angle_out)
    for (int k = 0; k < K; ++k) io->angle_out[us * K + k] = Phi[k];
  if (io->bprev_out && io->xprev_out) {
    if (L > 0) {
      const size_t il = ix_tok(d, b, L - 1, h), ilb = ix_bc(d, b, L - 1, h);
      for (int r = 0; r < R; ++r) {
        for (int k = 0; k < K; ++k) {
          double complex bt = io->B[ilb * R * N + r * N + 2 * k] + I * io->B[ilb * R * N + r * N + 2 * k + 1];
          double complex g = cexp(-I * Phi[k]) * bt;
          io->bprev_out[(us * R + r) * N + 2 * k] = creal(g);
          io->bprev_out[(us * R + r) * N + 2 * k + 1] = cimag(g);
        }
        for (int p = 0; p < P; ++p) io->xprev_out[(us * R + r) * P + p] = io->x[il * R * P + r * P + p];
      }
    } else {
      for (int i = 0; i < R * N; ++i) io->bprev_out[us * R * N + i] = io->bprev0 ? io->bprev0[us * R * N + i] : 0.0;
      for (int i = 0; i < R * P; ++i) io->xprev_out[us * R * P + i] = io->xprev0 ? io->xprev0[us * R * P + i] : 0.0;
    }
  }
  free(Hs); free(u_prev); free(u_cur); free(a); free(Phi);
}

/* ------------------------------------------------------------------------- */
/* real RoPE form                                                              */
/* ------------------------------------------------------------------------- */
/* rotate one pair (v0, v1) by -phi */
static void rot_neg(double phi, double v0, double v1, double* o0, double* o1) {
  *o0 = cos(phi) * v0 + sin(phi) * v1;
  *o1 = -sin(phi) * v0 + cos(phi) * v1;
}

static void unit_rope(const m3o_dims* d, const m3o_io* io, int b, int h) {
  const int L = d->seqlen, P = d->headdim, N = d->dstate, R = d->rank, K = N / 2;
  const double Dh = io->D ? io->D[h] : 0.0;
  double* hs = calloc((size_t)N * P, sizeof(double));
  double* u_prev = calloc((size_t)N * P, sizeof(double));
  double* u_cur = calloc((size_t)N * P, sizeof(double));
  double* Br = calloc((size_t)R * N, sizeof(double));
  double* Cr = calloc((size_t)R * N, sizeof(double));
  double* Phi = calloc((size_t)K, sizeof(double));
  const size_t us = ix_state(d, b, h);

  if (io->angle0)
    for (int k = 0; k < K; ++k) Phi[k] = io->angle0[us * K + k];
  if (io->h0) memcpy(hs, io->h0 + us * N * P, sizeof(double) * N * P);
  if (io->bprev0 && io->xprev0)
    for (int n = 0; n < N; ++n)
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int r = 0; r < R; ++r) s += io->bprev0[(us * R + r) * N + n] * io->xprev0[(us * R + r) * P + p];
        u_prev[n * P + p] = s;
      }

  for (int t = 0; t < L; ++t) {
    const size_t it = ix_tok(d, b, t, h);
    const double dt = io->dt[it], lam = io->lam[it];
    const double* x = io->x + it * R * P;
    for (int k = 0; k < K; ++k) Phi[k] += dt * io->theta[it * K + k];
    for (int r = 0; r < R; ++r)
      for (int k = 0; k < K; ++k) {
        const double* Bt = io->B + ix_bc(d, b, t, h) * R * N + r * N;
        const double* Ct = io->C + ix_bc(d, b, t, h) * R * N + r * N;
        rot_neg(Phi[k], Bt[2 * k], Bt[2 * k + 1], &Br[r * N + 2 * k], &Br[r * N + 2 * k + 1]);
        rot_neg(Phi[k], Ct[2 * k], Ct[2 * k + 1], &Cr[r * N + 2 * k], &Cr[r * N + 2 * k + 1]);
      }
    const double alpha = exp(dt * decay_rate(io, it, h));
    const double beta = (1.0 - lam) * dt * alpha;
    const double gamma = lam * dt;
    for (int n = 0; n < N; ++n)
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int r = 0; r < R; ++r) s += Br[r * N + n] * x[r * P + p];
        u_cur[n * P + p] = s;
        hs[n * P + p] = alpha * hs[n * P + p] + beta * u_prev[n * P + p] + gamma * s;
      }
    if (io->y)
      for (int r = 0; r < R; ++r)
        for (int p = 0; p < P; ++p) {
          double s = 0;
          for (int n = 0; n < N; ++n) s += Cr[r * N + n] * hs[n * P + p];
          io->y[it * R * P + r * P + p] = s + Dh * x[r * P + p];
        }
    double* tmp = u_prev;
    u_prev = u_cur;
    u_cur = tmp;
  }
  if (io->h_out) memcpy(io->h_out + us * N * P, hs, sizeof(double) * N * P);
  if (io->angle_out)
    for (int k = 0; k < K; ++k) io->angle_out[us * K + k] = Phi[k];
  if (io->bprev_out && io->xprev_out && L > 0) {
    const size_t il = ix_tok(d, b, L - 1, h);
    memcpy(io->bprev_out + us * R * N, Br, sizeof(double) * R * N);
    memcpy(io->xprev_out + us * R * P, io->x + il * R * P, sizeof(double) * R * P);
  }
  free(hs); free(u_prev); free(u_cur); free(Br); free(Cr); free(Phi);
}

/* ------------------------------------------------------------------------- */
/* quadratic (materialised L x L kernel) form                                  */
/* ------------------------------------------------------------------------- */
/*
 * Unrolling the three-term update gives h_t = sum_{s<=t} K(t,s) u_s
 * + e^{cum_t} hbar_0, where cum_t = sum_{q<=t} dt_q A,
 *   K(t,t)   = lam_t dt_t,
 *   K(t,s<t) = e^{cum_t - cum_s} (lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}),
 *   hbar_0   = h_0 + (1 - lam_1) dt_1 u_0 ,
 * because the lagged term of step s+1 carries e^{dt_{s+1} A} just like the
 * state, so it folds into the weight of column s.  Everything is in the
 * rotated real frame (u_s = sum_r B~_s[r]^T x_s[r]).  Brute force: the full
 * kernel matrix is materialised.
 */
static void unit_quadratic(const m3o_dims* d, const m3o_io* io, int b, int h) {
  const int L = d->seqlen, P = d->headdim, N = d->dstate, R = d->rank, K = N / 2;
  const double Dh = io->D ? io->D[h] : 0.0;
  const size_t us = ix_state(d, b, h);
  double* Br = calloc((size_t)L * R * N + 1, sizeof(double));
  double* Cr = calloc((size_t)L * R * N + 1, sizeof(double));
  double* cum = calloc((size_t)L + 1, sizeof(double));
  double* Km = calloc((size_t)L * L + 1, sizeof(double));
  double* hbar0 = calloc((size_t)N * P, sizeof(double));
  double* Phi = calloc((size_t)K, sizeof(double));

  if (io->angle0)
    for (int k = 0; k < K; ++k) Phi[k] = io->angle0[us * K + k];
  double c = 0;
  for (int t = 0; t < L; ++t) {
    const size_t it = ix_tok(d, b, t, h);
    for (int k = 0; k < K; ++k) Phi[k] += io->dt[it] * io->theta[it * K + k];
    for (int r = 0; r < R; ++r)
      for (int k = 0; k < K; ++k) {
        const double* Bt = io->B + ix_bc(d, b, t, h) * R * N + r * N;
        const double* Ct = io->C + ix_bc(d, b, t, h) * R * N + r * N;
        rot_neg(Phi[k], Bt[2 * k], Bt[2 * k + 1], &Br[(t * R + r) * N + 2 * k], &Br[(t * R + r) * N + 2 * k + 1]);
        rot_neg(Phi[k], Ct[2 * k], Ct[2 * k + 1], &Cr[(t * R + r) * N + 2 * k], &Cr[(t * R + r) * N + 2 * k + 1]);
      }
    c += io->dt[it] * decay_rate(io, it, h);
    cum[t] = c;
  }
  for (int t = 0; t < L; ++t)
    for (int s = 0; s <= t; ++s) {
      const size_t is = ix_tok(d, b, s, h);
      if (s == t) {
        Km[t * L + s] = io->lam[is] * io->dt[is];
      } else {
        const size_t in = ix_tok(d, b, s + 1, h);
        double w = io->lam[is] * io->dt[is] + (1.0 - io->lam[in]) * io->dt[in];
        Km[t * L + s] = exp(cum[t] - cum[s]) * w;
      }
    }
  if (io->h0) memcpy(hbar0, io->h0 + us * N * P, sizeof(double) * N * P);
  if (io->bprev0 && io->xprev0 && L > 0) {
    const size_t i1 = ix_tok(d, b, 0, h);
    const double mu1 = (1.0 - io->lam[i1]) * io->dt[i1];
    for (int n = 0; n < N; ++n)
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int r = 0; r < R; ++r) s += io->bprev0[(us * R + r) * N + n] * io->xprev0[(us * R + r) * P + p];
        hbar0[n * P + p] += mu1 * s;
      }
  }
  for (int t = 0; t < L; ++t) {
    const size_t it = ix_tok(d, b, t, h);
    for (int r = 0; r < R; ++r)
      for (int p = 0; p < P; ++p) {
        double acc = 0;
        for (int s = 0; s <= t; ++s) {
          const size_t is = ix_tok(d, b, s, h);
          for (int r2 = 0; r2 < R; ++r2) {
            double score = 0;
            for (int n = 0; n < N; ++n) score += Cr[(t * R + r) * N + n] * Br[(s * R + r2) * N + n];
            acc += Km[t * L + s] * score * io->x[is * R * P + r2 * P + p];
          }
        }
        double carry = 0;
        for (int n = 0; n < N; ++n) carry += Cr[(t * R + r) * N + n] * hbar0[n * P + p];
        acc += exp(cum[t]) * carry;
        io->y[it * R * P + r * P + p] = acc + Dh * io->x[it * R * P + r * P + p];
      }
  }
  free(Br); free(Cr); free(cum); free(Km); free(hbar0); free(Phi);
}

/* ------------------------------------------------------------------------- */
/* threading over independent (batch, head) units                             */
/* ------------------------------------------------------------------------- */
typedef void (*unit_fn)(const m3o_dims*, const m3o_io*, int, int);
typedef struct {
  const m3o_dims* d;
  const m3o_io* io;
  unit_fn fn;
  int first, step, count;
} worker_arg;

static void* worker(void* p) {
  worker_arg* w = (worker_arg*)p;
  for (int u = w->first; u < w->count; u += w->step) w->fn(w->d, w->io, u / w->d->nheads, u % w->d->nheads);
  return NULL;
}

static int run_units(const m3o_dims* d, const m3o_io* io, unit_fn fn, int nthreads, const int* units,
                     int nunits) {
  if (!d || !io || d->batch < 0 || d->seqlen < 0 || d->nheads <= 0 || d->headdim <= 0 || d->dstate <= 0 ||
      (d->dstate & 1) || d->rank <= 0)
    return -1;
  if (units) { /* explicit subset of (b*H + h) units, serial */
    for (int i = 0; i < nunits; ++i) fn(d, io, units[i] / d->nheads, units[i] % d->nheads);
    return 0;
  }
  const int total = d->batch * d->nheads;
  if (nthreads <= 1 || total <= 1) {
    for (int u = 0; u < total; ++u) fn(d, io, u / d->nheads, u % d->nheads);
    return 0;
  }
  if (nthreads > total) nthreads = total;
  pthread_t* th = malloc(sizeof(pthread_t) * nthreads);
  worker_arg* wa = malloc(sizeof(worker_arg) * nthreads);
  for (int i = 0; i < nthreads; ++i) {
    wa[i] = (worker_arg){d, io, fn, i, nthreads, total};
    pthread_create(&th[i], NULL, worker, &wa[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  free(th);
  free(wa);
  return 0;
}

/* units: optional list of flattened (b*H + h) indices to compute (NULL = all) */
int m3o_scan_complex(const m3o_dims* d, const m3o_io* io, int nthreads, const int* units, int nunits) {
  return run_units(d, io, unit_complex, nthreads, units, nunits);
}
int m3o_scan_rope(const m3o_dims* d, const m3o_io* io, int nthreads, const int* units, int nunits) {
  return run_units(d, io, unit_rope, nthreads, units, nunits);
}
int m3o_scan_quadratic(const m3o_dims* d, const m3o_io* io, int nthreads) {
  if (!io || !io->y) return -1;
  return run_units(d, io, unit_quadratic, nthreads, NULL, 0);
}
/* One decode step = the complex recurrence continued by one token from the
 * given state; d->seqlen must be 1. */
int m3o_decode_step(const m3o_dims* d, const m3o_io* io, int nthreads) {
  if (!d || d->seqlen != 1) return -1;
  return run_units(d, io, unit_complex, nthreads, NULL, 0);
}

/* ------------------------------------------------------------------------- */
/* B/C normalisation: for every row (b, t, h, r) of a raw projection Z
 * [b, L, H, R, N],
 *     out[n] = Z[n] / sqrt(mean_n' Z[n']^2 + eps) * w[h, r, n] + bias[h, r, n],
 * with w = 1 when NULL and bias = 0 when NULL (an all-zero row with eps = 0
 * gives bias: 0/0 is read as 0).  Same page, section 2 (RMS norm
 * of B and C, head-specific bias); the placement of eps inside the square root
 * and of the bias after the weight is the standard RMS-norm form. */
int m3o_bc_norm(const m3o_dims* d, const double* z, const double* w, const double* bias, double eps, double* out) {
  const int N = d->dstate, R = d->rank, H = d->nheads;
  const size_t rows = (size_t)d->batch * d->seqlen * H * R;
  for (size_t row = 0; row < rows; ++row) {
    const int r = (int)(row % R), h = (int)((row / R) % H);
    const double* zr = z + row * N;
    double ms = 0.0;
    for (int n = 0; n < N; ++n) ms += zr[n] * zr[n];
    ms /= N;
    /* an all-zero row with eps = 0 is 0/0; it normalises to 0 (then the bias) */
    const double inv = (ms + eps > 0.0) ? 1.0 / sqrt(ms + eps) : 0.0;
    for (int n = 0; n < N; ++n) {
      const size_t p = ((size_t)h * R + r) * N + n;
      out[row * N + n] = zr[n] * inv * (w ? w[p] : 1.0) + (bias ? bias[p] : 0.0);
    }
  }
  return 0;
}

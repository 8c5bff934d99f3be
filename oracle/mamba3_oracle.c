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
 * from a state; m3o_scan_rope_bwd, the gradients of the prefill by reverse-mode
 * differentiation of the RoPE form (the pages give no gradient formulas; it is
 * pinned against finite differences of m3o_scan_complex); and m3o_bc_norm, the RMS normalisation of raw B or C
 * projections over the state dimension with a per-(head, rank) weight and bias
 * (same page, section 2: "BC norm" and head-specific B/C bias), which the
 * recurrence then consumes; and m3o_gated_norm, the output side (grouped RMS
 * norm ahead of the silu gate, same page, section 2).
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
  const struct m3o_grad* grad; /* the backward pass's gradients (m3o_scan_rope_bwd only) */
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
/* backward: reverse-mode gradient of the RoPE-form recurrence                 */
/* ------------------------------------------------------------------------- */
/*
 * The pages give no gradient formulas; this is the chain rule applied to
 * unit_rope's steps, token by token from the last to the first, with the
 * forward states h_t kept from a first pass (gh = dL/dh_t, gu = dL/du_t):
 *   y_t = C~_t^T h_t + D x_t      gh_t += C~_t dy_t,  dC~_t[r] = h_t dy_t[r],  dD += <dy_t, x_t>
 *   h_t = alpha_t h_{t-1} + beta_t u_{t-1} + gamma_t u_t
 *                                 d alpha_t = <gh_t, h_{t-1}>, d beta_t = <gh_t, u_{t-1}>,
 *                                 d gamma_t = <gh_t, u_t>, gu_t += gamma_t gh_t,
 *                                 gu_{t-1} += beta_t gh_t, gh_{t-1} = alpha_t gh_t
 *   u_t = sum_r B~_t[r] x_t[r]^T  dB~_t[r] = gu_t x_t[r],  dx_t[r] += gu_t^T B~_t[r]
 *   alpha = exp(dt a), beta = (1 - lam) dt alpha, gamma = lam dt    (into dt, lam, a)
 *   (B~0, B~1) = rot(-Phi)(B0, B1) dB = rot(+Phi) dB~,  dPhi += dB~0 B~1 - dB~1 B~0  (B and C)
 *   Phi_t = Phi_{t-1} + dt_t theta_t
 *                                 S_t = d angle_out + sum_{s >= t} dPhi_s,
 *                                 dtheta_t = dt_t S_t,  ddt_t += <theta_t, S_t>
 * The exported state (h_{L-1}, B~_{L-1}, x_{L-1}, Phi_{L-1}) adds its gradients
 * at t = L - 1; those of the initial state (h_0, B~_0, x_0, Phi_0) come out after
 * t = 0.  dB and dC are written per head (a caller with grouped B, C sums them
 * over each group); dA and dD per (batch, head), or dA per token with A_t.
 */
typedef struct m3o_grad {
  const double* dy;                                              /* [b, L, H, R, P] */
  const double *dh_out, *dbprev_out, *dxprev_out, *dangle_out;   /* each NULL = zero */
  double* dx;                                                    /* [b, L, H, R, P] */
  double *dB, *dC;                                               /* per head [b, L, H, R, N] */
  double *dtheta, *ddt, *dlam;                                   /* [b, L, H, N/2], [b, L, H], [b, L, H] */
  double *dA, *dD;                                               /* [b, H] ([b, L, H] for dA with A_t) */
  double *dh0, *dbprev0, *dxprev0, *dangle0;                     /* each NULL = not wanted */
} m3o_grad;

/* u = sum_r Bt[r] x[r]^T */
static void outer_sum(int N, int P, int R, const double* Bt, const double* x, double* u) {
  for (int n = 0; n < N; ++n)
    for (int p = 0; p < P; ++p) {
      double s = 0;
      for (int r = 0; r < R; ++r) s += Bt[r * N + n] * x[r * P + p];
      u[n * P + p] = s;
    }
}

static double dot(const double* a, const double* b, size_t n) {
  double s = 0;
  for (size_t i = 0; i < n; ++i) s += a[i] * b[i];
  return s;
}

static void unit_rope_bwd(const m3o_dims* d, const m3o_io* io, int b, int h) {
  const m3o_grad* g = io->grad;
  const int L = d->seqlen, P = d->headdim, N = d->dstate, R = d->rank, K = N / 2;
  const size_t NP = (size_t)N * P;
  const double Dh = io->D ? io->D[h] : 0.0;
  const size_t us = ix_state(d, b, h);
  double* Hs = calloc((size_t)(L + 1) * NP, sizeof(double)); /* Hs[t + 1] = h_t, Hs[0] = h_{-1} */
  double* Bt = calloc((size_t)(L > 0 ? L : 1) * R * N, sizeof(double));
  double* Ct = calloc((size_t)(L > 0 ? L : 1) * R * N, sizeof(double));
  double* Ph = calloc((size_t)(L > 0 ? L : 1) * K, sizeof(double));
  double* Phi = calloc((size_t)K, sizeof(double));
  double* u0 = calloc(NP, sizeof(double)); /* u_{-1} = B~_0^T x_0 of the initial state */
  double* u_prev = calloc(NP, sizeof(double));
  double* u_cur = calloc(NP, sizeof(double));

  /* ---- forward: unit_rope's steps, keeping h_t, B~_t, C~_t, Phi_t ---- */
  if (io->angle0)
    for (int k = 0; k < K; ++k) Phi[k] = io->angle0[us * K + k];
  if (io->h0) memcpy(Hs, io->h0 + us * NP, sizeof(double) * NP);
  if (io->bprev0 && io->xprev0) outer_sum(N, P, R, io->bprev0 + us * R * N, io->xprev0 + us * R * P, u0);
  memcpy(u_prev, u0, sizeof(double) * NP);
  for (int t = 0; t < L; ++t) {
    const size_t it = ix_tok(d, b, t, h), ib = ix_bc(d, b, t, h);
    const double dt = io->dt[it], lam = io->lam[it];
    for (int k = 0; k < K; ++k) {
      Phi[k] += dt * io->theta[it * K + k];
      Ph[(size_t)t * K + k] = Phi[k];
    }
    for (int r = 0; r < R; ++r)
      for (int k = 0; k < K; ++k) {
        const double* Bv = io->B + ib * R * N + r * N;
        const double* Cv = io->C + ib * R * N + r * N;
        double* bo = Bt + ((size_t)t * R + r) * N;
        double* co = Ct + ((size_t)t * R + r) * N;
        rot_neg(Phi[k], Bv[2 * k], Bv[2 * k + 1], &bo[2 * k], &bo[2 * k + 1]);
        rot_neg(Phi[k], Cv[2 * k], Cv[2 * k + 1], &co[2 * k], &co[2 * k + 1]);
      }
    const double alpha = exp(dt * decay_rate(io, it, h));
    const double beta = (1.0 - lam) * dt * alpha, gamma = lam * dt;
    outer_sum(N, P, R, Bt + (size_t)t * R * N, io->x + it * R * P, u_cur);
    const double* hp = Hs + (size_t)t * NP;
    double* hn = Hs + (size_t)(t + 1) * NP;
    for (size_t i = 0; i < NP; ++i) hn[i] = alpha * hp[i] + beta * u_prev[i] + gamma * u_cur[i];
    double* tmp = u_prev;
    u_prev = u_cur;
    u_cur = tmp;
  }

  /* ---- backward ---- */
  double* gh = calloc(NP, sizeof(double));
  double* gu = calloc(NP, sizeof(double));   /* dL/du_t, collecting beta_{t+1} gh_{t+1} first */
  double* gup = calloc(NP, sizeof(double));  /* dL/du_{t-1} */
  double* S = calloc((size_t)K, sizeof(double));
  double* dBt = calloc((size_t)R * N, sizeof(double));
  double* dCt = calloc((size_t)R * N, sizeof(double));
  double* dPhi = calloc((size_t)K, sizeof(double));
  if (g->dh_out) memcpy(gh, g->dh_out + us * NP, sizeof(double) * NP);
  if (g->dangle_out)
    for (int k = 0; k < K; ++k) S[k] = g->dangle_out[us * K + k];
  double dA_unit = 0.0, dD_unit = 0.0;
  for (int t = L - 1; t >= 0; --t) {
    const size_t it = ix_tok(d, b, t, h);
    const double* x = io->x + it * R * P;
    const double* dy = g->dy + it * R * P;
    double* dx = g->dx + it * R * P;
    const double* Bv = Bt + (size_t)t * R * N;
    const double* Cv = Ct + (size_t)t * R * N;
    const double* h_t = Hs + (size_t)(t + 1) * NP;
    const double* h_p = Hs + (size_t)t * NP;
    const double dt = io->dt[it], lam = io->lam[it], a = decay_rate(io, it, h);
    const double alpha = exp(dt * a), beta = (1.0 - lam) * dt * alpha, gamma = lam * dt;
    /* u_t and u_{t-1} again (cheaper to recompute than to keep) */
    outer_sum(N, P, R, Bv, x, u_cur);
    if (t > 0)
      outer_sum(N, P, R, Bt + (size_t)(t - 1) * R * N, io->x + ix_tok(d, b, t - 1, h) * R * P, u_prev);
    else
      memcpy(u_prev, u0, sizeof(double) * NP);
    /* readout */
    for (int n = 0; n < N; ++n)
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int r = 0; r < R; ++r) s += Cv[r * N + n] * dy[r * P + p];
        gh[n * P + p] += s;
      }
    for (int r = 0; r < R; ++r)
      for (int n = 0; n < N; ++n) {
        double s = 0;
        for (int p = 0; p < P; ++p) s += h_t[n * P + p] * dy[r * P + p];
        dCt[r * N + n] = s;
      }
    for (int i = 0; i < R * P; ++i) {
      dx[i] = Dh * dy[i];
      dD_unit += dy[i] * x[i];
    }
    /* three-term update */
    const double d_alpha = dot(gh, h_p, NP), d_beta = dot(gh, u_prev, NP), d_gamma = dot(gh, u_cur, NP);
    for (size_t i = 0; i < NP; ++i) {
      gu[i] += gamma * gh[i];
      gup[i] = beta * gh[i];
    }
    /* u_t = sum_r B~_t[r] x_t[r]^T */
    for (int r = 0; r < R; ++r) {
      for (int n = 0; n < N; ++n) {
        double s = 0;
        for (int p = 0; p < P; ++p) s += gu[n * P + p] * x[r * P + p];
        dBt[r * N + n] = s;
      }
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int n = 0; n < N; ++n) s += gu[n * P + p] * Bv[r * N + n];
        dx[r * P + p] += s;
      }
    }
    if (t == L - 1) { /* the exported B~_{L-1} and x_{L-1} */
      if (g->dbprev_out)
        for (int i = 0; i < R * N; ++i) dBt[i] += g->dbprev_out[us * R * N + i];
      if (g->dxprev_out)
        for (int i = 0; i < R * P; ++i) dx[i] += g->dxprev_out[us * R * P + i];
    }
    /* scalars: alpha = exp(dt a), beta = (1 - lam) dt alpha, gamma = lam dt */
    const double d_alpha_all = d_alpha + d_beta * (1.0 - lam) * dt;
    double ddt = d_alpha_all * alpha * a + d_beta * (1.0 - lam) * alpha + d_gamma * lam;
    g->dlam[it] = -d_beta * dt * alpha + d_gamma * dt;
    const double da = d_alpha_all * alpha * dt;
    if (io->A_t)
      g->dA[it] = da;
    else
      dA_unit += da;
    /* rotation back, and the angle's share */
    for (int k = 0; k < K; ++k) dPhi[k] = 0.0;
    for (int r = 0; r < R; ++r)
      for (int k = 0; k < K; ++k) {
        const double ph = Ph[(size_t)t * K + k], c = cos(ph), sn = sin(ph);
        const double* db = dBt + r * N + 2 * k;
        const double* dc = dCt + r * N + 2 * k;
        const double* bt = Bv + r * N + 2 * k;
        const double* ct = Cv + r * N + 2 * k;
        double* oB = g->dB + it * R * N + r * N + 2 * k;
        double* oC = g->dC + it * R * N + r * N + 2 * k;
        oB[0] = c * db[0] - sn * db[1];
        oB[1] = sn * db[0] + c * db[1];
        oC[0] = c * dc[0] - sn * dc[1];
        oC[1] = sn * dc[0] + c * dc[1];
        dPhi[k] += db[0] * bt[1] - db[1] * bt[0] + dc[0] * ct[1] - dc[1] * ct[0];
      }
    for (int k = 0; k < K; ++k) {
      S[k] += dPhi[k];
      g->dtheta[it * K + k] = dt * S[k];
      ddt += io->theta[it * K + k] * S[k];
    }
    g->ddt[it] = ddt;
    for (size_t i = 0; i < NP; ++i) gh[i] *= alpha;
    double* tmp = gu;
    gu = gup;
    gup = tmp;
  }
  /* initial state: h_{-1} = h_0, u_{-1} = B~_0^T x_0, Phi_{-1} = Phi_0 */
  if (g->dh0) memcpy(g->dh0 + us * NP, gh, sizeof(double) * NP);
  if (g->dbprev0 && g->dxprev0) {
    const double* b0 = io->bprev0 ? io->bprev0 + us * R * N : NULL;
    const double* x0 = io->xprev0 ? io->xprev0 + us * R * P : NULL;
    for (int r = 0; r < R; ++r) {
      for (int n = 0; n < N; ++n) {
        double s = 0;
        for (int p = 0; p < P; ++p) s += gu[n * P + p] * (x0 ? x0[r * P + p] : 0.0);
        g->dbprev0[(us * R + r) * N + n] = s;
      }
      for (int p = 0; p < P; ++p) {
        double s = 0;
        for (int n = 0; n < N; ++n) s += gu[n * P + p] * (b0 ? b0[r * N + n] : 0.0);
        g->dxprev0[(us * R + r) * P + p] = s;
      }
    }
  }
  if (g->dangle0)
    for (int k = 0; k < K; ++k) g->dangle0[us * K + k] = S[k];
  if (!io->A_t) g->dA[us] = dA_unit;
  g->dD[us] = dD_unit;
  free(Hs); free(Bt); free(Ct); free(Ph); free(Phi); free(u0); free(u_prev); free(u_cur);
  free(gh); free(gu); free(gup); free(S); free(dBt); free(dCt); free(dPhi);
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
/* Gradients of the prefill (see unit_rope_bwd); io->grad must be set. */
int m3o_scan_rope_bwd(const m3o_dims* d, const m3o_io* io, int nthreads) {
  if (!io || !io->grad || !io->grad->dy || !io->grad->dx || !io->grad->dB || !io->grad->dC ||
      !io->grad->dtheta || !io->grad->ddt || !io->grad->dlam || !io->grad->dA || !io->grad->dD)
    return -1;
  return run_units(d, io, unit_rope_bwd, nthreads, NULL, 0);
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

/* ------------------------------------------------------------------------- */
/* Output side: pre-gate grouped RMS norm and the gate                         */
/* ------------------------------------------------------------------------- */
/*
 * Same page, section 2: hybrids add a grouped RMS norm in front of the output
 * gate.  For every token (b, t) and norm group g of H / G consecutive heads,
 * over the group's channels c = (h, r, p):
 *     out[c] = y[c] / sqrt(mean_c y[c]^2 + eps) * w[h, r, p] * silu(z[c]),
 * silu(z) = z / (1 + e^{-z}) (the gate of the Mamba line; the pages do not name
 * it).  y, z, out [b, L, H, R, P]; w [H, R, P] or NULL (weight 1).  An all-zero
 * group with eps = 0 gives 0.
 */
int m3o_gated_norm(const m3o_dims* d, int groups, const double* y, const double* z, const double* w, double eps,
                   double* out) {
  const int H = d->nheads, R = d->rank, P = d->headdim;
  if (groups <= 0 || H % groups != 0) return -1;
  const size_t hpg = (size_t)(H / groups), gsize = hpg * R * P;
  const size_t rows = (size_t)d->batch * d->seqlen * groups; /* (b, t, g) in order */
  for (size_t row = 0; row < rows; ++row) {
    const size_t g = row % groups;
    const double* yr = y + row * gsize;
    double ms = 0.0;
    for (size_t c = 0; c < gsize; ++c) ms += yr[c] * yr[c];
    ms /= (double)gsize;
    const double inv = (ms + eps) > 0.0 ? 1.0 / sqrt(ms + eps) : 0.0;
    for (size_t c = 0; c < gsize; ++c) {
      const size_t h = g * hpg + c / ((size_t)R * P), rp = c % ((size_t)R * P);
      const double wt = w ? w[h * R * P + rp] : 1.0;
      const double zv = z[row * gsize + c];
      out[row * gsize + c] = yr[c] * inv * wt * (zv / (1.0 + exp(-zv)));
    }
  }
  return 0;
}

/* ------------------------------------------------------------------------- */
/* MIMO rank-R projections around the recurrence.
 *
 * Same page, section 1.3: MIMO raises the rank of the input and output
 * projections to R, so that x_t is P x R (and B_t N x R) and the state update
 * becomes a matrix product.  The page prints no weights; the plainest reading
 * taken here is one dense matrix per head on each side of the recurrence:
 *   up:    x[b,t,h,r,p] = sum_q Wx[h, r P + p, q] u[b,t,h,q]
 *          u [b, L, H, P],  Wx [H, R P, P],  x [b, L, H, R, P]
 *   down:  o[b,t,h,p]   = sum_r sum_q Wy[h, p, r P + q] y[b,t,h,r,q]
 *          y [b, L, H, R, P],  Wy [H, P, R P],  o [b, L, H, P]
 * (R = 1 with identity weights leaves u and y unchanged: SISO.)  Plain loops,
 * fp64; d->dstate is ignored.
 */
int m3o_mimo_up(const m3o_dims* d, const double* u, const double* Wx, double* x) {
  const int H = d->nheads, R = d->rank, P = d->headdim;
  const size_t tokens = (size_t)d->batch * d->seqlen;
  for (size_t t = 0; t < tokens; ++t)
    for (int h = 0; h < H; ++h) {
      const double* ut = u + (t * H + h) * P;
      const double* W = Wx + (size_t)h * R * P * P;
      double* xt = x + (t * H + h) * (size_t)R * P;
      for (int rp = 0; rp < R * P; ++rp) {
        double acc = 0.0;
        for (int q = 0; q < P; ++q) acc += W[(size_t)rp * P + q] * ut[q];
        xt[rp] = acc;
      }
    }
  return 0;
}

int m3o_mimo_down(const m3o_dims* d, const double* y, const double* Wy, double* o) {
  const int H = d->nheads, R = d->rank, P = d->headdim;
  const size_t tokens = (size_t)d->batch * d->seqlen;
  for (size_t t = 0; t < tokens; ++t)
    for (int h = 0; h < H; ++h) {
      const double* yt = y + (t * H + h) * (size_t)R * P;
      const double* W = Wy + (size_t)h * P * R * P;
      double* ot = o + (t * H + h) * P;
      for (int p = 0; p < P; ++p) {
        double acc = 0.0;
        for (int rq = 0; rq < R * P; ++rq) acc += W[(size_t)p * R * P + rq] * yt[rq];
        ot[p] = acc;
      }
    }
  return 0;
}

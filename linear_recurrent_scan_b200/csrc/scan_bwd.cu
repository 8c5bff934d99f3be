// Backward pass of the chunked prefill on the SIMT pipes (fp32 FMA).
//
// The pages (the Mamba-3 articles) give no gradient formulas; these follow from
// the chain rule on the chunked form of the prefill (see scan_simt.cu): with
// hbar the carried state, u_j = sum_r B~_j[r]^T x_j[r], cum the chunk-local sum
// of the log-decays a = dt A, and the kernel
//   K(t, t) = gamma_t,   K(t, j < t) = e^{cum_t - cum_j} w_j,
// a chunk computes
//   y_t      = C~_t^T (e^{cum_t} hbar_in + sum_{j<=t} K(t, j) u_j) + D x_t
//   hbar_out = e^{cum_end} hbar_in + sum_j e^{cum_end - cum_j} w_j u_j .
// Given G = dL/dhbar_out (from the later chunk, or the exported state's
// gradient at the end), and writing P1 = C~ B~^T, P2 = dY X^T (rows x rows),
// S = K o P1, W = K o P2 (the kernel spread over the rank rows of each token):
//   dC~ = diag(e^{cum}) dY hbar_in^T + W B~
//   dB~ = diag(w e^{cum_end - cum}) X G^T + W^T C~
//   dX  = diag(w e^{cum_end - cum}) B~ G + S^T dY + D dY
//   dL/dhbar_in = e^{cum_end} G + C~^T diag(e^{cum}) dY
// and, with Z(t, j) = sum over the two tokens' rank rows of P1 o P2,
//   d gamma_t = Z(t, t)
//   d w_j     = e^{cum_end - cum_j} <u_j, G> + sum_{t > j} e^{cum_t - cum_j} Z(t, j)
//   d a_i     = sum of every path that crosses token i's decay: from hbar_in
//               or u_j (j < i) to y_t (t >= i) or to hbar_out.
// The lagged weight (1 - lam_{j+1}) dt_{j+1} inside w_j belongs to the next
// token, which for a chunk's last token sits in the chunk processed before it
// (the sweep runs backwards); its dt and lam gradients wait one chunk.  The
// rotation goes back with rot(+Phi); dPhi = dB~_0 B~_1 - dB~_1 B~_0 (and C)
// summed from the end gives dtheta = dt S and the angle's share of ddt.
//
// One CTA per (batch, head).  A first pass runs the chunk recurrence forward
// and stores hbar and Phi at every chunk start in the workspace; the second
// pass walks the chunks backwards with dL/dhbar in shared memory.
#include "common.cuh"
#include "internal.h"

namespace m3 {
namespace {

constexpr int kThreads = 512;
constexpr int kRows = 32;  // M = Q * R rows per chunk
constexpr int kNScal = 15;  // per-token scalar arrays of the backward chunk

struct BwdLayout {
  int M, Q;
  size_t off_hb, off_G, off_B, off_C, off_dB, off_dC, off_X, off_dY, off_S, off_W, off_Q, off_phi, off_th, off_T,
      off_sc, off_ang, off_misc, total;
};

BwdLayout bwd_layout(int P, int N, int R) {
  BwdLayout l;
  l.Q = kRows / R;
  l.M = l.Q * R;
  const int K = N / 2;
  size_t o = 0;
  auto take = [&](size_t n) {
    size_t r = o;
    o += (n + 3) & ~size_t(3);
    return r;
  };
  // rows of hbar, G, X, dY padded to P + 1 floats and of B~, C~ to N + 1, so that a
  // warp walking down a column (one lane per row) hits 32 different banks
  l.off_hb = take((size_t)N * (P + 1));
  l.off_G = take((size_t)N * (P + 1));
  l.off_B = take((size_t)l.M * (N + 1));
  l.off_C = take((size_t)l.M * (N + 1));
  l.off_dB = take((size_t)l.M * N);
  l.off_dC = take((size_t)l.M * N);
  l.off_X = take((size_t)l.M * (P + 1));
  l.off_dY = take((size_t)l.M * (P + 1));
  l.off_S = take((size_t)l.M * l.M);
  l.off_W = take((size_t)l.M * l.M);
  l.off_Q = take((size_t)l.M * l.M);
  l.off_phi = take((size_t)l.Q * K);
  l.off_th = take((size_t)l.Q * K);
  l.off_T = take((size_t)l.Q * l.Q);
  l.off_sc = take((size_t)kNScal * (l.Q + 1));
  l.off_ang = take((size_t)2 * K);
  l.off_misc = take(16);
  l.total = o * sizeof(float);
  return l;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide sum of one float per thread, added to *dst (shared memory).
__device__ __forceinline__ void block_add(float v, float* dst) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) atomicAdd(dst, v);
}

// NT, PT, RT: N, P, R fixed at compile time (inner loops unrolled), or 0 to take
// them from the arguments.
template <typename T, int NT, int PT, int RT>
__global__ void __launch_bounds__(kThreads, 1) scan_bwd_kernel(BwdArgs g, BwdLayout lay) {
  extern __shared__ float sm[];
  __shared__ int s_pend_t;  // first token of the chunk processed last, its lagged-weight share pending
  __shared__ float s_erow[kRows];  // e^{cum} of each row's token
  const ScanArgs& a = g.f;
  const int P = PT ? PT : a.P, N = NT ? NT : a.N, R = RT ? RT : a.R;
  const int Q = RT ? kRows / RT : lay.Q, L = a.seqlen, K = N / 2, NP = N * P;
  const int PS = P + 1, NS = N + 1;  // padded row strides (hbar, G, X, dY; B~, C~)
  const int unit = blockIdx.x;
  const int b = unit / a.nheads, hh = unit % a.nheads;
  const int tid = threadIdx.x;
  float* hb = sm + lay.off_hb;     // [N][PS] hbar at the chunk start
  float* G = sm + lay.off_G;       // [N][PS] dL/dhbar at the chunk end
  float* sB = sm + lay.off_B;      // [M][NS] B~
  float* sC = sm + lay.off_C;      // [M][NS] C~
  float* dBt = sm + lay.off_dB;    // [M][N] dL/dB~
  float* dCt = sm + lay.off_dC;    // [M][N] dL/dC~
  float* sX = sm + lay.off_X;      // [M][PS]
  float* sdY = sm + lay.off_dY;    // [M][PS]
  float* sS = sm + lay.off_S;      // [M][M] K o (C~ B~^T)
  float* sW = sm + lay.off_W;      // [M][M] K o (dY X^T)
  float* sQ = sm + lay.off_Q;      // [M][M] (C~ B~^T) o (dY X^T)
  float* phit = sm + lay.off_phi;  // [Q][K] angle of each token of the chunk
  float* sth = sm + lay.off_th;    // [Q][K] theta of the chunk's tokens
  float* sT = sm + lay.off_T;      // [Q][Q] e^{cum_t - cum_j} Z(t, j) for t > j
  const int QS = Q + 1;
  float* sc = sm + lay.off_sc;
  float *s_dt = sc, *s_lam = sc + QS, *s_cum = sc + 2 * QS, *s_gam = sc + 3 * QS, *s_w = sc + 4 * QS;
  float *s_zin = sc + 5 * QS, *s_zue = sc + 6 * QS, *s_dg = sc + 7 * QS, *s_cZu = sc + 8 * QS;
  float *s_cT = sc + 9 * QS, *s_rT = sc + 10 * QS, *s_dth = sc + 11 * QS, *s_ecum = sc + 12 * QS;
  float* s_eend = sc + 13 * QS;
  float* s_at = sc + 14 * QS;  // decay rate of each token (A_t, or A of the head)
  float* phi = sm + lay.off_ang;  // [K] running angle (pass 1) or angle at the chunk start (pass 2)
  float* Sang = phi + K;          // [K] dL/dPhi summed from the end
  float* misc = sm + lay.off_misc;  // [0] <hbar_in, G>, [1] dD, [2] initial lagged share, [3..4] pending ddt, dlam

  const T* X = static_cast<const T*>(a.x);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  const T* TH = static_cast<const T*>(a.theta);
  const T* DT = static_cast<const T*>(a.dt);
  const T* LM = static_cast<const T*>(a.lam);
  const T* DY = static_cast<const T*>(g.dy);
  T* dXg = static_cast<T*>(g.dx);
  T* dBg = static_cast<T*>(g.dB);
  T* dCg = static_cast<T*>(g.dC);
  T* dTHg = static_cast<T*>(g.dtheta);
  T* dDTg = static_cast<T*>(g.ddt);
  T* dLMg = static_cast<T*>(g.dlam);
  const T* AT = static_cast<const T*>(a.A_t);  // time-varying decay [b, L, H], or null
  T* dATg = static_cast<T*>(g.dA_t);
  const float Ah = AT ? 0.f : a.A[hh];
  const float Dh = a.D ? a.D[hh] : 0.f;
  const size_t us = (size_t)unit;
  auto tok = [&](int t) { return ((size_t)b * L + t) * a.nheads + hh; };
  const int gh = hh / (a.nheads / a.ngroups);  // B, C row of this head
  auto tok_bc = [&](int t) { return ((size_t)b * L + t) * a.ngroups + gh; };
  const bool has_init = a.h0 != nullptr;

  if (L == 0) {  // the exported state is the initial state: its gradients pass through
    if (g.dh0) {
      for (int i = tid; i < NP; i += kThreads) g.dh0[us * NP + i] = g.dh_out ? g.dh_out[us * NP + i] : 0.f;
      for (int i = tid; i < R * N; i += kThreads)
        g.dbprev0[us * R * N + i] = g.dbprev_out ? g.dbprev_out[us * R * N + i] : 0.f;
      for (int i = tid; i < R * P; i += kThreads)
        g.dxprev0[us * R * P + i] = g.dxprev_out ? g.dxprev_out[us * R * P + i] : 0.f;
      for (int k = tid; k < K; k += kThreads) g.dangle0[us * K + k] = g.dangle_out ? g.dangle_out[us * K + k] : 0.f;
    }
    return;
  }
  const int nchunks = (L + Q - 1) / Q;
  float* ck = g.ckpt + us * (size_t)nchunks * (NP + K);

  // scalars of tokens t0 .. t0 + q (the token after the chunk: dt 0, lam 1 past the end) and the rows
  auto load_chunk = [&](int t0, int q, bool backward) {
    for (int i = tid; i <= q; i += kThreads) {
      if (t0 + i < L) {
        s_dt[i] = ld1(DT + tok(t0 + i));
        s_lam[i] = ld1(LM + tok(t0 + i));
      } else {
        s_dt[i] = 0.f;
        s_lam[i] = 1.f;
      }
    }
    const int M = q * R;
    for (int i = tid; i < M * N; i += kThreads) {
      const int m = i / N, n = i % N;
      const size_t gi = tok_bc(t0 + m / R) * R * N + (size_t)(m % R) * N + n;
      sB[m * NS + n] = ld1(Bg + gi);
      if (backward) sC[m * NS + n] = ld1(Cg + gi);
    }
    for (int i = tid; i < M * P; i += kThreads) {
      const int m = i / P, p = i % P;
      const size_t gi = tok(t0 + m / R) * R * P + (size_t)(m % R) * P + p;
      sX[m * PS + p] = ld1(X + gi);
      if (backward) sdY[m * PS + p] = ld1(DY + gi);
    }
    for (int i = tid; i < q * K; i += kThreads) sth[i] = ld1(TH + tok(t0 + i / K) * K + i % K);
    for (int i = tid; i < q; i += kThreads) s_at[i] = AT ? ld1(AT + tok(t0 + i)) : Ah;
  };
  // decay scan of the chunk (warp 0, one lane per token, q <= 32): cum, gamma, w,
  // e^{cum}, e^{cum_end - cum}
  auto decay_scalars = [&](int q) {
    if (tid < 32) {
      const int i = tid;
      float c = i < q ? s_dt[i] * s_at[i] : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float v = __shfl_up_sync(0xffffffffu, c, o);
        if (i >= o) c += v;
      }
      const float cend = __shfl_sync(0xffffffffu, c, q - 1);
      if (i < q) {
        s_cum[i] = c;
        s_gam[i] = s_lam[i] * s_dt[i];
        s_w[i] = s_gam[i] + (1.f - s_lam[i + 1]) * s_dt[i + 1];
        s_ecum[i] = expf(c);
        s_eend[i] = expf(cend - c);
      }
    }
  };
  // rotate the chunk's B (and C) rows by -Phi, keeping each token's angle; advance phi
  auto rotate_chunk = [&](int t0, int q, bool backward) {
    for (int k = tid; k < K; k += kThreads) {
      float local = 0.f;
      for (int i = 0; i < q; ++i) {
        local += s_dt[i] * sth[i * K + k];
        const float ph = phi[k] + local;
        phit[i * K + k] = ph;
        float sn, cs;
        sincosf(ph, &sn, &cs);
        for (int r = 0; r < R; ++r) {
          float* bb = sB + (i * R + r) * NS + 2 * k;
          const float b0 = bb[0], b1 = bb[1];
          bb[0] = cs * b0 + sn * b1;
          bb[1] = -sn * b0 + cs * b1;
          if (backward) {
            float* cc = sC + (i * R + r) * NS + 2 * k;
            const float c0 = cc[0], c1 = cc[1];
            cc[0] = cs * c0 + sn * c1;
            cc[1] = -sn * c0 + cs * c1;
          }
        }
      }
      phi[k] = wrap_angle(phi[k] + local);
    }
  };

  // St[n][p] = scale St[n][p] + sum_{j < M} f_j A[j][n] Bm[j][p]  (f = 1 when f_row is null).
  // With N, P fixed at compile time a thread keeps N/16 rows x 2 columns in registers.
  auto state_update = [&](float* St, const float* A, const float* Bm, const float* f_row, float scale, int M) {
    if constexpr (NT != 0 && PT == 64 && kThreads == 512) {
      constexpr int NR = NT / 16;
      const int n0 = tid >> 5, p0 = tid & 31;
      float acc[NR][2];
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        acc[i][0] = scale * St[(n0 + 16 * i) * PS + p0];
        acc[i][1] = scale * St[(n0 + 16 * i) * PS + p0 + 32];
      }
#pragma unroll 4
      for (int j = 0; j < M; ++j) {
        const float f = f_row ? f_row[j] : 1.f;
        const float d0 = f * Bm[j * PS + p0], d1 = f * Bm[j * PS + p0 + 32];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const float c = A[j * NS + n0 + 16 * i];
          acc[i][0] += c * d0;
          acc[i][1] += c * d1;
        }
      }
#pragma unroll
      for (int i = 0; i < NR; ++i) {
        St[(n0 + 16 * i) * PS + p0] = acc[i][0];
        St[(n0 + 16 * i) * PS + p0 + 32] = acc[i][1];
      }
    } else {
      for (int i = tid; i < NP; i += kThreads) {
        const int n = i / P, p = i % P;
        float acc = scale * St[n * PS + p];
#pragma unroll 8
        for (int j = 0; j < M; ++j) acc += (f_row ? f_row[j] : 1.f) * A[j * NS + n] * Bm[j * PS + p];
        St[n * PS + p] = acc;
      }
    }
  };

  // ---------------- pass 1: hbar and Phi at every chunk start ----------------
  const float mu1 = (1.f - ld1(LM + tok(0))) * ld1(DT + tok(0));  // weight of the initial lagged term
  for (int i = tid; i < NP; i += kThreads) {
    const int n = i / P, p = i % P;
    float v = 0.f;
    if (has_init) {
      v = a.h0[us * NP + i];
      float u = 0.f;
      for (int r = 0; r < R; ++r) u += a.bprev0[(us * R + r) * N + n] * a.xprev0[(us * R + r) * P + p];
      v += mu1 * u;
    }
    hb[n * PS + p] = v;
  }
  for (int k = tid; k < K; k += kThreads) phi[k] = has_init ? a.angle0[us * K + k] : 0.f;
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * Q, q = min(Q, L - t0), M = q * R;
    float* cp = ck + (size_t)c * (NP + K);
    for (int i = tid; i < NP; i += kThreads) cp[i] = hb[(i / P) * PS + i % P];
    for (int k = tid; k < K; k += kThreads) cp[NP + k] = phi[k];
    load_chunk(t0, q, false);
    __syncthreads();
    decay_scalars(q);
    rotate_chunk(t0, q, false);
    __syncthreads();
    for (int i = tid; i < M * P; i += kThreads) {  // x rows times their weight e^{cum_end - cum} w
      const int m = i / P, p = i % P;
      sX[m * PS + p] *= s_eend[m / R] * s_w[m / R];
    }
    __syncthreads();
    state_update(hb, sB, sX, nullptr, expf(s_cum[q - 1]), M);
    __syncthreads();
  }

  // ---------------- pass 2: chunks from the last to the first ----------------
  for (int i = tid; i < NP; i += kThreads) G[(i / P) * PS + i % P] = g.dh_out ? g.dh_out[us * NP + i] : 0.f;
  for (int k = tid; k < K; k += kThreads) Sang[k] = g.dangle_out ? g.dangle_out[us * K + k] : 0.f;
  if (tid == 0) {
    s_pend_t = -1;
    misc[1] = 0.f;
  }
  float dA_acc = 0.f;  // thread 0
  float dD_acc = 0.f;
  __syncthreads();
  for (int c = nchunks - 1; c >= 0; --c) {
    const int t0 = c * Q, q = min(Q, L - t0), M = q * R;
    const float* cp = ck + (size_t)c * (NP + K);
    for (int i = tid; i < NP; i += kThreads) hb[(i / P) * PS + i % P] = cp[i];
    for (int k = tid; k < K; k += kThreads) phi[k] = cp[NP + k];
    for (int i = tid; i < Q; i += kThreads) {
      s_zin[i] = 0.f;
      s_zue[i] = 0.f;
      s_dth[i] = 0.f;
    }
    if (tid == 0) misc[0] = 0.f;
    load_chunk(t0, q, true);
    __syncthreads();
    decay_scalars(q);
    rotate_chunk(t0, q, true);
    __syncthreads();
    const float ecend = expf(s_cum[q - 1]);

    // (1) row pairs (token of j <= token of m): S = K o P1, W = K o P2, P1 o P2
    for (int m = tid; m < M; m += kThreads) s_erow[m] = s_ecum[m / R];
    for (int i = tid; i < M * M; i += kThreads) {
      const int m = i / M, j = i % M, tm = m / R, tj = j / R;
      float vs = 0.f, vw = 0.f, vq = 0.f;
      if (tj <= tm) {
        float p1 = 0.f, p2 = 0.f;
#pragma unroll 8
        for (int n = 0; n < N; ++n) p1 += sC[m * NS + n] * sB[j * NS + n];
#pragma unroll 8
        for (int p = 0; p < P; ++p) p2 += sdY[m * PS + p] * sX[j * PS + p];
        const float kern = (tj == tm) ? s_gam[tm] : expf(s_cum[tm] - s_cum[tj]) * s_w[tj];
        vs = kern * p1;
        vw = kern * p2;
        vq = p1 * p2;
      }
      sS[i] = vs;
      sW[i] = vw;
      sQ[i] = vq;
    }
    __syncthreads();

    // (2) token pairs: Z(t, j) over the rank rows; its diagonal is d gamma
    for (int i = tid; i < q * q; i += kThreads) {
      const int t = i / q, j = i % q;
      float z = 0.f;
      if (j <= t)
        for (int r = 0; r < R; ++r)
          for (int r2 = 0; r2 < R; ++r2) z += sQ[(t * R + r) * M + j * R + r2];
      if (t == j) s_dg[t] = z;
      sT[t * Q + j] = (j < t) ? expf(s_cum[t] - s_cum[j]) * z : 0.f;
    }
    // (3) dX, and per token the paths hbar_in -> y_t and u_j -> hbar_out
    // (yi = (C~ hbar_in)[m][p] and bg = (B~ G)[m][p] come in from the loops below)
    auto dx_out = [&](int m, int p, float yi, float bg, float& zin_c, float& zue_c) {
      const int t = m / R, r = m % R;
      float sdy = 0.f;
      for (int j = t * R; j < M; ++j) sdy += sS[j * M + m] * sdY[j * PS + p];
      const float dy = sdY[m * PS + p], xv = sX[m * PS + p];
      float dxv = s_w[t] * s_eend[t] * bg + sdy + Dh * dy;
      if (t0 + t == L - 1 && g.dxprev_out) dxv += g.dxprev_out[(us * R + r) * P + p];
      st1(dXg + tok(t0 + t) * R * P + (size_t)r * P + p, dxv);
      zin_c = s_ecum[t] * dy * yi;
      zue_c = s_eend[t] * xv * bg;
      dD_acc += dy * xv;
    };
    if constexpr (NT != 0 && PT == 64 && kThreads == 512) {
      const int m0 = tid >> 5, p0 = tid & 31;  // rows m0, m0 + 16; columns p0, p0 + 32
      float yi[2][2] = {}, bg[2][2] = {};
#pragma unroll 4
      for (int n = 0; n < NT; ++n) {
        const float c0 = sC[m0 * NS + n], c1 = sC[(m0 + 16) * NS + n];
        const float b0 = sB[m0 * NS + n], b1 = sB[(m0 + 16) * NS + n];
        const float h0 = hb[n * PS + p0], h1 = hb[n * PS + p0 + 32];
        const float g0 = G[n * PS + p0], g1 = G[n * PS + p0 + 32];
        yi[0][0] += c0 * h0;
        yi[0][1] += c0 * h1;
        yi[1][0] += c1 * h0;
        yi[1][1] += c1 * h1;
        bg[0][0] += b0 * g0;
        bg[0][1] += b0 * g1;
        bg[1][0] += b1 * g0;
        bg[1][1] += b1 * g1;
      }
      // a warp holds one row (one token): sum its lanes before the shared atomics
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int m = m0 + 16 * a2;
        float zi = 0.f, zu = 0.f;
        if (m < M)
#pragma unroll
          for (int b2 = 0; b2 < 2; ++b2) {
            float ci, cu;
            dx_out(m, p0 + 32 * b2, yi[a2][b2], bg[a2][b2], ci, cu);
            zi += ci;
            zu += cu;
          }
        zi = warp_sum(zi);
        zu = warp_sum(zu);
        if (p0 == 0 && m < M) {
          atomicAdd(&s_zin[m / R], zi);
          atomicAdd(&s_zue[m / R], zu);
        }
      }
    } else {
      for (int i = tid; i < M * P; i += kThreads) {
        const int m = i / P, p = i % P;
        float yi = 0.f, bg = 0.f;
#pragma unroll 8
        for (int n = 0; n < N; ++n) {
          yi += sC[m * NS + n] * hb[n * PS + p];
          bg += sB[m * NS + n] * G[n * PS + p];
        }
        float ci, cu;
        dx_out(m, p, yi, bg, ci, cu);
        atomicAdd(&s_zin[m / R], ci);
        atomicAdd(&s_zue[m / R], cu);
      }
    }
    {
      float part = 0.f;
      for (int i = tid; i < NP; i += kThreads) part += hb[(i / P) * PS + i % P] * G[(i / P) * PS + i % P];
      block_add(part, &misc[0]);
    }
    __syncthreads();

    // (4) dC~ = diag(e^cum) dY hbar_in^T + W B~,  dB~ = diag(w e^{cum_end - cum}) X G^T + W^T C~
    if constexpr (NT != 0 && PT == 64 && kThreads == 512) {
      constexpr int NC = NT / 32;
      const int m0 = tid >> 5, n0 = tid & 31;  // rows m0, m0 + 16; columns n0 + 32 c
      float dc[2][NC] = {}, db[2][NC] = {};
#pragma unroll 4
      for (int p = 0; p < PT; ++p) {
        const float y0 = sdY[m0 * PS + p], y1 = sdY[(m0 + 16) * PS + p];
        const float x0 = sX[m0 * PS + p], x1 = sX[(m0 + 16) * PS + p];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float h = hb[(n0 + 32 * c) * PS + p], gg = G[(n0 + 32 * c) * PS + p];
          dc[0][c] += y0 * h;
          dc[1][c] += y1 * h;
          db[0][c] += x0 * gg;
          db[1][c] += x1 * gg;
        }
      }
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int t = (m0 + 16 * a2) / R;  // rows past M are computed but never stored
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          dc[a2][c] *= s_ecum[t];
          db[a2][c] *= s_w[t] * s_eend[t];
        }
      }
      // W is zero outside the causal triangle, so j runs over every row
#pragma unroll 4
      for (int j = 0; j < M; ++j) {
        const float wa0 = sW[m0 * M + j], wa1 = sW[(m0 + 16) * M + j];
        const float wb0 = sW[j * M + m0], wb1 = sW[j * M + m0 + 16];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float bj = sB[j * NS + n0 + 32 * c], cj = sC[j * NS + n0 + 32 * c];
          dc[0][c] += wa0 * bj;
          dc[1][c] += wa1 * bj;
          db[0][c] += wb0 * cj;
          db[1][c] += wb1 * cj;
        }
      }
#pragma unroll
      for (int a2 = 0; a2 < 2; ++a2) {
        const int m = m0 + 16 * a2, t = m / R, r = m % R;
        if (m < M)
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const int n = n0 + 32 * c;
            float dbv = db[a2][c];
            if (t0 + t == L - 1 && g.dbprev_out) dbv += g.dbprev_out[(us * R + r) * N + n];
            dBt[m * N + n] = dbv;
            dCt[m * N + n] = dc[a2][c];
          }
      }
    } else {
      for (int i = tid; i < M * N; i += kThreads) {
        const int m = i / N, n = i % N, t = m / R, r = m % R;
        float dc = 0.f, db = 0.f;
#pragma unroll 8
        for (int p = 0; p < P; ++p) {
          dc += sdY[m * PS + p] * hb[n * PS + p];
          db += sX[m * PS + p] * G[n * PS + p];
        }
        dc *= s_ecum[t];
        db *= s_w[t] * s_eend[t];
        for (int j = 0; j < (t + 1) * R; ++j) dc += sW[m * M + j] * sB[j * NS + n];
        for (int j = t * R; j < M; ++j) db += sW[j * M + m] * sC[j * NS + n];
        if (t0 + t == L - 1 && g.dbprev_out) db += g.dbprev_out[(us * R + r) * N + n];
        dBt[i] = db;
        dCt[i] = dc;
      }
    }
    __syncthreads();

    // (5) dL/dhbar_in = e^{cum_end} G + C~^T diag(e^cum) dY (in place)
    state_update(G, sC, sdY, s_erow, ecend, M);
    // rotation back (dB = rot(+Phi) dB~) and the angle's share, from the chunk's last token
    for (int k = tid; k < K; k += kThreads) {
      float Sk = Sang[k];
      for (int i = q - 1; i >= 0; --i) {
        float sn, cs;
        sincosf(phit[i * K + k], &sn, &cs);
        float dphi = 0.f;
        for (int r = 0; r < R; ++r) {
          const int m = i * R + r;
          const float db0 = dBt[m * N + 2 * k], db1 = dBt[m * N + 2 * k + 1];
          const float dc0 = dCt[m * N + 2 * k], dc1 = dCt[m * N + 2 * k + 1];
          dphi += db0 * sB[m * NS + 2 * k + 1] - db1 * sB[m * NS + 2 * k] + dc0 * sC[m * NS + 2 * k + 1] -
                  dc1 * sC[m * NS + 2 * k];
          const size_t gi = tok(t0 + i) * R * N + (size_t)r * N + 2 * k;
          if (g.dBh) {  // grouped: this head's share added to the group's fp32 sum
            const size_t gg = tok_bc(t0 + i) * R * N + (size_t)r * N + 2 * k;
            atomicAdd(g.dBh + gg, cs * db0 - sn * db1);
            atomicAdd(g.dBh + gg + 1, sn * db0 + cs * db1);
            atomicAdd(g.dCh + gg, cs * dc0 - sn * dc1);
            atomicAdd(g.dCh + gg + 1, sn * dc0 + cs * dc1);
          } else {
            st1(dBg + gi, cs * db0 - sn * db1);
            st1(dBg + gi + 1, sn * db0 + cs * db1);
            st1(dCg + gi, cs * dc0 - sn * dc1);
            st1(dCg + gi + 1, sn * dc0 + cs * dc1);
          }
        }
        Sk += dphi;
        const size_t ti = tok(t0 + i) * K + k;
        st1(dTHg + ti, s_dt[i] * Sk);
        if constexpr (NT != 0) {  // K a multiple of 32: whole warps walk the tokens together
          const float v = warp_sum(sth[i * K + k] * Sk);
          if ((tid & 31) == 0) atomicAdd(&s_dth[i], v);
        } else {
          atomicAdd(&s_dth[i], sth[i * K + k] * Sk);
        }
      }
      Sang[k] = Sk;
    }
    // column and row sums of the token-pair paths
    for (int j = tid; j < q; j += kThreads) {
      float cz = 0.f, rt = 0.f;
      for (int t = j + 1; t < q; ++t) cz += sT[t * Q + j];
      for (int j2 = 0; j2 < j; ++j2) rt += s_w[j2] * sT[j * Q + j2];
      s_cZu[j] = cz;
      s_cT[j] = s_w[j] * cz;
      s_rT[j] = rt;
    }
    __syncthreads();

    // (6) per token: d a (every path across the token's decay), d gamma, d w -> ddt, dlam, dA
    if (tid == 0) {
      const float c0 = ecend * misc[0];
      float suf_zin = 0.f;
      for (int i = 0; i < q; ++i) suf_zin += s_zin[i];
      float pre = 0.f, F = 0.f, dw_prev = 0.f, first_ddt = 0.f, first_dlm = 0.f;
      for (int i = 0; i < q; ++i) {
        const float da = c0 + suf_zin + pre + F;
        const float dw = s_zue[i] + s_cZu[i];
        const float dgt = s_dg[i] + dw;  // gamma_i enters K(i, i) and w_i
        float ddt = da * s_at[i] + dgt * s_lam[i] + s_dth[i];
        float dlm = dgt * s_dt[i];
        if (AT)
          st1(dATg + tok(t0 + i), da * s_dt[i]);
        else
          dA_acc += da * s_dt[i];
        if (i > 0) {  // token i's lagged weight (1 - lam_i) dt_i sits in w_{i-1}
          ddt += dw_prev * (1.f - s_lam[i]);
          dlm -= dw_prev * s_dt[i];
          st1(dDTg + tok(t0 + i), ddt);
          st1(dLMg + tok(t0 + i), dlm);
        } else {
          first_ddt = ddt;
          first_dlm = dlm;
        }
        suf_zin -= s_zin[i];
        pre += s_w[i] * s_zue[i];
        F += s_cT[i] - s_rT[i];
        dw_prev = dw;
      }
      if (s_pend_t >= 0) {  // the chunk after this one: its first token's lagged weight sits in w_{q-1}
        st1(dDTg + tok(s_pend_t), misc[3] + dw_prev * (1.f - s_lam[q]));
        st1(dLMg + tok(s_pend_t), misc[4] - dw_prev * s_dt[q]);
      }
      s_pend_t = t0;
      misc[3] = first_ddt;
      misc[4] = first_dlm;
    }
    __syncthreads();
  }

  // ---------------- the initial state ----------------
  // hbar_{-1} = h_0 + mu1 B~_0^T x_0: dh_0 = G; mu1 = (1 - lam_0) dt_0 is token 0's lagged weight
  {
    float part = 0.f;
    if (has_init)
      for (int i = tid; i < NP; i += kThreads) {
        const int n = i / P, p = i % P;
        float u = 0.f;
        for (int r = 0; r < R; ++r) u += a.bprev0[(us * R + r) * N + n] * a.xprev0[(us * R + r) * P + p];
        part += u * G[n * PS + p];
      }
    if (tid == 0) misc[2] = 0.f;
    __syncthreads();
    block_add(part, &misc[2]);
    block_add(dD_acc, &misc[1]);
    __syncthreads();
  }
  if (tid == 0) {
    const float dmu = misc[2];
    st1(dDTg + tok(0), misc[3] + dmu * (1.f - s_lam[0]));
    st1(dLMg + tok(0), misc[4] - dmu * s_dt[0]);
    if (!AT) atomicAdd(g.dA + hh, dA_acc);
    if (g.dD) atomicAdd(g.dD + hh, misc[1]);
  }
  if (g.dh0) {
    for (int i = tid; i < NP; i += kThreads) g.dh0[us * NP + i] = G[(i / P) * PS + i % P];
    for (int i = tid; i < R * N; i += kThreads) {
      const int r = i / N, n = i % N;
      float s = 0.f;
      if (has_init)
        for (int p = 0; p < P; ++p) s += G[n * PS + p] * a.xprev0[(us * R + r) * P + p];
      g.dbprev0[us * R * N + i] = mu1 * s;
    }
    for (int i = tid; i < R * P; i += kThreads) {
      const int r = i / P, p = i % P;
      float s = 0.f;
      if (has_init)
        for (int n = 0; n < N; ++n) s += G[n * PS + p] * a.bprev0[(us * R + r) * N + n];
      g.dxprev0[us * R * P + i] = mu1 * s;
    }
    for (int k = tid; k < K; k += kThreads) g.dangle0[us * K + k] = Sang[k];
  }
}

// dB, dC [b, t, g] in the input dtype from the groups' fp32 sums
template <typename T>
__global__ void __launch_bounds__(256) bc_group_convert_kernel(const float* dBs, const float* dCs, T* dB, T* dC,
                                                               long long total) {
  for (long long e = (long long)blockIdx.x * 256 + threadIdx.x; e < total; e += (long long)gridDim.x * 256) {
    st1(dB + e, dBs[e]);
    st1(dC + e, dCs[e]);
  }
}

}  // namespace

// grouped B, C: the fp32 sums of dB and dC over each group's heads, [b, L, G, R, N] each
size_t bwd_group_bytes(const ScanArgs& a) {
  if (a.ngroups >= a.nheads) return 0;
  return 2 * (size_t)a.batch * a.seqlen * a.ngroups * a.R * a.N * sizeof(float);
}

size_t bwd_checkpoint_bytes(const ScanArgs& a) {
  const BwdLayout l = bwd_layout(a.P, a.N, a.R);
  const size_t nchunks = ((size_t)a.seqlen + l.Q - 1) / l.Q;
  return (size_t)a.batch * a.nheads * nchunks * ((size_t)a.N * a.P + a.N / 2) * sizeof(float);
}

int bwd_supported(const ScanArgs& a) {
  if (a.ngroups < 1 || a.nheads % a.ngroups != 0) return MAMBA3_ERR_INVALID;
  // A per head or A_t per token; B, C per head or grouped; no fused norm
  if (a.bcnorm || (!a.A && !a.A_t)) return MAMBA3_ERR_UNSUPPORTED;
  if (a.R > kRows) return MAMBA3_ERR_UNSUPPORTED;
  if (bwd_layout(a.P, a.N, a.R).total > 220 * 1024) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

int launch_scan_bwd(const BwdArgs& g, cudaStream_t s) {
  const ScanArgs& a = g.f;
  if (g.dA && cudaMemsetAsync(g.dA, 0, sizeof(float) * a.nheads, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (g.dD && cudaMemsetAsync(g.dD, 0, sizeof(float) * a.nheads, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  const int units = a.batch * a.nheads;
  if (units == 0) return MAMBA3_OK;
  const BwdLayout lay = bwd_layout(a.P, a.N, a.R);
  using KFn = void (*)(BwdArgs, BwdLayout);
  KFn k = nullptr;
  if (a.dtype == MAMBA3_BF16 && a.P == 64 && (a.N == 64 || a.N == 128) && (a.R == 1 || a.R == 2 || a.R == 4)) {
    using B16 = __nv_bfloat16;
    if (a.N == 128)
      k = a.R == 1 ? scan_bwd_kernel<B16, 128, 64, 1> : (a.R == 2 ? scan_bwd_kernel<B16, 128, 64, 2>
                                                                  : scan_bwd_kernel<B16, 128, 64, 4>);
    else
      k = a.R == 1 ? scan_bwd_kernel<B16, 64, 64, 1> : (a.R == 2 ? scan_bwd_kernel<B16, 64, 64, 2>
                                                                 : scan_bwd_kernel<B16, 64, 64, 4>);
  } else {
    k = a.dtype == MAMBA3_F32 ? scan_bwd_kernel<float, 0, 0, 0> : scan_bwd_kernel<__nv_bfloat16, 0, 0, 0>;
  }
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  const long long total = (long long)a.batch * a.seqlen * a.ngroups * a.R * a.N;
  if (g.dBh && cudaMemsetAsync(g.dBh, 0, bwd_group_bytes(a), s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  k<<<units, kThreads, lay.total, s>>>(g, lay);
  if (cudaGetLastError() != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (g.dBh && total > 0) {
    long long blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (a.dtype == MAMBA3_F32)
      bc_group_convert_kernel<float><<<(int)blocks, 256, 0, s>>>(g.dBh, g.dCh, static_cast<float*>(g.dB),
                                                                 static_cast<float*>(g.dC), total);
    else
      bc_group_convert_kernel<__nv_bfloat16><<<(int)blocks, 256, 0, s>>>(
          g.dBh, g.dCh, static_cast<__nv_bfloat16*>(g.dB), static_cast<__nv_bfloat16*>(g.dC), total);
  }
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // namespace m3

// Chunked prefill of the Mamba-3 recurrence on the SIMT pipes (fp32 FMA).
//
// This is the path for fp32 inputs (and for bf16 shapes that the tensor-core
// kernel does not cover): every product is an fp32 FMA, so it meets a 1e-4
// relative tolerance against the fp64 definition.
//
// Chunked form (derived from the three-term update of section 1.1 of
// "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation)).  With
// u_s = sum_r B~_s[r]^T x_s[r] and cum_t = sum_{q<=t} dt_q A inside a chunk,
// the lagged term of step s+1 carries the same decay as the state, so it folds
// into the weight of column s:
//   w_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}         (0-th order next token)
//   h_t = e^{cum_t} hbar_in + sum_{s<t} e^{cum_t - cum_s} w_s u_s + lam_t dt_t u_t
//   hbar_out = e^{cum_end} hbar_in + sum_{s<=end} e^{cum_end - cum_s} w_s u_s
// where hbar = h + (1 - lam_next) dt_next u (the state with the next token's
// lagged term already added); at the end of the sequence the next token does
// not exist and hbar = h.  Within a chunk only differences of chunk-local
// cumulative sums are exponentiated, so nothing overflows for long sequences.
// The angles are carried across chunks wrapped to [-pi, pi].
//
// One CTA per (batch, head) marches over the chunks; the state hbar stays in
// shared memory in fp32.
#include "common.cuh"
#include "internal.h"

namespace m3 {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxRows = 64;  // M = Q * R rows per chunk

struct SimtLayout {
  int M, Q;
  size_t off_h, off_B, off_C, off_X, off_S, off_cum, off_w, off_g, off_dt, off_phi, total;
};

SimtLayout simt_layout(int P, int N, int R, int Q) {
  SimtLayout l;
  l.Q = Q;
  l.M = Q * R;
  size_t o = 0;
  auto take = [&](size_t n) {
    size_t r = o;
    o += (n + 3) & ~size_t(3);
    return r;
  };
  l.off_h = take((size_t)N * P);
  l.off_B = take((size_t)l.M * N);
  l.off_C = take((size_t)l.M * N);
  l.off_X = take((size_t)l.M * P);
  l.off_S = take((size_t)l.M * l.M);
  l.off_cum = take(Q);
  l.off_w = take(Q);
  l.off_g = take(Q);
  l.off_dt = take(Q + 1);
  l.off_phi = take(N / 2);
  l.total = o * sizeof(float);
  return l;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) scan_simt_kernel(ScanArgs a, SimtLayout lay) {
  extern __shared__ float sm[];
  const int P = a.P, N = a.N, R = a.R, Q = a.Q, L = a.seqlen, K = N / 2;
  const int unit = blockIdx.x;
  const int b = unit / a.nheads, hh = unit % a.nheads;
  const int tid = threadIdx.x;
  float* hbar = sm + lay.off_h;  // [N][P]
  float* sB = sm + lay.off_B;    // [M][N]
  float* sC = sm + lay.off_C;    // [M][N]
  float* sX = sm + lay.off_X;    // [M][P]
  float* sS = sm + lay.off_S;    // [M][M]
  float* cum = sm + lay.off_cum;
  float* w = sm + lay.off_w;
  float* gam = sm + lay.off_g;
  float* sdt = sm + lay.off_dt;  // dt then lam of the chunk + the next token
  float* phi = sm + lay.off_phi;
  __shared__ float s_lam[kMaxRows + 1];

  const float Ah = a.A ? a.A[hh] : 0.f;
  const T* AT = static_cast<const T*>(a.A_t);  // time-varying decay [b, L, H], or null
  const float Dh = a.D ? a.D[hh] : 0.f;
  const T* X = static_cast<const T*>(a.x);
  const T* Bg = static_cast<const T*>(a.B);
  const T* Cg = static_cast<const T*>(a.C);
  const T* TH = static_cast<const T*>(a.theta);
  const T* DT = static_cast<const T*>(a.dt);
  const T* LM = static_cast<const T*>(a.lam);
  T* Y = static_cast<T*>(a.y);
  const size_t us = (size_t)unit;
  auto tok = [&](int t) { return ((size_t)b * L + t) * a.nheads + hh; };
  const int gh = hh / (a.nheads / a.ngroups);  // B, C row of this head
  auto tok_bc = [&](int t) { return ((size_t)b * L + t) * a.ngroups + gh; };

  // ---- initial state: hbar_0 = h_0 + (1 - lam_1) dt_1 B~_0^T x_0 ----
  const bool has_init = a.h0 != nullptr;
  float mu1 = 0.f;
  if (L > 0) mu1 = (1.f - ld1(LM + tok(0))) * ld1(DT + tok(0));
  for (int i = tid; i < N * P; i += kThreads) {
    const int n = i / P, p = i % P;
    float v = 0.f;
    if (has_init) {
      v = a.h0[us * N * P + i];
      float c = 0.f;
      for (int r = 0; r < R; ++r) c += a.bprev0[(us * R + r) * N + n] * a.xprev0[(us * R + r) * P + p];
      v += mu1 * c;
    }
    hbar[i] = v;
  }
  for (int k = tid; k < K; k += kThreads) phi[k] = has_init ? a.angle0[us * K + k] : 0.f;
  __syncthreads();

  if (L == 0) {  // nothing to scan: the exported state is the initial state
    if (a.h_out) {
      for (int i = tid; i < N * P; i += kThreads) a.h_out[us * N * P + i] = has_init ? a.h0[us * N * P + i] : 0.f;
      for (int i = tid; i < R * N; i += kThreads) a.bprev_out[us * R * N + i] = has_init ? a.bprev0[us * R * N + i] : 0.f;
      for (int i = tid; i < R * P; i += kThreads) a.xprev_out[us * R * P + i] = has_init ? a.xprev0[us * R * P + i] : 0.f;
      for (int k = tid; k < K; k += kThreads) a.angle_out[us * K + k] = phi[k];
    }
    return;
  }

  for (int t0 = 0; t0 < L; t0 += Q) {
    const int q = min(Q, L - t0);
    const int M = q * R;
    // ---- scalars of the chunk (and the next token, if any) ----
    for (int i = tid; i <= q; i += kThreads) {
      if (t0 + i < L) {
        sdt[i] = ld1(DT + tok(t0 + i));
        s_lam[i] = ld1(LM + tok(t0 + i));
      } else {  // past the end of the sequence: no lagged term
        sdt[i] = 0.f;
        s_lam[i] = 1.f;
      }
    }
    // ---- raw B, C, x rows ----
    for (int i = tid; i < M * N; i += kThreads) {
      const int m = i / N, n = i % N;
      const size_t g = tok_bc(t0 + m / R) * R * N + (size_t)(m % R) * N + n;
      sB[i] = ld1(Bg + g);
      sC[i] = ld1(Cg + g);
    }
    for (int i = tid; i < M * P; i += kThreads) {
      const int m = i / P, p = i % P;
      sX[i] = ld1(X + tok(t0 + m / R) * R * P + (size_t)(m % R) * P + p);
    }
    __syncthreads();
    if (tid == 0) {
      float c = 0.f;
      for (int i = 0; i < q; ++i) {
        c += sdt[i] * (AT ? ld1(AT + tok(t0 + i)) : Ah);
        cum[i] = c;
        gam[i] = s_lam[i] * sdt[i];
        w[i] = gam[i] + (1.f - s_lam[i + 1]) * sdt[i + 1];
      }
    }
    // ---- rotation by the accumulated angle (one thread per pair) ----
    for (int k = tid; k < K; k += kThreads) {
      float local = 0.f;
      for (int i = 0; i < q; ++i) {
        local += sdt[i] * ld1(TH + tok(t0 + i) * K + k);
        float s, c;
        sincosf(phi[k] + local, &s, &c);
        for (int r = 0; r < R; ++r) {
          float* bb = sB + (i * R + r) * N + 2 * k;
          float* cc = sC + (i * R + r) * N + 2 * k;
          const float b0 = bb[0], b1 = bb[1], c0 = cc[0], c1 = cc[1];
          bb[0] = c * b0 + s * b1;
          bb[1] = -s * b0 + c * b1;
          cc[0] = c * c0 + s * c1;
          cc[1] = -s * c0 + c * c1;
        }
      }
      phi[k] = wrap_angle(phi[k] + local);
    }
    __syncthreads();
    // ---- masked scores S[m][j] = (C~_m . B~_j) * kernel(t_m, t_j) ----
    for (int i = tid; i < M * M; i += kThreads) {
      const int m = i / M, j = i % M;
      const int tm = m / R, tj = j / R;
      float v = 0.f;
      if (tj <= tm) {
        float d = 0.f;
        for (int n = 0; n < N; ++n) d += sC[m * N + n] * sB[j * N + n];
        const float kern = (tj == tm) ? gam[tm] : expf(cum[tm] - cum[tj]) * w[tj];
        v = d * kern;
      }
      sS[i] = v;
    }
    __syncthreads();
    // ---- y = S x + e^{cum} C~ hbar_in + D x ----
    for (int i = tid; i < M * P; i += kThreads) {
      const int m = i / P, p = i % P;
      float acc = 0.f;
      for (int j = 0; j < M; ++j) acc += sS[m * M + j] * sX[j * P + p];
      float inter = 0.f;
      for (int n = 0; n < N; ++n) inter += sC[m * N + n] * hbar[n * P + p];
      acc += expf(cum[m / R]) * inter + Dh * sX[i];
      st1(Y + tok(t0 + m / R) * R * P + (size_t)(m % R) * P + p, acc);
    }
    __syncthreads();
    // ---- hbar_out = e^{cum_end} hbar_in + sum_j e^{cum_end - cum_j} w_j B~_j^T x_j ----
    const float cend = cum[q - 1];
    for (int i = tid; i < N * P; i += kThreads) {
      const int n = i / P, p = i % P;
      float acc = expf(cend) * hbar[i];
      for (int j = 0; j < M; ++j) acc += expf(cend - cum[j / R]) * w[j / R] * sB[j * N + n] * sX[j * P + p];
      hbar[i] = acc;
    }
    __syncthreads();
  }

  // ---- export: h_L (= hbar at the end), B~_L, x_L, Phi_L ----
  if (a.h_out) {
    const int qlast = L - ((L - 1) / Q) * Q;  // tokens in the last chunk
    for (int i = tid; i < N * P; i += kThreads) a.h_out[us * N * P + i] = hbar[i];
    for (int i = tid; i < R * N; i += kThreads) a.bprev_out[us * R * N + i] = sB[(qlast - 1) * R * N + i];
    for (int i = tid; i < R * P; i += kThreads) a.xprev_out[us * R * P + i] = sX[(qlast - 1) * R * P + i];
    for (int k = tid; k < K; k += kThreads) a.angle_out[us * K + k] = phi[k];
  }
}

int default_q(const ScanArgs& a) { return a.Q > 0 ? a.Q : kMaxRows / a.R; }

}  // namespace

int simt_scan_supported(const ScanArgs& a) {
  if (a.ngroups < 1 || a.nheads % a.ngroups != 0) return MAMBA3_ERR_INVALID;  // B, C rows per token
  const int Q = default_q(a);
  if (Q < 1 || Q * a.R > kMaxRows) return MAMBA3_ERR_UNSUPPORTED;
  if (simt_layout(a.P, a.N, a.R, Q).total > 220 * 1024) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

int launch_scan_simt(const ScanArgs& a0, cudaStream_t s) {
  ScanArgs a = a0;
  a.Q = default_q(a0);
  const SimtLayout lay = simt_layout(a.P, a.N, a.R, a.Q);
  const int units = a.batch * a.nheads;
  if (units == 0) return MAMBA3_OK;
  if (a.dtype == MAMBA3_F32) {
    auto k = scan_simt_kernel<float>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total) != cudaSuccess)
      return MAMBA3_ERR_CUDA;
    k<<<units, kThreads, lay.total, s>>>(a, lay);
  } else {
    auto k = scan_simt_kernel<__nv_bfloat16>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lay.total) != cudaSuccess)
      return MAMBA3_ERR_CUDA;
    k<<<units, kThreads, lay.total, s>>>(a, lay);
  }
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // namespace m3

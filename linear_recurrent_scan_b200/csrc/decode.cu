// Fused single-token decode step of the Mamba-3 recurrence (sm_100a).
//
// Per (batch, head) unit, in place on the fp32 state:
//   Phi   <- wrap(Phi + dt * theta)                      (RoPE trick, section 1.2)
//   B~, C~ = B, C with each pair (2k, 2k+1) rotated by -Phi_k
//   h     <- alpha h + beta B~_prev^T x_prev + gamma B~^T x (section 1.1, rank R per 1.3)
//   y[r]  = C~[r] h + D x[r]
//   B~_prev <- B~, x_prev <- x
// Sources: "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation)
// sections 1.1-1.3; the decode step is memory-bound (section 1.3: about 2.5
// ops per byte for standard SSM decoding), so the kernel is organised around
// streaming the N x P fp32 state exactly once with 16-byte loads and stores.
//
// Work split: one CTA of 128 threads per (b, h).  A thread owns four
// consecutive columns p..p+3 of h and the rows n = ty, ty + G, ... (G = 128 /
// (P/4) row groups); it issues all of its state loads before any arithmetic
// so that up to 16 independent 16-byte loads are in flight per thread.  The
// rank-R update and the readout partial sums stay in registers; the readout is
// reduced over the G row groups through shared memory.
#include "common.cuh"
#include "internal.h"

namespace m3 {
namespace {

constexpr int kThreads = 128;
constexpr int kMaxRows = 16;  // rows of h per thread (N <= kMaxRows * G)

template <typename T, int R>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeArgs a) {
  const int P = a.P, N = a.N, K = N / 2;
  const int unit = blockIdx.x;
  const int h_idx = unit % a.nheads;
  const int tpr = P / 4;  // threads per row
  const int G = kThreads / tpr;
  const int tid = threadIdx.x;
  const int p4 = tid % tpr;
  const int ty = tid / tpr;

  extern __shared__ float sm[];
  float* sB = sm;                 // [R][N]  B~ of this token
  float* sC = sB + R * N;         // [R][N]  C~ of this token
  float* sBp = sC + R * N;        // [R][N]  B~ of the previous token
  float* sX = sBp + R * N;        // [R][P]
  float* sXp = sX + R * P;        // [R][P]
  float* sRed = sXp + R * P;      // [G][R][P] readout partial sums
  __shared__ float sCoef[3];      // alpha, beta, gamma

  float* hu = a.h + (size_t)unit * N * P;

  // 1. issue the state loads first (streaming: h is larger than L2)
  float4 hv[kMaxRows];
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j) {
    const int n = ty + j * G;
    if (n < N) hv[j] = __ldcs(reinterpret_cast<const float4*>(hu + (size_t)n * P + 4 * p4));
  }

  // 2. per-token scalars, angles and rotated B, C into shared memory
  const T* xu = static_cast<const T*>(a.x) + (size_t)unit * R * P;
  const T* Bu = static_cast<const T*>(a.B) + (size_t)unit * R * N;
  const T* Cu = static_cast<const T*>(a.C) + (size_t)unit * R * N;
  const T* thu = static_cast<const T*>(a.theta) + (size_t)unit * K;
  const float dt = ld1(static_cast<const T*>(a.dt) + unit);
  if (tid == 0) {
    const float lam = ld1(static_cast<const T*>(a.lam) + unit);
    const float alpha = expf(dt * a.A[h_idx]);
    sCoef[0] = alpha;
    sCoef[1] = (1.f - lam) * dt * alpha;
    sCoef[2] = lam * dt;
  }
  float* angu = a.angle + (size_t)unit * K;
  for (int k = tid; k < K; k += kThreads) {
    const float phi = wrap_angle(angu[k] + dt * ld1(thu + k));
    float s, c;
    sincosf(phi, &s, &c);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float b0 = ld1(Bu + r * N + 2 * k), b1 = ld1(Bu + r * N + 2 * k + 1);
      const float c0 = ld1(Cu + r * N + 2 * k), c1 = ld1(Cu + r * N + 2 * k + 1);
      sB[r * N + 2 * k] = c * b0 + s * b1;
      sB[r * N + 2 * k + 1] = -s * b0 + c * b1;
      sC[r * N + 2 * k] = c * c0 + s * c1;
      sC[r * N + 2 * k + 1] = -s * c0 + c * c1;
    }
    angu[k] = phi;  // each angle is read and written by the same thread
  }
  float* bpu = a.bprev + (size_t)unit * R * N;
  float* xpu = a.xprev + (size_t)unit * R * P;
  for (int i = tid; i < R * N; i += kThreads) sBp[i] = bpu[i];
  for (int i = tid; i < R * P; i += kThreads) {
    sXp[i] = xpu[i];
    sX[i] = ld1(xu + i);
  }
  __syncthreads();
  // the carry for the next step (all reads of the old carry are done)
  for (int i = tid; i < R * N; i += kThreads) bpu[i] = sB[i];
  for (int i = tid; i < R * P; i += kThreads) xpu[i] = sX[i];

  // 3. state update and readout partial sums in registers
  const float alpha = sCoef[0], beta = sCoef[1], gamma = sCoef[2];
  float4 xr[R], xpr[R], yacc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    xr[r] = *reinterpret_cast<const float4*>(sX + r * P + 4 * p4);
    xpr[r] = *reinterpret_cast<const float4*>(sXp + r * P + 4 * p4);
    yacc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int j = 0; j < kMaxRows; ++j) {
    const int n = ty + j * G;
    if (n < N) {
      float4 hn;
      hn.x = alpha * hv[j].x;
      hn.y = alpha * hv[j].y;
      hn.z = alpha * hv[j].z;
      hn.w = alpha * hv[j].w;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float bp = beta * sBp[r * N + n], bc = gamma * sB[r * N + n];
        hn.x += bp * xpr[r].x + bc * xr[r].x;
        hn.y += bp * xpr[r].y + bc * xr[r].y;
        hn.z += bp * xpr[r].z + bc * xr[r].z;
        hn.w += bp * xpr[r].w + bc * xr[r].w;
      }
      __stcs(reinterpret_cast<float4*>(hu + (size_t)n * P + 4 * p4), hn);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float cr = sC[r * N + n];
        yacc[r].x += cr * hn.x;
        yacc[r].y += cr * hn.y;
        yacc[r].z += cr * hn.z;
        yacc[r].w += cr * hn.w;
      }
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) *reinterpret_cast<float4*>(sRed + (ty * R + r) * P + 4 * p4) = yacc[r];
  __syncthreads();

  // 4. reduce the readout over row groups, add D x, store y
  const float Dh = a.D ? a.D[h_idx] : 0.f;
  T* yu = static_cast<T*>(a.y) + (size_t)unit * R * P;
  for (int i = tid; i < R * P; i += kThreads) {
    float s = 0.f;
    for (int g = 0; g < G; ++g) s += sRed[g * R * P + i];
    st1(yu + i, s + Dh * sX[i]);
  }
}

size_t decode_smem_bytes(int P, int N, int R) {
  const int G = kThreads / (P / 4);
  return sizeof(float) * (size_t)(3 * R * N + 2 * R * P + G * R * P);
}

template <typename T, int R>
int launch_t(const DecodeArgs& a, cudaStream_t s) {
  const size_t smem = decode_smem_bytes(a.P, a.N, a.R);
  auto k = decode_kernel<T, R>;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  k<<<a.batch * a.nheads, kThreads, smem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

template <typename T>
int launch_r(const DecodeArgs& a, cudaStream_t s) {
  switch (a.R) {
    case 1: return launch_t<T, 1>(a, s);
    case 2: return launch_t<T, 2>(a, s);
    case 4: return launch_t<T, 4>(a, s);
    case 8: return launch_t<T, 8>(a, s);
  }
  return MAMBA3_ERR_UNSUPPORTED;
}

}  // namespace

int decode_supported(const DecodeArgs& a) {
  if (a.P % 4 != 0 || a.P / 4 > kThreads || kThreads % (a.P / 4) != 0) return MAMBA3_ERR_UNSUPPORTED;
  const int G = kThreads / (a.P / 4);
  if (a.N > kMaxRows * G) return MAMBA3_ERR_UNSUPPORTED;
  if (!(a.R == 1 || a.R == 2 || a.R == 4 || a.R == 8)) return MAMBA3_ERR_UNSUPPORTED;
  if (decode_smem_bytes(a.P, a.N, a.R) > 200 * 1024) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.batch * a.nheads == 0) return MAMBA3_OK;
  return a.dtype == MAMBA3_F32 ? launch_r<float>(a, s) : launch_r<__nv_bfloat16>(a, s);
}

}  // namespace m3

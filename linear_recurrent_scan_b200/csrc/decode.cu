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
// Two kernels.  decode_stream_kernel (second half of this file) is the main
// path for P = 64, N in {64, 128}, R in {1, 2, 4}: persistent CTAs stream the
// (b, h) units through a 2-stage shared-memory ring filled and drained by bulk
// copies, and can fuse the B/C RMS norm.  decode_kernel below covers every
// other supported shape (and unaligned pointers).
//
// decode_kernel work split: one CTA of 128 threads per (b, h).  A thread owns four
// consecutive columns p..p+3 of h and the rows n = ty, ty + G, ... (G = 128 /
// (P/4) row groups); it issues all of its state loads before any arithmetic
// so that up to 16 independent 16-byte loads are in flight per thread.  The
// rank-R update and the readout partial sums stay in registers; the readout is
// reduced over the G row groups through shared memory.
#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace m3 {
namespace {

// Row of B and C that unit (b, h) = (u / H, u % H) reads: u itself with one row
// per head; b * G + h / (H / G) when G groups of heads share B and C.
__device__ __forceinline__ size_t bc_row(const DecodeArgs& a, int u) {
  return (size_t)(u / a.nheads) * a.ngroups + (u % a.nheads) / (a.nheads / a.ngroups);
}

constexpr int kThreads = 128;
constexpr int kMaxRows = 16;  // rows of h per thread (N <= kMaxRows * G)

// Status word of the decode step, one per device (the decode entry points take
// no workspace).  A timed-out wait records MAMBA3_ERR_TIMEOUT here; it stays set
// until mamba3_decode_status reads and clears it.
__device__ DeviceStatus g_decode_status;

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
  const T* Bu = static_cast<const T*>(a.B) + bc_row(a, unit) * R * N;
  const T* Cu = static_cast<const T*>(a.C) + bc_row(a, unit) * R * N;
  const T* thu = static_cast<const T*>(a.theta) + (size_t)unit * K;
  const float dt = ld1(static_cast<const T*>(a.dt) + unit);
  if (tid == 0) {
    const float lam = ld1(static_cast<const T*>(a.lam) + unit);
    const float rate = a.A_t ? ld1(static_cast<const T*>(a.A_t) + unit) : a.A[h_idx];  // A_t [b, H] or A [H]
    const float alpha = expf(dt * rate);
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


// ------------------------------------------------------------------ streaming version
// Persistent CTAs stream (batch, head) units: while unit i is computed in
// shared memory, the TMA engine brings unit i+1 (its N x P state slab and the
// small per-unit inputs) into the other stage of a 2-stage ring, and a bulk
// store writes unit i-1's new state back.  HBM traffic therefore does not wait
// on the SIMT work.  Used for P = 64, N in {64, 128}.
constexpr int kSThreads = 256;
constexpr int kSP = 64;

template <typename T, int N, int R>
struct DStage {  // byte offsets inside one stage; every region is a multiple of 16 bytes
  static constexpr int H = 0;                                   // state      N x P f32
  static constexpr int BP = H + N * kSP * 4;                    // b_prev     R x N f32
  static constexpr int XP = BP + R * N * 4;                     // x_prev     R x P f32
  static constexpr int ANG = XP + R * kSP * 4;                  // angle      N/2 f32
  static constexpr int B = ANG + (N / 2) * 4;                   // B          R x N T
  static constexpr int C = B + R * N * (int)sizeof(T);          // C          R x N T
  static constexpr int X = C + R * N * (int)sizeof(T);          // x          R x P T
  static constexpr int TH = X + R * kSP * (int)sizeof(T);       // theta      N/2 T
  static constexpr int LOADED = TH + (N / 2) * (int)sizeof(T);  // bytes brought by the bulk loads
  static constexpr int BYTES = (LOADED + 127) & ~127;
  // shared by both stages: rotated B, C (f32), readout partial sums per warp
  static constexpr int SB = 2 * BYTES;
  static constexpr int SC = SB + R * N * 4;
  static constexpr int RED = SC + R * N * 4;
  static constexpr int BAR = RED + (kSThreads / 32) * R * kSP * 4;
  static constexpr int TOTAL = BAR + 64;
};

template <typename T, int N, int R, bool BCN>
__global__ void __launch_bounds__(kSThreads) decode_stream_kernel(DecodeArgs a) {
  using S = DStage<T, N, R>;
  constexpr int K2 = N / 2, ROWS = N / 16;
  extern __shared__ __align__(128) uint8_t dsm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + S::BAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dsm + S::BAR + 16);
  float* sB = reinterpret_cast<float*>(dsm + S::SB);
  float* sC = reinterpret_cast<float*>(dsm + S::SC);
  float* red = reinterpret_cast<float*>(dsm + S::RED);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p4 = tid & 15, ty = tid >> 4;
  const int units = a.batch * a.nheads;

  if (tid == 0) {
    ptx::mbar_init(&bars[0], 1);
    ptx::mbar_init(&bars[1], 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();
  // Launched with programmatic stream serialization: let the next step's grid
  // be scheduled now (its CTAs take SM slots as ours exit and run their
  // prologue), then wait until the previous grid in the stream has completed
  // and its writes are visible.  Every global access below follows the wait,
  // so the ordering is that of a plain stream launch.
  ptx::grid_launch_dependents();
  ptx::grid_dependency_wait();

  // stage -> 1 + iteration whose loads were issued into it and not yet waited for
  int inflight[2] = {0, 0};
  auto issue_loads = [&](int u, int stage, int iter) {
    if (a.test_withhold) return;  // testing the timeout path only: the wait below must give up
    inflight[stage] = iter + 1;
    uint8_t* st = dsm + stage * S::BYTES;
    uint64_t* bar = &bars[stage];
    ptx::mbar_arrive_expect_tx(bar, S::LOADED);
    ptx::bulk_load(st + S::H, a.h + (size_t)u * N * kSP, N * kSP * 4, bar);
    ptx::bulk_load(st + S::BP, a.bprev + (size_t)u * R * N, R * N * 4, bar);
    ptx::bulk_load(st + S::XP, a.xprev + (size_t)u * R * kSP, R * kSP * 4, bar);
    ptx::bulk_load(st + S::ANG, a.angle + (size_t)u * K2, K2 * 4, bar);
    ptx::bulk_load(st + S::B, static_cast<const T*>(a.B) + bc_row(a, u) * R * N, R * N * sizeof(T), bar);
    ptx::bulk_load(st + S::C, static_cast<const T*>(a.C) + bc_row(a, u) * R * N, R * N * sizeof(T), bar);
    ptx::bulk_load(st + S::X, static_cast<const T*>(a.x) + (size_t)u * R * kSP, R * kSP * sizeof(T), bar);
    ptx::bulk_load(st + S::TH, static_cast<const T*>(a.theta) + (size_t)u * K2, K2 * sizeof(T), bar);
  };

  int it = 0;
  int u = blockIdx.x;
  if (tid == 0 && u < units) issue_loads(u, 0, 0);
  for (; u < units; u += gridDim.x, ++it) {
    const int s = it & 1;
    uint8_t* st = dsm + s * S::BYTES;
    const int un = u + gridDim.x;
    if (tid == 0 && un < units) {
      ptx::bulk_wait_read<0>();  // the other stage's previous state store has read its source
      issue_loads(un, s ^ 1, it + 1);
    }
    const int hh = u % a.nheads;
    const float dt = ld1(static_cast<const T*>(a.dt) + u);
    const float lam = ld1(static_cast<const T*>(a.lam) + u);
    const float rate = a.A_t ? ld1(static_cast<const T*>(a.A_t) + u) : a.A[hh];  // A_t [b, H] or A [H]
    const float alpha = expf(dt * rate);
    const float beta = (1.f - lam) * dt * alpha, gamma = lam * dt;
    const float Dh = a.D ? a.D[hh] : 0.f;
    ptx::mbar_wait(&bars[s], (it >> 1) & 1, abort_flag, &g_decode_status, 1, a.wait_limit);
    if (__syncthreads_or(*abort_flag != 0)) break;
    if (tid == 0) inflight[s] = 0;
    float* rinv = reinterpret_cast<float*>(dsm + S::BAR + 32);  // fused norm: 1/RMS of B rows, then C rows
    if constexpr (BCN) {  // warp w < 2R: raw row w % R of B (w < R) or of C
      if (warp < 2 * R) {
        const T* row = reinterpret_cast<const T*>(st + (warp < R ? S::B : S::C)) + (warp % R) * N;
        float ss = 0.f;
        for (int n = lane; n < N; n += 32) {
          const float v = ld1(row + n);
          ss += v * v;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float v = ss * (1.f / N) + a.neps;
        if (lane == 0) rinv[warp] = v > 0.f ? rsqrtf(v) : 0.f;  // all-zero row, eps = 0: 0, not 0/0
      }
      __syncthreads();
    }

    // ---- rotation of B and C by the updated angle; the carry for the next step ----
    const float* ang = reinterpret_cast<const float*>(st + S::ANG);
    const T* Bs = reinterpret_cast<const T*>(st + S::B);
    const T* Cs = reinterpret_cast<const T*>(st + S::C);
    const T* Xs = reinterpret_cast<const T*>(st + S::X);
    const T* THs = reinterpret_cast<const T*>(st + S::TH);
    for (int i = tid; i < R * K2; i += kSThreads) {
      const int r = i / K2, k = i % K2;
      const float phi = wrap_angle(ang[k] + dt * ld1(THs + k));
      float sn, cs;
      __sincosf(phi, &sn, &cs);  // |phi| <= pi
      float b0 = ld1(Bs + r * N + 2 * k), b1 = ld1(Bs + r * N + 2 * k + 1);
      float c0 = ld1(Cs + r * N + 2 * k), c1 = ld1(Cs + r * N + 2 * k + 1);
      if constexpr (BCN) {  // normalised row times the head's weight, plus its bias
        const size_t q = ((size_t)hh * R + r) * N + 2 * k;
        const float ib = rinv[r], ic = rinv[R + r];
        b0 = b0 * ib * (a.nw_B ? a.nw_B[q] : 1.f) + (a.nb_B ? a.nb_B[q] : 0.f);
        b1 = b1 * ib * (a.nw_B ? a.nw_B[q + 1] : 1.f) + (a.nb_B ? a.nb_B[q + 1] : 0.f);
        c0 = c0 * ic * (a.nw_C ? a.nw_C[q] : 1.f) + (a.nb_C ? a.nb_C[q] : 0.f);
        c1 = c1 * ic * (a.nw_C ? a.nw_C[q + 1] : 1.f) + (a.nb_C ? a.nb_C[q + 1] : 0.f);
      }
      const float rb0 = cs * b0 + sn * b1, rb1 = -sn * b0 + cs * b1;
      sB[r * N + 2 * k] = rb0;
      sB[r * N + 2 * k + 1] = rb1;
      sC[r * N + 2 * k] = cs * c0 + sn * c1;
      sC[r * N + 2 * k + 1] = -sn * c0 + cs * c1;
      *reinterpret_cast<float2*>(a.bprev + ((size_t)u * R + r) * N + 2 * k) = make_float2(rb0, rb1);
      if (r == 0) a.angle[(size_t)u * K2 + k] = phi;
    }
    for (int i = tid; i < R * kSP; i += kSThreads) a.xprev[(size_t)u * R * kSP + i] = ld1(Xs + i);
    __syncthreads();

    // ---- state update in shared memory and readout partial sums ----
    const float* bp = reinterpret_cast<const float*>(st + S::BP);
    const float* xp = reinterpret_cast<const float*>(st + S::XP);
    float* hs = reinterpret_cast<float*>(st + S::H);
    float4 xr[R], xpr[R], yacc[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      xr[r] = ld4(Xs + r * kSP + 4 * p4);
      xpr[r] = *reinterpret_cast<const float4*>(xp + r * kSP + 4 * p4);
      yacc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < ROWS; ++j) {
      const int n = ty + 16 * j;
      float4* hp = reinterpret_cast<float4*>(hs + n * kSP + 4 * p4);
      const float4 hv = *hp;
      float4 hn = make_float4(alpha * hv.x, alpha * hv.y, alpha * hv.z, alpha * hv.w);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float cb = beta * bp[r * N + n], cc = gamma * sB[r * N + n];
        hn.x += cb * xpr[r].x + cc * xr[r].x;
        hn.y += cb * xpr[r].y + cc * xr[r].y;
        hn.z += cb * xpr[r].z + cc * xr[r].z;
        hn.w += cb * xpr[r].w + cc * xr[r].w;
      }
      *hp = hn;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float cr = sC[r * N + n];
        yacc[r].x += cr * hn.x;
        yacc[r].y += cr * hn.y;
        yacc[r].z += cr * hn.z;
        yacc[r].w += cr * hn.w;
      }
    }
    ptx::fence_proxy_async_smem();  // the new state is read by the bulk store
#pragma unroll
    for (int r = 0; r < R; ++r) {  // the two row groups of this warp
      yacc[r].x += __shfl_xor_sync(0xffffffffu, yacc[r].x, 16);
      yacc[r].y += __shfl_xor_sync(0xffffffffu, yacc[r].y, 16);
      yacc[r].z += __shfl_xor_sync(0xffffffffu, yacc[r].z, 16);
      yacc[r].w += __shfl_xor_sync(0xffffffffu, yacc[r].w, 16);
      if (lane < 16) *reinterpret_cast<float4*>(red + (warp * R + r) * kSP + 4 * p4) = yacc[r];
    }
    __syncthreads();
    if (tid == 0) {
      ptx::bulk_store(a.h + (size_t)u * N * kSP, hs, N * kSP * 4);
      ptx::bulk_commit();
    }
    T* yu = static_cast<T*>(a.y) + (size_t)u * R * kSP;
    for (int i = tid; i < R * kSP; i += kSThreads) {
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < kSThreads / 32; ++w) acc += red[w * R * kSP + i];
      st1(yu + i, acc + Dh * ld1(Xs + i));
    }
    __syncthreads();  // stage s and the partial sums may be reused
  }
  if (tid == 0) {
    // after an abort: the loads already issued land before the CTA exits
    for (int st2 = 0; st2 < 2; ++st2)
      if (inflight[st2] && !ptx::mbar_wait_drain(&bars[st2], ((inflight[st2] - 1) >> 1) & 1))
        report_timeout(&g_decode_status, 2);
    ptx::bulk_wait_all();
  }
}

template <typename T, int N, int R, bool BCN>
int launch_stream_k(const DecodeArgs& a, cudaStream_t s) {
  using S = DStage<T, N, R>;
  auto k = decode_stream_kernel<T, N, R, BCN>;
  static int blocks_per_sm = 0, sms = 0;
  if (blocks_per_sm == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, S::TOTAL) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, k, kSThreads, S::TOTAL) != cudaSuccess ||
        blocks_per_sm < 1)
      return MAMBA3_ERR_CUDA;
  }
  const int units = a.batch * a.nheads;
  const int grid = units < blocks_per_sm * sms ? units : blocks_per_sm * sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = S::TOTAL;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, k, a) != cudaSuccess) return MAMBA3_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

template <typename T, int N, int R>
int launch_stream_t(const DecodeArgs& a, cudaStream_t s) {
  return a.bcnorm ? launch_stream_k<T, N, R, true>(a, s) : launch_stream_k<T, N, R, false>(a, s);
}

bool stream_ok(const DecodeArgs& a) {
  if (a.P != kSP || (a.N != 64 && a.N != 128) || !(a.R == 1 || a.R == 2 || a.R == 4)) return false;
  const uintptr_t all = reinterpret_cast<uintptr_t>(a.h) | reinterpret_cast<uintptr_t>(a.bprev) |
                        reinterpret_cast<uintptr_t>(a.xprev) | reinterpret_cast<uintptr_t>(a.angle) |
                        reinterpret_cast<uintptr_t>(a.B) | reinterpret_cast<uintptr_t>(a.C) |
                        reinterpret_cast<uintptr_t>(a.x) | reinterpret_cast<uintptr_t>(a.theta);
  return (all & 15u) == 0;
}

template <typename T>
int launch_stream(const DecodeArgs& a, cudaStream_t s) {
  if (a.N == 128) {
    if (a.R == 1) return launch_stream_t<T, 128, 1>(a, s);
    if (a.R == 2) return launch_stream_t<T, 128, 2>(a, s);
    return launch_stream_t<T, 128, 4>(a, s);
  }
  if (a.R == 1) return launch_stream_t<T, 64, 1>(a, s);
  if (a.R == 2) return launch_stream_t<T, 64, 2>(a, s);
  return launch_stream_t<T, 64, 4>(a, s);
}

}  // namespace

int decode_status_read_and_clear(int* code) {
  DeviceStatus st, zero = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(&st, g_decode_status, sizeof(st)) != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (st.code != 0 && cudaMemcpyToSymbol(g_decode_status, &zero, sizeof(zero)) != cudaSuccess) return MAMBA3_ERR_CUDA;
  *code = st.code;
  return MAMBA3_OK;
}

int decode_supported(const DecodeArgs& a) {
  if (a.ngroups < 1 || a.nheads % a.ngroups != 0) return MAMBA3_ERR_INVALID;  // B, C rows per token
  if (a.bcnorm && !stream_ok(a)) return MAMBA3_ERR_UNSUPPORTED;  // the fused norm lives in the streaming kernel
  if (a.P % 4 != 0 || a.P / 4 > kThreads || kThreads % (a.P / 4) != 0) return MAMBA3_ERR_UNSUPPORTED;
  const int G = kThreads / (a.P / 4);
  if (a.N > kMaxRows * G) return MAMBA3_ERR_UNSUPPORTED;
  if (!(a.R == 1 || a.R == 2 || a.R == 4 || a.R == 8)) return MAMBA3_ERR_UNSUPPORTED;
  if (decode_smem_bytes(a.P, a.N, a.R) > 200 * 1024) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.batch * a.nheads == 0) return MAMBA3_OK;
  if (stream_ok(a)) return a.dtype == MAMBA3_F32 ? launch_stream<float>(a, s) : launch_stream<__nv_bfloat16>(a, s);
  return a.dtype == MAMBA3_F32 ? launch_r<float>(a, s) : launch_r<__nv_bfloat16>(a, s);
}

}  // namespace m3

// Output side of the layer: pre-gate grouped RMS norm and the gate.
//
// "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section 2:
// hybrids put a grouped RMS norm in front of the output gate.  Per token and
// norm group g (nheads / groups consecutive heads), over the group's channels
// c = (h, r, p), which are contiguous in [b, L, H, R, P]:
//   out[c] = y[c] * rsqrt(mean_c y[c]^2 + eps) * w[h, r, p] * silu(z[c]),
// silu(z) = z / (1 + e^{-z}).  A group of S channels is S contiguous values of y
// and z, and its weights are the S contiguous values w[g * S ...].
//
// HBM-bound: y and z are read once and out written once, 16 bytes per access.
// Groups of up to 128 vectors (power-of-two counts) go to a team of lanes inside
// a warp (shuffle reduction); other groups get one CTA each (shared-memory
// reduction, y and z read again from L2 for the second sweep).
#include "common.cuh"
#include "internal.h"

namespace m3 {
namespace {

constexpr int kTeamThreads = 256;
constexpr int kRowThreads = 256;

template <typename T>
struct Vec;  // one 16-byte access
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  using U = uint4;
  __device__ static void unpack(const U& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 v = __bfloat1622float2(h[i]);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
  __device__ static U pack(const float* f) {
    U u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  using U = float4;
  __device__ static void unpack(const U& u, float* f) {
    f[0] = u.x;
    f[1] = u.y;
    f[2] = u.z;
    f[3] = u.w;
  }
  __device__ static U pack(const float* f) { return make_float4(f[0], f[1], f[2], f[3]); }
};

// silu with the fast exponential and division intrinsics (a few ulp at the sizes
// that reach the gate); for z below about -88 the exponential overflows and the
// quotient is 0, the limit of silu
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// n weights (n a multiple of 4) from a 16-byte aligned address, or 1 without weights
template <int n>
__device__ __forceinline__ void load_w(const float* w, float* out) {
  if (!w) {
#pragma unroll
    for (int e = 0; e < n; ++e) out[e] = 1.f;
    return;
  }
#pragma unroll
  for (int q = 0; q < n / 4; ++q) {
    const float4 t = reinterpret_cast<const float4*>(w)[q];
    out[4 * q] = t.x;
    out[4 * q + 1] = t.y;
    out[4 * q + 2] = t.z;
    out[4 * q + 3] = t.w;
  }
}

// group of a row (rows are (token, group) in order), in 32 bits when the count fits
__device__ __forceinline__ int group_of(long long row, const GatedNormArgs& a) {
  return a.rows <= 0xffffffffLL ? (int)((unsigned)row % (unsigned)a.groups) : (int)(row % a.groups);
}

__device__ __forceinline__ float inv_rms(float sumsq, int S, float eps) {
  const float v = sumsq / (float)S + eps;
  return v > 0.f ? rsqrtf(v) : 0.f;  // an all-zero group with eps = 0 gives 0
}

// Team kernel: TEAM lanes (a power of two <= 32) hold one group, NV vectors each
// (lane m takes vectors m, m + TEAM, ...: coalesced); a lane works on U groups per
// iteration so that 2 U NV loads are in flight before the first reduction.
template <typename T, int TEAM, int NV, int U>
__global__ void __launch_bounds__(kTeamThreads) gated_norm_team_kernel(GatedNormArgs a) {
  using V = Vec<T>;
  constexpr int TPW = 32 / TEAM;  // groups per warp and iteration step
  constexpr int S = TEAM * NV * V::N;
  const int lane = threadIdx.x & 31, member = lane % TEAM, sub = lane / TEAM;
  const long long warp = ((long long)blockIdx.x * kTeamThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kTeamThreads) >> 5;
  const typename V::U* Y = static_cast<const typename V::U*>(a.y);
  const typename V::U* Z = static_cast<const typename V::U*>(a.z);
  typename V::U* O = static_cast<typename V::U*>(a.out);
  // every lane of a warp runs the same iterations (the shuffles need them all)
  for (long long base = warp * TPW * U; base < a.rows; base += nwarps * TPW * U) {
    typename V::U yv[U][NV], zv[U][NV];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * TPW + sub;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        if (row < a.rows) {
          yv[u][v] = Y[row * (TEAM * NV) + v * TEAM + member];
          zv[u][v] = Z[row * (TEAM * NV) + v * TEAM + member];
        } else {
          float zero[V::N] = {};
          yv[u][v] = zv[u][v] = V::pack(zero);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long row = base + u * TPW + sub;
      float ss = 0.f;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float y[V::N];
        V::unpack(yv[u][v], y);
#pragma unroll
        for (int e = 0; e < V::N; ++e) ss += y[e] * y[e];
      }
#pragma unroll
      for (int o = TEAM / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = inv_rms(ss, S, a.eps);
      if (row < a.rows) {
        const float* w = a.w ? a.w + (size_t)group_of(row, a) * S : nullptr;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          float y[V::N], z[V::N], wt[V::N], o[V::N];
          V::unpack(yv[u][v], y);
          V::unpack(zv[u][v], z);
          load_w<V::N>(w ? w + (v * TEAM + member) * V::N : nullptr, wt);
#pragma unroll
          for (int e = 0; e < V::N; ++e) o[e] = y[e] * inv * wt[e] * silu(z[e]);
          O[row * (TEAM * NV) + v * TEAM + member] = V::pack(o);
        }
      }
    }
  }
}

// Row kernel: one CTA per group (grid-stride), any group size; VEC-wide
// accesses when the group size allows, else one element at a time.  The block
// is sized to the group (a multiple of 32 threads, at most kRowThreads).
template <typename T, bool VEC>
__global__ void __launch_bounds__(kRowThreads) gated_norm_row_kernel(GatedNormArgs a) {
  using V = Vec<T>;
  __shared__ float red[kRowThreads / 32];
  __shared__ float s_inv;
  const int S = a.group_size;
  const int W = VEC ? V::N : 1;
  const int nv = S / W;
  const int tid = threadIdx.x, nt = blockDim.x;
  for (long long row = blockIdx.x; row < a.rows; row += gridDim.x) {
    const T* yr = static_cast<const T*>(a.y) + row * S;
    const T* zr = static_cast<const T*>(a.z) + row * S;
    T* orow = static_cast<T*>(a.out) + row * S;
    const float* w = a.w ? a.w + (size_t)group_of(row, a) * S : nullptr;
    float ss = 0.f;
    for (int v = tid; v < nv; v += nt) {
      if (VEC) {
        float y[V::N];
        V::unpack(reinterpret_cast<const typename V::U*>(yr)[v], y);
#pragma unroll
        for (int e = 0; e < V::N; ++e) ss += y[e] * y[e];
      } else {
        const float y = ld1(yr + v);
        ss += y * y;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
      float t = 0.f;
      for (int i = 0; i < nt / 32; ++i) t += red[i];
      s_inv = inv_rms(t, S, a.eps);
    }
    __syncthreads();
    const float inv = s_inv;
    for (int v = tid; v < nv; v += nt) {
      if (VEC) {
        float y[V::N], z[V::N], wt[V::N], o[V::N];
        V::unpack(reinterpret_cast<const typename V::U*>(yr)[v], y);
        V::unpack(reinterpret_cast<const typename V::U*>(zr)[v], z);
        load_w<V::N>(w ? w + v * V::N : nullptr, wt);
#pragma unroll
        for (int e = 0; e < V::N; ++e) o[e] = y[e] * inv * wt[e] * silu(z[e]);
        reinterpret_cast<typename V::U*>(orow)[v] = V::pack(o);
      } else {
        st1(orow + v, ld1(yr + v) * inv * (w ? w[v] : 1.f) * silu(ld1(zr + v)));
      }
    }
    __syncthreads();  // red and s_inv are reused by the next row
  }
}

int grid_for(long long work_blocks) {
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                  cudaSuccess)
      sms = 148;
  }
  const long long cap = 8LL * sms;
  return (int)(work_blocks < cap ? (work_blocks > 0 ? work_blocks : 1) : cap);
}

template <typename T, int TEAM, int NV, int U>
void launch_team(const GatedNormArgs& a, cudaStream_t s) {
  const long long groups_per_block = (long long)(kTeamThreads / TEAM) * U;
  gated_norm_team_kernel<T, TEAM, NV, U>
      <<<grid_for((a.rows + groups_per_block - 1) / groups_per_block), kTeamThreads, 0, s>>>(a);
}

template <typename T>
int launch_t(const GatedNormArgs& a, cudaStream_t s) {
  using V = Vec<T>;
  const int S = a.group_size;
  const int nv = S % V::N == 0 ? S / V::N : 0;  // 16-byte vectors per group
  switch (nv) {
    case 1: launch_team<T, 1, 1, 4>(a, s); break;
    case 2: launch_team<T, 2, 1, 4>(a, s); break;
    case 4: launch_team<T, 4, 1, 4>(a, s); break;
    case 8: launch_team<T, 8, 1, 4>(a, s); break;
    case 16: launch_team<T, 16, 1, 4>(a, s); break;
    case 32: launch_team<T, 32, 1, 4>(a, s); break;
    case 64: launch_team<T, 32, 2, 2>(a, s); break;
    case 128: launch_team<T, 32, 4, 1>(a, s); break;
    default: {
      const int work = nv ? nv : S;
      int threads = (work + 31) / 32 * 32;
      threads = threads < kRowThreads ? threads : kRowThreads;
      if (nv)
        gated_norm_row_kernel<T, true><<<grid_for(a.rows), threads, 0, s>>>(a);
      else
        gated_norm_row_kernel<T, false><<<grid_for(a.rows), threads, 0, s>>>(a);
    }
  }
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // namespace

int launch_gated_norm(const GatedNormArgs& a, cudaStream_t s) {
  if (a.rows == 0) return MAMBA3_OK;
  return a.dtype == MAMBA3_F32 ? launch_t<float>(a, s) : launch_t<__nv_bfloat16>(a, s);
}

}  // namespace m3

// Shared device helpers for the Mamba-3 recurrence kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mamba3.h"

namespace m3 {

constexpr float kPi = 3.14159265358979323846f;
constexpr float kTwoPi = 6.28318530717958647692f;
constexpr float kInvTwoPi = 0.15915494309189533577f;
constexpr float kLog2e = 1.44269504088896340736f;

// Element loads/stores for the two input dtypes.
__device__ __forceinline__ float ld1(const float* p) { return *p; }
__device__ __forceinline__ float ld1(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void st1(float* p, float v) { *p = v; }
__device__ __forceinline__ void st1(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

// Four consecutive elements (16-byte aligned for float, 8-byte for bf16).
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  return make_float4(fa.x, fa.y, fb.x, fb.y);
}
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
  __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// Wrap an angle to [-pi, pi] with one fp32 reduction step; the angles fed to
// it are sums of a wrapped angle and a bounded increment, so one step suffices.
__device__ __forceinline__ float wrap_angle(float a) { return a - kTwoPi * rintf(a * kInvTwoPi); }

// Device status word at the start of the prefill workspace.
struct DeviceStatus {
  int code;   // MAMBA3_OK or MAMBA3_ERR_TIMEOUT
  int where;  // which wait gave up (kernel-specific tag)
  int block;  // blockIdx.x of the first reporter
  int pad;
};

__device__ __forceinline__ void report_timeout(DeviceStatus* st, int where) {
  if (st && atomicCAS(&st->code, 0, (int)MAMBA3_ERR_TIMEOUT) == 0) {
    st->where = where;
    st->block = (int)blockIdx.x;
  }
}

}  // namespace m3

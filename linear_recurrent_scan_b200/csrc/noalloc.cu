// mamba3_scan_fwd_noalloc: the prefill with library-owned scratch, for callers
// that cannot allocate device memory themselves.  The scratch is a file-scope
// device array; nothing here allocates or frees.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

// Shared by every call on a device; holds the device status word at offset 0.
static __device__ __align__(256) unsigned char g_scan_scratch[MAMBA3_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices];  // device address per device ordinal, null until looked up

// In host code `g_scan_scratch` is only a host-side stand-in for the device
// array; a kernel must be given the device address, looked up once per device
// with that device current.
int scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MAMBA3_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scan_scratch) != cudaSuccess || p == nullptr) return MAMBA3_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MAMBA3_OK;
}

}  // namespace

extern "C" int mamba3_scan_fwd_noalloc(const mamba3_dims* dims, const void* x, const void* B, const void* C,
                                       const void* theta, const void* dt, const void* lam, const float* A,
                                       const float* D, const mamba3_state* init, void* y,
                                       const mamba3_state* final_state, void* stream) {
  const size_t need = mamba3_scan_workspace_bytes(dims);
  if (need == 0) return MAMBA3_ERR_INVALID;
  if (need > MAMBA3_NOALLOC_SCRATCH_BYTES) return MAMBA3_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = scratch_for_current_device(&scratch);
  if (rc != MAMBA3_OK) return rc;
  // mamba3_scan_fwd clears the status word on `stream` before its kernels run
  return m3::scan_fwd_shared_scratch(dims, x, B, C, theta, dt, lam, A, D, init, y, final_state, scratch,
                                     MAMBA3_NOALLOC_SCRATCH_BYTES, stream);
}

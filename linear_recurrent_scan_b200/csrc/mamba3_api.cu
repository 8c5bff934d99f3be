// C ABI of the Mamba-3 recurrence library: argument validation and dispatch.
// Every check runs on the host before anything is enqueued; the library never
// allocates and never synchronises (except mamba3_device_status).
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kStatusBytes = m3::kStatusBlockBytes;

// Process-wide settings of the bounded device waits (mamba3_set_wait_limit,
// mamba3_test_withhold_loads), read at every launch.
constexpr long long kDefaultWaitLimit = 4000000000LL;  // SM cycles, about 2 s at 1.9 GHz
volatile long long g_wait_limit = kDefaultWaitLimit;
volatile int g_test_withhold = 0;
volatile int g_test_segments = 0;  // mamba3_test_set_segments: 0 = the library's choice

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_dims(const mamba3_dims* d, bool need_seqlen) {
  if (!d) return MAMBA3_ERR_INVALID;
  if (d->batch < 1 || d->nheads < 1 || d->headdim < 4 || d->dstate < 2) return MAMBA3_ERR_INVALID;
  if (need_seqlen && d->seqlen < 0) return MAMBA3_ERR_INVALID;
  if (d->headdim % 4 != 0 || d->dstate % 2 != 0) return MAMBA3_ERR_INVALID;
  if (!(d->rank == 1 || d->rank == 2 || d->rank == 4 || d->rank == 8)) return MAMBA3_ERR_INVALID;
  if (d->in_dtype != MAMBA3_F32 && d->in_dtype != MAMBA3_BF16) return MAMBA3_ERR_INVALID;
  if (need_seqlen && d->chunk < 0) return MAMBA3_ERR_INVALID;
  if (d->ngroups < 0 || (d->ngroups > 0 && d->nheads % d->ngroups != 0)) return MAMBA3_ERR_INVALID;
  // every flattened index must fit comfortably in 64 bits and the grid in 31
  const double tokens = (double)d->batch * (need_seqlen ? (d->seqlen > 0 ? d->seqlen : 1) : 1) * d->nheads;
  const double row = (double)d->rank * (d->dstate > d->headdim ? d->dstate : d->headdim);
  if (tokens * row > 9.0e15 || (double)d->batch * d->nheads > 2.0e9) return MAMBA3_ERR_INVALID;
  if (d->dstate > 1024 || d->headdim > 1024) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

// B, C rows per (batch, token): 0 in the dims means one per head.
int bc_groups(const mamba3_dims* d) { return d->ngroups > 0 ? d->ngroups : d->nheads; }

int check_state(const mamba3_state* s) {
  if (!s) return MAMBA3_OK;
  if (!s->h || !s->b_prev || !s->x_prev || !s->angle) return MAMBA3_ERR_INVALID;
  if (!aligned16(s->h) || !aligned16(s->b_prev) || !aligned16(s->x_prev) || !aligned4(s->angle))
    return MAMBA3_ERR_INVALID;
  return MAMBA3_OK;
}

int check_inputs(const void* x, const void* B, const void* C, const void* theta, const void* dt,
                 const void* lam, const float* A, const float* D, const void* y) {
  if (!x || !B || !C || !theta || !dt || !lam || !A || !y) return MAMBA3_ERR_INVALID;
  if (!aligned16(x) || !aligned16(B) || !aligned16(C) || !aligned16(theta) || !aligned16(y))
    return MAMBA3_ERR_INVALID;
  if (!aligned4(dt) || !aligned4(lam) || !aligned4(A) || (D && !aligned4(D))) return MAMBA3_ERR_INVALID;
  return MAMBA3_OK;
}

bool norm_ok(const mamba3_bc_norm* n) {
  if (!n || !(n->eps >= 0.f)) return false;
  return aligned4(n->w_B) && aligned4(n->w_C) && aligned4(n->bias_B) && aligned4(n->bias_C);
}

// mamba3_test_set_segments: S when it divides seqlen and the shape has the
// segmented path, else 0
int forced_segments(const m3::ScanArgs& a) {
  const int S = g_test_segments;
  if (S < 2 || a.seqlen % S != 0 || m3::tc_scan_supported(a) != MAMBA3_OK || m3::bwd_tc_supported(a) != MAMBA3_OK ||
      a.bcnorm)
    return 0;
  return S;
}

template <typename Args>
void set_norm(Args& a, const mamba3_bc_norm* n) {
  a.bcnorm = 1;
  a.nw_B = n->w_B; a.nw_C = n->w_C; a.nb_B = n->bias_B; a.nb_C = n->bias_C;
  a.neps = n->eps;
}

}  // namespace

extern "C" {

int mamba3_version(void) { return 200; }

const char* mamba3_status_string(int status) {
  switch (status) {
    case MAMBA3_OK: return "ok";
    case MAMBA3_ERR_INVALID: return "invalid argument (null pointer, bad size or misaligned pointer)";
    case MAMBA3_ERR_UNSUPPORTED: return "shape not supported by the compiled kernels";
    case MAMBA3_ERR_WORKSPACE: return "workspace missing or too small";
    case MAMBA3_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MAMBA3_ERR_TIMEOUT: return "a bounded on-device wait gave up";
  }
  return "unknown status";
}

size_t mamba3_scan_workspace_bytes(const mamba3_dims* d) {
  if (check_dims(d, true) != MAMBA3_OK) return 0;
  return kStatusBytes;
}

}  // extern "C"

namespace {
// The forward arguments common to the prefill and its backward pass.
m3::ScanArgs scan_args(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                       const void* dt, const void* lam, const float* A, const float* D, const mamba3_state* init) {
  m3::ScanArgs a;
  memset(&a, 0, sizeof(a));
  a.batch = d->batch;
  a.seqlen = d->seqlen;
  a.nheads = d->nheads;
  a.P = d->headdim;
  a.N = d->dstate;
  a.R = d->rank;
  a.Q = d->chunk;
  a.ngroups = bc_groups(d);
  a.dtype = d->in_dtype;
  a.x = x; a.B = B; a.C = C; a.theta = theta; a.dt = dt; a.lam = lam; a.A = A; a.D = D;
  if (init) { a.h0 = init->h; a.bprev0 = init->b_prev; a.xprev0 = init->x_prev; a.angle0 = init->angle; }
  a.wait_limit = g_wait_limit;
  a.test_withhold = g_test_withhold;
  return a;
}

// The prefill behind mamba3_scan_fwd (A per head), mamba3_scan_fwd_at (A_t per
// token; A null) and mamba3_scan_fwd_bcnorm (norm non-null, already checked).
int scan_fwd_impl(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                  const void* dt, const void* lam, const float* A, const void* A_t, const float* D,
                  const mamba3_bc_norm* norm, const mamba3_state* init, void* y,
                  const mamba3_state* final_state, void* workspace, size_t workspace_bytes, void* stream,
                  bool allow_split = true) {
  int rc = check_dims(d, true);
  if (rc) return rc;
  const float* A_chk = A ? A : static_cast<const float*>(A_t);  // the rate array that must be present
  if (d->seqlen > 0 && (rc = check_inputs(x, B, C, theta, dt, lam, A_chk, D, y))) return rc;
  if (d->seqlen == 0 && !A_chk) return MAMBA3_ERR_INVALID;
  if ((rc = check_state(init)) || (rc = check_state(final_state))) return rc;
  if (!workspace || !aligned16(workspace)) return MAMBA3_ERR_WORKSPACE;
  if (workspace_bytes < mamba3_scan_workspace_bytes(d)) return MAMBA3_ERR_WORKSPACE;

  m3::ScanArgs a = scan_args(d, x, B, C, theta, dt, lam, A, D, init);
  a.A_t = A_t;
  a.y = y;
  if (final_state) {
    a.h_out = final_state->h; a.bprev_out = final_state->b_prev;
    a.xprev_out = final_state->x_prev; a.angle_out = final_state->angle;
  }
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  if (norm && d->seqlen > 0) set_norm(a, norm);  // with no tokens there is nothing to normalise

  const bool use_tc = m3::tc_scan_supported(a) == MAMBA3_OK;
  if (!use_tc && a.bcnorm) return MAMBA3_ERR_UNSUPPORTED;  // the fused form is tensor-core only
  if (!use_tc && (rc = m3::simt_scan_supported(a))) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc) {  // a long sequence over few units runs in segments when the workspace allows it
    const int S = g_test_segments ? forced_segments(a) : m3::seg_count(a, m3::kSMs);
    if (S > 0 && workspace_bytes >= kStatusBytes + m3::seg_workspace_bytes(a, S)) {
      if (cudaMemsetAsync(workspace, 0, sizeof(m3::DeviceStatus), s) != cudaSuccess) return MAMBA3_ERR_CUDA;
      return m3::launch_scan_segmented(a, S, s);
    }
  }
  // otherwise the tensor-core prefill splits its last wave when the workspace allows it
  size_t zero = sizeof(m3::DeviceStatus);
  if (use_tc && allow_split && d->seqlen > 0) {
    const size_t sb = m3::tc_split_bytes(a);
    if (sb > 0 && workspace_bytes >= kStatusBytes + sb) {
      a.split = 1;
      zero = m3::tc_split_zero_bytes(a);
    }
  }
  if (cudaMemsetAsync(workspace, 0, zero, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  return use_tc ? m3::launch_scan_tc(a, s) : m3::launch_scan_simt(a, s);
}

// The decode step behind mamba3_decode_step, mamba3_decode_step_at and
// mamba3_decode_step_bcnorm (norm non-null, already checked).
int decode_impl(const mamba3_dims* d, const mamba3_state* state, const void* x, const void* B, const void* C,
                const void* theta, const void* dt, const void* lam, const float* A, const void* A_t,
                const float* D, const mamba3_bc_norm* norm, void* y, void* stream) {
  int rc = check_dims(d, false);
  if (rc) return rc;
  if (!state) return MAMBA3_ERR_INVALID;
  if ((rc = check_state(state))) return rc;
  const float* A_chk = A ? A : static_cast<const float*>(A_t);
  if ((rc = check_inputs(x, B, C, theta, dt, lam, A_chk, D, y))) return rc;
  m3::DecodeArgs a;
  memset(&a, 0, sizeof(a));
  a.batch = d->batch;
  a.nheads = d->nheads;
  a.P = d->headdim;
  a.N = d->dstate;
  a.R = d->rank;
  a.ngroups = bc_groups(d);
  a.dtype = d->in_dtype;
  a.h = state->h; a.bprev = state->b_prev; a.xprev = state->x_prev; a.angle = state->angle;
  a.x = x; a.B = B; a.C = C; a.theta = theta; a.dt = dt; a.lam = lam; a.A = A; a.A_t = A_t; a.D = D; a.y = y;
  if (norm) set_norm(a, norm);
  a.wait_limit = g_wait_limit;
  a.test_withhold = g_test_withhold;
  if ((rc = m3::decode_supported(a))) return rc;
  return m3::launch_decode(a, static_cast<cudaStream_t>(stream));
}
}  // namespace

extern "C" {

int mamba3_scan_fwd(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                    const void* dt, const void* lam, const float* A, const float* D,
                    const mamba3_state* init, void* y, const mamba3_state* final_state, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return scan_fwd_impl(d, x, B, C, theta, dt, lam, A, nullptr, D, nullptr, init, y, final_state, workspace,
                       workspace_bytes, stream);
}

}  // extern "C"

namespace m3 {
int scan_fwd_shared_scratch(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                            const void* dt, const void* lam, const float* A, const float* D,
                            const mamba3_state* init, void* y, const mamba3_state* final_state, void* scratch,
                            size_t scratch_bytes, void* stream) {
  return scan_fwd_impl(d, x, B, C, theta, dt, lam, A, nullptr, D, nullptr, init, y, final_state, scratch,
                       scratch_bytes, stream, /*allow_split=*/false);
}
}  // namespace m3

extern "C" {

int mamba3_scan_fwd_at(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                       const void* dt, const void* lam, const void* A_t, const float* D, const mamba3_state* init,
                       void* y, const mamba3_state* final_state, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!A_t) return MAMBA3_ERR_INVALID;
  return scan_fwd_impl(d, x, B, C, theta, dt, lam, nullptr, A_t, D, nullptr, init, y, final_state, workspace,
                       workspace_bytes, stream);
}

int mamba3_decode_step_at(const mamba3_dims* d, const mamba3_state* state, const void* x, const void* B,
                          const void* C, const void* theta, const void* dt, const void* lam, const void* A_t,
                          const float* D, void* y, void* stream) {
  if (!A_t) return MAMBA3_ERR_INVALID;
  return decode_impl(d, state, x, B, C, theta, dt, lam, nullptr, A_t, D, nullptr, y, stream);
}

int mamba3_scan_fwd_bcnorm(const mamba3_dims* d, const void* x, const void* B_raw, const void* C_raw,
                           const void* theta, const void* dt, const void* lam, const float* A, const float* D,
                           const mamba3_bc_norm* norm, const mamba3_state* init, void* y,
                           const mamba3_state* final_state, void* workspace, size_t workspace_bytes, void* stream) {
  if (!norm_ok(norm)) return MAMBA3_ERR_INVALID;
  return scan_fwd_impl(d, x, B_raw, C_raw, theta, dt, lam, A, nullptr, D, norm, init, y, final_state, workspace,
                       workspace_bytes, stream);
}

int mamba3_decode_step_bcnorm(const mamba3_dims* d, const mamba3_state* state, const void* x, const void* B_raw,
                              const void* C_raw, const void* theta, const void* dt, const void* lam, const float* A,
                              const float* D, const mamba3_bc_norm* norm, void* y, void* stream) {
  if (!norm_ok(norm)) return MAMBA3_ERR_INVALID;
  return decode_impl(d, state, x, B_raw, C_raw, theta, dt, lam, A, nullptr, D, norm, y, stream);
}

int mamba3_decode_step(const mamba3_dims* d, const mamba3_state* state, const void* x, const void* B,
                       const void* C, const void* theta, const void* dt, const void* lam, const float* A,
                       const float* D, void* y, void* stream) {
  return decode_impl(d, state, x, B, C, theta, dt, lam, A, nullptr, D, nullptr, y, stream);
}

int mamba3_library_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MAMBA3_ERR_CUDA;
  int dec = 0, proj = 0;
  int rc = m3::decode_status_read_and_clear(&dec);
  if (rc == MAMBA3_OK) rc = m3::proj_status_read_and_clear(&proj);
  if (rc != MAMBA3_OK) return rc;
  return dec != 0 ? dec : proj;
}

namespace {
int mimo_proj_impl(const mamba3_dims* d, int up, const void* in, const void* weight, const void* z, const float* w,
                   float eps, void* out, void* stream) {
  if (!d || d->batch < 1 || d->seqlen < 0 || d->nheads < 1) return MAMBA3_ERR_INVALID;
  if (!(d->rank == 1 || d->rank == 2 || d->rank == 4 || d->rank == 8)) return MAMBA3_ERR_INVALID;
  if (d->in_dtype != MAMBA3_F32 && d->in_dtype != MAMBA3_BF16) return MAMBA3_ERR_INVALID;
  if (!(eps >= 0.f)) return MAMBA3_ERR_INVALID;
  const double tokens = (double)d->batch * d->seqlen;
  if (tokens * d->nheads * d->rank * d->headdim > 9.0e15 || tokens > 2.0e9) return MAMBA3_ERR_INVALID;
  if (d->in_dtype != MAMBA3_BF16 || d->headdim != 64 || d->rank == 8) return MAMBA3_ERR_UNSUPPORTED;
  if (tokens > 0) {
    if (!in || !weight || !out || !aligned16(in) || !aligned16(weight) || !aligned16(out)) return MAMBA3_ERR_INVALID;
    if (z && !aligned16(z)) return MAMBA3_ERR_INVALID;
    if (w && !aligned4(w)) return MAMBA3_ERR_INVALID;
  }
  m3::ProjArgs a;
  memset(&a, 0, sizeof(a));
  a.tokens = (long long)d->batch * d->seqlen;
  a.nheads = d->nheads;
  a.R = d->rank;
  a.up = up;
  a.in = in; a.weight = weight; a.out = out; a.z = z; a.w = w; a.eps = eps;
  a.wait_limit = g_wait_limit;
  a.test_withhold = g_test_withhold;
  return m3::launch_mimo_proj(a, static_cast<cudaStream_t>(stream));
}
}  // namespace

int mamba3_mimo_up(const mamba3_dims* d, const void* u, const void* Wx, void* x, void* stream) {
  return mimo_proj_impl(d, 1, u, Wx, nullptr, nullptr, 0.f, x, stream);
}

int mamba3_mimo_down(const mamba3_dims* d, const void* y, const void* Wy, const void* z, const float* w, float eps,
                     void* out, void* stream) {
  return mimo_proj_impl(d, 0, y, Wy, z, w, eps, out, stream);
}

int mamba3_set_wait_limit(long long cycles) {
  if (cycles < 1000) return MAMBA3_ERR_INVALID;
  g_wait_limit = cycles;
  return MAMBA3_OK;
}

int mamba3_test_withhold_loads(int on) {
  g_test_withhold = on ? 1 : 0;
  return MAMBA3_OK;
}

size_t mamba3_scan_segmented_workspace_bytes(const mamba3_dims* d) {
  if (check_dims(d, true) != MAMBA3_OK) return 0;
  m3::ScanArgs a = scan_args(d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  const int S = g_test_segments ? forced_segments(a) : m3::seg_count(a, m3::kSMs);
  return kStatusBytes + m3::seg_workspace_bytes(a, S);
}

size_t mamba3_scan_fwd_workspace_bytes(const mamba3_dims* d) {
  if (check_dims(d, true) != MAMBA3_OK) return 0;
  m3::ScanArgs a = scan_args(d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  const int S = g_test_segments ? forced_segments(a) : m3::seg_count(a, m3::kSMs);
  if (S > 0) return kStatusBytes + m3::seg_workspace_bytes(a, S);
  return kStatusBytes + (d->seqlen > 0 ? m3::tc_split_bytes(a) : 0);
}

int mamba3_test_set_split(int k, int c1) {
  if (k > 0 && c1 < 1) return MAMBA3_ERR_INVALID;
  m3::tc_force_split(k, c1);
  return MAMBA3_OK;
}

int mamba3_test_set_segments(int S) {
  if (S < 0) return MAMBA3_ERR_INVALID;
  g_test_segments = S;
  return MAMBA3_OK;
}

int mamba3_device_status(const void* workspace, void* stream) {
  if (!workspace) return MAMBA3_ERR_INVALID;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  m3::DeviceStatus st;
  if (cudaMemcpy(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return MAMBA3_ERR_CUDA;
  return st.code;
}

}  // extern "C"

namespace {
// The backward pass behind mamba3_scan_bwd (A per head, dA) and mamba3_scan_bwd_at
// (A_t per token, dA_t); the rate and its gradient were checked by the caller.
int scan_bwd_impl(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                  const void* dt, const void* lam, const float* A, const void* A_t, const float* D,
                  const mamba3_state* init, const void* dy, const mamba3_state* d_final, void* dx, void* dB,
                  void* dC, void* dtheta, void* ddt, void* dlam, float* dA, void* dA_t, float* dD,
                  const mamba3_state* d_init, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(d, true);
  if (rc) return rc;
  if (dD && !aligned4(dD)) return MAMBA3_ERR_INVALID;
  const float* rate = A ? A : static_cast<const float*>(A_t);  // the rate array that must be present
  if (d->seqlen > 0) {
    if ((rc = check_inputs(x, B, C, theta, dt, lam, rate, D, dy))) return rc;
    if ((rc = check_inputs(dx, dB, dC, dtheta, ddt, dlam, rate, D, dy))) return rc;  // the gradients' layouts
  }
  if ((rc = check_state(init)) || (rc = check_state(d_final)) || (rc = check_state(d_init))) return rc;
  if (!workspace || !aligned16(workspace)) return MAMBA3_ERR_WORKSPACE;
  m3::ScanArgs sizes = scan_args(d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                                 nullptr);
  const bool use_tc = m3::bwd_tc_supported(sizes) == MAMBA3_OK;
  const size_t ckpt_bytes = m3::bwd_checkpoint_bytes(sizes);
  const size_t need = use_tc ? m3::bwd_tc_workspace_bytes(sizes) : ckpt_bytes + m3::bwd_group_bytes(sizes);
  if (workspace_bytes < kStatusBytes + need) return MAMBA3_ERR_WORKSPACE;
  m3::BwdArgs g;
  memset(&g, 0, sizeof(g));
  g.f = scan_args(d, x, B, C, theta, dt, lam, A, D, init);
  g.f.A_t = A_t;
  g.f.workspace = workspace;
  g.f.workspace_bytes = workspace_bytes;
  if ((rc = m3::bwd_supported(g.f))) return rc;
  g.dy = dy;
  if (d_final) {
    g.dh_out = d_final->h; g.dbprev_out = d_final->b_prev; g.dxprev_out = d_final->x_prev; g.dangle_out = d_final->angle;
  }
  g.dx = dx; g.dB = dB; g.dC = dC; g.dtheta = dtheta; g.ddt = ddt; g.dlam = dlam; g.dA = dA; g.dA_t = dA_t; g.dD = dD;
  if (d_init) { g.dh0 = d_init->h; g.dbprev0 = d_init->b_prev; g.dxprev0 = d_init->x_prev; g.dangle0 = d_init->angle; }
  g.ckpt = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc) {
    // the chunk kernel splits its last wave when the workspace holds the hand-over
    const size_t sb = d->seqlen > 0 ? m3::bwd_tc_split_bytes(sizes) : 0;
    g.split = sb > 0 && workspace_bytes >= kStatusBytes + need + sb;
    if (cudaMemsetAsync(workspace, 0, sizeof(m3::DeviceStatus), s) != cudaSuccess) return MAMBA3_ERR_CUDA;
    return m3::launch_scan_bwd_tc(g, s);
  }
  if (m3::bwd_group_bytes(sizes)) {
    g.dBh = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes + ckpt_bytes);
    g.dCh = g.dBh + (size_t)d->batch * d->seqlen * bc_groups(d) * d->rank * d->dstate;
  }
  if (cudaMemsetAsync(workspace, 0, sizeof(m3::DeviceStatus), s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  return m3::launch_scan_bwd(g, s);
}
}  // namespace

extern "C" {

size_t mamba3_scan_bwd_workspace_bytes(const mamba3_dims* d) {
  if (check_dims(d, true) != MAMBA3_OK) return 0;
  const m3::ScanArgs a = scan_args(d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  if (m3::bwd_tc_supported(a) == MAMBA3_OK)  // (with the split last wave's hand-over where it applies)
    return kStatusBytes + m3::bwd_tc_workspace_bytes(a) + (d->seqlen > 0 ? m3::bwd_tc_split_bytes(a) : 0);
  return kStatusBytes + m3::bwd_checkpoint_bytes(a) + m3::bwd_group_bytes(a);
}

int mamba3_scan_bwd(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                    const void* dt, const void* lam, const float* A, const float* D, const mamba3_state* init,
                    const void* dy, const mamba3_state* d_final, void* dx, void* dB, void* dC, void* dtheta,
                    void* ddt, void* dlam, float* dA, float* dD, const mamba3_state* d_init, void* workspace,
                    size_t workspace_bytes, void* stream) {
  if (!A || !dA || !aligned4(dA)) return MAMBA3_ERR_INVALID;
  return scan_bwd_impl(d, x, B, C, theta, dt, lam, A, nullptr, D, init, dy, d_final, dx, dB, dC, dtheta, ddt, dlam,
                       dA, nullptr, dD, d_init, workspace, workspace_bytes, stream);
}

int mamba3_scan_bwd_at(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                       const void* dt, const void* lam, const void* A_t, const float* D, const mamba3_state* init,
                       const void* dy, const mamba3_state* d_final, void* dx, void* dB, void* dC, void* dtheta,
                       void* ddt, void* dlam, void* dA_t, float* dD, const mamba3_state* d_init, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (!A_t || !dA_t || !aligned4(A_t) || !aligned4(dA_t)) return MAMBA3_ERR_INVALID;
  return scan_bwd_impl(d, x, B, C, theta, dt, lam, nullptr, A_t, D, init, dy, d_final, dx, dB, dC, dtheta, ddt, dlam,
                       nullptr, dA_t, dD, d_init, workspace, workspace_bytes, stream);
}

int mamba3_gated_norm(const mamba3_dims* d, int groups, const void* y, const void* z, const float* w, float eps,
                      void* out, void* stream) {
  if (!d || d->batch < 1 || d->seqlen < 0 || d->nheads < 1 || d->headdim < 1 || d->rank < 1) return MAMBA3_ERR_INVALID;
  if (d->in_dtype != MAMBA3_F32 && d->in_dtype != MAMBA3_BF16) return MAMBA3_ERR_INVALID;
  if (groups < 1 || d->nheads % groups != 0 || !(eps >= 0.f)) return MAMBA3_ERR_INVALID;
  const double total = (double)d->batch * d->seqlen * d->nheads * d->rank * d->headdim;
  if (total > 9.0e15 || (double)d->nheads / groups * d->rank * d->headdim > 2.0e9) return MAMBA3_ERR_INVALID;
  m3::GatedNormArgs a;
  a.rows = (long long)d->batch * d->seqlen * groups;
  a.groups = groups;
  a.group_size = d->nheads / groups * d->rank * d->headdim;
  a.dtype = d->in_dtype;
  a.y = y; a.z = z; a.w = w; a.eps = eps; a.out = out;
  if (a.rows > 0) {
    if (!y || !z || !out || !aligned16(y) || !aligned16(z) || !aligned16(out)) return MAMBA3_ERR_INVALID;
    if (w && !aligned16(w)) return MAMBA3_ERR_INVALID;
  }
  return m3::launch_gated_norm(a, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------- the prefill from host buffers
namespace {

constexpr int kHostSplits = 8;  // sub-batches the host prefill cycles through the stage

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// The sub-batches of mamba3_scan_fwd_host (bs batch rows each, nb of them) and the
// device stage: the status word, then two slots of one sub-batch's x, y, B, C,
// theta, dt and lam.
struct HostLayout {
  int nb, bs;
  size_t x_row, bc_row, th_row, dl_row;  // bytes of one batch row of x (and y), B (and C), theta, dt (and lam)
  size_t x, bc, th, dl;                  // aligned bytes of one sub-batch of each
  size_t slot, total;
};

HostLayout host_layout(const mamba3_dims* d) {
  HostLayout l;
  l.nb = d->batch < kHostSplits ? d->batch : kHostSplits;
  l.bs = (d->batch + l.nb - 1) / l.nb;
  l.nb = (d->batch + l.bs - 1) / l.bs;
  const size_t es = d->in_dtype == MAMBA3_BF16 ? 2 : 4;
  const size_t L = d->seqlen, H = d->nheads, R = d->rank, P = d->headdim, N = d->dstate, G = bc_groups(d);
  l.x_row = L * H * R * P * es;
  l.bc_row = L * G * R * N * es;
  l.th_row = L * H * (N / 2) * es;
  l.dl_row = L * H * es;
  l.x = align256(l.bs * l.x_row);
  l.bc = align256(l.bs * l.bc_row);
  l.th = align256(l.bs * l.th_row);
  l.dl = align256(l.bs * l.dl_row);
  l.slot = 2 * l.x + 2 * l.bc + l.th + 2 * l.dl;
  l.total = kStatusBytes + 2 * l.slot;
  return l;
}

// Streams and events of one call (created per call, so that calls on different
// streams never share them; destroying them does not wait for their work).
struct HostPipe {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr, in[2] = {nullptr, nullptr}, done[2] = {nullptr, nullptr}, out[2] = {nullptr, nullptr};
  bool ok = true;
  HostPipe() {
    const unsigned f = cudaEventDisableTiming;
    ok = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&start, f) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaEventCreateWithFlags(&in[i], f) == cudaSuccess && cudaEventCreateWithFlags(&done[i], f) == cudaSuccess &&
           cudaEventCreateWithFlags(&out[i], f) == cudaSuccess;
  }
  ~HostPipe() {
    for (int i = 0; i < 2; ++i) {
      if (in[i]) cudaEventDestroy(in[i]);
      if (done[i]) cudaEventDestroy(done[i]);
      if (out[i]) cudaEventDestroy(out[i]);
    }
    if (start) cudaEventDestroy(start);
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
  }
};

mamba3_state state_rows(const mamba3_state* s, const mamba3_dims* d, int r0) {
  mamba3_state o;
  const size_t H = d->nheads, N = d->dstate, P = d->headdim, R = d->rank;
  o.h = s->h + r0 * H * N * P;
  o.b_prev = s->b_prev + r0 * H * R * N;
  o.x_prev = s->x_prev + r0 * H * R * P;
  o.angle = s->angle + r0 * H * (N / 2);
  return o;
}

}  // namespace

extern "C" {

size_t mamba3_scan_fwd_host_stage_bytes(const mamba3_dims* d) {
  if (check_dims(d, true) != MAMBA3_OK) return 0;
  return host_layout(d).total;
}

int mamba3_scan_fwd_host(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                         const void* dt, const void* lam, const float* A, const float* D, const mamba3_state* init,
                         void* y, const mamba3_state* final_state, void* stage, size_t stage_bytes, void* stream) {
  int rc = check_dims(d, true);
  if (rc) return rc;
  if (!A || !aligned4(A) || (D && !aligned4(D))) return MAMBA3_ERR_INVALID;
  if ((rc = check_state(init)) || (rc = check_state(final_state))) return rc;
  if (!stage || !aligned16(stage)) return MAMBA3_ERR_WORKSPACE;
  const HostLayout l = host_layout(d);
  if (stage_bytes < l.total) return MAMBA3_ERR_WORKSPACE;
  if (d->seqlen == 0)  // nothing to copy: the state passes through as in the device call
    return scan_fwd_impl(d, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, A, nullptr, D, nullptr, init,
                         nullptr, final_state, stage, stage_bytes, stream);
  if (!x || !B || !C || !theta || !dt || !lam || !y) return MAMBA3_ERR_INVALID;
  // the kernel family for the whole problem (every sub-batch takes the same one)
  uint8_t* base = static_cast<uint8_t*>(stage);
  m3::ScanArgs probe = scan_args(d, base, base, base, base, base, base, A, D, init);
  const bool use_tc = m3::tc_scan_supported(probe) == MAMBA3_OK;
  if (!use_tc && (rc = m3::simt_scan_supported(probe))) return rc;

  HostPipe p;
  if (!p.ok) return MAMBA3_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaMemcpyKind h2d = cudaMemcpyHostToDevice, d2h = cudaMemcpyDeviceToHost;
  bool ok = cudaMemsetAsync(stage, 0, sizeof(m3::DeviceStatus), s) == cudaSuccess &&
            cudaEventRecord(p.start, s) == cudaSuccess && cudaStreamWaitEvent(p.up, p.start, 0) == cudaSuccess &&
            cudaStreamWaitEvent(p.down, p.start, 0) == cudaSuccess;
  for (int i = 0; ok && i < l.nb; ++i) {
    const int r0 = i * l.bs, rows = (d->batch - r0) < l.bs ? (d->batch - r0) : l.bs, slot = i & 1;
    uint8_t* sx = base + kStatusBytes + slot * l.slot;
    uint8_t* sy = sx + l.x;
    uint8_t* sB = sy + l.x;
    uint8_t* sC = sB + l.bc;
    uint8_t* sth = sC + l.bc;
    uint8_t* sdt = sth + l.th;
    uint8_t* slm = sdt + l.dl;
    // inputs of sub-batch i into the slot once the prefill of sub-batch i - 2 has read it
    if (i >= 2) ok = cudaStreamWaitEvent(p.up, p.done[slot], 0) == cudaSuccess;
    ok = ok && cudaMemcpyAsync(sx, static_cast<const uint8_t*>(x) + r0 * l.x_row, rows * l.x_row, h2d, p.up) == cudaSuccess &&
         cudaMemcpyAsync(sB, static_cast<const uint8_t*>(B) + r0 * l.bc_row, rows * l.bc_row, h2d, p.up) == cudaSuccess &&
         cudaMemcpyAsync(sC, static_cast<const uint8_t*>(C) + r0 * l.bc_row, rows * l.bc_row, h2d, p.up) == cudaSuccess &&
         cudaMemcpyAsync(sth, static_cast<const uint8_t*>(theta) + r0 * l.th_row, rows * l.th_row, h2d, p.up) == cudaSuccess &&
         cudaMemcpyAsync(sdt, static_cast<const uint8_t*>(dt) + r0 * l.dl_row, rows * l.dl_row, h2d, p.up) == cudaSuccess &&
         cudaMemcpyAsync(slm, static_cast<const uint8_t*>(lam) + r0 * l.dl_row, rows * l.dl_row, h2d, p.up) == cudaSuccess &&
         cudaEventRecord(p.in[slot], p.up) == cudaSuccess && cudaStreamWaitEvent(s, p.in[slot], 0) == cudaSuccess;
    // its y buffer once the copy-out of sub-batch i - 2 has read it
    if (ok && i >= 2) ok = cudaStreamWaitEvent(s, p.out[slot], 0) == cudaSuccess;
    if (!ok) break;
    mamba3_dims ds = *d;
    ds.batch = rows;
    mamba3_state is, fs;
    if (init) is = state_rows(init, d, r0);
    if (final_state) fs = state_rows(final_state, d, r0);
    m3::ScanArgs a = scan_args(&ds, sx, sB, sC, sth, sdt, slm, A, D, init ? &is : nullptr);
    a.y = sy;
    if (final_state) {
      a.h_out = fs.h; a.bprev_out = fs.b_prev; a.xprev_out = fs.x_prev; a.angle_out = fs.angle;
    }
    a.workspace = stage;
    a.workspace_bytes = kStatusBytes;
    if ((rc = use_tc ? m3::launch_scan_tc(a, s) : m3::launch_scan_simt(a, s)) != MAMBA3_OK) return rc;
    ok = cudaEventRecord(p.done[slot], s) == cudaSuccess && cudaStreamWaitEvent(p.down, p.done[slot], 0) == cudaSuccess &&
         cudaMemcpyAsync(static_cast<uint8_t*>(y) + r0 * l.x_row, sy, rows * l.x_row, d2h, p.down) == cudaSuccess &&
         cudaEventRecord(p.out[slot], p.down) == cudaSuccess;
  }
  // the caller's stream resumes after the last copies out
  for (int i = l.nb - 2; ok && i < l.nb; ++i)
    if (i >= 0) ok = cudaStreamWaitEvent(s, p.out[i & 1], 0) == cudaSuccess;
  return ok ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // extern "C"

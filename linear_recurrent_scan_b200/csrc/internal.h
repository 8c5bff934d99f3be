// Internal launcher interface between the C ABI (mamba3_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/mamba3.h"

namespace m3 {

struct ScanArgs {
  int batch, seqlen, nheads, P, N, R, Q;
  int ngroups;  // B, C rows per (batch, token): nheads, or G dividing it (head h reads row h / (nheads / G))
  mamba3_dtype dtype;
  const void *x, *B, *C, *theta, *dt, *lam;
  const float *A, *D;  // A null when A_t is given
  const void* A_t;     // time-varying decay [b, L, H] (dtype of x), or null: A[h] per head
  const float *h0, *bprev0, *xprev0, *angle0;  // all null = zero state
  void* y;
  float *h_out, *bprev_out, *xprev_out, *angle_out;  // all null = no export
  void* workspace;  // device status word at offset 0
  size_t workspace_bytes;
  // fused B/C normalisation (bcnorm != 0): B and C are the raw projections
  int bcnorm;
  const float *nw_B, *nw_C, *nb_B, *nb_C;  // [H, R, N], each nullable
  float neps;
  // bounded device waits: give up after about this many SM cycles (mamba3_set_wait_limit)
  long long wait_limit;
  int test_withhold;  // testing the timeout path only: issue no input loads
  float* decay_out;   // segment aggregates: sum of dt * A over each sequence [b, H], or null
  int split;          // the tensor-core prefill may split its last wave (the workspace holds
                      // tc_split_bytes after the status block, the first bytes zeroed)
};

struct DecodeArgs {
  int batch, nheads, P, N, R;
  int ngroups;  // as in ScanArgs
  mamba3_dtype dtype;
  float *h, *bprev, *xprev, *angle;
  const void *x, *B, *C, *theta, *dt, *lam;
  const float *A, *D;  // A null when A_t is given
  const void* A_t;     // time-varying decay of the token [b, H] (dtype of x), or null
  void* y;
  int bcnorm;  // as in ScanArgs
  const float *nw_B, *nw_C, *nb_B, *nb_C;
  float neps;
  long long wait_limit;  // as in ScanArgs
  int test_withhold;
};

// Backward of the prefill: the forward's arguments in `f` (its y and final
// state unused), the output gradient and the gradients to produce.
struct BwdArgs {
  ScanArgs f;
  const void* dy;                                                // layout of y
  const float *dh_out, *dbprev_out, *dxprev_out, *dangle_out;    // all null = no exported-state gradient
  void *dx, *dB, *dC, *dtheta, *ddt, *dlam;                      // layouts and dtype of the inputs
  float *dA, *dD;                                                // [H], zeroed by the launcher; dD nullable
  void* dA_t;  // with f.A_t: the decay-rate gradient per token (layout of dt, dtype of x); dA null
  float *dh0, *dbprev0, *dxprev0, *dangle0;                      // all null = not wanted
  float* ckpt;  // [units][chunks][N*P + N/2]: hbar and Phi at every chunk start
  int split;         // the tensor-core backward may split its last wave (bwd_tc_split_bytes fit)
  float *dBh, *dCh;  // grouped B, C: fp32 scratch for their gradients (SIMT path: per head
                     // [b, L, H, R, N], summed afterwards; tensor-core path: the group sums
                     // [b, L, G, R, N] themselves); null with one row per head
};

// Pre-gate grouped RMS norm and gate of the layer output: rows = tokens x groups
// contiguous groups of group_size values each.
struct GatedNormArgs {
  long long rows;
  int groups, group_size;
  mamba3_dtype dtype;
  const void *y, *z;
  const float* w;  // [groups * group_size] (= [H, R, P]) or null
  float eps;
  void* out;
};
int launch_gated_norm(const GatedNormArgs& a, cudaStream_t s);

size_t bwd_checkpoint_bytes(const ScanArgs& a);
size_t bwd_group_bytes(const ScanArgs& a);  // per-head B, C gradients when B, C are grouped
int bwd_supported(const ScanArgs& a);
int launch_scan_bwd(const BwdArgs& g, cudaStream_t s);
// The tensor-core backward (scan_bwd_tc.cu): bf16, P = 64, N in {64, 128}, R in
// {1, 2, 4}, seqlen >= 1.  Its workspace after the status word: the state
// checkpoints, then (grouped B/C) the fp32 group sums of dB and dC.
int bwd_tc_supported(const ScanArgs& a);
size_t bwd_tc_workspace_bytes(const ScanArgs& a);
int launch_scan_bwd_tc(BwdArgs g, cudaStream_t s);

// Each launcher returns MAMBA3_OK, MAMBA3_ERR_UNSUPPORTED (shape not compiled)
// or MAMBA3_ERR_CUDA (launch failure).
int decode_supported(const DecodeArgs& a);
int launch_decode(const DecodeArgs& a, cudaStream_t s);

int simt_scan_supported(const ScanArgs& a);
int launch_scan_simt(const ScanArgs& a, cudaStream_t s);

// Device status words of the entry points without a workspace (one per device
// and kernel file, sticky until read): the decode step and the MIMO projections.
int decode_status_read_and_clear(int* code);
int proj_status_read_and_clear(int* code);

// MIMO rank-R projections (mimo_proj.cu): up u [T, H, P] -> x [T, H, R, P] with
// Wx [H, R P, P]; down y [T, H, R, P] -> out [T, H, P] with Wy [H, P, R P], then
// (z non-null) the RMS norm over P with weight w [H, P] (nullable) and the silu
// gate.  bf16, P = 64, R in {1, 2, 4}.
struct ProjArgs {
  long long tokens;
  int nheads, R, up;
  const void *in, *weight;
  void* out;
  const void* z;
  const float* w;
  float eps;
  long long wait_limit;
  int test_withhold;
};
int launch_mimo_proj(const ProjArgs& a, cudaStream_t s);

// TMA tensor maps over the prefill's inputs (scan_tc.cu): a [batch, L, heads, R,
// inner] bf16 tensor with box {64, R, 1, Q, 1} and 128-byte swizzle; dt or lam
// [batch, L, H] with box {8, rows, 1}; theta [batch, L, H, N/2] with box
// {N/2, 1, Q, 1}.  Each returns false when the driver rejects the map.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn();  // cuTensorMapEncodeTiled from the driver, or null
bool make_map(CUtensorMap* m, const void* base, int inner, int heads, const ScanArgs& a, int Q);
bool make_dl_map(CUtensorMap* m, const void* base, const ScanArgs& a, int rows);
bool make_theta_map(CUtensorMap* m, const ScanArgs& a, int Q, bool swizzle = false);

// Long sequences with few (batch, head) units (scan_seg.cu): segments per unit
// (0 = run unsegmented), the workspace they need after the status word, and the
// segmented prefill.
constexpr int kSMs = 148;
// the device status block at the start of every prefill workspace
constexpr size_t kStatusBlockBytes = 256;

// The tensor-core prefill's split last wave (scan_tc.cu): units that run in two
// CTAs and where they split (k = 0: none), the workspace it needs after the
// status block (0 without a split) and the part of it that must be zero before
// the launch; tc_force_split(k, c1) fixes the plan for tests (k = 0: the
// library's plan, k < 0: never split).
struct SplitPlan {
  int k, c1;
};
SplitPlan tc_split_plan(const ScanArgs& a);
// the cached plan for `units` units of `nchunks` chunks each (tc_force_split applies;
// c1 counts the chunks of the kernel that asks)
SplitPlan split_plan(int units, int nchunks);
// the backward chunk kernel's split (scan_bwd_tc.cu): workspace after the checkpoints
// and group sums, 0 without a split
size_t bwd_tc_split_bytes(const ScanArgs& a);
size_t tc_split_bytes(const ScanArgs& a);
size_t tc_split_zero_bytes(const ScanArgs& a);
void tc_force_split(int k, int c1);

// mamba3_scan_fwd on a scratch that every call on the device shares (the no-alloc
// entry point): never splits the last wave, whose tickets and hand-over flags would
// then be shared by overlapping calls (mamba3_api.cu).
int scan_fwd_shared_scratch(const mamba3_dims* d, const void* x, const void* B, const void* C, const void* theta,
                            const void* dt, const void* lam, const float* A, const float* D,
                            const mamba3_state* init, void* y, const mamba3_state* final_state, void* scratch,
                            size_t scratch_bytes, void* stream);
int seg_count(const ScanArgs& a, int sms);
// CTAs of the segment-state kernel that share an SM for these sizes (1 or 2)
int seg_state_ctas_per_sm(const ScanArgs& a);
size_t seg_workspace_bytes(const ScanArgs& a, int S);
int launch_scan_segmented(const ScanArgs& a, int S, cudaStream_t s);
// Every sequence's end state from a zero state and zero angle (the segments'
// aggregates), one streaming tensor-core reduction per sequence (seg_state.cu).
int launch_seg_state(const ScanArgs& a, cudaStream_t s);

int tc_scan_supported(const ScanArgs& a);
int launch_scan_tc(const ScanArgs& a, cudaStream_t s);

}  // namespace m3

// Long single sequences with few (batch, head) units: the prefill split into S
// segments per unit, so that S times as many CTAs share the GPU.
//
// The state is constant in size and the cost linear in the sequence length
// ("Mamba-3 paper review" (no1joon.github.io), Table 7 discussion), and the
// rotation angles are sums over time steps ("Mamba-3: 2x smaller state ..."
// (MarkTechPost, Korean translation), section 1.2), so a segment's effect on
// the state is a decay, a rotation and an additive term:
//   1. launch_seg_state: every segment's end state from a zero state and a
//      zero angle (h_loc, the rotated B and the x of its last token, its angle
//      sum Phi_loc), on the sequence viewed as batch b S of length L / S, as one
//      streaming tensor-core reduction per segment (seg_state.cu);
//   2. seg_combine_kernel: per unit (four CTAs, a quarter of the rotation pairs
//      each), in segment order, the state entering
//      segment s + 1 from the one entering segment s (frame rotated by -Phi_in):
//        h     = e^{sum_seg dt A} (h_in + (1 - lam_f) dt_f sum_r b_in[r] x_in[r]^T)
//                + rot(-Phi_in) h_loc
//        b_prev = rot(-Phi_in) b_loc,  x_prev = x_loc,  Phi = wrap(Phi_in + Phi_loc)
//      (f = the segment's first token; rot acts on the (2k, 2k+1) pairs of the
//      state dimension), written as the initial states of the segments and, for
//      the last one, as the exported final state;
//   3. the tensor-core prefill on the b S segments from those initial states.
// Passes 1 and 3 both read B, x, theta, dt, lam: the price of the parallelism.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace m3 {
namespace {

constexpr int kThreads = 256;

struct SegParams {
  ScanArgs a;        // the unsegmented problem (its init and final state, inputs)
  int S, Ls;         // segments per unit and their length
  const float *loc_h, *loc_b, *loc_x, *loc_ang;  // [b S, H, ...] segment aggregates
  const float* loc_decay;                        // [b S, H] sum of dt * A over each segment
  float *in_h, *in_b, *in_x, *in_ang;            // [b S, H, ...] initial state of every segment
};

template <typename T>
__device__ __forceinline__ float ldv(const void* p, size_t i) {
  return ld1(static_cast<const T*>(p) + i);
}

// kSplit CTAs per unit (b, h), each owning a quarter of the rotation pairs k (the
// rows 2k, 2k+1 of h and b_prev and the angles k): the update acts within pairs, so
// the parts are independent.  Part 0 also carries x_prev.  The running state of
// the part lives in shared memory.
constexpr int kSplit = 4;

template <typename T>
__global__ void __launch_bounds__(kThreads) seg_combine_kernel(const SegParams sp) {
  extern __shared__ float sm[];
  const ScanArgs& a = sp.a;
  const int N = a.N, P = a.P, R = a.R, K2 = N / 2, NP = N * P;
  const int H = a.nheads, L = a.seqlen, S = sp.S, Ls = sp.Ls;
  const int unit = blockIdx.x / kSplit, part = blockIdx.x % kSplit;
  const int b = unit / H, hh = unit % H;
  const int KP = K2 / kSplit, k0 = part * KP;  // this part's pairs k0 .. k0 + KP - 1
  const int tid = threadIdx.x;
  float* h = sm;               // [2 KP][P]: rows 2 k0 .. 2 (k0 + KP) - 1 of h
  float* bp = h + 2 * KP * P;  // [R][2 KP]
  float* xp = bp + R * 2 * KP; // [R][P]
  float* ang = xp + R * P;     // [KP]
  float* red = ang + KP;       // [S] decay sums
  const size_t us = (size_t)unit;
  const int row0 = 2 * k0, rows = 2 * KP;

  for (int i = tid; i < S; i += kThreads) red[i] = sp.loc_decay[((size_t)b * S + i) * H + hh];
  // the state entering segment 0: the caller's initial state, or zero
  for (int i = tid; i < rows * P; i += kThreads) h[i] = a.h0 ? a.h0[us * NP + row0 * P + i] : 0.f;
  for (int i = tid; i < R * rows; i += kThreads) {
    const int r = i / rows, n = row0 + i % rows;
    bp[i] = a.bprev0 ? a.bprev0[(us * R + r) * N + n] : 0.f;
  }
  for (int i = tid; i < R * P; i += kThreads) xp[i] = a.xprev0 ? a.xprev0[us * R * P + i] : 0.f;
  for (int i = tid; i < KP; i += kThreads) ang[i] = a.angle0 ? a.angle0[us * K2 + k0 + i] : 0.f;
  __syncthreads();

  // Per thread: its (pair, column) steps of h, and (tid < R KP) one pair of b_prev,
  // (tid < R P) one x_prev entry, (tid < KP) one angle.  Segment s + 1's aggregates
  // are loaded while segment s is combined, so the chain waits on no global load.
  constexpr int kMaxPer = 4;  // (pair, column) steps per thread: KP P / 256 <= 4 (N <= 128, P = 64)
  struct Agg {
    float h0[kMaxPer], h1[kMaxPer], b0, b1, x, ang, lam, dt;
  };
  auto fetch = [&](int s, Agg& g) {
    if (s >= S) return;
    const size_t su = ((size_t)b * S + s) * H + hh;
    const float* lh = sp.loc_h + su * NP + row0 * P;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
      const int i = tid + j * kThreads;
      if (i < KP * P) {
        const int k = i / P, p = i % P;
        g.h0[j] = lh[(2 * k) * P + p];
        g.h1[j] = lh[(2 * k + 1) * P + p];
      }
    }
    if (tid < R * KP) {
      const int r = tid / KP, k = tid % KP;
      const float* lb = sp.loc_b + (su * R + r) * N + row0;
      g.b0 = lb[2 * k];
      g.b1 = lb[2 * k + 1];
    }
    if (tid < R * P) g.x = sp.loc_x[su * R * P + tid];
    if (tid < KP) g.ang = sp.loc_ang[su * K2 + k0 + tid];
    const size_t f = ((size_t)b * L + (size_t)s * Ls) * H + hh;  // the segment's first token
    g.lam = ldv<T>(a.lam, f);
    g.dt = ldv<T>(a.dt, f);
  };
  Agg cur, nxt;
  fetch(0, cur);
  for (int s = 0; s < S; ++s) {
    const size_t su = ((size_t)b * S + s) * H + hh;  // the segment's unit in the b S x H view
    fetch(s + 1, nxt);
    // the initial state of segment s (this part's rows)
    for (int i = tid; i < rows * P; i += kThreads) sp.in_h[su * NP + row0 * P + i] = h[i];
    for (int i = tid; i < R * rows; i += kThreads) {
      const int r = i / rows, n = row0 + i % rows;
      sp.in_b[(su * R + r) * N + n] = bp[i];
    }
    if (part == 0)
      for (int i = tid; i < R * P; i += kThreads) sp.in_x[su * R * P + i] = xp[i];
    for (int i = tid; i < KP; i += kThreads) sp.in_ang[su * K2 + k0 + i] = ang[i];
    // the copy above reads h in another thread-to-element map than the update below
    // writes it: every thread has to finish the copy first
    __syncthreads();
    // the state leaving it
    const float mu = (1.f - cur.lam) * cur.dt;
    const float decay = expf(red[s]);
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {  // one (pair k, column p) per step
      const int i = tid + j * kThreads;
      if (i < KP * P) {
        const int k = i / P, p = i % P;
        float sn, cs;
        sincosf(ang[k], &sn, &cs);
        float c0 = h[(2 * k) * P + p], c1 = h[(2 * k + 1) * P + p];
        for (int r = 0; r < R; ++r) {
          const float xr = mu * xp[r * P + p];
          c0 += bp[r * rows + 2 * k] * xr;
          c1 += bp[r * rows + 2 * k + 1] * xr;
        }
        const float l0 = cur.h0[j], l1 = cur.h1[j];
        h[(2 * k) * P + p] = decay * c0 + cs * l0 + sn * l1;
        h[(2 * k + 1) * P + p] = decay * c1 + cs * l1 - sn * l0;
      }
    }
    __syncthreads();  // every thread has read bp, xp, ang of the entering state
    if (tid < R * KP) {
      const int r = tid / KP, k = tid % KP;
      float sn, cs;
      sincosf(ang[k], &sn, &cs);
      bp[r * rows + 2 * k] = cs * cur.b0 + sn * cur.b1;
      bp[r * rows + 2 * k + 1] = cs * cur.b1 - sn * cur.b0;
    }
    if (tid < R * P) xp[tid] = cur.x;
    __syncthreads();  // bp rotated with the entering angle before it moves on
    if (tid < KP) ang[tid] = wrap_angle(ang[tid] + cur.ang);
    __syncthreads();
    cur = nxt;
  }
  if (a.h_out) {  // the state after the whole sequence (this part's rows)
    for (int i = tid; i < rows * P; i += kThreads) a.h_out[us * NP + row0 * P + i] = h[i];
    for (int i = tid; i < R * rows; i += kThreads) {
      const int r = i / rows, n = row0 + i % rows;
      a.bprev_out[(us * R + r) * N + n] = bp[i];
    }
    if (part == 0)
      for (int i = tid; i < R * P; i += kThreads) a.xprev_out[us * R * P + i] = xp[i];
    for (int i = tid; i < KP; i += kThreads) a.angle_out[us * K2 + k0 + i] = ang[i];
  }
}

// per (b S x H) unit: h, b_prev, x_prev, angle (floats)
size_t seg_state_floats(const ScanArgs& a) {
  return (size_t)a.N * a.P + (size_t)a.R * a.N + (size_t)a.R * a.P + (size_t)a.N / 2;
}

}  // namespace

// Segments per unit for `a`, or 0 when the plain prefill is the better choice:
// only the tensor-core shapes, long sequences (at least 1024 tokens per
// segment) and fewer units than SMs; S divides L and is chosen so that the b S H
// CTAs fill the SMs' waves as evenly as possible.
int seg_count(const ScanArgs& a, int sms) {
  if (tc_scan_supported(a) != MAMBA3_OK || bwd_tc_supported(a) != MAMBA3_OK || a.bcnorm) return 0;
  const long long units = (long long)a.batch * a.nheads;
  if (units >= sms || a.seqlen < 2048) return 0;
  // Time model: the prefill runs one CTA per SM, the segment-state pass
  // seg_state_ctas_per_sm; each CTA costs its tokens plus about two chunks of
  // pipeline fill and drain, the state pass about half as much per token.
  const double fill = 2.0 * (128 / a.R);
  const long long slots2 = (long long)sms * seg_state_ctas_per_sm(a);
  int best = 0;
  double best_cost = 0.0;
  for (int S = 2; S <= 64; S *= 2) {
    if (a.seqlen % S != 0 || a.seqlen / S < 1024) break;
    const long long ctas = units * S;
    if (ctas < sms) continue;
    const double per = (double)(a.seqlen / S) + fill;
    const double cost = (double)((ctas + sms - 1) / sms) * per + 0.5 * (double)((ctas + slots2 - 1) / slots2) * per;
    if (best == 0 || cost < best_cost - 1e-9) {
      best = S;
      best_cost = cost;
    }
  }
  return best;
}

size_t seg_workspace_bytes(const ScanArgs& a, int S) {
  if (S <= 0) return 0;
  return (2 * seg_state_floats(a) + 1) * (size_t)a.batch * S * a.nheads * sizeof(float);
}

// The prefill of `a` in S segments (workspace: the status word, then the segment
// aggregates and the segments' initial states).
int launch_scan_segmented(const ScanArgs& a, int S, cudaStream_t s) {
  const size_t per = seg_state_floats(a);
  const size_t units_s = (size_t)a.batch * S * a.nheads;
  float* loc = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + 256);
  float* ini = loc + units_s * per;
  SegParams sp;
  memset(&sp, 0, sizeof(sp));
  sp.a = a;
  sp.S = S;
  sp.Ls = a.seqlen / S;
  // [b S H] arrays of each field, one after the other
  sp.loc_h = loc;
  sp.loc_b = loc + units_s * a.N * a.P;
  sp.loc_x = sp.loc_b + units_s * a.R * a.N;
  sp.loc_ang = sp.loc_x + units_s * a.R * a.P;
  sp.in_h = ini;
  sp.in_b = ini + units_s * a.N * a.P;
  sp.in_x = sp.in_b + units_s * a.R * a.N;
  sp.in_ang = sp.in_x + units_s * a.R * a.P;
  float* decay = ini + units_s * per;  // [b S, H]
  sp.loc_decay = decay;

  // 1. segment aggregates
  ScanArgs a1 = a;
  a1.batch = a.batch * S;
  a1.seqlen = sp.Ls;
  a1.h0 = a1.bprev0 = a1.xprev0 = a1.angle0 = nullptr;
  a1.h_out = const_cast<float*>(sp.loc_h);
  a1.bprev_out = const_cast<float*>(sp.loc_b);
  a1.xprev_out = const_cast<float*>(sp.loc_x);
  a1.angle_out = const_cast<float*>(sp.loc_ang);
  a1.decay_out = decay;
  a1.y = nullptr;
  int rc = launch_seg_state(a1, s);
  if (rc != MAMBA3_OK) return rc;
  // 2. the segments' initial states (and the final state)
  // the combine's register prefetch and pair split: K2 a multiple of kSplit, K2 P / kSplit <= 4 x 256
  if (a.N / 2 % kSplit != 0 || a.N / 2 / kSplit * a.P > 4 * kThreads) return MAMBA3_ERR_UNSUPPORTED;
  const int kp = a.N / 2 / kSplit;
  const size_t smem = ((size_t)2 * kp * a.P + (size_t)a.R * 2 * kp + (size_t)a.R * a.P + kp + S) * sizeof(float);
  auto kc = a.dtype == MAMBA3_F32 ? seg_combine_kernel<float> : seg_combine_kernel<__nv_bfloat16>;
  if (smem > 48 * 1024 && cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  kc<<<a.batch * a.nheads * kSplit, kThreads, smem, s>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return MAMBA3_ERR_CUDA;
  // 3. the prefill of every segment from its initial state
  ScanArgs a3 = a;
  a3.batch = a.batch * S;
  a3.seqlen = sp.Ls;
  a3.h0 = sp.in_h;
  a3.bprev0 = sp.in_b;
  a3.xprev0 = sp.in_x;
  a3.angle0 = sp.in_ang;
  a3.h_out = a3.bprev_out = a3.xprev_out = a3.angle_out = nullptr;
  return launch_scan_tc(a3, s);
}

}  // namespace m3

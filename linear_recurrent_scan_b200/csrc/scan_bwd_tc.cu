// Backward pass of the chunked prefill on the 5th-generation tensor cores
// (tcgen05, accumulators in TMEM, operands staged by TMA; bf16 inputs, sm_100a).
//
// The pages on Mamba-3 print no gradient formulas ("Mamba-3 technical summary"
// (digitalbourgeois.tistory.com), "3 key changes", item 3, notes only that MIMO
// raises the training cost).  The gradients below are the chain rule on the
// chunked form of the three-term update ("Mamba-3: 2x smaller state ..."
// (MarkTechPost, Korean translation), section 1.1), its rotation (section 1.2)
// and its rank-R products (section 1.3).  A chunk holds M = 64 rows = Q tokens
// x R ranks.  With B~, C~ the rotated rows, hbar the carried state at the chunk
// start, G = dL/dhbar at the chunk end, cum the chunk-local cumulative log decay,
// w the trapezoid weight of a column, f_j = w_j e^{cum_end - cum_j} and the
// kernel K(t, t) = gamma_t, K(t, j < t) = e^{cum_t - cum_j} w_j:
//   P1 = C~ B~^T,  P2 = dY X^T,  S = K o P1 (+ D on the diagonal),  W = K o P2
//   dC~ = diag(e^cum) dY hbar^T + W B~
//   dB~ = diag(f) X G^T + W^T C~
//   dX  = diag(f) B~ G + S^T dY            (S carries D: + D dY)
//   dL/dhbar_in = e^{cum_end} G + C~^T diag(e^cum) dY
// and the per-token sums of the decay, gamma and w gradients from the rank-summed
// Z = P1 o P2, the paths hbar_in -> y (zin), u -> hbar_out (zue) and
// <hbar_in, G>.  The rotation goes back by +Phi; the angle gradient summed from
// the end of the sequence gives dtheta = dt S and the angle's share of ddt.
//
// Two kernels.
//   bwd_state_kernel  one CTA per (batch, head) marches the chunks forward and
//                     writes the carried state hbar at every chunk start (a bf16
//                     image of the swizzled shared-memory tile the MMAs read) and
//                     the wrapped angle there.  Per chunk one MMA, B~^T X_w.
//   bwd_chunk_kernel  one CTA per (batch, head) marches the chunks backwards
//                     with G in fp32 registers (the TMEM lane of its state row).
//                     Per chunk two MMA batches:
//                       1) P1, P2, dC~ = dY_e hbar^T, dB~ = X_w G^T, BG = B~ G,
//                          Gacc = C~^T dY_e   (dY_e = diag(e^cum) dY, X_w = diag(f) X)
//                       2) dC~ += W B~,  dB~ += W^T C~,  dX = f BG + S^T dY
//                     between them the epilogue forms S, W (bf16 tiles), the
//                     token sums and G <- e^{cum_end} G + Gacc; after them it
//                     rotates dB~, dC~ back and stores every gradient.  The TMA
//                     loads of the next chunk (in reverse order) overlap the
//                     current one.
// M = 64 accumulators occupy TMEM lanes 0..15 of each 32-lane quadrant (row
// m -> lane 32 (m / 16) + m % 16); N x P ones with N = 128 all 128 lanes.
// Every wait is bounded; on expiry the CTA reports MAMBA3_ERR_TIMEOUT in the
// status word, lets its copies and MMAs land, frees TMEM and returns.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace m3 {
namespace {

using namespace ptx;

constexpr int kP = 64;        // head dim handled here
constexpr int kM = 64;        // rows per chunk
constexpr int kBlk = 8192;    // one 64-row x 128-byte swizzled tile
constexpr int kNScal = 16;    // per-token scalar arrays
constexpr int kScalStride = 80;  // >= Q + 1

enum Tag { kTagFull = 21, kTagMma1, kTagMma2, kTagDrain2, kTagHand2, kTagTicket2 };

// split last wave of the chunk kernel (k = 0: one CTA per unit)
struct BwdSplit {
  int k, c1;
  int* ticket;  // zeroed before the launch
  int* flags;   // [k], zeroed
  float* hand;  // [k][N P + N/2 + 4]
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// byte offset of 16-byte chunk c (0..7) of row `row` inside a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// 16 TMEM lanes, two 8-column halves: threads 0..15 read lanes base .. base + 15 at
// columns [col, col + 8), threads 16..31 the same lanes at [col + 8, col + 16) -- the
// layout that lets every lane of a warp carry a row of an M = 64 accumulator (whose
// rows sit in lanes 0..15 of each 32-lane quadrant)
__device__ __forceinline__ void tmem_ld_16x2(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], 8;"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// per-token scalar arrays in shared memory ([kNScal][kScalStride] floats)
enum Scal {
  sDt = 0, sLam, sAt, sC2, sGam, sW, sE, sF, sZin, sZue, sDg, sCZu, sRT, sDth, sEend, sSpare
};

// Sizes shared by the two kernels.
template <int N, int R>
struct BCfg {
  static constexpr int Q = kM / R;       // tokens per chunk
  static constexpr int NKB = N / 64;     // 64-wide blocks of the state dimension
  static constexpr int K2 = N / 2;       // rotation pairs
  static constexpr int NG = K2 / 4;      // 16-byte groups (4 pairs) of a row
  static constexpr int TH_BYTES = Q * K2 * 2;
  static constexpr int HB_BYTES = N * 128;  // N x P bf16 state tile (128-byte rows)
  static constexpr int CK_BYTES = HB_BYTES + K2 * 4;  // one checkpoint: state tile + angle
};

__device__ __forceinline__ size_t tok_index(const ScanArgs& a, int b, int t, int h) {
  return ((size_t)b * a.seqlen + t) * a.nheads + h;
}

// every thread waits on the barrier; one decision for the block afterwards
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           DeviceStatus* st, int tag, long long limit) {
  mbar_wait(bar, parity, abort_flag, st, tag, limit);
  return __syncthreads_or(*abort_flag != 0) == 0;
}

// ====================================================================== state kernel
// 256 threads.  Per chunk: write the checkpoint of the chunk start, wait for the
// chunk's tiles, scalars, angles + RoPE of B in place, X_w, one MMA, state update.
constexpr int kSThreads = 256;

template <int N, int R>
struct SCfg : BCfg<N, R> {
  using B = BCfg<N, R>;
  static constexpr int NPART = kSThreads / B::NG;     // token parts of the angle scan
  static constexpr int NPA = NPART < B::Q ? NPART : B::Q;  // parts in use
  static constexpr int TPP = B::Q / NPA;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_X = B::NKB * kBlk;
  static constexpr int OFF_TH = OFF_X + kBlk;
  static constexpr int STAGE = OFF_TH + ((B::TH_BYTES + 1023) & ~1023);
  static constexpr int OFF_XW = 2 * STAGE;
  static constexpr int OFF_SC = OFF_XW + kBlk;                      // scalars
  static constexpr int OFF_PART = OFF_SC + kNScal * kScalStride * 4;  // angle partials [NPA][K2]
  static constexpr int OFF_PHI = OFF_PART + NPA * B::K2 * 4;        // running angle [K2]
  static constexpr int OFF_BAR = OFF_PHI + B::K2 * 4;               // 4 barriers
  static constexpr int OFF_MISC = OFF_BAR + 32;                     // tmem slot, abort flag
  static constexpr int SMEM = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(B::Q % NPA == 0, "parts");
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
};

template <int N, int R, bool TVA>
__global__ void __launch_bounds__(kSThreads) bwd_state_kernel(const __grid_constant__ CUtensorMap tmB,
                                                              const __grid_constant__ CUtensorMap tmX,
                                                              const __grid_constant__ CUtensorMap tmT,
                                                              const ScanArgs a, uint8_t* ckpt, int nchunks) {
  using K = SCfg<N, R>;
  constexpr int Q = K::Q, K2 = K::K2, NG = K::NG, NPA = K::NPA, TPP = K::TPP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x;
  const int b = unit / a.nheads, hh = unit % a.nheads;
  const int L = a.seqlen, H = a.nheads;
  const int gh = hh / (a.nheads / a.ngroups);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);  // full0, full1, mma
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.workspace);
  float* sc = reinterpret_cast<float*>(smem + K::OFF_SC);
  float* part_sum = reinterpret_cast<float*>(smem + K::OFF_PART);
  float* phi = reinterpret_cast<float*>(smem + K::OFF_PHI);
  const __nv_bfloat16* DT = static_cast<const __nv_bfloat16*>(a.dt);
  const __nv_bfloat16* LM = static_cast<const __nv_bfloat16*>(a.lam);
  const __nv_bfloat16* AT = static_cast<const __nv_bfloat16*>(a.A_t);
  const float Ah = TVA ? 0.f : a.A[hh];

  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init(&bars[2], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmT);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  if (tid < K2) phi[tid] = a.angle0 ? a.angle0[(size_t)unit * K2 + tid] : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // epilogue geometry: state row n, 32 columns (half) of the N x 64 accumulator
  const int quad = warp & 3, half = warp >> 2;
  const int n = (N == 128) ? quad * 32 + lane : (lane < 16 ? quad * 16 + lane : -1);
  const uint32_t lane_base = (uint32_t)(quad * 32) << 16;

  // carried state hbar_0 = h_0 + (1 - lam_1) dt_1 sum_r B~_0[r]^T x_0[r]
  float hb[32];
#pragma unroll
  for (int p = 0; p < 32; ++p) hb[p] = 0.f;
  if (n >= 0 && a.h0 != nullptr) {
    const size_t i0 = tok_index(a, b, 0, hh);
    const float mu1 = (1.f - __bfloat162float(LM[i0])) * __bfloat162float(DT[i0]);
    const float* h0 = a.h0 + ((size_t)unit * N + n) * kP + 32 * half;
#pragma unroll
    for (int p = 0; p < 32; ++p) hb[p] = h0[p];
    for (int r = 0; r < R; ++r) {
      const float bp = mu1 * a.bprev0[((size_t)unit * R + r) * N + n];
      const float* xp = a.xprev0 + ((size_t)unit * R + r) * kP + 32 * half;
#pragma unroll
      for (int p = 0; p < 32; ++p) hb[p] += bp * xp[p];
    }
  }

  auto issue = [&](int c) {
    const int s = c & 1;
    uint8_t* st = smem + s * K::STAGE;
    const int t0 = c * Q;
    mbar_arrive_expect_tx(&bars[s], (uint32_t)(K::NKB * kBlk + kBlk + K::TH_BYTES));
#pragma unroll
    for (int kb = 0; kb < K::NKB; ++kb) tma_load_5d(st + K::OFF_B + kb * kBlk, &tmB, &bars[s], kb * 64, 0, gh, t0, b);
    tma_load_5d(st + K::OFF_X, &tmX, &bars[s], 0, 0, hh, t0, b);
    tma_load_4d(st + K::OFF_TH, &tmT, &bars[s], 0, hh, t0, b);
  };
  // scalars of tokens t0 .. t0 + Q (the token after the chunk: dt 0, lam 1 past the end)
  float r_dt = 0.f, r_lm = 1.f, r_at = Ah;
  auto load_scalars = [&](int c) {
    const int t = c * Q + tid;
    r_dt = 0.f; r_lm = 1.f; r_at = Ah;
    if (tid <= Q && c < nchunks && t < L) {
      const size_t i = tok_index(a, b, t, hh);
      r_dt = __bfloat162float(DT[i]);
      r_lm = __bfloat162float(LM[i]);
      if constexpr (TVA) r_at = __bfloat162float(AT[i]);
    }
  };
  int issued = 0;  // chunks whose loads were issued
  if (tid == 0 && !a.test_withhold) { issue(0); issued = 1; }
  load_scalars(0);
  int abort_c = -1, abort_mma = 0;  // chunk and stage of an abort
  const size_t ck_unit = (size_t)unit * nchunks;
  const int g = tid % NG, part = tid / NG;   // angle scan: 4-pair group, token part
  const int kb = g / 8, c8 = g % 8;

  for (int c = 0; c < nchunks; ++c) {
    const int s = c & 1;
    uint8_t* st = smem + s * K::STAGE;
    const int t0 = c * Q;
    if (tid == 0 && c + 1 < nchunks && !a.test_withhold) {
      fence_proxy_async_smem();  // the stage's previous generic reads before the TMA refill
      issue(c + 1);
      issued = c + 2;
    }
    if (tid <= Q) {
      sc[sDt * kScalStride + tid] = r_dt;
      sc[sLam * kScalStride + tid] = r_lm;
      sc[sAt * kScalStride + tid] = r_at;
    }
    load_scalars(c + 1);
    // checkpoint of the chunk start: the bf16 state tile image and the angle
    uint8_t* ck = ckpt + (ck_unit + c) * (size_t)K::HB_BYTES;
    if (n >= 0) {
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint4 q;
        q.x = pack_bf16(hb[8 * q4 + 0], hb[8 * q4 + 1]);
        q.y = pack_bf16(hb[8 * q4 + 2], hb[8 * q4 + 3]);
        q.z = pack_bf16(hb[8 * q4 + 4], hb[8 * q4 + 5]);
        q.w = pack_bf16(hb[8 * q4 + 6], hb[8 * q4 + 7]);
        *reinterpret_cast<uint4*>(ck + swz(n, 4 * half + q4)) = q;
      }
    }
    if (tid < K2) {
      float* ckphi = reinterpret_cast<float*>(ckpt + (size_t)gridDim.x * nchunks * K::HB_BYTES) + (ck_unit + c) * K2;
      ckphi[tid] = phi[tid];
    }
    __syncthreads();
    // decay scan (warp 0, two tokens per lane): log2 of the chunk-local decay, gamma, w
    if (warp == 0) {
      const int i0 = 2 * lane, i1 = 2 * lane + 1;
      const float a0 = i0 < Q ? sc[sDt * kScalStride + i0] * sc[sAt * kScalStride + i0] * kLog2e : 0.f;
      const float a1 = i1 < Q ? sc[sDt * kScalStride + i1] * sc[sAt * kScalStride + i1] * kLog2e : 0.f;
      float v = a0 + a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      const float c1 = v, c0 = v - a1;
      const float cend = __shfl_sync(0xffffffffu, v, (Q - 1) / 2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = e ? i1 : i0;
        if (i < Q) {
          const float dt = sc[sDt * kScalStride + i], lm = sc[sLam * kScalStride + i];
          const float gam = lm * dt;
          const float w = gam + (1.f - sc[sLam * kScalStride + i + 1]) * sc[sDt * kScalStride + i + 1];
          sc[sC2 * kScalStride + i] = e ? c1 : c0;
          sc[sF * kScalStride + i] = w * ex2(cend - (e ? c1 : c0));
        }
      }
      if (lane == 0) sc[sSpare * kScalStride] = cend;
    }
    if (!block_wait(&bars[s], (c >> 1) & 1, abort_flag, status, kTagFull, a.wait_limit)) { abort_c = c; break; }

    // angles: partial sums of dt theta per (part, 4-pair group)
    const __nv_bfloat16* th = reinterpret_cast<const __nv_bfloat16*>(st + K::OFF_TH);
    float run[4] = {0.f, 0.f, 0.f, 0.f};
    if (part < NPA) {
      float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < TPP; ++i) {
        const int t = part * TPP + i;
        const float d = sc[sDt * kScalStride + t];
        const uint2 tv = *reinterpret_cast<const uint2*>(th + t * K2 + 4 * g);
        const float2 t01 = unpack_bf16(tv.x), t23 = unpack_bf16(tv.y);
        loc[0] += d * t01.x; loc[1] += d * t01.y; loc[2] += d * t23.x; loc[3] += d * t23.y;
      }
      *reinterpret_cast<float4*>(part_sum + part * K2 + 4 * g) = make_float4(loc[0], loc[1], loc[2], loc[3]);
    }
    __syncthreads();
    if (part < NPA) {
      const float4 base = *reinterpret_cast<const float4*>(phi + 4 * g);
      run[0] = base.x; run[1] = base.y; run[2] = base.z; run[3] = base.w;
      for (int p2 = 0; p2 < part; ++p2) {
        const float4 ps = *reinterpret_cast<const float4*>(part_sum + p2 * K2 + 4 * g);
        run[0] += ps.x; run[1] += ps.y; run[2] += ps.z; run[3] += ps.w;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) run[k] = wrap_angle(run[k]);
#pragma unroll
      for (int i = 0; i < TPP; ++i) {
        const int t = part * TPP + i;
        const float d = sc[sDt * kScalStride + t];
        const uint2 tv = *reinterpret_cast<const uint2*>(th + t * K2 + 4 * g);
        const float2 t01 = unpack_bf16(tv.x), t23 = unpack_bf16(tv.y);
        run[0] += d * t01.x; run[1] += d * t01.y; run[2] += d * t23.x; run[3] += d * t23.y;
        float sn[4], cs[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) __sincosf(run[k], &sn[k], &cs[k]);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          uint4* p = reinterpret_cast<uint4*>(st + K::OFF_B + kb * kBlk + swz(t * R + r, c8));
          const uint4 q = *p;
          const uint32_t bw[4] = {q.x, q.y, q.z, q.w};
          uint32_t bo[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 v = unpack_bf16(bw[k]);
            bo[k] = pack_bf16(cs[k] * v.x + sn[k] * v.y, cs[k] * v.y - sn[k] * v.x);
          }
          *p = make_uint4(bo[0], bo[1], bo[2], bo[3]);
        }
      }
    }
    // X_w = diag(f) X (two 16-byte chunks per thread)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int idx = tid + kSThreads * i;
      const int row = idx >> 3, cc = idx & 7;
      const float f = sc[sF * kScalStride + row / R];
      const uint4 xq = *reinterpret_cast<const uint4*>(st + K::OFF_X + swz(row, cc));
      const float2 f0 = unpack_bf16(xq.x), f1 = unpack_bf16(xq.y), f2 = unpack_bf16(xq.z), f3 = unpack_bf16(xq.w);
      *reinterpret_cast<uint4*>(smem + K::OFF_XW + swz(row, cc)) =
          make_uint4(pack_bf16(f * f0.x, f * f0.y), pack_bf16(f * f1.x, f * f1.y), pack_bf16(f * f2.x, f * f2.y),
                     pack_bf16(f * f3.x, f * f3.y));
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (part == NPA - 1 && part < NPA) {  // the last part's running angle is the chunk's end angle
      *reinterpret_cast<float4*>(phi + 4 * g) =
          make_float4(wrap_angle(run[0]), wrap_angle(run[1]), wrap_angle(run[2]), wrap_angle(run[3]));
    }
    if (tid == 0) {  // Hacc = B~^T X_w  (N x 64, K = 64 rows)
      tc_fence_after();
      const uint32_t iH = idesc_bf16(N, kP, 1, 1);
      const uint32_t cB = smem_u32(st + K::OFF_B), cXw = smem_u32(smem + K::OFF_XW);
#pragma unroll
      for (int kk = 0; kk < kM / 16; ++kk)
        mma_bf16_ss(tmem, smem_desc_sw128(cB + kk * 2048, kBlk, 1024), smem_desc_sw128(cXw + kk * 2048, kBlk, 1024),
                    iH, kk > 0);
      mma_commit(&bars[2]);
    }
    if (!block_wait(&bars[2], c & 1, abort_flag, status, kTagMma1, a.wait_limit)) {
      abort_c = c;
      abort_mma = 1;
      break;
    }
    tc_fence_after();
    const float e_end = ex2(sc[sSpare * kScalStride]);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      float acc[16];
      tmem_ld16(tmem + lane_base + 32 * half + 16 * h2, acc);
      tmem_ld_wait();
#pragma unroll
      for (int p = 0; p < 16; ++p) hb[16 * h2 + p] = e_end * hb[16 * h2 + p] + acc[p];
    }
    tc_fence_before();
    __syncthreads();  // stage s, X_w and the scalars may be reused
  }
  if (abort_c >= 0 && tid == 0) {
    // Let what was issued land before TMEM is freed and the CTA exits: the loads of
    // chunk abort_c (unless the wait for them was passed) and of the chunk after
    // it, and the MMA of chunk abort_c when the abort came while waiting for it.
    for (int c2 = abort_c + abort_mma; c2 < issued; ++c2)
      if (!mbar_wait_drain(&bars[c2 & 1], (c2 >> 1) & 1)) report_timeout(status, kTagDrain2);
    if (abort_mma && !mbar_wait_drain(&bars[2], abort_c & 1)) report_timeout(status, kTagDrain2);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}


// ====================================================================== chunk kernel
constexpr int kCThreads = 512;

template <int N, int R>
struct CCfg : BCfg<N, R> {
  using B = BCfg<N, R>;
  // angle scan of the prep phase: thread = (4-pair group, token part)
  static constexpr int NPART = kCThreads / B::NG;
  static constexpr int NPA = NPART < B::Q ? NPART : B::Q;
  static constexpr int TPP = B::Q / NPA;
  // angle-gradient suffix: thread = (pair, token part)
  static constexpr int NPART2 = kCThreads / B::K2;
  static constexpr int TPP2 = (B::Q + NPART2 - 1) / NPART2;
  // per stage: B, C, X, dY tiles (TMA), the checkpointed state tile and angle (bulk copies), theta (TMA)
  static constexpr int OFF_B = 0;
  static constexpr int OFF_C = B::NKB * kBlk;
  static constexpr int OFF_X = 2 * B::NKB * kBlk;
  static constexpr int OFF_DY = OFF_X + kBlk;
  static constexpr int OFF_HB = OFF_DY + kBlk;
  static constexpr int OFF_TH = OFF_HB + B::HB_BYTES;
  static constexpr int OFF_PH = OFF_TH + ((B::TH_BYTES + 127) & ~127);
  static constexpr int STAGE = (OFF_PH + B::K2 * 4 + 1023) & ~1023;
  static constexpr int LOAD_BYTES = 2 * B::NKB * kBlk + 2 * kBlk + B::HB_BYTES + B::TH_BYTES + B::K2 * 4;
  // single buffers
  static constexpr int OFF_DYE = 2 * STAGE;               // diag(e^cum) dY
  static constexpr int OFF_XW = OFF_DYE + kBlk;           // diag(f) X
  static constexpr int OFF_G = OFF_XW + kBlk;             // G (bf16 state tile)
  static constexpr int OFF_S = OFF_G + B::HB_BYTES;       // S, then W; later the angle gradients [Q][K2] f32
  static constexpr int OFF_W = OFF_S + kBlk;
  static constexpr int QP = B::Q + 1;                     // odd row stride of the angle table
  static constexpr int OFF_PHT = OFF_W + kBlk;            // angle of every token [K2][QP] f32
  static constexpr int OFF_SC = OFF_PHT + B::K2 * QP * 4;
  static constexpr int PART_FLOATS = (NPA > NPART2 ? NPA : NPART2) * B::K2;
  static constexpr int OFF_PART = OFF_SC + kNScal * kScalStride * 4;
  static constexpr int OFF_SANG = OFF_PART + PART_FLOATS * 4;  // angle gradient from the end [2][K2] (by chunk parity)
  static constexpr int OFF_RED = OFF_SANG + 2 * B::K2 * 4;     // block sums [32]
  static constexpr int OFF_BAR = OFF_RED + 128;                // full0, full1, mma1, mma2
  static constexpr int OFF_MISC = OFF_BAR + 64;                // tmem slot, abort flag
  static constexpr int SMEM = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(B::Q * B::K2 * 4 <= 2 * kBlk, "angle gradients fit in S, W");
  static_assert(B::Q % NPA == 0, "angle parts");
  static_assert(N * kP * 4 <= 2 * STAGE, "final G staging fits in the stages");
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
  // TMEM columns
  static constexpr uint32_t kColP1 = 0, kColP2 = 64, kColDC = 128, kColDB = 128 + N, kColDX = 128 + 2 * N,
                            kColGA = 192 + 2 * N;
};

template <int N, int R, bool TVA, bool GRP>
__global__ void __launch_bounds__(kCThreads, 1)
    bwd_chunk_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                     const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmDY,
                     const __grid_constant__ CUtensorMap tmT, const BwdArgs g, const uint8_t* ckpt, int nchunks,
                     const BwdSplit sp) {
  using K = CCfg<N, R>;
  constexpr int Q = K::Q, K2 = K::K2, NG = K::NG, NPA = K::NPA, TPP = K::TPP, NKB = K::NKB;
  constexpr int NPART2 = K::NPART2, TPP2 = K::TPP2, QP = K::QP;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const ScanArgs& a = g.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int units = a.batch * a.nheads;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 8);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.workspace);
  // this CTA's work: a whole unit (blockIdx), or with a split last wave the next
  // ticket (0..k-1: the end of units 0..k-1, chunks [c1, n), marched first; k..U-1:
  // whole units; U..U+k-1: chunks [0, c1) of units 0..k-1, from the hand-over of the
  // adjoint state, the running angle-gradient sum and the pending token)
  if (tid == 0) {
    *abort_flag = 0;
    int item = blockIdx.x;
    if (sp.k > 0) {
      item = atomicAdd(sp.ticket, 1);
      if (item >= units + sp.k) {  // only a workspace shared by overlapping calls gives one
        *abort_flag = 1;
        report_timeout(status, kTagTicket2);
        item = 0;
      } else if (item >= units) {
        const int* f = sp.flags + (item - units);
        const long long t_start = clock64();
        while (ld_acquire_gpu(f) == 0) {
          if (clock64() - t_start > a.wait_limit) {
            *abort_flag = 1;
            report_timeout(status, kTagHand2);
            break;
          }
          __nanosleep(256);
        }
      }
    }
    *item_slot = item;
  }
  __syncthreads();
  const int item = *item_slot;
  const bool skip = *abort_flag != 0;
  int unit = item, c_top = nchunks - 1, r_end = nchunks;
  const float* hand_in = nullptr;
  float* hand_out = nullptr;
  constexpr int kSlot = N * kP + K::K2 + 4;  // G, the angle-gradient sum, the pending ddt and dlam
  if (sp.k > 0 && !skip) {
    if (item < sp.k) {  // the end of the sequence: chunks [c1, n), then the hand-over
      r_end = nchunks - sp.c1;
      hand_out = sp.hand + (size_t)item * kSlot;
    } else if (item >= units) {  // chunks [0, c1) from the hand-over
      unit = item - units;
      c_top = sp.c1 - 1;
      r_end = sp.c1;
      hand_in = sp.hand + (size_t)unit * kSlot;
    }
  }
  if (skip) r_end = 0;
  const int b = unit / a.nheads, hh = unit % a.nheads;
  const int L = a.seqlen;
  const int gh = hh / (a.nheads / a.ngroups);
  float* sc = reinterpret_cast<float*>(smem + K::OFF_SC);
  float* part_sum = reinterpret_cast<float*>(smem + K::OFF_PART);
  float* sang = reinterpret_cast<float*>(smem + K::OFF_SANG);
  float* red = reinterpret_cast<float*>(smem + K::OFF_RED);
  float* pht = reinterpret_cast<float*>(smem + K::OFF_PHT);  // [K2][QP]: consecutive tokens, consecutive banks
  float* dphi_s = reinterpret_cast<float*>(smem + K::OFF_S);
  // angle gradient of (token t, pair k): rows of K2, the pairs XOR-swizzled in groups of
  // four by the row, so that the 16 rows a warp stores at once fall in different banks
  // and a row read by 32 consecutive pairs stays conflict-free
  auto dphi_at = [](int t, int k) { return t * K::K2 + (k ^ ((t & 7) << 2)); };
  const __nv_bfloat16* DT = static_cast<const __nv_bfloat16*>(a.dt);
  const __nv_bfloat16* LM = static_cast<const __nv_bfloat16*>(a.lam);
  const __nv_bfloat16* AT = static_cast<const __nv_bfloat16*>(a.A_t);
  __nv_bfloat16* dXg = static_cast<__nv_bfloat16*>(g.dx);
  __nv_bfloat16* dBg = static_cast<__nv_bfloat16*>(g.dB);
  __nv_bfloat16* dCg = static_cast<__nv_bfloat16*>(g.dC);
  __nv_bfloat16* dTHg = static_cast<__nv_bfloat16*>(g.dtheta);
  __nv_bfloat16* dDTg = static_cast<__nv_bfloat16*>(g.ddt);
  __nv_bfloat16* dLMg = static_cast<__nv_bfloat16*>(g.dlam);
  __nv_bfloat16* dATg = static_cast<__nv_bfloat16*>(g.dA_t);
  const float Ah = TVA ? 0.f : a.A[hh];
  const float Dh = a.D ? a.D[hh] : 0.f;
  const size_t ck_unit = (size_t)unit * nchunks;
  const float* ckphi = reinterpret_cast<const float*>(ckpt + (size_t)units * nchunks * K::HB_BYTES);

  if (tid == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmDY);
    prefetch_tmap(&tmT);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid < K2)
    sang[tid] = hand_in ? __ldcg(hand_in + N * kP + tid) : (g.dangle_out ? g.dangle_out[(size_t)unit * K2 + tid] : 0.f);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // geometry: M = 64 accumulators (row m, valid on lanes 0..15), N x 64 (state row n)
  const int quad = warp & 3, sl = warp >> 2;
  const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
  // M = 64 accumulators through tmem_ld_16x2: every lane carries row m, half selects
  // the 8-column half of the warp's 16-column slice
  const int half = lane >> 4;
  const int m = 16 * quad + (lane & 15);
  const int tm = m / R, rm = m % R;
  const int n = (N == 128) ? quad * 32 + lane : (lane < 16 ? quad * 16 + lane : -1);
  const int p0 = 16 * sl;  // this thread's 16 columns of a 64-column accumulator

  // G = dL/dhbar at the end of the chunk being processed (fp32, this thread's 16 columns of row n)
  float G[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) G[i] = 0.f;
  if (n >= 0 && hand_in) {
#pragma unroll
    for (int i = 0; i < 16; ++i) G[i] = __ldcg(hand_in + n * kP + p0 + i);
  } else if (n >= 0 && g.dh_out) {
#pragma unroll
    for (int i = 0; i < 16; ++i) G[i] = g.dh_out[((size_t)unit * N + n) * kP + p0 + i];
  }
  auto store_G = [&]() {  // bf16 copy of G into its swizzled tile (row n, columns p0 .. p0 + 15)
    if (n < 0) return;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      uint4 q;
      q.x = pack_bf16(G[8 * h2 + 0], G[8 * h2 + 1]);
      q.y = pack_bf16(G[8 * h2 + 2], G[8 * h2 + 3]);
      q.z = pack_bf16(G[8 * h2 + 4], G[8 * h2 + 5]);
      q.w = pack_bf16(G[8 * h2 + 6], G[8 * h2 + 7]);
      *reinterpret_cast<uint4*>(smem + K::OFF_G + swz(n, p0 / 8 + h2)) = q;
    }
  };
  store_G();

  // loads of chunk c (reverse index r = c_top - c: stage r & 1, phase (r >> 1) & 1)
  auto issue = [&](int c) {
    const int r = c_top - c, s = r & 1;
    uint8_t* st = smem + s * K::STAGE;
    const int t0 = c * Q;
    mbar_arrive_expect_tx(&bars[s], (uint32_t)K::LOAD_BYTES);
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb) {
      tma_load_5d(st + K::OFF_B + kb * kBlk, &tmB, &bars[s], kb * 64, 0, gh, t0, b);
      tma_load_5d(st + K::OFF_C + kb * kBlk, &tmC, &bars[s], kb * 64, 0, gh, t0, b);
    }
    tma_load_5d(st + K::OFF_X, &tmX, &bars[s], 0, 0, hh, t0, b);
    tma_load_5d(st + K::OFF_DY, &tmDY, &bars[s], 0, 0, hh, t0, b);
    tma_load_4d(st + K::OFF_TH, &tmT, &bars[s], 0, hh, t0, b);
    bulk_load(st + K::OFF_HB, ckpt + (ck_unit + c) * (size_t)K::HB_BYTES, K::HB_BYTES, &bars[s]);
    bulk_load(st + K::OFF_PH, ckphi + (ck_unit + c) * K2, K2 * 4, &bars[s]);
  };
  float r_dt = 0.f, r_lm = 1.f, r_at = Ah;
  auto load_scalars = [&](int c) {
    const int t = c * Q + tid;
    r_dt = 0.f; r_lm = 1.f; r_at = Ah;
    if (tid <= Q && c >= 0 && t < L) {
      const size_t i = tok_index(a, b, t, hh);
      r_dt = __bfloat162float(DT[i]);
      r_lm = __bfloat162float(LM[i]);
      if constexpr (TVA) r_at = __bfloat162float(AT[i]);
    }
  };
  int issued = 0;  // chunks (in reverse order) whose loads were issued
  if (tid == 0 && !a.test_withhold && r_end > 0) { issue(c_top); issued = 1; }
  load_scalars(c_top);
  // pending (thread 0): ddt, dlam of the first token of the chunk processed last,
  // without its lagged share, which the next chunk processed (the one before it) supplies
  float pend_ddt = 0.f, pend_dlm = 0.f, dA_acc = 0.f, dD_acc = 0.f;
  int pend_t = -1;
  if (hand_in && tid == 0) {  // the first token after this part waits for its lagged share
    pend_t = (c_top + 1) * Q;
    pend_ddt = __ldcg(hand_in + N * kP + K2);
    pend_dlm = __ldcg(hand_in + N * kP + K2 + 1);
  }
  int abort_r = -1, abort_stage = 0;  // where an abort happened (0: loads, 1: batch 1, 2: batch 2)
  const int ag = tid % NG, apart = tid / NG;   // angle scan: 4-pair group, token part
  const int akb = ag / 8, ac8 = ag % 8;

  for (int r = 0; r < r_end; ++r) {
    const int c = c_top - r, s = r & 1;
    uint8_t* st = smem + s * K::STAGE;
    const int t0 = c * Q;
    if (tid == 0 && r + 1 < r_end && !a.test_withhold) {
      fence_proxy_async_smem();  // the stage's previous generic reads before the TMA refill
      issue(c - 1);
      issued = r + 2;
    }
    if (tid <= Q) {
      sc[sDt * kScalStride + tid] = r_dt;
      sc[sLam * kScalStride + tid] = r_lm;
      sc[sAt * kScalStride + tid] = r_at;
    }
    if (tid < Q) {
      sc[sZin * kScalStride + tid] = 0.f;
      sc[sZue * kScalStride + tid] = 0.f;
      sc[sDg * kScalStride + tid] = 0.f;
      sc[sCZu * kScalStride + tid] = 0.f;
      sc[sRT * kScalStride + tid] = 0.f;
      sc[sDth * kScalStride + tid] = 0.f;
    }
    if (tid == 0) red[0] = 0.f;
    load_scalars(c - 1);
    __syncthreads();
    // ---- decay scan (warp 0, two tokens per lane) ----
    if (warp == 0) {
      const int i0 = 2 * lane, i1 = 2 * lane + 1;
      const float a0 = i0 < Q ? sc[sDt * kScalStride + i0] * sc[sAt * kScalStride + i0] * kLog2e : 0.f;
      const float a1 = i1 < Q ? sc[sDt * kScalStride + i1] * sc[sAt * kScalStride + i1] * kLog2e : 0.f;
      float v = a0 + a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
      }
      const float cum1 = v, cum0 = v - a1;
      const float cend = __shfl_sync(0xffffffffu, v, (Q - 1) / 2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = e ? i1 : i0;
        if (i < Q) {
          const float cu = e ? cum1 : cum0;
          const float dt = sc[sDt * kScalStride + i], lm = sc[sLam * kScalStride + i];
          const float gam = lm * dt;
          const float w = gam + (1.f - sc[sLam * kScalStride + i + 1]) * sc[sDt * kScalStride + i + 1];
          const float ee = ex2(cend - cu);
          sc[sC2 * kScalStride + i] = cu;
          sc[sGam * kScalStride + i] = gam;
          sc[sW * kScalStride + i] = w;
          sc[sE * kScalStride + i] = ex2(cu);
          sc[sEend * kScalStride + i] = ee;
          sc[sF * kScalStride + i] = w * ee;
        }
      }
      if (lane == 0) sc[sSpare * kScalStride] = cend;
    }
    if (!block_wait(&bars[s], (r >> 1) & 1, abort_flag, status, kTagFull, a.wait_limit)) {
      abort_r = r;
      abort_stage = 0;
      break;
    }

    // ---- angles of every token (wrapped) and RoPE of B and C in place ----
    const __nv_bfloat16* th = reinterpret_cast<const __nv_bfloat16*>(st + K::OFF_TH);
    const float* phs = reinterpret_cast<const float*>(st + K::OFF_PH);
    if (apart < NPA) {
      float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < TPP; ++i) {
        const int t = apart * TPP + i;
        const float d = sc[sDt * kScalStride + t];
        const uint2 tv = *reinterpret_cast<const uint2*>(th + t * K2 + 4 * ag);
        const float2 t01 = unpack_bf16(tv.x), t23 = unpack_bf16(tv.y);
        loc[0] += d * t01.x; loc[1] += d * t01.y; loc[2] += d * t23.x; loc[3] += d * t23.y;
      }
      *reinterpret_cast<float4*>(part_sum + apart * K2 + 4 * ag) = make_float4(loc[0], loc[1], loc[2], loc[3]);
    }
    __syncthreads();
    if (apart < NPA) {
      const float4 base = *reinterpret_cast<const float4*>(phs + 4 * ag);
      float run[4] = {base.x, base.y, base.z, base.w};
      for (int p2 = 0; p2 < apart; ++p2) {
        const float4 ps = *reinterpret_cast<const float4*>(part_sum + p2 * K2 + 4 * ag);
        run[0] += ps.x; run[1] += ps.y; run[2] += ps.z; run[3] += ps.w;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) run[k] = wrap_angle(run[k]);
#pragma unroll
      for (int i = 0; i < TPP; ++i) {
        const int t = apart * TPP + i;
        const float d = sc[sDt * kScalStride + t];
        const uint2 tv = *reinterpret_cast<const uint2*>(th + t * K2 + 4 * ag);
        const float2 t01 = unpack_bf16(tv.x), t23 = unpack_bf16(tv.y);
        run[0] += d * t01.x; run[1] += d * t01.y; run[2] += d * t23.x; run[3] += d * t23.y;
#pragma unroll
        for (int k = 0; k < 4; ++k) pht[(4 * ag + k) * QP + t] = wrap_angle(run[k]);
        float sn[4], cs[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) __sincosf(run[k], &sn[k], &cs[k]);
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
          const uint32_t off = akb * kBlk + swz(t * R + rr, ac8);
          uint4* pb = reinterpret_cast<uint4*>(st + K::OFF_B + off);
          uint4* pc = reinterpret_cast<uint4*>(st + K::OFF_C + off);
          const uint4 qb = *pb, qc = *pc;
          const uint32_t bw[4] = {qb.x, qb.y, qb.z, qb.w}, cw[4] = {qc.x, qc.y, qc.z, qc.w};
          uint32_t bo[4], co[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 bv = unpack_bf16(bw[k]), cv = unpack_bf16(cw[k]);
            bo[k] = pack_bf16(cs[k] * bv.x + sn[k] * bv.y, cs[k] * bv.y - sn[k] * bv.x);
            co[k] = pack_bf16(cs[k] * cv.x + sn[k] * cv.y, cs[k] * cv.y - sn[k] * cv.x);
          }
          *pb = make_uint4(bo[0], bo[1], bo[2], bo[3]);
          *pc = make_uint4(co[0], co[1], co[2], co[3]);
        }
      }
    }
    // ---- dY_e = diag(e^cum) dY and X_w = diag(f) X (one 16-byte chunk of each per thread) ----
    {
      const int row = tid >> 3, cc = tid & 7;
      const float e = sc[sE * kScalStride + row / R], f = sc[sF * kScalStride + row / R];
      const uint4 yq = *reinterpret_cast<const uint4*>(st + K::OFF_DY + swz(row, cc));
      const uint4 xq = *reinterpret_cast<const uint4*>(st + K::OFF_X + swz(row, cc));
      const uint32_t yw[4] = {yq.x, yq.y, yq.z, yq.w}, xw[4] = {xq.x, xq.y, xq.z, xq.w};
      uint32_t yo[4], xo[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 yv = unpack_bf16(yw[k]), xv = unpack_bf16(xw[k]);
        yo[k] = pack_bf16(e * yv.x, e * yv.y);
        xo[k] = pack_bf16(f * xv.x, f * xv.y);
      }
      *reinterpret_cast<uint4*>(smem + K::OFF_DYE + swz(row, cc)) = make_uint4(yo[0], yo[1], yo[2], yo[3]);
      *reinterpret_cast<uint4*>(smem + K::OFF_XW + swz(row, cc)) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- MMA batch 1 ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t cB = smem_u32(st + K::OFF_B), cC = smem_u32(st + K::OFF_C), cX = smem_u32(st + K::OFF_X),
                     cY = smem_u32(st + K::OFF_DY), cHB = smem_u32(st + K::OFF_HB);
      const uint32_t cYe = smem_u32(smem + K::OFF_DYE), cXw = smem_u32(smem + K::OFF_XW),
                     cG = smem_u32(smem + K::OFF_G);
      const uint32_t iPP = idesc_bf16(kM, kM, 0, 0);      // P1 = C~ B~^T, P2 = dY X^T
      const uint32_t iMN = idesc_bf16(kM, N, 0, 0);       // dY_e hbar^T, X_w G^T  (K = P)
      const uint32_t iBG = idesc_bf16(kM, kP, 0, 1);      // B~ G                  (K = N)
      const uint32_t iGA = idesc_bf16(N, kP, 1, 1);       // C~^T dY_e             (K = M)
#pragma unroll
      for (int kk = 0; kk < N / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
        mma_bf16_ss(tmem + K::kColP1, smem_desc_sw128(cC + off, 16, 1024), smem_desc_sw128(cB + off, 16, 1024), iPP,
                    kk > 0);
        mma_bf16_ss(tmem + K::kColDX, smem_desc_sw128(cB + off, 16, 1024),
                    smem_desc_sw128(cG + kk * 2048, K::HB_BYTES, 1024), iBG, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < kP / 16; ++kk) {
        mma_bf16_ss(tmem + K::kColP2, smem_desc_sw128(cY + kk * 32, 16, 1024), smem_desc_sw128(cX + kk * 32, 16, 1024),
                    iPP, kk > 0);
        mma_bf16_ss(tmem + K::kColDC, smem_desc_sw128(cYe + kk * 32, 16, 1024),
                    smem_desc_sw128(cHB + kk * 32, 16, 1024), iMN, kk > 0);
        mma_bf16_ss(tmem + K::kColDB, smem_desc_sw128(cXw + kk * 32, 16, 1024),
                    smem_desc_sw128(cG + kk * 32, 16, 1024), iMN, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < kM / 16; ++kk)
        mma_bf16_ss(tmem + K::kColGA, smem_desc_sw128(cC + kk * 2048, kBlk, 1024),
                    smem_desc_sw128(cYe + kk * 2048, kBlk, 1024), iGA, kk > 0);
      mma_commit(&bars[2]);
    }
    if (!block_wait(&bars[2], r & 1, abort_flag, status, kTagMma1, a.wait_limit)) {
      abort_r = r;
      abort_stage = 1;
      break;
    }
    tc_fence_after();

    // ---- epilogue A: S, W (bf16 tiles), token sums, G update ----
    {
      const float* c2 = sc + sC2 * kScalStride;
      const float* wv = sc + sW * kScalStride;
      const float c2m = c2[tm], gam_m = sc[sGam * kScalStride + tm];
      const int c0 = 16 * sl + 8 * half;  // this thread's 8 columns of P1, P2
      float p1[8], p2[8];
      tmem_ld_16x2(tmem + lane_base + K::kColP1 + 16 * sl, p1);
      tmem_ld_16x2(tmem + lane_base + K::kColP2 + 16 * sl, p2);
      tmem_ld_wait();
      float z_diag = 0.f, z_row = 0.f, colz[8];
      uint32_t sp[4], wp[4];
#pragma unroll
      for (int jj = 0; jj < 8; jj += 2) {
        float sv[2], wvv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = c0 + jj + e, tj = j / R;
          const float q = p1[jj + e] * p2[jj + e];
          float kf = 0.f, ez = 0.f;
          if (tj < tm) {
            ez = ex2(c2m - c2[tj]);
            kf = ez * wv[tj];
            z_row += kf * q;
          } else if (tj == tm) {
            kf = gam_m;
            z_diag += q;
          }
          colz[jj + e] = ez * q;
          sv[e] = kf * p1[jj + e] + (j == m ? Dh : 0.f);
          wvv[e] = kf * p2[jj + e];
          if (j == m) dD_acc += p2[jj + e];
        }
        sp[jj / 2] = pack_bf16(sv[0], sv[1]);
        wp[jj / 2] = pack_bf16(wvv[0], wvv[1]);
      }
      *reinterpret_cast<uint4*>(smem + K::OFF_S + swz(m, c0 / 8)) = make_uint4(sp[0], sp[1], sp[2], sp[3]);
      *reinterpret_cast<uint4*>(smem + K::OFF_W + swz(m, c0 / 8)) = make_uint4(wp[0], wp[1], wp[2], wp[3]);
      // the two halves hold the same row
      z_diag += __shfl_xor_sync(0xffffffffu, z_diag, 16);
      z_row += __shfl_xor_sync(0xffffffffu, z_row, 16);
      if (half == 0) {
        atomicAdd(&sc[sDg * kScalStride + tm], z_diag);
        atomicAdd(&sc[sRT * kScalStride + tm], z_row);
      }
      // column sums over the 16 rows of each half
      float mine = 0.f;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        float v = colz[jj];
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if ((lane & 15) == jj) mine = v;
      }
      if ((lane & 15) < 8 && mine != 0.f) atomicAdd(&sc[sCZu * kScalStride + (c0 + (lane & 15)) / R], mine);

      // zin: sum_n C~[m][n] dC~1[m][n] over the warp's N / 4 columns (8 per thread and piece)
      {
        constexpr int NCW = N / 4;
        float zin = 0.f;
#pragma unroll
        for (int pc = 0; pc < NCW / 16; ++pc) {
          const int cb = NCW * sl + 16 * pc;
          float dc[8];
          tmem_ld_16x2(tmem + lane_base + K::kColDC + cb, dc);
          tmem_ld_wait();
          const int nn = cb + 8 * half;
          const uint4 cq = *reinterpret_cast<const uint4*>(st + K::OFF_C + (nn / 64) * kBlk + swz(m, (nn % 64) / 8));
          const uint32_t cw[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 cv = unpack_bf16(cw[k]);
            zin += cv.x * dc[2 * k] + cv.y * dc[2 * k + 1];
          }
        }
        zin += __shfl_xor_sync(0xffffffffu, zin, 16);
        if (half == 0) atomicAdd(&sc[sZin * kScalStride + tm], zin);
      }
      // zue: e^{cum_end - cum} sum_p X[m][p] (B~ G)[m][p] (B~ G is scaled by f in epilogue B)
      {
        float bg[8];
        tmem_ld_16x2(tmem + lane_base + K::kColDX + 16 * sl, bg);
        tmem_ld_wait();
        const uint4 xq = *reinterpret_cast<const uint4*>(st + K::OFF_X + swz(m, (16 * sl + 8 * half) / 8));
        const uint32_t xw[4] = {xq.x, xq.y, xq.z, xq.w};
        float zue = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 xv = unpack_bf16(xw[k]);
          zue += xv.x * bg[2 * k] + xv.y * bg[2 * k + 1];
        }
        zue += __shfl_xor_sync(0xffffffffu, zue, 16);
        if (half == 0) atomicAdd(&sc[sZue * kScalStride + tm], zue * sc[sEend * kScalStride + tm]);
      }
      // G <- e^{cum_end} G + C~^T dY_e; <hbar_in, G_out> for the decay of every token
      {
        float acc[16];
        tmem_ld16(tmem + lane_base + K::kColGA + p0, acc);
        tmem_ld_wait();
        const float ecend = ex2(sc[sSpare * kScalStride]);
        float hg = 0.f;
        if (n >= 0) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const uint4 hq = *reinterpret_cast<const uint4*>(st + K::OFF_HB + swz(n, p0 / 8 + h2));
            const uint32_t hw[4] = {hq.x, hq.y, hq.z, hq.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float2 hv = unpack_bf16(hw[k]);
              hg += hv.x * G[8 * h2 + 2 * k] + hv.y * G[8 * h2 + 2 * k + 1];
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) G[i] = ecend * G[i] + acc[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) hg += __shfl_xor_sync(0xffffffffu, hg, o);
        if (lane == 0) atomicAdd(&red[0], hg);
        store_G();
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();

    // ---- MMA batch 2 ----
    if (tid == 0) {
      tc_fence_after();
      const uint32_t cB = smem_u32(st + K::OFF_B), cC = smem_u32(st + K::OFF_C), cY = smem_u32(st + K::OFF_DY);
      const uint32_t cS = smem_u32(smem + K::OFF_S), cW = smem_u32(smem + K::OFF_W);
      const uint32_t iWB = idesc_bf16(kM, N, 0, 1);    // W B~      (A K-major, B MN-major)
      const uint32_t iWC = idesc_bf16(kM, N, 1, 1);    // W^T C~    (both MN-major)
      const uint32_t iSY = idesc_bf16(kM, kP, 1, 1);   // S^T dY    (both MN-major; into P1's columns)
#pragma unroll
      for (int kk = 0; kk < kM / 16; ++kk) {
        mma_bf16_ss(tmem + K::kColDC, smem_desc_sw128(cW + kk * 32, 16, 1024),
                    smem_desc_sw128(cB + kk * 2048, kBlk, 1024), iWB, 1u);
        mma_bf16_ss(tmem + K::kColDB, smem_desc_sw128(cW + kk * 2048, kBlk, 1024),
                    smem_desc_sw128(cC + kk * 2048, kBlk, 1024), iWC, 1u);
        mma_bf16_ss(tmem + K::kColP1, smem_desc_sw128(cS + kk * 2048, kBlk, 1024),
                    smem_desc_sw128(cY + kk * 2048, kBlk, 1024), iSY, kk > 0 ? 1u : 0u);
      }
      mma_commit(&bars[3]);
    }
    if (!block_wait(&bars[3], r & 1, abort_flag, status, kTagMma2, a.wait_limit)) {
      abort_r = r;
      abort_stage = 2;
      break;
    }
    tc_fence_after();

    // ---- epilogue B: dX = f B~G + S^T dY; dB~, dC~ rotated back by +Phi; the angle gradient ----
    {
      const int t = t0 + tm;
      const bool store = t < L;
      const bool last = (t == L - 1);
      {
        float bg[8], sx[8];
        tmem_ld_16x2(tmem + lane_base + K::kColDX + 16 * sl, bg);
        tmem_ld_16x2(tmem + lane_base + K::kColP1 + 16 * sl, sx);
        tmem_ld_wait();
        const float f = sc[sF * kScalStride + tm];
        const int c0 = 16 * sl + 8 * half;
        float dx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) dx[i] = f * bg[i] + sx[i];
        if (last && g.dxprev_out) {
#pragma unroll
          for (int i = 0; i < 8; ++i) dx[i] += g.dxprev_out[((size_t)unit * R + rm) * kP + c0 + i];
        }
        if (store)
          *reinterpret_cast<uint4*>(dXg + (tok_index(a, b, t, hh) * R + rm) * kP + c0) =
              make_uint4(pack_bf16(dx[0], dx[1]), pack_bf16(dx[2], dx[3]), pack_bf16(dx[4], dx[5]),
                         pack_bf16(dx[6], dx[7]));
      }
      constexpr int NCW = N / 4;
#pragma unroll 1
      for (int pc = 0; pc < NCW / 16; ++pc) {
        const int cb = NCW * sl + 16 * pc;
        const int nn = cb + 8 * half;  // this thread's 8 state columns (4 pairs)
        float dc[8], db[8];
        tmem_ld_16x2(tmem + lane_base + K::kColDC + cb, dc);
        tmem_ld_16x2(tmem + lane_base + K::kColDB + cb, db);
        tmem_ld_wait();
        if (last && g.dbprev_out) {
#pragma unroll
          for (int i = 0; i < 8; ++i) db[i] += g.dbprev_out[((size_t)unit * R + rm) * N + nn + i];
        }
        float bt[8], ct[8];
        {
          const uint32_t off = (nn / 64) * kBlk + swz(m, (nn % 64) / 8);
          const uint4 bq = *reinterpret_cast<const uint4*>(st + K::OFF_B + off);
          const uint4 cq = *reinterpret_cast<const uint4*>(st + K::OFF_C + off);
          const uint32_t bw[4] = {bq.x, bq.y, bq.z, bq.w}, cw[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 bv = unpack_bf16(bw[k]), cv = unpack_bf16(cw[k]);
            bt[2 * k] = bv.x; bt[2 * k + 1] = bv.y;
            ct[2 * k] = cv.x; ct[2 * k + 1] = cv.y;
          }
        }
        float dph[4], ob[8], oc[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float db0 = db[2 * i], db1 = db[2 * i + 1], dc0 = dc[2 * i], dc1 = dc[2 * i + 1];
          dph[i] = db0 * bt[2 * i + 1] - db1 * bt[2 * i] + dc0 * ct[2 * i + 1] - dc1 * ct[2 * i];
          float sn, cs;
          __sincosf(pht[(nn / 2 + i) * QP + tm], &sn, &cs);
          ob[2 * i] = cs * db0 - sn * db1;
          ob[2 * i + 1] = sn * db0 + cs * db1;
          oc[2 * i] = cs * dc0 - sn * dc1;
          oc[2 * i + 1] = sn * dc0 + cs * dc1;
        }
        if (store) {
          if constexpr (GRP) {  // shared rows: this head's share, summed over the group in fp32
            const size_t gi = ((((size_t)b * L + t) * a.ngroups + gh) * R + rm) * N + nn;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              atomicAdd(g.dBh + gi + i, ob[i]);
              atomicAdd(g.dCh + gi + i, oc[i]);
            }
          } else {
            const size_t gi = (tok_index(a, b, t, hh) * R + rm) * N + nn;
            *reinterpret_cast<uint4*>(dBg + gi) = make_uint4(pack_bf16(ob[0], ob[1]), pack_bf16(ob[2], ob[3]),
                                                             pack_bf16(ob[4], ob[5]), pack_bf16(ob[6], ob[7]));
            *reinterpret_cast<uint4*>(dCg + gi) = make_uint4(pack_bf16(oc[0], oc[1]), pack_bf16(oc[2], oc[3]),
                                                             pack_bf16(oc[4], oc[5]), pack_bf16(oc[6], oc[7]));
          }
        }
        // the angle gradient of the token: sum over its R rows (consecutive lanes of a half)
#pragma unroll
        for (int o = 1; o < R; o <<= 1)
#pragma unroll
          for (int i = 0; i < 4; ++i) dph[i] += __shfl_xor_sync(0xffffffffu, dph[i], o);
        if (rm == 0)  // row tm, pairs XOR-swizzled by the row (see dphi_at)
          *reinterpret_cast<float4*>(dphi_s + dphi_at(tm, nn / 2)) = make_float4(dph[0], dph[1], dph[2], dph[3]);
      }
    }
    tc_fence_before();  // P1, DC, DB, DX are rewritten by the next chunk's first batch
    __syncthreads();

    // ---- the angle gradient summed from the end: dtheta = dt S, and sum_k theta S per token ----
    {
      const int k = tid % K2, part = tid / K2;
      const int tb = part * TPP2;
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < TPP2; ++i)
        if (tb + i < Q) ps += dphi_s[dphi_at(tb + i, k)];
      part_sum[part * K2 + k] = ps;
      __syncthreads();
      // running sum from the end of the sequence, double-buffered by chunk parity
      float S = sang[(r & 1) * K2 + k];
      for (int p2 = part + 1; p2 < NPART2; ++p2) S += part_sum[p2 * K2 + k];
      float v[TPP2];  // theta S of this thread's pair at each of its tokens
#pragma unroll
      for (int i = TPP2 - 1; i >= 0; --i) {
        const int t = tb + i;
        v[i] = 0.f;
        if (t < Q) {
          S += dphi_s[dphi_at(t, k)];
          const float dtv = sc[sDt * kScalStride + t];
          const int tg = t0 + t;
          if (tg < L) dTHg[tok_index(a, b, tg, hh) * K2 + k] = __float2bfloat16_rn(dtv * S);
          v[i] = __bfloat162float(th[t * K2 + k]) * S;
        }
      }
      // the sums over the warp's 32 pairs of all TPP2 tokens at once: each butterfly
      // step halves the values a lane holds (it keeps the half its lane bit selects
      // and adds the partner's copy of it), then the last steps reduce the one left
      constexpr int HB = TPP2 >= 16 ? 4 : (TPP2 >= 8 ? 3 : (TPP2 >= 4 ? 2 : (TPP2 >= 2 ? 1 : 0)));
      static_assert((1 << HB) == TPP2, "tokens per part: a power of two");
#pragma unroll
      for (int st2 = 0; st2 < HB; ++st2) {
        const int off = 16 >> st2, hlf = TPP2 >> (st2 + 1);
        const bool up = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < TPP2 / 2; ++i)
          if (i < hlf) {
            const float send = up ? v[i] : v[i + hlf];
            const float keep = up ? v[i + hlf] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
      }
#pragma unroll
      for (int off = 16 >> HB; off > 0; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
      int j = 0;  // the token whose sum this lane holds
#pragma unroll
      for (int st2 = 0; st2 < HB; ++st2)
        if (lane & (16 >> st2)) j += TPP2 >> (st2 + 1);
      if ((lane & ((32 >> HB) - 1)) == 0 && tb + j < Q) atomicAdd(&sc[sDth * kScalStride + tb + j], v[0]);
      if (part == 0) sang[((r + 1) & 1) * K2 + k] = S;
    }
    __syncthreads();

    // ---- per token: the decay, gamma and w gradients -> ddt, dlam, dA (warp 0) ----
    if (warp == 0) {
      const int i0 = 2 * lane, i1 = 2 * lane + 1;
      auto V = [&](int arr, int i) { return i < Q ? sc[arr * kScalStride + i] : 0.f; };
      const float zin0 = V(sZin, i0), zin1 = V(sZin, i1);
      float suf = zin0 + zin1;  // suffix over lanes of the pair sums
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += u;
      }
      const float suf0 = suf, suf1 = suf - zin0;
      const float w0 = V(sW, i0), w1 = V(sW, i1);
      const float dw0 = V(sZue, i0) + V(sCZu, i0), dw1 = V(sZue, i1) + V(sCZu, i1);
      const float g0 = w0 * dw0 - V(sRT, i0), g1 = w1 * dw1 - V(sRT, i1);
      float pre = g0 + g1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, pre, o);
        if (lane >= o) pre += u;
      }
      const float ex0 = pre - g0 - g1, ex1 = pre - g1;  // exclusive prefixes at tokens i0, i1
      const float c0 = ex2(sc[sSpare * kScalStride]) * red[0];
      const float da0 = c0 + suf0 + ex0, da1 = c0 + suf1 + ex1;
      const float dt0 = V(sDt, i0), dt1 = V(sDt, i1), lm0 = V(sLam, i0), lm1 = V(sLam, i1);
      const float at0 = V(sAt, i0), at1 = V(sAt, i1);
      const float dgam0 = V(sDg, i0) + dw0, dgam1 = V(sDg, i1) + dw1;
      const float dwp = __shfl_up_sync(0xffffffffu, dw1, 1);  // dw of token i0 - 1
      float ddt0 = da0 * at0 + dgam0 * lm0 + V(sDth, i0), dlm0 = dgam0 * dt0;
      if (lane > 0) {
        ddt0 += dwp * (1.f - lm0);
        dlm0 -= dwp * dt0;
      }
      const float ddt1 = da1 * at1 + dgam1 * lm1 + V(sDth, i1) + dw0 * (1.f - lm1);
      const float dlm1 = dgam1 * dt1 - dw0 * dt1;
      if (i1 < Q && t0 + i1 < L) {
        const size_t ti = tok_index(a, b, t0 + i1, hh);
        dDTg[ti] = __float2bfloat16_rn(ddt1);
        dLMg[ti] = __float2bfloat16_rn(dlm1);
        if constexpr (TVA) dATg[ti] = __float2bfloat16_rn(da1 * dt1);
      }
      if (i0 < Q && t0 + i0 < L) {
        const size_t ti = tok_index(a, b, t0 + i0, hh);
        if (lane > 0) {
          dDTg[ti] = __float2bfloat16_rn(ddt0);
          dLMg[ti] = __float2bfloat16_rn(dlm0);
        }
        if constexpr (TVA) dATg[ti] = __float2bfloat16_rn(da0 * dt0);
      }
      float dap = da0 * dt0 + da1 * dt1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dap += __shfl_xor_sync(0xffffffffu, dap, o);
      const float dw_last = __shfl_sync(0xffffffffu, dw1, (Q - 1) / 2);  // token Q - 1
      if (lane == 0) {
        dA_acc += dap;
        if (pend_t >= 0) {  // the first token of the chunk after this one: its lagged weight sits in w_{Q-1}
          const size_t ti = tok_index(a, b, pend_t, hh);
          dDTg[ti] = __float2bfloat16_rn(pend_ddt + dw_last * (1.f - sc[sLam * kScalStride + Q]));
          dLMg[ti] = __float2bfloat16_rn(pend_dlm - dw_last * sc[sDt * kScalStride + Q]);
        }
        pend_t = t0;
        pend_ddt = ddt0;
        pend_dlm = dlm0;
      }
    }
    __syncthreads();
  }

  if (skip) {
    // (no ticket in range, or the hand-over never came: nothing was issued)
  } else if (abort_r >= 0) {
    if (tid == 0) {
      // let what was issued land before TMEM is freed and the CTA exits: the
      // loads not yet waited for and the MMA batch the abort interrupted
      for (int r2 = abort_r + (abort_stage > 0 ? 1 : 0); r2 < issued; ++r2)
        if (!mbar_wait_drain(&bars[r2 & 1], (r2 >> 1) & 1)) report_timeout(status, kTagDrain2);
      if (abort_stage > 0 && !mbar_wait_drain(&bars[1 + abort_stage], abort_r & 1))
        report_timeout(status, kTagDrain2);
    }
  } else if (hand_out) {
    // ---- the end of a split unit: its dA and dD shares into the globals; G, the
    // running angle-gradient sum and the pending token's ddt, dlam to the hand-over ----
    if (tid < 4) red[1 + tid] = 0.f;
    __syncthreads();
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, o);
    if (lane == 0) atomicAdd(&red[2], dD_acc);
    if (n >= 0) {
#pragma unroll
      for (int i = 0; i < 16; ++i) hand_out[n * kP + p0 + i] = G[i];
    }
    for (int k = tid; k < K2; k += kCThreads) hand_out[N * kP + k] = sang[(r_end & 1) * K2 + k];
    __syncthreads();
    if (tid == 0) {
      hand_out[N * kP + K2] = pend_ddt;
      hand_out[N * kP + K2 + 1] = pend_dlm;
      if (!TVA) atomicAdd(g.dA + hh, dA_acc);
      if (g.dD) atomicAdd(g.dD + hh, red[2]);
    }
    __threadfence();
  } else {
    // ---- the initial state: hbar_in of the first chunk = h_0 + mu1 sum_r b_prev0[r]^T x_prev0[r] ----
    float* Gs = reinterpret_cast<float*>(smem);  // [N][P] f32 in the stage buffers (no loads pending)
    if (n >= 0) {
#pragma unroll
      for (int i = 0; i < 16; ++i) Gs[n * kP + p0 + i] = G[i];
    }
    if (tid < 4) red[1 + tid] = 0.f;
    __syncthreads();
    const bool has_init = a.h0 != nullptr;
    const size_t i0 = tok_index(a, b, 0, hh);
    const float dt_0 = __bfloat162float(DT[i0]), lm_0 = __bfloat162float(LM[i0]);
    const float mu1 = (1.f - lm_0) * dt_0;
    float part = 0.f;
    if (has_init)
      for (int i = tid; i < N * kP; i += kCThreads) {
        const int nn = i / kP, pp = i % kP;
        float u = 0.f;
        for (int rr = 0; rr < R; ++rr)
          u += a.bprev0[((size_t)unit * R + rr) * N + nn] * a.xprev0[((size_t)unit * R + rr) * kP + pp];
        part += u * Gs[i];
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      part += __shfl_xor_sync(0xffffffffu, part, o);
      dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, o);
    }
    if (lane == 0) {
      atomicAdd(&red[1], part);
      atomicAdd(&red[2], dD_acc);
    }
    __syncthreads();
    if (tid == 0) {
      const float dmu = red[1];
      dDTg[i0] = __float2bfloat16_rn(pend_ddt + dmu * (1.f - lm_0));
      dLMg[i0] = __float2bfloat16_rn(pend_dlm - dmu * dt_0);
      if (!TVA) atomicAdd(g.dA + hh, dA_acc);
      if (g.dD) atomicAdd(g.dD + hh, red[2]);
    }
    if (g.dh0) {
      for (int i = tid; i < N * kP; i += kCThreads) g.dh0[(size_t)unit * N * kP + i] = Gs[i];
      for (int i = tid; i < R * N; i += kCThreads) {
        const int rr = i / N, nn = i % N;
        float s2 = 0.f;
        if (has_init)
          for (int pp = 0; pp < kP; ++pp) s2 += Gs[nn * kP + pp] * a.xprev0[((size_t)unit * R + rr) * kP + pp];
        g.dbprev0[(size_t)unit * R * N + i] = mu1 * s2;
      }
      for (int i = tid; i < R * kP; i += kCThreads) {
        const int rr = i / kP, pp = i % kP;
        float s2 = 0.f;
        if (has_init)
          for (int nn = 0; nn < N; ++nn) s2 += Gs[nn * kP + pp] * a.bprev0[((size_t)unit * R + rr) * N + nn];
        g.dxprev0[(size_t)unit * R * kP + i] = mu1 * s2;
      }
      for (int k = tid; k < K2; k += kCThreads) g.dangle0[(size_t)unit * K2 + k] = sang[(r_end & 1) * K2 + k];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  // the end of a split unit releases its hand-over (also after an abort, so that the
  // CTA of the unit's start never waits for one that has ended)
  if (tid == 0 && hand_out != nullptr) {
    __threadfence();
    st_release_gpu(sp.flags + item, 1);
  }
}

// dB[b, t, g] (dtype of the inputs) from the fp32 group sums
__global__ void __launch_bounds__(256) bc_group_convert_kernel(const float* dBs, const float* dCs, __nv_bfloat16* dB,
                                                               __nv_bfloat16* dC, long long total4) {
  for (long long e = (long long)blockIdx.x * 256 + threadIdx.x; e < total4; e += (long long)gridDim.x * 256) {
    const float4 vb = reinterpret_cast<const float4*>(dBs)[e];
    const float4 vc = reinterpret_cast<const float4*>(dCs)[e];
    reinterpret_cast<uint2*>(dB)[e] = make_uint2(pack_bf16(vb.x, vb.y), pack_bf16(vb.z, vb.w));
    reinterpret_cast<uint2*>(dC)[e] = make_uint2(pack_bf16(vc.x, vc.y), pack_bf16(vc.z, vc.w));
  }
}

// ------------------------------------------------------------------ host side
template <int N, int R, bool TVA, bool GRP>
int launch_nr(const BwdArgs& g, cudaStream_t s) {
  using SK = SCfg<N, R>;
  using CK = CCfg<N, R>;
  const ScanArgs& a = g.f;
  constexpr int Q = BCfg<N, R>::Q;
  const int nchunks = (a.seqlen + Q - 1) / Q;
  const int units = a.batch * a.nheads;
  uint8_t* ckpt = static_cast<uint8_t*>(a.workspace) + 256;
  CUtensorMap tmB, tmC, tmX, tmDY, tmT;
  if (!make_map(&tmB, a.B, N, a.ngroups, a, Q) || !make_map(&tmC, a.C, N, a.ngroups, a, Q) ||
      !make_map(&tmX, a.x, kP, a.nheads, a, Q) || !make_map(&tmDY, g.dy, kP, a.nheads, a, Q) ||
      !make_theta_map(&tmT, a, Q))
    return MAMBA3_ERR_CUDA;
  auto ks = bwd_state_kernel<N, R, TVA>;
  auto kc = bwd_chunk_kernel<N, R, TVA, GRP>;
  if (cudaFuncSetAttribute(ks, cudaFuncAttributeMaxDynamicSharedMemorySize, SK::SMEM_ALLOC) != cudaSuccess ||
      cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, CK::SMEM_ALLOC) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  ks<<<units, kSThreads, SK::SMEM_ALLOC, s>>>(tmB, tmX, tmT, a, ckpt, nchunks);
  if (cudaGetLastError() != cudaSuccess) return MAMBA3_ERR_CUDA;
  BwdSplit sp;
  memset(&sp, 0, sizeof(sp));
  if (g.split) {  // the region after the checkpoints and group sums (bwd_tc_split_bytes)
    const SplitPlan p = split_plan(units, nchunks);
    if (p.k > 0) {
      uint8_t* region = static_cast<uint8_t*>(a.workspace) + 256 + ((bwd_tc_workspace_bytes(a) + 255) & ~(size_t)255);
      const size_t flag_bytes = ((size_t)(p.k + 1) * 4 + 255) & ~(size_t)255;
      sp.k = p.k;
      sp.c1 = p.c1;
      sp.ticket = reinterpret_cast<int*>(region);
      sp.flags = sp.ticket + 1;
      sp.hand = reinterpret_cast<float*>(region + flag_bytes);
      if (cudaMemsetAsync(region, 0, flag_bytes, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
    }
  }
  kc<<<units + sp.k, kCThreads, CK::SMEM_ALLOC, s>>>(tmB, tmC, tmX, tmDY, tmT, g, ckpt, nchunks, sp);
  if (cudaGetLastError() != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (GRP) {
    const long long total4 = (long long)a.batch * a.seqlen * a.ngroups * R * N / 4;
    long long blocks = (total4 + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    if (blocks > 0)
      bc_group_convert_kernel<<<(int)blocks, 256, 0, s>>>(g.dBh, g.dCh, static_cast<__nv_bfloat16*>(g.dB),
                                                          static_cast<__nv_bfloat16*>(g.dC), total4);
  }
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

template <int N, int R>
int launch_r(const BwdArgs& g, cudaStream_t s) {
  const bool tva = g.f.A_t != nullptr, grp = g.f.ngroups < g.f.nheads;
  if (tva) return grp ? launch_nr<N, R, true, true>(g, s) : launch_nr<N, R, true, false>(g, s);
  return grp ? launch_nr<N, R, false, true>(g, s) : launch_nr<N, R, false, false>(g, s);
}

}  // namespace

int bwd_tc_supported(const ScanArgs& a) {
  if (a.dtype != MAMBA3_BF16 || a.P != kP || a.seqlen < 1 || a.bcnorm) return MAMBA3_ERR_UNSUPPORTED;
  if (a.N != 64 && a.N != 128) return MAMBA3_ERR_UNSUPPORTED;
  if (a.R != 1 && a.R != 2 && a.R != 4) return MAMBA3_ERR_UNSUPPORTED;
  if (a.nheads % a.ngroups != 0) return MAMBA3_ERR_INVALID;
  return MAMBA3_OK;
}

size_t bwd_tc_split_bytes(const ScanArgs& a) {
  if (bwd_tc_supported(a) != MAMBA3_OK) return 0;
  const int Q = 64 / a.R, nchunks = (a.seqlen + Q - 1) / Q;
  const SplitPlan p = split_plan(a.batch * a.nheads, nchunks);
  if (p.k == 0) return 0;
  const size_t slot = ((size_t)a.N * kP + a.N / 2 + 4) * sizeof(float);
  return 256 + (((size_t)(p.k + 1) * 4 + 255) & ~(size_t)255) + (size_t)p.k * slot;  // (256: alignment)
}

size_t bwd_tc_workspace_bytes(const ScanArgs& a) {
  const size_t Q = kM / a.R, nchunks = ((size_t)a.seqlen + Q - 1) / Q;
  const size_t ck = (size_t)a.batch * a.nheads * nchunks * ((size_t)a.N * 128 + (size_t)a.N / 2 * 4);
  const size_t grp = a.ngroups < a.nheads ? 2 * (size_t)a.batch * a.seqlen * a.ngroups * a.R * a.N * 4 : 0;
  return ((ck + 255) & ~(size_t)255) + grp;
}

// Workspace after the 256-byte status word: the checkpoints (state tiles, then
// angles), then with grouped B/C the fp32 group sums of dB and dC.
int launch_scan_bwd_tc(BwdArgs g, cudaStream_t s) {
  const ScanArgs& a = g.f;
  if (g.dA && cudaMemsetAsync(g.dA, 0, sizeof(float) * a.nheads, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (g.dD && cudaMemsetAsync(g.dD, 0, sizeof(float) * a.nheads, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  const size_t Q = kM / a.R, nchunks = ((size_t)a.seqlen + Q - 1) / Q;
  const size_t ck = (size_t)a.batch * a.nheads * nchunks * ((size_t)a.N * 128 + (size_t)a.N / 2 * 4);
  if (a.ngroups < a.nheads) {
    const size_t gb = (size_t)a.batch * a.seqlen * a.ngroups * a.R * a.N * 4;
    g.dBh = reinterpret_cast<float*>(static_cast<uint8_t*>(a.workspace) + 256 + ((ck + 255) & ~(size_t)255));
    g.dCh = g.dBh + gb / 4;
    if (cudaMemsetAsync(g.dBh, 0, 2 * gb, s) != cudaSuccess) return MAMBA3_ERR_CUDA;
  } else {
    g.dBh = g.dCh = nullptr;
  }
  if (a.N == 128) {
    if (a.R == 1) return launch_r<128, 1>(g, s);
    if (a.R == 2) return launch_r<128, 2>(g, s);
    if (a.R == 4) return launch_r<128, 4>(g, s);
  } else {
    if (a.R == 1) return launch_r<64, 1>(g, s);
    if (a.R == 2) return launch_r<64, 2>(g, s);
    if (a.R == 4) return launch_r<64, 4>(g, s);
  }
  return MAMBA3_ERR_UNSUPPORTED;
}

}  // namespace m3

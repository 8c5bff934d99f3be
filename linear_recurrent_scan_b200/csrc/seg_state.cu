// End state of every segment of a long sequence from a zero state and a zero
// angle (the segment aggregates of the segmented prefill, scan_seg.cu), as one
// streaming tensor-core reduction per segment (tcgen05 + TMA, bf16, sm_100a).
//
// In the frame rotated by -Phi the decay is real ("Mamba-3: 2x smaller state ..."
// (MarkTechPost, Korean translation), sections 1.1-1.2), so the state after the
// last token of a segment is one sum over its tokens,
//   h_end = sum_s e^{cum_end - cum_s} w_s B~_s^T x_s        (cum inclusive, from the
//                                                             segment start)
// with the trapezoid weight w_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1} (the last
// token's next one lies outside the segment: w = gamma).  Every 128-row chunk adds
// B~^T X_w (K = 128) to ONE TMEM accumulator, with X_w = diag(e^{cum_end - cum} w)
// X weighted to the segment's end: no per-chunk epilogue, so the MMAs run behind
// the chunk preparation (decay prefix, angles, RoPE of B in place, X_w written over
// X in place) through a TMA ring of 3-5 stages; where three stages fit in half an
// SM's shared memory, two CTAs share the SM and hide each other's waits.
// cum_end - cum_s is the difference of two fp32 sums over the
// segment (<= 1.6 per token here), a relative error near 1e-4 in the weight; a
// weight that underflows belongs to a term below fp32 resolution.
// 256 threads; at the end the accumulator becomes h (fp32), with the B of the
// last token rotated by its angle (fp32), its x and the angle.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace m3 {
namespace {

using namespace ptx;

constexpr int kP = 64;
constexpr int kM = 128;          // rows per chunk
constexpr int kTile = 16384;     // 128 rows x 128 bytes, 128-byte swizzle
constexpr int kThreads = 256;
// Besides its share of every chunk's preparation, one lane issues the TMA loads (warp
// 7), one warp loads the next chunks' scalars (warp 6) and one lane issues the MMAs
// (thread 0), so that no warp carries more than one of these to the chunk's barrier.
constexpr int kLoader = kThreads - 32;  // lane 0 of warp 7
constexpr int kScalarWarp = 6;

enum Tag { kTagFull = 41, kTagMma, kTagDrain };

__device__ __forceinline__ uint32_t swz(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// NST stages of inputs; chunk c + NST - 1 is loaded in the middle of chunk c, into the
// stage that the MMA of chunk c - 1 read.  Two CTAs per SM with three stages where
// they fit in half of the SM's 228 KB (less 1 KB per CTA), else one CTA with as many
// stages (up to 5) as fit.
template <int N, int R>
struct GCfg {
  static constexpr int Q = kM / R;
  static constexpr int NKB = N / 64;
  static constexpr int K2 = N / 2;
  static constexpr int NG = K2 / 4;                     // 16-byte groups of a row
  static constexpr int TH_BYTES = Q * K2 * 2;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_X = NKB * kTile;             // X, then X_w in place
  static constexpr int OFF_TH = OFF_X + kTile;
  static constexpr int STAGE = OFF_TH + ((TH_BYTES + 1023) & ~1023);
  // final angle, sums, barriers, misc, and the per-token scalars of two chunks
  // ([2][3][Q + 1] floats: dt, lam, A_t of the chunk's tokens and the next one)
  static constexpr int TAIL = (K2 * 4 + 64 + 2 * 5 * 8 + 16 + 24 * (Q + 1) + 64 + 1023) & ~1023;
  static constexpr int fit(int st) { return st * STAGE + TAIL + 1024; }
  static constexpr int CPS = fit(2) <= 233472 / 3 - 1024 ? 3 : (fit(3) <= 233472 / 2 - 1024 ? 2 : 1);  // CTAs per SM
  static constexpr int NST = CPS == 3 ? 2 : (CPS == 2 ? 3 : (fit(5) <= 232448 ? 5 : (fit(4) <= 232448 ? 4 : (fit(3) <= 232448 ? 3 : 2))));
  static constexpr int D = NST - 1;                     // chunks loaded ahead
  static constexpr int OFF_PHI = NST * STAGE;           // final angle [K2]
  static constexpr int OFF_RED = OFF_PHI + K2 * 4;      // [8] warp sums
  static constexpr int OFF_BAR = (OFF_RED + 64 + 7) & ~7;  // full[NST], mma[NST]
  static constexpr int OFF_MISC = OFF_BAR + 2 * NST * 8;
  static constexpr int OFF_SCL = OFF_MISC + 16;
  static constexpr int SMEM = OFF_SCL + 24 * (Q + 1);
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static_assert(SMEM - OFF_PHI <= TAIL && SMEM_ALLOC <= 232448 && NST >= 2, "shared memory");
};

template <int N, int R, bool TVA>
__global__ void __launch_bounds__(kThreads, GCfg<N, R>::CPS) seg_state_kernel(const __grid_constant__ CUtensorMap tmB,
                                                             const __grid_constant__ CUtensorMap tmX,
                                                             const __grid_constant__ CUtensorMap tmT,
                                                             const ScanArgs a) {
  using K = GCfg<N, R>;
  constexpr int Q = K::Q, K2 = K::K2, NG = K::NG, NST = K::NST, D = K::D;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int unit = blockIdx.x, b = unit / a.nheads, hh = unit % a.nheads;
  const int L = a.seqlen, H = a.nheads;
  const int gh = hh / (a.nheads / a.ngroups);
  const int nchunks = (L + Q - 1) / Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.workspace);
  float* phi = reinterpret_cast<float*>(smem + K::OFF_PHI);
  float* red = reinterpret_cast<float*>(smem + K::OFF_RED);
  const __nv_bfloat16* DT = static_cast<const __nv_bfloat16*>(a.dt);
  const __nv_bfloat16* LM = static_cast<const __nv_bfloat16*>(a.lam);
  const __nv_bfloat16* AT = static_cast<const __nv_bfloat16*>(a.A_t);
  const float Ah = TVA ? 0.f : a.A[hh];
  auto tok = [&](int t) { return ((size_t)b * L + t) * H + hh; };

  if (tid == 0) {
    for (int i = 0; i < 2 * NST; ++i) mbar_init(&bars[i], 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto issue = [&](int c) {
    const int s = c % NST;
    uint8_t* st = smem + s * K::STAGE;
    const int t0 = c * Q;
    mbar_arrive_expect_tx(&bars[s], (uint32_t)(K::NKB * kTile + kTile + K::TH_BYTES));
#pragma unroll
    for (int kb = 0; kb < K::NKB; ++kb) tma_load_5d(st + K::OFF_B + kb * kTile, &tmB, &bars[s], kb * 64, 0, gh, t0, b);
    tma_load_5d(st + K::OFF_X, &tmX, &bars[s], 0, 0, hh, t0, b);
    tma_load_4d(st + K::OFF_TH, &tmT, &bars[s], 0, hh, t0, b);
  };
  int issued = 0;  // (the loader's) chunks whose loads were issued
  if (tid == kLoader && !a.test_withhold)
    for (; issued < D && issued < nchunks; ++issued) issue(issued);

  // the segment's total log2 decay (block reduction over its tokens)
  float tot = 0.f;
  for (int t = tid; t < L; t += kThreads) {
    const size_t i = tok(t);
    tot += __bfloat162float(DT[i]) * (TVA ? __bfloat162float(AT[i]) : Ah);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  if (lane == 0) red[warp] = tot;
  __syncthreads();
  float total = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) total += red[w];
  if (tid == 0 && a.decay_out) a.decay_out[unit] = total;
  total *= kLog2e;

  // Warp w owns the 4-pair groups w GPW .. w GPW + GPW - 1 of every row; lane l owns the
  // tokens l TPL .. l TPL + TPL - 1 of every chunk.  The decay prefix and the angle
  // prefix are warp scans over the lanes, so a chunk needs one block barrier, before
  // its MMA.  Every warp keeps the decay carry and its groups' running angles.
  constexpr int TPL = Q / 32, GPW = NG / (kThreads / 32);
  static_assert(TPL >= 1 && Q % 32 == 0 && TPL * R == 4 && GPW >= 1 && NG % (kThreads / 32) == 0, "lanes and warps");
  // dt, lam (and A_t) of a chunk's tokens and the next one: one warp loads chunk c + 2's
  // into registers while chunk c is prepared and stores them into buffer c & 1 ... of
  // chunk c + 1 at its end, so that every warp reads them from shared memory (one set of
  // global loads instead of one per warp, and no warp waits on them)
  constexpr int E = (Q + 1 + 31) / 32;
  float* scl = reinterpret_cast<float*>(smem + K::OFF_SCL);  // [2][3][Q + 1]
  float e_dt[E], e_lm[E], e_at[E];
  auto load_pre = [&](int c) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int k = lane + 32 * e, t = c * Q + k;
      e_dt[e] = 0.f;
      e_lm[e] = 1.f;
      e_at[e] = Ah;
      if (k <= Q && t < L) {
        const size_t ti = tok(t);
        e_dt[e] = __bfloat162float(DT[ti]);
        e_lm[e] = __bfloat162float(LM[ti]);
        if constexpr (TVA) e_at[e] = __bfloat162float(AT[ti]);
      }
    }
  };
  auto store_pre = [&](int buf) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int k = lane + 32 * e;
      if (k <= Q) {
        scl[(buf * 3 + 0) * (Q + 1) + k] = e_dt[e];
        scl[(buf * 3 + 1) * (Q + 1) + k] = e_lm[e];
        scl[(buf * 3 + 2) * (Q + 1) + k] = e_at[e];
      }
    }
  };
  if (warp == kScalarWarp) {
    load_pre(0);
    store_pre(0);
    load_pre(1);
  }
  __syncthreads();
  float carry = 0.f;       // log2 decay through the end of the previous chunk
  float phw[GPW][4];       // running angle of this warp's pair groups
#pragma unroll
  for (int q = 0; q < GPW; ++q)
#pragma unroll
    for (int k = 0; k < 4; ++k) phw[q][k] = 0.f;
  int abort_c = -1;

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % NST;
    uint8_t* st = smem + s * K::STAGE;
    float dt[TPL + 1], lm[TPL + 1], at[TPL];
    {
      const float* sb = scl + (c & 1) * 3 * (Q + 1);
#pragma unroll
      for (int i = 0; i <= TPL; ++i) {
        dt[i] = sb[lane * TPL + i];
        lm[i] = sb[(Q + 1) + lane * TPL + i];
        if (i < TPL) at[i] = TVA ? sb[2 * (Q + 1) + lane * TPL + i] : Ah;
      }
    }
    // decay prefix over the chunk (lane-local, then a warp scan) and the X_w weight f
    float f[TPL];
    {
      float v[TPL], run = 0.f;
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        v[i] = dt[i] * at[i] * kLog2e;
        run += v[i];
      }
      float incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      float acc = carry + incl - run;
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        acc += v[i];
        const float w = lm[i] * dt[i] + (1.f - lm[i + 1]) * dt[i + 1];
        f[i] = w * ex2(total - acc);
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (!mbar_wait(&bars[s], (c / NST) & 1, abort_flag, status, kTagFull, a.wait_limit)) {}
    if (*abort_flag) {  // block-wide decision at the barrier below
    }
    // angles of this warp's pair groups at this lane's tokens, RoPE of B in place
    const __nv_bfloat16* th = reinterpret_cast<const __nv_bfloat16*>(st + K::OFF_TH);
#pragma unroll
    for (int q = 0; q < GPW; ++q) {
      const int g = warp * GPW + q, kb = g / 8, c8 = g % 8;
      float inc[TPL][4], tot4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < TPL; ++i) {
        const int t = lane * TPL + i;
        // 8 bytes at byte 8 g of row t, through the tile's 64- / 128-byte swizzle (a
        // warp reads one column of the tile; unswizzled that is a 16-way bank conflict)
        const int chunk = (g >> 1) ^ (K2 == 32 ? ((t >> 1) & 3) : (t & 7));
        const uint2 tv = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(th) + t * (2 * K2) +
                                                         chunk * 16 + (g & 1) * 8);
        const float2 t01 = unpack_bf16(tv.x), t23 = unpack_bf16(tv.y);
        inc[i][0] = dt[i] * t01.x; inc[i][1] = dt[i] * t01.y; inc[i][2] = dt[i] * t23.x; inc[i][3] = dt[i] * t23.y;
#pragma unroll
        for (int k = 0; k < 4; ++k) tot4[k] += inc[i][k];
      }
      float ex[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x = tot4[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float u = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += u;
        }
        ex[k] = wrap_angle(phw[q][k] + x - tot4[k]);  // angle before this lane's first token
        phw[q][k] = wrap_angle(phw[q][k] + __shfl_sync(0xffffffffu, x, 31));
      }
      float sn[TPL][4], cs[TPL][4];
#pragma unroll
      for (int i = 0; i < TPL; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          ex[k] += inc[i][k];
          __sincosf(ex[k], &sn[i][k], &cs[i][k]);
        }
      // The lane's rows are 4 lane .. 4 lane + 3 (TPL R = 4).  Taken in the same order
      // by every lane, a warp's 32 accesses would fall on 2 of the 8 16-byte columns
      // of the 128-byte swizzle (row & 7 in {j, j + 4}); starting each lane pair one
      // row further spreads them over all 8.
      const int rot = (lane >> 1) & 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int jl = (j + rot) & 3, it = jl / R;
        float s4[4], c4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          s4[k] = sn[0][k];
          c4[k] = cs[0][k];
        }
#pragma unroll
        for (int ii = 1; ii < TPL; ++ii)
          if (it == ii) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              s4[k] = sn[ii][k];
              c4[k] = cs[ii][k];
            }
          }
        uint4* p = reinterpret_cast<uint4*>(st + K::OFF_B + kb * kTile + swz(lane * 4 + jl, c8));
        const uint4 qv = *p;
        const uint32_t bw[4] = {qv.x, qv.y, qv.z, qv.w};
        uint32_t bo[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 vv = unpack_bf16(bw[k]);
          bo[k] = pack_bf16(c4[k] * vv.x + s4[k] * vv.y, c4[k] * vv.y - s4[k] * vv.x);
        }
        *p = make_uint4(bo[0], bo[1], bo[2], bo[3]);
      }
    }
    // load chunk c + D into the stage of chunk c - 1 once that chunk's MMA has read it
    if (tid == kLoader && c + D < nchunks && !a.test_withhold) {
      const int prev = c + D - NST;
      if (prev < 0 ||
          mbar_wait(&bars[NST + prev % NST], (prev / NST) & 1, abort_flag, status, kTagMma, a.wait_limit)) {
        fence_proxy_async_smem();
        issue(c + D);
        issued = c + D + 1;
      }
    }
    // X_w = diag(f) X over X in place (each thread rewrites the 16-byte pieces it
    // read): warp w writes rows 16 w .. 16 w + 15; the weight of row m is token m / R's
    // f, held by lane (m / R) / TPL
    uint8_t* xw = st + K::OFF_X;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int u = warp * 128 + lane + 32 * i;
      const int row = u >> 3, cc = u & 7;
      const int tk = row / R;
      float fsel = 0.f;
#pragma unroll
      for (int j = 0; j < TPL; ++j) {
        const float fj = __shfl_sync(0xffffffffu, f[j], tk / TPL);
        if (tk % TPL == j) fsel = fj;
      }
      const uint4 xq = *reinterpret_cast<const uint4*>(st + K::OFF_X + swz(row, cc));
      const float2 f0 = unpack_bf16(xq.x), f1 = unpack_bf16(xq.y), f2 = unpack_bf16(xq.z), f3 = unpack_bf16(xq.w);
      *reinterpret_cast<uint4*>(xw + swz(row, cc)) =
          make_uint4(pack_bf16(fsel * f0.x, fsel * f0.y), pack_bf16(fsel * f1.x, fsel * f1.y),
                     pack_bf16(fsel * f2.x, fsel * f2.y), pack_bf16(fsel * f3.x, fsel * f3.y));
    }
    if (warp == kScalarWarp) {  // chunk c + 1's scalars for the next iteration; chunk c + 2's in flight
      store_pre((c + 1) & 1);
      load_pre(c + 2);
    }
    fence_proxy_async_smem();
    if (__syncthreads_or(*abort_flag != 0)) {
      abort_c = c;
      break;
    }
    if (tid == 0) {  // Hacc += B~^T X_w  (N x 64, K = 128 rows)
      tc_fence_after();
      const uint32_t iH = idesc_bf16(N, kP, 1, 1);
      const uint32_t cB = smem_u32(st + K::OFF_B), cX = smem_u32(xw);
#pragma unroll
      for (int kk = 0; kk < kM / 16; ++kk)
        mma_bf16_ss(tmem, smem_desc_sw128(cB + kk * 2048, kTile, 1024), smem_desc_sw128(cX + kk * 2048, kTile, 1024),
                    iH, (c > 0 || kk > 0) ? 1u : 0u);
      mma_commit(&bars[NST + s]);
    }
  }
  // the final angle of every pair, for the export and the last token's rotation
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < GPW; ++q)
#pragma unroll
      for (int k = 0; k < 4; ++k) phi[4 * (warp * GPW + q) + k] = phw[q][k];
  }
  __syncthreads();

  // chunks whose MMA was issued; a commit covers every earlier MMA of this thread
  const int mma_issued = abort_c >= 0 ? abort_c : nchunks;
  if (tid == 0) {
    if (abort_c < 0 && nchunks > 0)
      mbar_wait(&bars[NST + (nchunks - 1) % NST], ((nchunks - 1) / NST) & 1, abort_flag, status, kTagMma,
                a.wait_limit);
    // after an abort, let the MMAs issued land before TMEM is freed and the CTA exits
    if (*abort_flag && mma_issued > 0 &&
        !mbar_wait_drain(&bars[NST + (mma_issued - 1) % NST], ((mma_issued - 1) / NST) & 1))
      report_timeout(status, kTagDrain);
  }
  __syncthreads();  // the abort flag as thread 0 left it
  if (tid == kLoader && *abort_flag) {  // and the copies issued land before the CTA exits
    for (int c2 = abort_c >= 0 ? abort_c : nchunks; c2 < issued; ++c2)
      if (!mbar_wait_drain(&bars[c2 % NST], (c2 / NST) & 1)) report_timeout(status, kTagDrain);
  }
  if (__syncthreads_or(*abort_flag != 0)) {
    // aborted: outputs undefined, the status word says so
  } else if (L > 0) {
    tc_fence_after();
    // h_end from the accumulator: state row n, 32 columns per thread
    const int quad = warp & 3, half = warp >> 2;
    const int n = (N == 128) ? quad * 32 + lane : (lane < 16 ? quad * 16 + lane : -1);
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float hv[32];
    tmem_ld32(tmem + lane_base + 32 * half, hv);
    tmem_ld_wait();
    if (n >= 0) {
      float* ho = a.h_out + ((size_t)unit * N + n) * kP + 32 * half;
#pragma unroll
      for (int p = 0; p < 32; p += 4) *reinterpret_cast<float4*>(ho + p) = make_float4(hv[p], hv[p + 1], hv[p + 2], hv[p + 3]);
    }
    const size_t il = tok(L - 1);
    const size_t ib = ((size_t)b * L + (L - 1)) * a.ngroups + gh;
    const __nv_bfloat16* Bl = static_cast<const __nv_bfloat16*>(a.B) + ib * R * N;
    const __nv_bfloat16* Xl = static_cast<const __nv_bfloat16*>(a.x) + il * R * kP;
    for (int i = tid; i < R * K2; i += kThreads) {  // B of the last token rotated by its angle, in fp32
      const int r = i / K2, k = i % K2;
      float sn, cs;
      sincosf(phi[k], &sn, &cs);
      const float b0 = __bfloat162float(Bl[r * N + 2 * k]), b1 = __bfloat162float(Bl[r * N + 2 * k + 1]);
      a.bprev_out[((size_t)unit * R + r) * N + 2 * k] = cs * b0 + sn * b1;
      a.bprev_out[((size_t)unit * R + r) * N + 2 * k + 1] = cs * b1 - sn * b0;
    }
    for (int i = tid; i < R * kP; i += kThreads) a.xprev_out[(size_t)unit * R * kP + i] = __bfloat162float(Xl[i]);
    if (tid < K2) a.angle_out[(size_t)unit * K2 + tid] = phi[tid];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

template <int N, int R, bool TVA>
int launch_nr(const ScanArgs& a, cudaStream_t s) {
  using K = GCfg<N, R>;
  constexpr int Q = K::Q;
  CUtensorMap tmB, tmX, tmT;
  if (!make_map(&tmB, a.B, N, a.ngroups, a, Q) || !make_map(&tmX, a.x, kP, a.nheads, a, Q) ||
      !make_theta_map(&tmT, a, Q, true))
    return MAMBA3_ERR_CUDA;
  auto k = seg_state_kernel<N, R, TVA>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM_ALLOC) != cudaSuccess ||
      cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  k<<<a.batch * a.nheads, kThreads, K::SMEM_ALLOC, s>>>(tmB, tmX, tmT, a);
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

template <int N, int R>
int launch_r(const ScanArgs& a, cudaStream_t s) {
  return a.A_t ? launch_nr<N, R, true>(a, s) : launch_nr<N, R, false>(a, s);
}

}  // namespace

int seg_state_ctas_per_sm(const ScanArgs& a) {
  if (a.N == 128) return a.R == 1 ? GCfg<128, 1>::CPS : (a.R == 2 ? GCfg<128, 2>::CPS : GCfg<128, 4>::CPS);
  return a.R == 1 ? GCfg<64, 1>::CPS : (a.R == 2 ? GCfg<64, 2>::CPS : GCfg<64, 4>::CPS);
}

int launch_seg_state(const ScanArgs& a, cudaStream_t s) {
  if (bwd_tc_supported(a) != MAMBA3_OK || a.h0 || a.angle0) return MAMBA3_ERR_UNSUPPORTED;
  if (a.N == 128) {
    if (a.R == 1) return launch_r<128, 1>(a, s);
    if (a.R == 2) return launch_r<128, 2>(a, s);
    if (a.R == 4) return launch_r<128, 4>(a, s);
  } else {
    if (a.R == 1) return launch_r<64, 1>(a, s);
    if (a.R == 2) return launch_r<64, 2>(a, s);
    if (a.R == 4) return launch_r<64, 4>(a, s);
  }
  return MAMBA3_ERR_UNSUPPORTED;
}

}  // namespace m3

// Chunked prefill of the Mamba-3 recurrence on the 5th-generation tensor
// cores (tcgen05, accumulators in TMEM) fed by TMA (sm_100a, bf16 inputs).
//
// Method (derived from the three-term update of section 1.1, the RoPE trick of
// section 1.2 and the MIMO shapes of section 1.3 of "Mamba-3: 2x smaller state
// ..." (MarkTechPost, Korean translation)).  A chunk holds M = 128 rows, i.e.
// Q = 128 / R tokens of R ranks each, row m = (token t = m / R, rank r = m % R).
// With B~, C~ rotated by -Phi, the per-token log decay a_t = dt_t A, the
// chunk-local cumulative sum cum_t, the trapezoid weight of column s
//   w_s = lam_s dt_s + (1 - lam_{s+1}) dt_{s+1}
// (the lagged term of step s+1 carries the same decay as the state, so it folds
// into column s; at the end of the sequence the next token is absent) and the
// carried state hbar (the state plus the next token's lagged term):
//   S      = C~ B~^T                                         (M x M, K = N)
//   P[m,j] = S[m,j] * { e^{cum_tm - cum_tj} w_tj  if t_j < t_m
//                       lam_tm dt_tm               if t_j = t_m   (all rank pairs)
//                       0                          if t_j > t_m }  + D [m = j]
//   Y      = P X  +  diag(e^{cum_t}) C~ hbar_in                   (M x P)
//   hbar_out = e^{cum_end} hbar_in + B~^T diag(e^{cum_end - cum_t} w_t) X
// Every exponent is a difference of chunk-local sums (<= 0), so nothing
// overflows.  The skip term D x rides on the diagonal of P.
//
// Design: one CTA per (batch, head) marches over its chunks; the state stays on
// chip, in fp32 registers of the epilogue warps.  18 warps:
//   warp 0       TMA producer: B, C, X tiles of chunk c into a 2-stage ring (3 for N = 64)
//                (128-byte swizzle, the layout the MMA descriptors read); B and C
//                of a stage are refilled once the state MMAs have read them, X
//                once the Y MMA has; theta (+ dt, lam) into single tiles.
//   warp 1       TMEM allocator and single-thread MMA issuer.
//   warps 2..9   prep: decay scalars, the row scale of X_w and the rank-1 decay
//                factors of the mask, accumulated angles (wrapped) and RoPE of
//                B and C in place, 16 bytes per access.  Prep bounds the chunk.
//   warps 10..17 epilogue, two warps per TMEM lane quadrant: X_w =
//                diag(e^{cum_end - cum_t} w_t) X while the S MMA runs, S -> P
//                (bf16, back into TMEM; the two warps take alternate 16-column
//                pieces), hbar update (column halves) and its bf16 copy for the
//                next chunk's inter-chunk MMA, y = Y + e^{cum} Yi (with R = 1 for
//                the previous chunk, so that the Y MMA's latency is off the
//                epilogue's path).
// With more units than SMs the last wave can be split (see the split plan below).
// MMAs per chunk: S = C~ B~^T; Yi = C~ hbar_in; Hacc = B~^T X_w (smem operands);
// Y = P X (P from TMEM).  TMEM columns: S [0,128), P [128,192) (bf16 pairs),
// Y [192,256), Yi [256,320), Hacc [320,384); with R = 1 a second Y, Yi buffer at
// [384,448), [448,512) (y written one chunk late).
// Variants (template V): the plain recurrence; the fused B/C RMS norm in front of
// the rotation; a time-varying decay A_t per token in place of A per head.
// Every wait is bounded: on expiry the CTA raises an abort flag, reports
// MAMBA3_ERR_TIMEOUT in the device status word, drains and returns.
#include <cuda.h>
#include <string.h>

#include <map>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace m3 {

// ------------------------------------------------------------------ TMA tensor maps (shared with the backward pass)
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// [batch, L, H, R, inner] bf16 tensor, box = {64, R, 1, Q, 1}, 128-byte swizzle,
// zero fill past the end of the sequence.
bool make_map(CUtensorMap* m, const void* base, int inner, int heads, const ScanArgs& a, int Q) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[5] = {(cuuint64_t)inner, (cuuint64_t)a.R, (cuuint64_t)heads, (cuuint64_t)a.seqlen,
                              (cuuint64_t)a.batch};
  const cuuint64_t e = 2;
  const cuuint64_t strides[4] = {e * inner, e * inner * a.R, e * inner * a.R * heads,
                                 e * inner * a.R * heads * a.seqlen};
  const cuuint32_t box[5] = {64, (cuuint32_t)a.R, 1, (cuuint32_t)Q, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// dt or lam [batch, L, H] bf16, box = {8, Q + 1, 1}: the 8 heads of a 16-byte
// group over the chunk's tokens and the next one, zero fill past the end.
// Needs H a multiple of 8 (16-byte row stride) and a 16-byte aligned base.
bool make_dl_map(CUtensorMap* m, const void* base, const ScanArgs& a, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || a.nheads % 8 != 0 || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)a.nheads, (cuuint64_t)a.seqlen, (cuuint64_t)a.batch};
  const cuuint64_t strides[2] = {2ull * a.nheads, 2ull * a.nheads * a.seqlen};
  const cuuint32_t box[3] = {8, (cuuint32_t)rows, 1};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// theta [batch, L, H, N/2] bf16, box = {N/2, 1, Q, 1}, zero fill past the end; no
// swizzle, or (swizzle) the 64-byte (N = 64) or 128-byte (N = 128) pattern, which
// moves 16-byte chunk c of row t to c ^ ((t >> 1) & 3) or c ^ (t & 7).
bool make_theta_map(CUtensorMap* m, const ScanArgs& a, int Q, bool swizzle) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int K2 = a.N / 2;
  const cuuint64_t dims[4] = {(cuuint64_t)K2, (cuuint64_t)a.nheads, (cuuint64_t)a.seqlen, (cuuint64_t)a.batch};
  const cuuint64_t strides[3] = {2ull * K2, 2ull * K2 * a.nheads, 2ull * K2 * a.nheads * a.seqlen};
  const cuuint32_t box[4] = {(cuuint32_t)K2, 1, (cuuint32_t)Q, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  const CUtensorMapSwizzle sw =
      !swizzle ? CU_TENSOR_MAP_SWIZZLE_NONE : (K2 == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.theta), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


namespace {

using namespace ptx;

constexpr int kP = 64;          // head dim handled by this kernel
constexpr int kM = 128;         // rows per chunk (MMA M)
constexpr int kTile = 16384;    // one 128-row x 128-byte swizzled tile
constexpr int kThreads = 576;   // 18 warps
constexpr int kPrep0 = 64;      // first prep thread
constexpr int kNPrep = 256;
constexpr int kEpi0 = kPrep0 + kNPrep;
constexpr int kNEpi = 256;
constexpr uint32_t kTmemCols = 512;
// With R = 1, Y and Yi are double-buffered (chunk c at + (c % 2) * kColYBuf) and
// the epilogue writes y of chunk c while the MMAs of chunk c + 1 run.
constexpr uint32_t kColS = 0, kColP = 128, kColY = 192, kColYi = 256, kColH = 320, kColYBuf = 192;

enum Tag {
  kTagEmpty = 1, kTagFull, kTagPrep1, kTagSFull, kTagAcc, kTagEpiDone, kTagP, kTagY, kTagDrain, kTagTh, kTagHand, kTagXw,
  kTagNorm, kTagTicket
};

// kernel variants: the plain recurrence, the fused B/C norm, the time-varying decay A_t
enum Variant { kPlain = 0, kBCNorm = 1, kTimeA = 2 };

template <int N, int R, int V>
struct Cfg {
  static constexpr int Q = kM / R;     // tokens per chunk
  static constexpr int NKB = N / 64;   // 64-wide blocks of the state dimension
  static constexpr int K2 = N / 2;     // rotation pairs
  static constexpr int NG = K2 / 4;    // groups of 4 pairs (16 bytes of a row)
  static constexpr int NPART = kNPrep / NG;  // token parts of the angle scan
  static constexpr int TPP = Q / NPART;  // tokens per part
  static constexpr int TB = (R == 1 && TPP % 2 == 0) ? 2 : 1;  // tokens per rotation batch
  // y one chunk late (double-buffered Y, Yi): shortens the epilogue's chain;
  // measured faster for R = 1 only
  static constexpr bool DEFER_Y = (R == 1);
  static constexpr int STAGE_BYTES = (2 * NKB + 1) * kTile;  // B, C, X
  // input stages: three where they fit (N = 64: 48 KB each), so that a stage's
  // refill has a chunk more of lead time; two for N = 128 (80 KB each)
  static constexpr int NST = N == 64 ? 3 : 2;
  static constexpr int TMA_BYTES = STAGE_BYTES;
  static constexpr int OFF_B = 0, OFF_C = NKB * kTile, OFF_X = 2 * NKB * kTile;
  static constexpr int OFF_XW = NST * STAGE_BYTES;      // X_w (single buffer)
  static constexpr int OFF_TH = OFF_XW + kTile;          // theta tile [Q][N/2] bf16 (single buffer)
  static constexpr int TH_BYTES = Q * K2 * 2;
  static constexpr int OFF_H = OFF_TH + ((TH_BYTES + 1023) & ~1023);  // hbar bf16, N rows x 128 bytes
  static constexpr int OFF_SC = OFF_H + N * 128;       // scalars
  // per stage (floats): c2[Q] (log2 of the chunk-local decay), gam[Q], wv[Q],
  // wsc[Q] (X_w row scale), colf[192] (rank-1 column factors of the mask)
  static constexpr int SC_PER_STAGE = 4 * Q + 192;
  static constexpr int OFF_PART = OFF_SC + NST * SC_PER_STAGE * 4;  // angle partials [NPART][K2]
  static constexpr int OFF_PHI = OFF_PART + NPART * K2 * 4;            // running base angle [K2]
  static constexpr int OFF_WARP = OFF_PHI + K2 * 4;                     // scan scratch [8]
  static constexpr int OFF_BAR = (OFF_WARP + 32 + 7) & ~7;
  static constexpr int NBAR = 24;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;  // tmem base, abort flag
  // dt and lam of tokens [t0, t0 + Q] for the 8 heads of this head's 16-byte
  // group (TMA tiles [Q + 1][8] bf16, single buffer, refilled with theta)
  static constexpr int DL_BYTES = (Q + 1) * 16;
  static constexpr int DL_PAD = (DL_BYTES + 127) & ~127;
  static constexpr int OFF_DL = (OFF_MISC + 16 + 127) & ~127;
  static constexpr int OFF_SINK = OFF_DL + 2 * DL_PAD;  // [Q] floats: consumes the tile reads
  // fused B/C normalisation (V = kBCNorm): w_B, bias_B, w_C, bias_C of this head,
  // [R][N] floats each;
  // time-varying decay by TMA (V = kTimeA): the A_t tile [Q][8] bf16 (refilled with
  // theta); nothing for the plain variant
  static constexpr int OFF_NRM = (OFF_SINK + Q * 4 + 127) & ~127;
  static constexpr int AT_BYTES = Q * 16;
  // (R = 1: the epilogue warps normalise the raw rows in place two chunks ahead; R > 1,
  // where the epilogue has no time to spare: prep applies the norm in its rotation,
  // from 1 / RMS of every raw row [2][128] computed first)
  static constexpr bool EPI_NORM = V == kBCNorm && R == 1;
  // X_w by the epilogue warps, except with the epilogue-side norm, which leaves the
  // epilogue the longer role: then prep writes it (after the previous state MMA)
  static constexpr bool XW_PREP = EPI_NORM;
  // the exported B~ of the last token computed after the rotation loop (fewer live
  // registers in the loop) rather than inside it: measured faster for N = 128 with
  // R = 1 and N = 64 with R = 4 (2 % each), slower for the other shapes (register
  // allocation differs); never with the epilogue-side norm (the raw row is gone)
  static constexpr bool EXPORT_AFTER = !EPI_NORM && ((N == 128 && R == 1) || (N == 64 && R == 4));
  static constexpr bool PREP_NORM = V == kBCNorm && R > 1;
  static constexpr int OFF_RINV = OFF_NRM + 4 * R * N * 4;
  static constexpr int NRM_BYTES = V == kBCNorm ? 4 * R * N * 4 + (PREP_NORM ? 2 * kM * 4 : 0)
                                                : (V == kTimeA ? AT_BYTES : 0);
  // y staging where shared memory allows (N = 64; N = 128 with R = 4 except the
  // fused norm): per epilogue warp one or two
  // 32-row x 64-byte tiles (64-byte swizzle) that the warp writes out with a TMA store
  static constexpr int OFF_Y = (OFF_NRM + NRM_BYTES + 1023) & ~1023;
  static constexpr int Y_TILE = 32 * 64;
  static constexpr int YBUF = OFF_Y + 16 * Y_TILE + 1024 <= 232448 ? 2 : (OFF_Y + 8 * Y_TILE + 1024 <= 232448 ? 1 : 0);
  static constexpr int SMEM = YBUF ? OFF_Y + 8 * YBUF * Y_TILE : OFF_NRM + NRM_BYTES;
  static constexpr int SMEM_ALLOC = SMEM + 1024;       // slack for 1024-byte alignment
  static_assert(NG * NPART == kNPrep && TPP * NPART == Q, "angle partition");
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// barrier slots
enum Bar {
  bFull0 = 0, bEmptyBC0 = 3, bPrep0 = 6, bEmptyX0 = 9, bNorm0 = 12,  // one per stage (up to 3)
  bSFull = 15, bAcc, bEpiDone, bPReady, bYFull, bDone, bThFull, bThFree, bXw
};

struct TcParams {
  ScanArgs a;
  int nchunks;
  int dl_tma;  // dt and lam arrive by TMA with theta (else: global loads one chunk ahead)
  int at_tma;  // a time-varying decay A_t arrives by TMA with theta (needs dl_tma)
  // split last wave (split_k > 0): units 0 .. split_k - 1 run in two CTAs, chunks
  // [0, split_c1) and [split_c1, nchunks); a CTA's work comes from a ticket
  // (tickets 0 .. k-1: first parts; k .. U-1: whole units; U .. U+k-1: second parts)
  int split_k, split_c1;
  int* ticket;  // zeroed before the launch
  int* flags;   // [split_k], zeroed: set once a first part has handed over
  float* hand;  // [split_k][N P + N/2]: the carried state hbar and the angle at chunk split_c1
};

// acquire / release accesses of the hand-over flags (gpu scope)
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_gpu(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ size_t tok_index(const ScanArgs& a, int b, int t, int h) {
  return ((size_t)b * a.seqlen + t) * a.nheads + h;
}

// stage of chunk c in an NST-stage ring and the ring's round (for the mbarrier
// parity); unsigned, so that a two-stage ring compiles to a mask and a shift
template <int NST>
__device__ __forceinline__ int stage_of(int c) { return (int)((unsigned)c % NST); }
template <int NST>
__device__ __forceinline__ int round_of(int c) { return (int)((unsigned)c / NST); }

// byte offset of 16-byte chunk `c` (0..7) of row `row` inside a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_bf16(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// named barrier over the 256 prep threads (id 1) that also ORs a predicate,
// so that every prep thread takes the same abort decision
__device__ __forceinline__ bool prep_sync_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 256, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void prep_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// X_w = diag(wsc) X of one chunk: thread i of 256 scales 16-byte chunks i, i + 256,
// i + 512, i + 768 of the swizzled x tile (row = token rank row, wsc per token)
template <int R>
__device__ __forceinline__ void write_xw(uint8_t* xw, const uint8_t* x, const float* wsc, int i0) {
  uint4 xq[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = i0 + 256 * i;
    xq[i] = *reinterpret_cast<const uint4*>(x + swz(idx >> 3, idx & 7));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = i0 + 256 * i;
    const int row = idx >> 3, cc = idx & 7;
    const float f = wsc[row / R];
    const float2 f0 = unpack_bf16(xq[i].x), f1 = unpack_bf16(xq[i].y), f2 = unpack_bf16(xq[i].z),
                 f3 = unpack_bf16(xq[i].w);
    uint4 o;
    o.x = pack_bf16(f * f0.x, f * f0.y);
    o.y = pack_bf16(f * f1.x, f * f1.y);
    o.z = pack_bf16(f * f2.x, f * f2.y);
    o.w = pack_bf16(f * f3.x, f * f3.y);
    *reinterpret_cast<uint4*>(xw + swz(row, cc)) = o;
  }
}

// ------------------------------------------------------------------ prep warps
// Thread pt in [0,256).  Per chunk: decay scalars (thread = token), accumulated
// angles (thread = group g of 4 pairs x token part) and RoPE of B and C in
// place (16 bytes per shared-memory access, 2 rows in flight), the rank-1
// column factors of the mask and X_w.  dt and lam are prefetched one chunk
// ahead into registers; theta arrives by TMA.
template <int N, int R, int V, bool dl_tma>
__device__ __forceinline__ void prep_role(uint8_t* smem, const ScanArgs& a, int nchunks, int b, int hh,
                                          int c0, const float* hand_in, float* hand_out, float Ah, uint64_t* bars,
                                          volatile int* abort_flag, DeviceStatus* status) {
  constexpr bool BCN = V == kBCNorm, TVA = V == kTimeA;
  using K = Cfg<N, R, V>;
  constexpr int Q = K::Q, K2 = K::K2, NG = K::NG, TPP = K::TPP, TB = K::TB, NPART = K::NPART;
  const int pt = threadIdx.x - kPrep0;
  const int L = a.seqlen, H = a.nheads;
  float* part_sum = reinterpret_cast<float*>(smem + K::OFF_PART);
  float* phi = reinterpret_cast<float*>(smem + K::OFF_PHI);
  float* warp_tot = reinterpret_cast<float*>(smem + K::OFF_WARP);
  const uint8_t* th_tile = smem + K::OFF_TH;
  const size_t unit = (size_t)b * H + hh;
  const int g = pt % NG, part = pt / NG;  // 4-pair group (one 16-byte chunk of a row), token part
  const int kb = g / 8, c8 = g % 8;       // 64-element block and 16-byte chunk of the group
  // dt, lam (and A_t) of this (batch, head): element t at [t * H]
  const __nv_bfloat16* DTu = static_cast<const __nv_bfloat16*>(a.dt) + (size_t)b * L * H + hh;
  const __nv_bfloat16* LMu = static_cast<const __nv_bfloat16*>(a.lam) + (size_t)b * L * H + hh;


  if (pt < K2) phi[pt] = hand_in ? __ldcg(hand_in + N * kP + pt) : (a.angle0 ? a.angle0[unit * K2 + pt] : 0.f);
  // (this CTA's chunks start at chunk c0 of the sequence; only a part that ends the
  // sequence exports the final state, a first part hands hbar and phi over instead)
  const int t_last = (hand_out == nullptr && a.bprev_out != nullptr) ? L - 1 - c0 * Q : -1;

  // prefetched per chunk: (scan threads) dt, lam of token pt and of the next
  // token, and its decay rate (A_t, else A); (angle threads) dt of this part's tokens
  float s_dt, s_lm, s_dtn, s_lmn, s_at, p_dt[TPP];
  auto load_scalars = [&](int cc, float& o_dt, float& o_lm, float& o_dtn, float& o_lmn, float& o_at,
                          float (&o_pdt)[TPP]) {
    const int tc0 = (c0 + cc) * Q;
    const int tg = tc0 + pt;
    const bool ok = pt < Q && cc < nchunks;
    o_at = Ah;
    if constexpr (TVA) {  // A_t sits at the same offset as dt
      const __nv_bfloat16* ATu = static_cast<const __nv_bfloat16*>(a.A_t) + (DTu - static_cast<const __nv_bfloat16*>(a.dt));
      o_at = (ok && tg < L) ? __bfloat162float(ATu[(size_t)tg * H]) : 0.f;
    }
    o_dt = (ok && tg < L) ? __bfloat162float(DTu[(size_t)tg * H]) : 0.f;
    o_lm = (ok && tg < L) ? __bfloat162float(LMu[(size_t)tg * H]) : 1.f;
    o_dtn = (ok && tg + 1 < L) ? __bfloat162float(DTu[(size_t)(tg + 1) * H]) : 0.f;
    o_lmn = (ok && tg + 1 < L) ? __bfloat162float(LMu[(size_t)(tg + 1) * H]) : 1.f;
#pragma unroll
    for (int i = 0; i < TPP; ++i) {
      const int tp = tc0 + part * TPP + i;
      o_pdt[i] = (cc < nchunks && tp < L) ? __bfloat162float(DTu[(size_t)tp * H]) : 0.f;
    }
  };
  if constexpr (dl_tma) {
    s_dt = s_dtn = 0.f;
    s_lm = s_lmn = 1.f;
    s_at = Ah;
#pragma unroll
    for (int i = 0; i < TPP; ++i) p_dt[i] = 0.f;
  } else {
    load_scalars(0, s_dt, s_lm, s_dtn, s_lmn, s_at, p_dt);
  }
  const __nv_bfloat16* ats = reinterpret_cast<const __nv_bfloat16*>(smem + K::OFF_NRM) + (hh & 7);
  const __nv_bfloat16* dts = reinterpret_cast<const __nv_bfloat16*>(smem + K::OFF_DL) + (hh & 7);
  const __nv_bfloat16* lms = reinterpret_cast<const __nv_bfloat16*>(smem + K::OFF_DL + K::DL_PAD) + (hh & 7);
  float* sink = reinterpret_cast<float*>(smem + K::OFF_SINK);
  const float* nrm = reinterpret_cast<const float*>(smem + K::OFF_NRM);
  if constexpr (K::PREP_NORM) {  // this head's normalisation weights and biases, [4][R][N]
    float* nw = reinterpret_cast<float*>(smem + K::OFF_NRM);
    const size_t base = (size_t)hh * R * N;
    for (int i = pt; i < R * N; i += kNPrep) {
      nw[i] = a.nw_B ? a.nw_B[base + i] : 1.f;
      nw[R * N + i] = a.nb_B ? a.nb_B[base + i] : 0.f;
      nw[2 * R * N + i] = a.nw_C ? a.nw_C[base + i] : 1.f;
      nw[3 * R * N + i] = a.nb_C ? a.nb_C[base + i] : 0.f;
    }
  }
  prep_sync();

  for (int c = 0; c < nchunks; ++c) {
    const int s = stage_of<K::NST>(c), u = round_of<K::NST>(c);
    const int t0 = c * Q;
    float* sc = reinterpret_cast<float*>(smem + K::OFF_SC) + s * K::SC_PER_STAGE;
    float *c2 = sc, *gm = sc + Q, *wv = sc + 2 * Q, *wsc = sc + 3 * Q, *colf = sc + 4 * Q;
    uint8_t* st = smem + s * K::STAGE_BYTES;
    const bool last_chunk = (c == nchunks - 1);

    // ---- phase A (no shared state): in-warp scan of dt*A*log2(e); theta of this part ----
    mbar_wait(&bars[bThFull], c & 1, abort_flag, status, kTagTh, a.wait_limit);
    if constexpr (dl_tma) {  // this chunk's dt and lam from the tile (rows past the sequence read 0)
      if (pt < Q) {
        s_dt = __bfloat162float(dts[pt * 8]);
        s_lm = __bfloat162float(lms[pt * 8]);
        s_dtn = __bfloat162float(dts[(pt + 1) * 8]);
        s_lmn = __bfloat162float(lms[(pt + 1) * 8]);
        if constexpr (TVA) s_at = __bfloat162float(ats[pt * 8]);
      }
#pragma unroll
      for (int i = 0; i < TPP; ++i) p_dt[i] = __bfloat162float(dts[(part * TPP + i) * 8]);
    }
    float v = (pt < Q) ? s_dt * (TVA ? s_at : Ah) * kLog2e : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, v, o);
      if ((pt & 31) >= o) v += n;
    }
    if ((pt & 31) == 31) warp_tot[pt >> 5] = v;
    uint2 thv[TPP];
    float loc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < TPP; ++i) {
      thv[i] = *reinterpret_cast<const uint2*>(th_tile + ((part * TPP + i) * K2 + 4 * g) * 2);
      const float2 t01 = unpack_bf16(thv[i].x), t23 = unpack_bf16(thv[i].y);
      loc[0] += p_dt[i] * t01.x;
      loc[1] += p_dt[i] * t01.y;
      loc[2] += p_dt[i] * t23.x;
      loc[3] += p_dt[i] * t23.y;
    }
    *reinterpret_cast<float4*>(part_sum + part * K2 + 4 * g) = make_float4(loc[0], loc[1], loc[2], loc[3]);
    if (dl_tma && pt < Q) sink[pt] = (s_dt + s_lm) + (s_dtn + s_lmn) + (TVA ? s_at : 0.f);
    // Release the theta (and dt, lam) tiles only after stores that consume
    // every value loaded from them: the arrive does not wait for shared-memory
    // loads still in flight, and the refill is an async-proxy write that is not
    // ordered after them, so arriving straight after the loads lets a slow
    // thread read the next chunk's values.
    mbar_arrive(&bars[bThFree]);
    const float4 base = *reinterpret_cast<const float4*>(phi + 4 * g);
    mbar_wait(&bars[bFull0 + s], u & 1, abort_flag, status, kTagFull, a.wait_limit);
    // (fused norm) the epilogue warps have normalised this chunk's raw B and C rows in place
    if constexpr (K::EPI_NORM) mbar_wait(&bars[bNorm0 + s], u & 1, abort_flag, status, kTagNorm, a.wait_limit);
    if (prep_sync_any(*abort_flag != 0)) return;  // barrier 1: one decision for all prep threads

    // ---- phase B: scalars, prefix of the angle, RoPE ----
    float* rinv = reinterpret_cast<float*>(smem + K::OFF_RINV);
    if constexpr (K::PREP_NORM) {
      // 1 / RMS of every raw row of the chunk, thread = row (B rows: pt < 128, C rows:
      // the rest): 16-byte reads of the whole row, no cross-lane reduction; an
      // all-zero row with eps = 0 (e.g. the padding past the sequence end) gives 0
      const int row = pt & (kM - 1);
      const uint8_t* tile = st + (pt < kM ? K::OFF_B : K::OFF_C);
      float ss = 0.f;
#pragma unroll
      for (int kb = 0; kb < K::NKB; ++kb)
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const uint4 q = *reinterpret_cast<const uint4*>(tile + kb * kTile + swz(row, c8));
          const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_bf16(qw[k]);
            ss += f.x * f.x + f.y * f.y;
          }
        }
      const float vr = ss * (1.f / N) + a.neps;
      rinv[pt] = vr > 0.f ? rsqrtf(vr) : 0.f;
      prep_sync();
    }
    for (int w = 0; w < (pt >> 5); ++w) v += warp_tot[w];
    if (pt < Q) {
      const float gam = s_lm * s_dt;
      c2[pt] = v;
      gm[pt] = gam;
      wv[pt] = gam + (1.f - s_lmn) * s_dtn;
    }
    float run[4] = {base.x, base.y, base.z, base.w};
#pragma unroll
    for (int p2 = 0; p2 < NPART - 1; ++p2) {
      if (p2 < part) {
        const float4 ps = *reinterpret_cast<const float4*>(part_sum + p2 * K2 + 4 * g);
        run[0] += ps.x;
        run[1] += ps.y;
        run[2] += ps.z;
        run[3] += ps.w;
      }
    }
    // wrap once at the start of the part; inside the part the angle grows by
    // TPP increments only, which __sincosf takes without a further wrap
#pragma unroll
    for (int k = 0; k < 4; ++k) run[k] = wrap_angle(run[k]);
    float pdt_cur[TPP];
#pragma unroll
    for (int i = 0; i < TPP; ++i) pdt_cur[i] = p_dt[i];
    // next chunk's scalars, in flight during the rotation (unless they come by TMA)
    if constexpr (!dl_tma) load_scalars(c + 1, s_dt, s_lm, s_dtn, s_lmn, s_at, p_dt);
#pragma unroll
    for (int i0 = 0; i0 < TPP; i0 += TB) {
      float sn[TB][4], cs[TB][4];
#pragma unroll
      for (int j = 0; j < TB; ++j) {
        const float2 t01 = unpack_bf16(thv[i0 + j].x), t23 = unpack_bf16(thv[i0 + j].y);
        const float d = pdt_cur[i0 + j];
        run[0] += d * t01.x;
        run[1] += d * t01.y;
        run[2] += d * t23.x;
        run[3] += d * t23.y;
#pragma unroll
        for (int k = 0; k < 4; ++k) __sincosf(run[k], &sn[j][k], &cs[j][k]);
      }
      uint4 bq[TB * R], cq[TB * R];
#pragma unroll
      for (int j = 0; j < TB * R; ++j) {  // every load of the batch before any store
        const uint32_t off = kb * kTile + swz((part * TPP + i0) * R + j, c8);
        bq[j] = *reinterpret_cast<const uint4*>(st + K::OFF_B + off);
        cq[j] = *reinterpret_cast<const uint4*>(st + K::OFF_C + off);
      }
#pragma unroll
      for (int j = 0; j < TB * R; ++j) {
        const int jt = j / R, r = j % R;
        const int t = part * TPP + i0 + jt;
        const bool export_row = !K::EXPORT_AFTER && last_chunk && (t0 + t == t_last);
        const uint32_t bw[4] = {bq[j].x, bq[j].y, bq[j].z, bq[j].w};
        const uint32_t cw[4] = {cq[j].x, cq[j].y, cq[j].z, cq[j].w};
        uint32_t bo[4], co[4];
        if constexpr (K::PREP_NORM) {
          // raw row (t, r): its 1 / RMS from the pass above, weight and bias, then the rotation
          float bv[8], cv[8];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 b2 = unpack_bf16(bw[k]), c2v = unpack_bf16(cw[k]);
            bv[2 * k] = b2.x; bv[2 * k + 1] = b2.y;
            cv[2 * k] = c2v.x; cv[2 * k + 1] = c2v.y;
          }
          const int rowi = t * R + r;
          const float ib = rinv[rowi], ic = rinv[kM + rowi];
          const float* wB = nrm + r * N + 8 * g;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            bv[e] = bv[e] * ib * wB[e] + wB[R * N + e];
            cv[e] = cv[e] * ic * wB[2 * R * N + e] + wB[3 * R * N + e];
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float b0 = cs[jt][k] * bv[2 * k] + sn[jt][k] * bv[2 * k + 1];
            const float b1 = cs[jt][k] * bv[2 * k + 1] - sn[jt][k] * bv[2 * k];
            bo[k] = pack_bf16(b0, b1);
            co[k] = pack_bf16(cs[jt][k] * cv[2 * k] + sn[jt][k] * cv[2 * k + 1],
                              cs[jt][k] * cv[2 * k + 1] - sn[jt][k] * cv[2 * k]);
            if (export_row) {
              a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k] = b0;
              a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k + 1] = b1;
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 bv = unpack_bf16(bw[k]), cv = unpack_bf16(cw[k]);
            const float b0 = cs[jt][k] * bv.x + sn[jt][k] * bv.y, b1 = cs[jt][k] * bv.y - sn[jt][k] * bv.x;
            bo[k] = pack_bf16(b0, b1);
            co[k] = pack_bf16(cs[jt][k] * cv.x + sn[jt][k] * cv.y, cs[jt][k] * cv.y - sn[jt][k] * cv.x);
            if (export_row) {
              a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k] = b0;
              a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k + 1] = b1;
            }
          }
        }
        const uint32_t off = kb * kTile + swz(t * R + r, c8);
        *reinterpret_cast<uint4*>(st + K::OFF_B + off) = make_uint4(bo[0], bo[1], bo[2], bo[3]);
        *reinterpret_cast<uint4*>(st + K::OFF_C + off) = make_uint4(co[0], co[1], co[2], co[3]);
      }
    }
    if (K::EXPORT_AFTER && last_chunk && t_last >= t0 && t_last < t0 + Q && (t_last - t0) / TPP == part) {
      // B~ of the sequence's last token in fp32 for the exported state: the part's
      // running angle is that token's (padding tokens add dt = 0), and its raw row
      // is read again from global memory, rotated with the loop's arithmetic
      const int tl = t_last - t0;
      const int gh = hh / (H / a.ngroups);
      float snl[4], csl[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) __sincosf(run[k], &snl[k], &csl[k]);
      const __nv_bfloat16* brow = static_cast<const __nv_bfloat16*>(a.B) +
                                  (((size_t)b * L + (size_t)(c0 * Q + t_last)) * a.ngroups + gh) * R * N + 8 * g;
      for (int r = 0; r < R; ++r) {
        const uint4 q = *reinterpret_cast<const uint4*>(brow + r * N);
        const uint32_t bw[4] = {q.x, q.y, q.z, q.w};
        float bv[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = unpack_bf16(bw[k]);
          bv[2 * k] = f.x;
          bv[2 * k + 1] = f.y;
        }
        if constexpr (K::PREP_NORM) {  // as in the loop: 1 / RMS of the row, weight and bias
          const float ib = reinterpret_cast<const float*>(smem + K::OFF_RINV)[tl * R + r];
          const float* wB = nrm + r * N + 8 * g;
#pragma unroll
          for (int e = 0; e < 8; ++e) bv[e] = bv[e] * ib * wB[e] + wB[R * N + e];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k] = csl[k] * bv[2 * k] + snl[k] * bv[2 * k + 1];
          a.bprev_out[(unit * R + r) * N + 8 * g + 2 * k + 1] = csl[k] * bv[2 * k + 1] - snl[k] * bv[2 * k];
        }
      }
    }
    if (part == NPART - 1) {  // the last part's running angle is the chunk's end angle
      *reinterpret_cast<float4*>(phi + 4 * g) =
          make_float4(wrap_angle(run[0]), wrap_angle(run[1]), wrap_angle(run[2]), wrap_angle(run[3]));
      if (last_chunk) {
        float* ad = hand_out ? hand_out + N * kP : (a.angle_out ? a.angle_out + unit * K2 : nullptr);
        if (ad)
          for (int k = 0; k < 4; ++k) ad[4 * g + k] = wrap_angle(run[k]);
        if (hand_out) __threadfence();
      }
    }
    prep_sync();  // barrier 2: scalars complete, every part has read phi

    // ---- phase C: mask factors, X_w (after the previous state MMA has read it) ----
    const float c2end = c2[Q - 1];
    if (pt < Q) wsc[pt] = wv[pt] * ex2(c2end - c2[pt]);
    if (pt < 192) {  // column factors e^{cum_ref - cum_tj} w_tj of the off-diagonal mask blocks
      const int qq = pt < 32 ? 1 : (pt < 96 ? 2 : 3);
      const int j = pt - (qq == 1 ? 0 : (qq == 2 ? 32 : 96));
      const int tj = j / R, tref = (32 * qq) / R;
      colf[pt] = ex2(c2[tref] - c2[tj]) * wv[tj];
    }
    if constexpr (K::XW_PREP) {
      if (c > 0) mbar_wait(&bars[bAcc], (c - 1) & 1, abort_flag, status, kTagAcc, a.wait_limit);
      if (prep_sync_any(*abort_flag != 0)) return;  // wsc visible, X_w free
      write_xw<R>(smem + K::OFF_XW, st + K::OFF_X, wsc, pt);
      fence_proxy_async_smem();
      mbar_arrive(&bars[bXw]);
    }
    fence_proxy_async_smem();
    mbar_arrive(&bars[bPrep0 + s]);  // (releases wsc and the mask factors to the epilogue)

    if (last_chunk && hand_out == nullptr && a.xprev_out && L > 0) {
      const __nv_bfloat16* xl =
          static_cast<const __nv_bfloat16*>(a.x) + tok_index(a, b, L - 1, hh) * R * kP;
      for (int i = pt; i < R * kP; i += kNPrep) a.xprev_out[unit * R * kP + i] = __bfloat162float(xl[i]);
    }
  }
}

// bf16 copy of this thread's 32 state columns into the swizzled hbar tile
__device__ __forceinline__ void store_hbar_bf16(const float (&hb)[32], uint8_t* Hs, int n, int ch) {
  if (n < 0) return;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    uint4 q;
    q.x = pack_bf16(hb[8 * q4 + 0], hb[8 * q4 + 1]);
    q.y = pack_bf16(hb[8 * q4 + 2], hb[8 * q4 + 3]);
    q.z = pack_bf16(hb[8 * q4 + 4], hb[8 * q4 + 5]);
    q.w = pack_bf16(hb[8 * q4 + 6], hb[8 * q4 + 7]);
    *reinterpret_cast<uint4*>(Hs + swz(n, 4 * ch + q4)) = q;
  }
}

// one 32-byte store (256-bit global store, sm_100): 8 packed words to a 32-byte aligned address
__device__ __forceinline__ void st_global_32b(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// y rows of one chunk from its Y and Yi accumulators: y = Y + e^{cum_t} Yi
// (this thread's 32 columns of row m, 32 bytes per store); rows past the sequence
// are not stored
__device__ __forceinline__ void store_y(const ScanArgs& a, uint32_t tY, uint32_t tYi, float e, int b, int hh, int tg,
                                        int rm, int R, int ch) {
  uint4* yr = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) +
                                       (tok_index(a, b, tg < a.seqlen ? tg : 0, hh) * R + rm) * kP + 32 * ch);
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float yv[16], yi[16];
    __syncwarp();
    tmem_ld16(tY + 32 * ch + 16 * half, yv);
    tmem_ld16(tYi + 32 * ch + 16 * half, yi);
    tmem_ld_wait();
    if (tg < a.seqlen) {
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) w[i] = pack_bf16(yv[2 * i] + e * yi[2 * i], yv[2 * i + 1] + e * yi[2 * i + 1]);
      st_global_32b(yr + 2 * half, w);
    }
  }
}

// The same rows through the warp's staging tile: lane l writes row l's 64 bytes (its
// 32 columns) into the 64-byte-swizzled 32 x 64 B tile `stg` (16-byte chunk c of row l
// at c ^ ((l >> 1) & 3), so a store instruction covers all 32 banks), then lane 0
// writes the tile out with one TMA store of the warp's 32 rows (rows past the sequence
// are clipped by the tensor map).  The tile is rewritten once the store that last
// read it has (PENDING younger stores may still be in flight).
template <int PENDING>
__device__ __forceinline__ void store_y_tma(const CUtensorMap* tmY, uint8_t* stg, uint32_t tY, uint32_t tYi, float e,
                                            int b, int hh, int t_first, int ch, int lane) {
  if (lane == 0) bulk_wait_read<PENDING>();
  __syncwarp();
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    float yv[16], yi[16];
    tmem_ld16(tY + 32 * ch + 16 * half, yv);
    tmem_ld16(tYi + 32 * ch + 16 * half, yi);
    tmem_ld_wait();
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const int o = 8 * q2, c = 2 * half + q2;
      uint4 q;
      q.x = pack_bf16(yv[o + 0] + e * yi[o + 0], yv[o + 1] + e * yi[o + 1]);
      q.y = pack_bf16(yv[o + 2] + e * yi[o + 2], yv[o + 3] + e * yi[o + 3]);
      q.z = pack_bf16(yv[o + 4] + e * yi[o + 4], yv[o + 5] + e * yi[o + 5]);
      q.w = pack_bf16(yv[o + 6] + e * yi[o + 6], yv[o + 7] + e * yi[o + 7]);
      *reinterpret_cast<uint4*>(stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) = q;
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_5d(tmY, stg, 32 * ch, 0, hh, t_first, b);
    bulk_commit();
  }
}

// Fused B/C norm of one chunk in place (raw -> w * row / RMS(row) + bias, bf16):
// thread et of the 256 epilogue threads owns row et of B (et < 128) or row et - 128
// of C, reads it whole in 16-byte pieces for its sum of squares (no cross-lane
// reduction), then rewrites it; all lanes of a warp read the same weights (R = 1)
// or R of them, so those reads are broadcasts.  An all-zero row with eps = 0 (the
// padding past the sequence end) gives 1 / RMS = 0.
template <int N, int R, int V>
__device__ __forceinline__ void bc_normalise(uint8_t* st, const float* nw, float eps, int et) {
  using K = Cfg<N, R, V>;
  const int row = et & (kM - 1);
  const bool is_c = et >= kM;
  uint8_t* tile = st + (is_c ? K::OFF_C : K::OFF_B);
  const float* w = nw + (is_c ? 2 : 0) * R * N + (row % R) * N;  // weight [n]; bias at + R N
  float ss = 0.f;
#pragma unroll
  for (int kb = 0; kb < K::NKB; ++kb)
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
      const uint4 q = *reinterpret_cast<const uint4*>(tile + kb * kTile + swz(row, c8));
      const uint32_t qw[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = unpack_bf16(qw[k]);
        ss += f.x * f.x + f.y * f.y;
      }
    }
  const float vr = ss * (1.f / N) + eps;
  const float ri = vr > 0.f ? rsqrtf(vr) : 0.f;
#pragma unroll 2
  for (int kb = 0; kb < K::NKB; ++kb)
#pragma unroll 2
    for (int c8 = 0; c8 < 8; ++c8) {
      uint4* p = reinterpret_cast<uint4*>(tile + kb * kTile + swz(row, c8));
      const uint4 q = *p;
      const int n0 = kb * 64 + c8 * 8;
      const float4 w0 = *reinterpret_cast<const float4*>(w + n0), w1 = *reinterpret_cast<const float4*>(w + n0 + 4);
      const float4 b0 = *reinterpret_cast<const float4*>(w + R * N + n0),
                   b1 = *reinterpret_cast<const float4*>(w + R * N + n0 + 4);
      const float2 f0 = unpack_bf16(q.x), f1 = unpack_bf16(q.y), f2 = unpack_bf16(q.z), f3 = unpack_bf16(q.w);
      uint4 o;
      o.x = pack_bf16(f0.x * ri * w0.x + b0.x, f0.y * ri * w0.y + b0.y);
      o.y = pack_bf16(f1.x * ri * w0.z + b0.z, f1.y * ri * w0.w + b0.w);
      o.z = pack_bf16(f2.x * ri * w1.x + b1.x, f2.y * ri * w1.y + b1.y);
      o.w = pack_bf16(f3.x * ri * w1.z + b1.z, f3.y * ri * w1.w + b1.w);
      *p = o;
    }
}

// ------------------------------------------------------------------ epilogue warps
// Two warps per TMEM lane quadrant: thread = (row m = 32 quad + lane, column
// half ch).  Row m of S, P, Y, Yi; state row n of Hacc / hbar (for N = 64 the
// M = 64 accumulator uses lanes 0..15 of each 32-lane quadrant).
template <int N, int R, int V>
__device__ __forceinline__ void epi_role(uint8_t* smem, const ScanArgs& a, int nchunks, int b, int hh, int c0,
                                         const float* hand_in, float* hand_out, uint64_t* bars,
                                         volatile int* abort_flag, DeviceStatus* status, uint32_t tmem,
                                         const CUtensorMap* tmY) {
  using K = Cfg<N, R, V>;
  constexpr int Q = K::Q;
  const int et = threadIdx.x - kEpi0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = warp & 3;
  const int ch = et >> 7;                // column half
  const int m = quad * 32 + lane;        // chunk row of S, P, Y, Yi
  const int tm = m / R, rm = m % R;      // token and rank of row m
  const int n = (N == 128) ? m : (lane < 16 ? quad * 16 + lane : -1);  // state row of hbar
  const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
  const int L = a.seqlen;
  const size_t unit = (size_t)b * a.nheads + hh;
  const float Dh = a.D ? a.D[hh] : 0.f;
  const int tref = (32 * quad) / R;      // first token of this quadrant's rows
  const int colf_off = quad == 1 ? 0 : (quad == 2 ? 32 : 96);
  uint8_t* Hs = smem + K::OFF_H;
  // (YBUF > 0) this warp's y staging tiles; the first token of its 32 rows in a chunk
  uint8_t* ystg = smem + K::OFF_Y + (et >> 5) * (K::YBUF > 0 ? K::YBUF : 1) * K::Y_TILE;
  const int trow = (32 * quad) / R;

  // ---- initial carried state hbar_0 = h_0 + (1 - lam_1) dt_1 B~_0^T x_0 (columns of this half) ----
  float hb[32];
#pragma unroll
  for (int p = 0; p < 32; ++p) hb[p] = 0.f;
  if (n >= 0 && hand_in != nullptr) {  // a second part: hbar as the first part left it
    const float* hi = hand_in + n * kP + 32 * ch;
#pragma unroll
    for (int p = 0; p < 32; ++p) hb[p] = __ldcg(hi + p);
  } else if (n >= 0 && a.h0 != nullptr) {
    const size_t i0 = tok_index(a, b, 0, hh);
    const float mu1 = (1.f - __bfloat162float(static_cast<const __nv_bfloat16*>(a.lam)[i0])) *
                      __bfloat162float(static_cast<const __nv_bfloat16*>(a.dt)[i0]);
    const float* h0 = a.h0 + (unit * N + n) * kP + 32 * ch;
#pragma unroll
    for (int p = 0; p < 32; ++p) hb[p] = h0[p];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float bp = mu1 * a.bprev0[(unit * R + r) * N + n];
      const float* xp = a.xprev0 + (unit * R + r) * kP + 32 * ch;
#pragma unroll
      for (int p = 0; p < 32; ++p) hb[p] += bp * xp[p];
    }
  }
  store_hbar_bf16(hb, Hs, n, ch);
  fence_proxy_async_smem();
  mbar_arrive(&bars[bEpiDone]);

  // (fused norm, R = 1) this head's weights and biases [4][R][N], then chunks 0 and 1;
  // chunk c + 2 follows at the end of chunk c, in the time the epilogue would wait for prep
  float* nw = reinterpret_cast<float*>(smem + K::OFF_NRM);
  auto normalise = [&](int cn) -> bool {
    const int sn = stage_of<K::NST>(cn);
    if (!mbar_wait(&bars[bFull0 + sn], round_of<K::NST>(cn) & 1, abort_flag, status, kTagFull, a.wait_limit)) return false;
    bc_normalise<N, R, V>(smem + sn * K::STAGE_BYTES, nw, a.neps, et);
    fence_proxy_async_smem();  // the stage is refilled by TMA later
    mbar_arrive(&bars[bNorm0 + sn]);
    return true;
  };
  if constexpr (K::EPI_NORM) {
    const size_t base = (size_t)hh * R * N;
    for (int i = et; i < R * N; i += kNEpi) {
      nw[i] = a.nw_B ? a.nw_B[base + i] : 1.f;
      nw[R * N + i] = a.nb_B ? a.nb_B[base + i] : 0.f;
      nw[2 * R * N + i] = a.nw_C ? a.nw_C[base + i] : 1.f;
      nw[3 * R * N + i] = a.nb_C ? a.nb_C[base + i] : 0.f;
    }
    asm volatile("bar.sync 2, 256;" ::: "memory");  // the epilogue warps' named barrier
    for (int cn = 0; cn < 2 && cn < nchunks; ++cn)
      if (!normalise(cn)) return;
  }

  float e_prev = 0.f;  // (deferred y) e^{cum} of row m in the previous chunk
  for (int c = 0; c < nchunks; ++c) {
    const int s = stage_of<K::NST>(c), u = round_of<K::NST>(c);
    const int t0 = (c0 + c) * Q;
    const float* sc = reinterpret_cast<const float*>(smem + K::OFF_SC) + s * K::SC_PER_STAGE;
    const float *c2 = sc, *gm = sc + Q, *wv = sc + 2 * Q, *colf = sc + 4 * Q + colf_off;

    mbar_wait(&bars[bPrep0 + s], u & 1, abort_flag, status, kTagPrep1, a.wait_limit);
    if constexpr (!K::XW_PREP) {
      // ---- X_w of this chunk (the buffer's last reader, the previous chunk's state
      // MMA, completed before this thread's previous state update), while S runs ----
      if (__any_sync(0xffffffffu, *abort_flag != 0)) return;
      write_xw<R>(smem + K::OFF_XW, smem + s * K::STAGE_BYTES + K::OFF_X, sc + 3 * Q, et);
      fence_proxy_async_smem();
      mbar_arrive(&bars[bXw]);
    }
    // ---- S -> P (bf16, into TMEM) ----
    mbar_wait(&bars[bSFull], c & 1, abort_flag, status, kTagSFull, a.wait_limit);
    if (__any_sync(0xffffffffu, *abort_flag != 0)) return;
    tc_fence_after();
    // every scalar this chunk needs is read now: prep may refill this stage's
    // scalars once P has been consumed
    const float my_c2 = c2[tm];
    const float my_gam = gm[tm];
    const float my_e = ex2(my_c2);
    const float e_end = ex2(c2[Q - 1]);
    const float rowf = ex2(my_c2 - c2[tref]);
    // the two warps of a lane quadrant take alternate 16-column pieces (piece k of
    // this warp: columns 32 k + 16 ch ..), so that each converts one half of the
    // diagonal block, the costly one, and half of every other block
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
      const int cb = k;                  // 32-column block of S
      const int j0 = 32 * cb + 16 * ch;  // first of this piece's 16 columns
      uint32_t pk[8];
      if (cb > quad) {  // warp-uniform: every column is a later token
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = 0u;
      } else {
        float sv[16];
        tmem_ld16(tmem + lane_base + kColS + j0, sv);
        tmem_ld_wait();
        if (cb < quad) {  // every column is an earlier token: rank-1 decay factors
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 cf = *reinterpret_cast<const float4*>(colf + j0 + 4 * j4);
            sv[4 * j4 + 0] *= cf.x * rowf;
            sv[4 * j4 + 1] *= cf.y * rowf;
            sv[4 * j4 + 2] *= cf.z * rowf;
            sv[4 * j4 + 3] *= cf.w * rowf;
          }
        } else {  // diagonal block: causal mask, trapezoid weights, D on the diagonal
          // one factor per column token (the piece's 16 columns are 16 / R tokens of R ranks)
#pragma unroll
          for (int q = 0; q < 16 / R; ++q) {
            const int tj = j0 / R + q;
            const float kf = tj < tm ? ex2(my_c2 - c2[tj]) * wv[tj] : (tj == tm ? my_gam : 0.f);
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const int jj = q * R + r;
              sv[jj] = sv[jj] * kf + (j0 + jj == m ? Dh : 0.f);
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16(sv[2 * i], sv[2 * i + 1]);
      }
      tmem_st8(tmem + lane_base + kColP + j0 / 2, pk);
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(&bars[bPReady]);

    // ---- state update hbar = e^{cum_end} hbar + Hacc (this half's 32 columns) ----
    mbar_wait(&bars[bAcc], c & 1, abort_flag, status, kTagAcc, a.wait_limit);
    if (__any_sync(0xffffffffu, *abort_flag != 0)) return;
    tc_fence_after();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float acc[16];
      tmem_ld16(tmem + lane_base + kColH + 32 * ch + 16 * half, acc);
      tmem_ld_wait();
#pragma unroll
      for (int p = 0; p < 16; ++p) hb[16 * half + p] = e_end * hb[16 * half + p] + acc[p];
    }
    store_hbar_bf16(hb, Hs, n, ch);
    if (c == nchunks - 1 && n >= 0 && (hand_out != nullptr || a.h_out != nullptr)) {
      float* ho = hand_out ? hand_out + n * kP + 32 * ch : a.h_out + (unit * N + n) * kP + 32 * ch;
#pragma unroll
      for (int p = 0; p < 32; p += 4)
        *reinterpret_cast<float4*>(ho + p) = make_float4(hb[p], hb[p + 1], hb[p + 2], hb[p + 3]);
      if (hand_out) __threadfence();
    }

    // ---- y = Y + e^{cum_t} Yi ----
    if constexpr (K::DEFER_Y) {  // the previous chunk's (its Y MMA completed before this chunk's S)
      if (c > 0) {
        if constexpr (K::YBUF > 0)
          store_y_tma<K::YBUF - 1>(tmY, ystg + ((c - 1) % K::YBUF) * K::Y_TILE,
                                   tmem + lane_base + kColY + ((c - 1) & 1) * kColYBuf,
                                   tmem + lane_base + kColYi + ((c - 1) & 1) * kColYBuf, e_prev, b, hh,
                                   t0 - Q + trow, ch, lane);
        else
          store_y(a, tmem + lane_base + kColY + ((c - 1) & 1) * kColYBuf,
                  tmem + lane_base + kColYi + ((c - 1) & 1) * kColYBuf, e_prev, b, hh, t0 - Q + tm, rm, R, ch);
      }
      e_prev = my_e;
    } else {
      mbar_wait(&bars[bYFull], c & 1, abort_flag, status, kTagY, a.wait_limit);
      if (__any_sync(0xffffffffu, *abort_flag != 0)) return;
      tc_fence_after();
      if constexpr (K::YBUF > 0) {
        store_y_tma<K::YBUF - 1>(tmY, ystg + (c % K::YBUF) * K::Y_TILE, tmem + lane_base + kColY,
                                 tmem + lane_base + kColYi, my_e, b, hh, t0 + trow, ch, lane);
      } else {
      const int tg = t0 + tm;
      uint4* yr = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) +
                                           (tok_index(a, b, tg < L ? tg : 0, hh) * R + rm) * kP + 32 * ch);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        float yv[16], yi[16];
        tmem_ld16(tmem + lane_base + kColY + 32 * ch + 16 * half, yv);
        tmem_ld16(tmem + lane_base + kColYi + 32 * ch + 16 * half, yi);
        tmem_ld_wait();
        if (tg < L) {
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = pack_bf16(yv[2 * i] + my_e * yi[2 * i], yv[2 * i + 1] + my_e * yi[2 * i + 1]);
          st_global_32b(yr + 2 * half, w);
        }
      }
      }
    }
    tc_fence_before();
    fence_proxy_async_smem();  // hbar (bf16) is read by the next chunk's MMA
    mbar_arrive(&bars[bEpiDone]);
    if constexpr (K::EPI_NORM) {
      if (c + 2 < nchunks && !normalise(c + 2)) return;
    }
  }
  if constexpr (K::DEFER_Y) {  // y of the last chunk (the Y barrier is committed for it alone)
    mbar_wait(&bars[bYFull], 0, abort_flag, status, kTagY, a.wait_limit);
    if (__any_sync(0xffffffffu, *abort_flag != 0)) return;
    tc_fence_after();
    const int cl = nchunks - 1;
    if constexpr (K::YBUF > 0)
      store_y_tma<K::YBUF - 1>(tmY, ystg + (cl % K::YBUF) * K::Y_TILE, tmem + lane_base + kColY + (cl & 1) * kColYBuf,
                               tmem + lane_base + kColYi + (cl & 1) * kColYBuf, e_prev, b, hh, (c0 + cl) * Q + trow, ch,
                               lane);
    else
      store_y(a, tmem + lane_base + kColY + (cl & 1) * kColYBuf, tmem + lane_base + kColYi + (cl & 1) * kColYBuf,
              e_prev, b, hh, (c0 + cl) * Q + tm, rm, R, ch);
    tc_fence_before();
  }
}

// DL: dt and lam arrive by TMA with theta (a compile-time choice, so that the
// global-load path's prefetch registers are not live in the TMA kernel's rotation)
template <int N, int R, int V, bool DL>
__global__ void __launch_bounds__(kThreads, 1)
    scan_tc_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmC,
                   const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmT,
                   const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmL,
                   const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmY,
                   const TcParams prm) {
  using K = Cfg<N, R, V>;
  constexpr int Q = K::Q;
  extern __shared__ uint8_t smem_raw[];
  // align to 1024 bytes by offsetting the __shared__ pointer itself, so that the
  // compiler keeps every access below in the shared state space
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const ScanArgs& a = prm.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 8);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(a.workspace);
  const int units = a.batch * a.nheads;

  if (tid == 0) {
    for (int i = 0; i < K::NST; ++i) {
      mbar_init(&bars[bFull0 + i], 1);
      mbar_init(&bars[bEmptyBC0 + i], 1);
      mbar_init(&bars[bEmptyX0 + i], 1);
      mbar_init(&bars[bPrep0 + i], kNPrep);
      mbar_init(&bars[bNorm0 + i], kNEpi);
    }
    mbar_init(&bars[bSFull], 1);
    mbar_init(&bars[bAcc], 1);
    mbar_init(&bars[bEpiDone], kNEpi);
    mbar_init(&bars[bPReady], kNEpi);
    mbar_init(&bars[bYFull], 1);
    mbar_init(&bars[bDone], 1);
    mbar_init(&bars[bThFull], 1);
    mbar_init(&bars[bThFree], kNPrep);
    mbar_init(&bars[bXw], kNEpi);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmC);
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmT);
    if (DL) {
      prefetch_tmap(&tmD);
      prefetch_tmap(&tmL);
    }
    if (prm.at_tma) prefetch_tmap(&tmA);
    // this CTA's work: a whole unit (blockIdx), or with a split last wave the next
    // ticket; a second part first waits (bounded) for its first part's hand-over
    int item = blockIdx.x;
    if (prm.split_k > 0) {
      item = atomicAdd(prm.ticket, 1);
      if (item >= units + prm.split_k) {
        // a ticket past this launch's range: another launch shares the workspace
        // (overlapping calls on one workspace race); compute nothing, touch no slot
        *abort_flag = 1;
        report_timeout(status, kTagTicket);
        item = 0;
      } else if (item >= units) {
        const int* f = prm.flags + (item - units);
        const long long t_start = clock64();
        while (ld_acquire_gpu(f) == 0) {
          if (clock64() - t_start > a.wait_limit) {
            *abort_flag = 1;
            report_timeout(status, kTagHand);
            break;
          }
          __nanosleep(256);
        }
      }
    }
    *item_slot = item;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int item = *item_slot;
  const bool skip = *abort_flag != 0;  // the hand-over never came: compute nothing
  int unit = item, c0 = 0, nchunks = prm.nchunks;
  const float* hand_in = nullptr;
  float* hand_out = nullptr;
  if (prm.split_k > 0 && !skip) {
    const size_t slot_floats = (size_t)N * kP + N / 2;
    if (item < prm.split_k) {  // first part: chunks [0, c1), hands hbar and phi over
      nchunks = prm.split_c1;
      hand_out = prm.hand + (size_t)item * slot_floats;
    } else if (item >= units) {  // second part: chunks [c1, n) from the hand-over
      unit = item - units;
      c0 = prm.split_c1;
      nchunks -= c0;
      hand_in = prm.hand + (size_t)unit * slot_floats;
    }
  }
  const int b = unit / a.nheads, hh = unit % a.nheads;

  if (skip) {
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // Three refill streams, each issued as soon as its buffer is free:
      //   B and C of chunk cb into stage cb % 2 once the state MMAs of chunk cb - 2 have read them,
      //   x of chunk cx once the Y MMA of chunk cx - 2 has read it,
      //   theta (+ dt, lam) of chunk ct once prep has read chunk ct - 1's.
      // One thread polls the three conditions (non-blocking), so no stream waits behind another.
      int cb = 0, cx = 0, ct = 0;
      const int gh = hh / (prm.a.nheads / prm.a.ngroups);  // the B/C row this head reads
      long long t_last = clock64();
      const uint32_t th_bytes =
          K::TH_BYTES + (DL ? 2u * K::DL_BYTES : 0u) + (prm.at_tma ? (uint32_t)K::AT_BYTES : 0u);
      // (test_withhold: issue nothing, so that every wait on a load must time out)
      while (!a.test_withhold && (cx < nchunks || ct < nchunks)) {
        bool progress = false;
        if (cb < nchunks && mbar_test(&bars[bEmptyBC0 + stage_of<K::NST>(cb)], (round_of<K::NST>(cb) & 1) ^ 1)) {
          const int s = stage_of<K::NST>(cb), t0 = (c0 + cb) * Q;
          uint8_t* st = smem + s * K::STAGE_BYTES;
          mbar_arrive_expect_tx(&bars[bFull0 + s], K::TMA_BYTES);  // B, C and x of chunk cb
#pragma unroll
          for (int kb = 0; kb < K::NKB; ++kb) {
            tma_load_5d(st + K::OFF_B + kb * kTile, &tmB, &bars[bFull0 + s], kb * 64, 0, gh, t0, b);
            tma_load_5d(st + K::OFF_C + kb * kTile, &tmC, &bars[bFull0 + s], kb * 64, 0, gh, t0, b);
          }
          ++cb;
          progress = true;
        }
        if (cx < cb && mbar_test(&bars[bEmptyX0 + stage_of<K::NST>(cx)], (round_of<K::NST>(cx) & 1) ^ 1)) {
          const int s = stage_of<K::NST>(cx);
          tma_load_5d(smem + s * K::STAGE_BYTES + K::OFF_X, &tmX, &bars[bFull0 + s], 0, 0, hh, (c0 + cx) * Q, b);
          ++cx;
          progress = true;
        }
        if (ct < nchunks && (ct == 0 || mbar_test(&bars[bThFree], (ct - 1) & 1))) {
          const int t0 = (c0 + ct) * Q;
          mbar_arrive_expect_tx(&bars[bThFull], th_bytes);
          tma_load_4d(smem + K::OFF_TH, &tmT, &bars[bThFull], 0, hh, t0, b);
          if (DL) {
            tma_load_3d(smem + K::OFF_DL, &tmD, &bars[bThFull], hh & ~7, t0, b);
            tma_load_3d(smem + K::OFF_DL + K::DL_PAD, &tmL, &bars[bThFull], hh & ~7, t0, b);
          }
          if (prm.at_tma) tma_load_3d(smem + K::OFF_NRM, &tmA, &bars[bThFull], hh & ~7, t0, b);
          ++ct;
          progress = true;
        }
        if (progress) {
          t_last = clock64();
        } else {
          if (*abort_flag) break;
          if (clock64() - t_last > a.wait_limit) {
            *abort_flag = 1;
            report_timeout(status, kTagEmpty);
            break;
          }
          __nanosleep(32);
        }
      }
      // drain: never leave this CTA with bulk copies still landing in its smem.  A
      // stage whose x load was never issued (abort) gets it now, so that its
      // full barrier can complete.
      for (; cx < cb; ++cx)
        tma_load_5d(smem + stage_of<K::NST>(cx) * K::STAGE_BYTES + K::OFF_X, &tmX,
                    &bars[bFull0 + stage_of<K::NST>(cx)], 0, 0, hh, (c0 + cx) * Q, b);
      for (int c = cb - K::NST; c < cb; ++c)
        if (c >= 0 && !mbar_wait_drain(&bars[bFull0 + stage_of<K::NST>(c)], round_of<K::NST>(c) & 1))
          report_timeout(status, kTagDrain);
      if (ct > 0 && !mbar_wait_drain(&bars[bThFull], (ct - 1) & 1)) report_timeout(status, kTagDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t iS = idesc_bf16(kM, kM, 0, 0);     // S = C~ B~^T        (both K-major)
      const uint32_t iYi = idesc_bf16(kM, kP, 0, 1);    // Yi = C~ hbar       (B MN-major)
      const uint32_t iH = idesc_bf16(N, kP, 1, 1);      // Hacc = B~^T X_w    (both MN-major)
      const uint32_t iY = idesc_bf16(kM, kP, 0, 1);     // Y = P X            (A in TMEM)
      const uint32_t sbase = smem_u32(smem);
      for (int c = 0; c < nchunks; ++c) {
        const int s = stage_of<K::NST>(c), u = round_of<K::NST>(c);
        const uint32_t st = sbase + s * K::STAGE_BYTES;
        const uint32_t cB = st + K::OFF_B, cC = st + K::OFF_C, cX = st + K::OFF_X, cXw = sbase + K::OFF_XW;
        const uint32_t ybuf = K::DEFER_Y ? (c & 1) * kColYBuf : 0u;  // Y, Yi buffer of this chunk
        if (!mbar_wait(&bars[bPrep0 + s], u & 1, abort_flag, status, kTagPrep1, a.wait_limit)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kTile + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColS, smem_desc_sw128(cC + off, 16, 1024), smem_desc_sw128(cB + off, 16, 1024), iS,
                      kk > 0);
        }
        mma_commit(&bars[bSFull]);
        if (!mbar_wait(&bars[bEpiDone], c & 1, abort_flag, status, kTagEpiDone, a.wait_limit)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < N / 16; ++kk) {
          const uint32_t offa = (kk >> 2) * kTile + (kk & 3) * 32;
          mma_bf16_ss(tmem + kColYi + ybuf, smem_desc_sw128(cC + offa, 16, 1024),
                      smem_desc_sw128(sbase + K::OFF_H + kk * 2048, N * 128, 1024), iYi, kk > 0);
        }
        // X_w comes from the epilogue warps
        if (!mbar_wait(&bars[bXw], c & 1, abort_flag, status, kTagXw, a.wait_limit)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kM / 16; ++kk) {
          mma_bf16_ss(tmem + kColH, smem_desc_sw128(cB + kk * 2048, kTile, 1024),
                      smem_desc_sw128(cXw + kk * 2048, kTile, 1024), iH, kk > 0);
        }
        mma_commit(&bars[bAcc]);
        mma_commit(&bars[bEmptyBC0 + s]);  // B~, C~ of this stage are no longer read
        if (!mbar_wait(&bars[bPReady], c & 1, abort_flag, status, kTagP, a.wait_limit)) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kM / 16; ++kk) {
          mma_bf16_ts(tmem + kColY + ybuf, tmem + kColP + 8 * kk, smem_desc_sw128(cX + kk * 2048, kTile, 1024), iY,
                      kk > 0);
        }
        // (deferred y: Y of chunk c is complete once S of chunk c + 1 is, since a
        // commit covers every earlier MMA; only the last chunk's Y gets the barrier)
        if (!K::DEFER_Y || c == nchunks - 1) mma_commit(&bars[bYFull]);
        mma_commit(&bars[bEmptyX0 + s]);    // x of this stage is no longer read
      }
      // every MMA this thread issued must be complete before TMEM is released
      mma_commit(&bars[bDone]);
      if (!mbar_wait_drain(&bars[bDone], 0)) report_timeout(status, kTagDrain);
    }
  } else if (tid < kEpi0) {
    prep_role<N, R, V, DL>(smem, a, nchunks, b, hh, c0, hand_in, hand_out, a.A ? a.A[hh] : 0.f, bars,
                       abort_flag, status);
  } else {
    epi_role<N, R, V>(smem, a, nchunks, b, hh, c0, hand_in, hand_out, bars, abort_flag, status, tmem, &tmY);
    // the y stores issued by this warp have read their staging tiles (and completed)
    if (K::YBUF > 0 && (tid & 31) == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  // a first part releases its hand-over (written and fenced by the prep and
  // epilogue threads before the barrier above), also after an abort, so that the
  // second part never waits for a CTA that has ended
  if (tid == 0 && hand_out != nullptr) {
    __threadfence();
    st_release_gpu(prm.flags + item, 1);
  }
}

// ------------------------------------------------------------------ host side
// y [batch, L, H, R, 64] bf16 for the epilogue warps' stores: box = {32, R, 1, 32 / R, 1}
// (a warp's 32 rows x 32 columns), 64-byte swizzle; rows past the sequence are clipped.
bool make_y_map(CUtensorMap* m, const ScanArgs& a) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || a.R > 32) return false;
  const cuuint64_t dims[5] = {(cuuint64_t)kP, (cuuint64_t)a.R, (cuuint64_t)a.nheads, (cuuint64_t)a.seqlen,
                              (cuuint64_t)a.batch};
  const cuuint64_t e = 2;
  const cuuint64_t strides[4] = {e * kP, e * kP * a.R, e * kP * a.R * a.nheads, e * kP * a.R * a.nheads * a.seqlen};
  const cuuint32_t box[5] = {32, (cuuint32_t)a.R, 1, (cuuint32_t)(32 / a.R), 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// ------------------------------------------------------------------ split last wave
// U units on S SMs (one CTA each) run in ceil(U / S) waves, the last holding only
// U mod S of them while the other SMs idle.  k units can instead run in two CTAs:
// chunks [0, c1) early (tickets 0 .. k-1, ahead of the whole units) and [c1, n)
// last (tickets U .. U+k-1), the second continuing from the carried state and
// angle the first hands over, so the result is the one-CTA result bit for bit.
// The plan minimises the makespan of the tickets' list schedule: a CTA takes its
// chunks plus kFillChunks, and a second part starts no earlier than its first part
// ends.  Plans are cached by (U, n).
constexpr double kFillChunks = 2.0;  // pipeline fill and drain of a CTA, in chunk times
constexpr size_t kSplitFlagBytes = 4;
constexpr size_t kSplitRegion = kStatusBlockBytes;  // the split's flags and hand-over slots start here

double split_makespan(int U, int n, int S, int k, int c1) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < S; ++i) free_at.push(0.0);
  std::vector<double> first_end((size_t)k);
  double span = 0.0;
  auto run = [&](double ready, int chunks) {
    double t = free_at.top();
    free_at.pop();
    if (t < ready) t = ready;
    const double e = t + kFillChunks + chunks;
    free_at.push(e);
    if (e > span) span = e;
    return e;
  };
  for (int i = 0; i < k; ++i) first_end[(size_t)i] = run(0.0, c1);
  for (int i = k; i < U; ++i) run(0.0, n);
  for (int i = 0; i < k; ++i) run(first_end[(size_t)i], n - c1);
  return span;
}

SplitPlan plan_split(int U, int n, int S) {
  SplitPlan best{0, 0};
  if (U <= S || n < 2 || U % S == 0) return best;
  const double base = split_makespan(U, n, S, 0, 0);
  double best_span = base;
  const int r = U % S;
  const int dk[] = {0, 2, 4, 8, 12, 16, 24, 32};
  const int step = n > 32 ? n / 32 : 1;
  for (int d : dk) {
    const int k = r + d;
    if (k > U) break;
    for (int c1 = step; c1 < n; c1 += step) {
      const double span = split_makespan(U, n, S, k, c1);
      if (span < best_span - 1e-9) {
        best_span = span;
        best = SplitPlan{k, c1};
      }
    }
  }
  // not worth two more CTAs' fill for less than 2 %
  if (best_span > 0.98 * base) best = SplitPlan{0, 0};
  return best;
}

std::mutex g_plan_mu;
std::map<std::pair<int, int>, SplitPlan> g_plans;
int g_force_k = 0, g_force_c1 = 0;

int tc_chunks(const ScanArgs& a) {
  const int Q = kM / a.R;
  return (a.seqlen + Q - 1) / Q;
}

size_t split_slot_bytes(const ScanArgs& a) { return ((size_t)a.N * kP + a.N / 2) * sizeof(float); }
size_t split_flag_region(int k) { return ((size_t)k * kSplitFlagBytes + 255) & ~(size_t)255; }

template <int N, int R>
int launch_nr(const ScanArgs& a, cudaStream_t s) {
  using K = Cfg<N, R, kPlain>;  // (Q does not depend on the variant)
  const int var = a.bcnorm ? kBCNorm : (a.A_t ? kTimeA : kPlain);
  const int smem_alloc = var == kBCNorm ? Cfg<N, R, kBCNorm>::SMEM_ALLOC
                                        : (var == kTimeA ? Cfg<N, R, kTimeA>::SMEM_ALLOC : K::SMEM_ALLOC);
  const int ybuf = var == kBCNorm ? Cfg<N, R, kBCNorm>::YBUF : (var == kTimeA ? Cfg<N, R, kTimeA>::YBUF : K::YBUF);
  CUtensorMap tmB, tmC, tmX, tmT;
  if (!make_map(&tmB, a.B, N, a.ngroups, a, K::Q) || !make_map(&tmC, a.C, N, a.ngroups, a, K::Q) ||
      !make_map(&tmX, a.x, kP, a.nheads, a, K::Q) ||
      !make_theta_map(&tmT, a, K::Q))
    return MAMBA3_ERR_CUDA;
  TcParams prm;
  prm.a = a;
  prm.nchunks = (a.seqlen + K::Q - 1) / K::Q;
  CUtensorMap tmD, tmL, tmA, tmY;
  memset(&tmY, 0, sizeof(tmY));
  if (ybuf > 0 && !make_y_map(&tmY, a)) return MAMBA3_ERR_CUDA;
  memset(&tmD, 0, sizeof(tmD));
  memset(&tmL, 0, sizeof(tmL));
  memset(&tmA, 0, sizeof(tmA));
  prm.dl_tma = make_dl_map(&tmD, a.dt, a, K::Q + 1) && make_dl_map(&tmL, a.lam, a, K::Q + 1);
  prm.at_tma = 0;
  if (a.A_t) {  // the A_t tile shares the region of the B/C norm table; all three tiles or none
    prm.at_tma = prm.dl_tma && !a.bcnorm && make_dl_map(&tmA, a.A_t, a, K::Q);
    if (!prm.at_tma) prm.dl_tma = 0;
  }
  prm.split_k = prm.split_c1 = 0;
  prm.ticket = prm.flags = nullptr;
  prm.hand = nullptr;
  if (a.split) {  // the caller zeroed the ticket and the flags
    const SplitPlan sp = tc_split_plan(a);
    if (sp.k > 0) {
      uint8_t* ws = static_cast<uint8_t*>(a.workspace);
      prm.split_k = sp.k;
      prm.split_c1 = sp.c1;
      prm.ticket = reinterpret_cast<int*>(ws + sizeof(DeviceStatus));
      prm.flags = reinterpret_cast<int*>(ws + kSplitRegion);
      prm.hand = reinterpret_cast<float*>(ws + kSplitRegion + split_flag_region(sp.k));
    }
  }
  auto kern = prm.dl_tma ? (var == kBCNorm ? scan_tc_kernel<N, R, kBCNorm, true>
                                           : (var == kTimeA ? scan_tc_kernel<N, R, kTimeA, true>
                                                            : scan_tc_kernel<N, R, kPlain, true>))
                        : (var == kBCNorm ? scan_tc_kernel<N, R, kBCNorm, false>
                                          : (var == kTimeA ? scan_tc_kernel<N, R, kTimeA, false>
                                                           : scan_tc_kernel<N, R, kPlain, false>));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_alloc) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  kern<<<a.batch * a.nheads + prm.split_k, kThreads, smem_alloc, s>>>(tmB, tmC, tmX, tmT, tmD, tmL, tmA, tmY, prm);
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // namespace

int tc_scan_supported(const ScanArgs& a) {
  if (a.ngroups < 1 || a.nheads % a.ngroups != 0) return MAMBA3_ERR_INVALID;  // B, C rows per token
  if (a.dtype != MAMBA3_BF16 || a.P != kP || a.seqlen < 1) return MAMBA3_ERR_UNSUPPORTED;
  if (a.N != 64 && a.N != 128) return MAMBA3_ERR_UNSUPPORTED;
  if (a.R != 1 && a.R != 2 && a.R != 4) return MAMBA3_ERR_UNSUPPORTED;
  if (a.Q != 0 && a.Q != kM / a.R) return MAMBA3_ERR_UNSUPPORTED;
  return MAMBA3_OK;
}

SplitPlan tc_split_plan(const ScanArgs& a) { return split_plan(a.batch * a.nheads, tc_chunks(a)); }

SplitPlan split_plan(int U, int n) {
  std::lock_guard<std::mutex> lock(g_plan_mu);
  if (g_force_k < 0) return SplitPlan{0, 0};
  if (g_force_k > 0)  // a forced plan that does not fit the shape means no split
    return (g_force_k <= U && g_force_c1 >= 1 && g_force_c1 < n) ? SplitPlan{g_force_k, g_force_c1} : SplitPlan{0, 0};
  const auto key = std::make_pair(U, n);
  auto it = g_plans.find(key);
  if (it != g_plans.end()) return it->second;
  const SplitPlan p = plan_split(U, n, kSMs);
  if (g_plans.size() >= 4096) g_plans.clear();  // (bounded: callers with ever-new shapes)
  g_plans[key] = p;
  return p;
}

size_t tc_split_bytes(const ScanArgs& a) {
  if (tc_scan_supported(a) != MAMBA3_OK) return 0;
  const SplitPlan p = tc_split_plan(a);
  if (p.k == 0) return 0;
  return split_flag_region(p.k) + (size_t)p.k * split_slot_bytes(a);
}

size_t tc_split_zero_bytes(const ScanArgs& a) {
  const SplitPlan p = tc_split_plan(a);
  return kSplitRegion + split_flag_region(p.k);
}

void tc_force_split(int k, int c1) {
  std::lock_guard<std::mutex> lock(g_plan_mu);
  g_force_k = k;
  g_force_c1 = c1;
}

int launch_scan_tc(const ScanArgs& a, cudaStream_t s) {
  if (a.N == 128) {
    if (a.R == 1) return launch_nr<128, 1>(a, s);
    if (a.R == 2) return launch_nr<128, 2>(a, s);
    if (a.R == 4) return launch_nr<128, 4>(a, s);
  } else {
    if (a.R == 1) return launch_nr<64, 1>(a, s);
    if (a.R == 2) return launch_nr<64, 2>(a, s);
    if (a.R == 4) return launch_nr<64, 4>(a, s);
  }
  return MAMBA3_ERR_UNSUPPORTED;
}

}  // namespace m3

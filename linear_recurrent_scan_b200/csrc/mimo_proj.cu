// MIMO rank-R projections of the Mamba-3 layer on the tcgen05 tensor cores
// (bf16 operands from TMA, fp32 accumulators in TMEM; sm_100a).
//
// "Mamba-3: 2x smaller state ..." (MarkTechPost, Korean translation), section
// 1.3: MIMO raises the rank of the input and output projections to R, so that
// x_t is P x R and the state update becomes a matrix product.  The page prints
// no weights; one dense matrix per head on each side of the recurrence is the
// reading implemented here:
//   up:    x[t, h, r, p] = sum_q Wx[h, r P + p, q] u[t, h, q]      (K = P, R P outputs)
//   down:  o[t, h, p]    = sum_k Wy[h, p, k] y[t, h, k], k = r P + q (K = R P, P outputs)
// optionally followed (down) by the pre-gate RMS norm over the head's P outputs
// and the silu gate of the output side (same page, section 2):
//   out = o / sqrt(mean_p o^2 + eps) * w[h, p] * silu(z[t, h, p]).
// t runs over every (batch, token) pair.
//
// One CTA per (head, range of 128-token tiles).  Warp 4 (one lane) loads the
// head's weight tile once, then streams the token tiles through a 2-stage TMA
// ring and issues one MMA chain per tile into one of two TMEM accumulators;
// warps 0..3 (one TMEM lane quadrant each, thread = token row) drain the other
// accumulator: fp32 -> (norm, gate) -> bf16 -> 16-byte stores.  The work is
// HBM-bound (about 50 FLOP per byte at R = 4, against a ridge near 250).
// Every wait is bounded; on expiry the CTA records MAMBA3_ERR_TIMEOUT in the
// library's status word, lets what it issued land, frees TMEM and returns.
#include <cuda.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "sm100_ptx.cuh"

namespace m3 {
namespace {

using namespace ptx;

constexpr int kP = 64;
constexpr int kRows = 128;   // tokens per tile (MMA M)
constexpr int kThreads = 160;  // warps 0..3 epilogue, warp 4 producer + MMA issuer

// Status word of the workspace-less projection calls (read by mamba3_library_status).
__device__ DeviceStatus g_proj_status;

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

struct ProjParams {
  long long tokens;  // batch * seqlen
  int nheads, tiles, tiles_per_cta;
  void* out;               // x [T, H, R, P] (up) or o [T, H, P] (down), bf16
  const void* z;           // down: gate [T, H, P] bf16, or null (no norm, no gate)
  const float* w;          // down with gate: norm weight [H, P] or null (1)
  float eps;
  long long wait_limit;
  int test_withhold;
};

// UP: A = u tile [128 x 64], B = Wx[h] [R P x 64]      -> D [128 x R P]
// DOWN: A = y tile [128 x R P] (R P / 64 blocks), B = Wy[h] [64 x R P] -> D [128 x 64]
template <int R, bool UP>
struct PCfg {
  static constexpr int KB = UP ? 1 : R;                   // 64-wide K blocks
  static constexpr int NOUT = UP ? R * kP : kP;           // accumulator columns
  static constexpr int IN_BYTES = KB * kRows * 128;       // one token tile
  static constexpr int W_BYTES = UP ? R * kP * 128 : R * kP * 128;  // (R P rows x 128 B) or (64 rows x R blocks)
  static constexpr int OFF_W = 0;
  static constexpr int OFF_IN = OFF_W + W_BYTES;
  static constexpr int OFF_BAR = OFF_IN + 2 * IN_BYTES;   // full[2], empty[2], accf[2], acce[2], wfull
  static constexpr int OFF_MISC = OFF_BAR + 128;
  static constexpr int SMEM = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * NOUT <= 32 ? 32 : (2 * NOUT <= 64 ? 64 : (2 * NOUT <= 128 ? 128 : (2 * NOUT <= 256 ? 256 : 512)));
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
  static_assert(NOUT <= 256, "one MMA per tile");
};

enum { bFull = 0, bEmpty = 2, bAccF = 4, bAccE = 6, bW = 8 };

template <int R, bool UP, bool GATE>
__global__ void __launch_bounds__(kThreads) mimo_proj_kernel(const __grid_constant__ CUtensorMap tmIn,
                                                             const __grid_constant__ CUtensorMap tmW,
                                                             const ProjParams prm) {
  using K = PCfg<R, UP>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  const int ctas_per_head = (prm.tiles + prm.tiles_per_cta - 1) / prm.tiles_per_cta;
  const int h = blockIdx.x / ctas_per_head;
  const int tile0 = (blockIdx.x % ctas_per_head) * prm.tiles_per_cta;
  const int ntile = min(prm.tiles_per_cta, prm.tiles - tile0);

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[bFull + i], 1);
      mbar_init(&bars[bEmpty + i], 1);
      mbar_init(&bars[bAccF + i], 1);
      mbar_init(&bars[bAccE + i], 128);
    }
    mbar_init(&bars[bW], 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmIn);
    prefetch_tmap(&tmW);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, K::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ---- producer and MMA issuer ----
      int loaded = 0, done = 0;  // tiles whose loads were issued / whose MMAs were issued
      int wload = 0;
      if (!prm.test_withhold) {
        mbar_arrive_expect_tx(&bars[bW], K::W_BYTES);
        if (UP) {
          tma_load_3d(smem + K::OFF_W, &tmW, &bars[bW], 0, 0, h);
        } else {
#pragma unroll
          for (int kb = 0; kb < R; ++kb) tma_load_3d(smem + K::OFF_W + kb * kP * 128, &tmW, &bars[bW], kb * 64, 0, h);
        }
        wload = 1;
      }
      const uint32_t idesc = idesc_bf16(kRows, K::NOUT, 0, 0);
      bool ok = true;
      long long t_last = clock64();
      while (ok && done < ntile) {
        bool progress = false;
        // load tile `loaded` into stage loaded & 1 once its previous MMA has read it
        if (!prm.test_withhold && loaded < ntile && loaded < done + 2 &&
            (loaded < 2 || mbar_test(&bars[bEmpty + (loaded & 1)], ((loaded >> 1) - 1) & 1))) {
          const int s = loaded & 1;
          const long long row0 = (long long)(tile0 + loaded) * kRows;
          mbar_arrive_expect_tx(&bars[bFull + s], K::IN_BYTES);
#pragma unroll
          for (int kb = 0; kb < K::KB; ++kb)
            tma_load_3d(smem + K::OFF_IN + s * K::IN_BYTES + kb * kRows * 128, &tmIn, &bars[bFull + s], kb * 64, h,
                        (int)row0);
          ++loaded;
          progress = true;
        }
        // MMA of tile `done` once its input landed and its accumulator is free
        if (done < loaded && mbar_test(&bars[bFull + (done & 1)], (done >> 1) & 1) &&
            (done < 2 || mbar_test(&bars[bAccE + (done & 1)], ((done >> 1) - 1) & 1)) &&
            (done > 0 || mbar_test(&bars[bW], 0))) {
          tc_fence_after();
          const int s = done & 1;
          const uint32_t cIn = smem_u32(smem + K::OFF_IN + s * K::IN_BYTES), cW = smem_u32(smem + K::OFF_W);
          const uint32_t d = tmem + (uint32_t)(s * K::NOUT);
#pragma unroll
          for (int kk = 0; kk < K::KB * 4; ++kk) {
            const uint32_t offa = (kk >> 2) * kRows * 128 + (kk & 3) * 32;
            const uint32_t offb = (kk >> 2) * kP * 128 + (kk & 3) * 32;
            mma_bf16_ss(d, smem_desc_sw128(cIn + offa, 16, 1024), smem_desc_sw128(cW + offb, 16, 1024), idesc,
                        kk > 0);
          }
          mma_commit(&bars[bEmpty + s]);
          mma_commit(&bars[bAccF + s]);
          ++done;
          progress = true;
        }
        if (progress) {
          t_last = clock64();
        } else {
          if (*abort_flag) ok = false;
          else if (clock64() - t_last > prm.wait_limit) {
            *abort_flag = 1;
            report_timeout(&g_proj_status, 31);
            ok = false;
          }
        }
      }
      // let the copies and MMAs issued land before TMEM is freed and the CTA exits
      if (wload && !mbar_wait_drain(&bars[bW], 0)) report_timeout(&g_proj_status, 32);
      for (int i = done; i < loaded; ++i)
        if (!mbar_wait_drain(&bars[bFull + (i & 1)], (i >> 1) & 1)) report_timeout(&g_proj_status, 32);
      if (done > 0 && !mbar_wait_drain(&bars[bAccF + ((done - 1) & 1)], ((done - 1) >> 1) & 1))
        report_timeout(&g_proj_status, 32);
    }
  } else {
    // ---- epilogue: warp w reads TMEM lanes 32 w .. 32 w + 31 (thread = token row) ----
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(prm.out);
    for (int i = 0; i < ntile; ++i) {
      const int s = i & 1;
      if (!mbar_wait(&bars[bAccF + s], (i >> 1) & 1, abort_flag, &g_proj_status, 33, prm.wait_limit)) break;
      tc_fence_after();
      const long long tok = (long long)(tile0 + i) * kRows + warp * 32 + lane;
      const bool valid = tok < prm.tokens;
      const uint32_t tacc = tmem + lane_base + (uint32_t)(s * K::NOUT);
      if constexpr (UP) {
        uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)(valid ? tok : 0) * prm.nheads + h) * (R * kP));
#pragma unroll 1
        for (int c = 0; c < K::NOUT / 32; ++c) {
          float v[32];
          tmem_ld32(tacc + 32 * c, v);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[4 * c + q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                          pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
          }
        }
      } else {
        float v[64];
        tmem_ld32(tacc, v);
        tmem_ld32(tacc + 32, v + 32);
        tmem_ld_wait();
        if (GATE) {
          float ms = 0.f;
#pragma unroll
          for (int p = 0; p < 64; ++p) ms += v[p] * v[p];
          const float var = ms * (1.f / kP) + prm.eps;
          const float inv = var > 0.f ? rsqrtf(var) : 0.f;  // an all-zero row with eps = 0 gives 0
          const uint4* zr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(prm.z) +
                                                          ((size_t)(valid ? tok : 0) * prm.nheads + h) * kP);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 zq = valid ? zr[q] : make_uint4(0, 0, 0, 0);
            const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const float z0 = __uint_as_float(zw[k] << 16), z1 = __uint_as_float(zw[k] & 0xffff0000u);
              const int p = 8 * q + 2 * k;
              const float w0 = prm.w ? prm.w[h * kP + p] : 1.f, w1 = prm.w ? prm.w[h * kP + p + 1] : 1.f;
              v[p] = v[p] * inv * w0 * __fdividef(z0, 1.f + __expf(-z0));
              v[p + 1] = v[p + 1] * inv * w1 * __fdividef(z1, 1.f + __expf(-z1));
            }
          }
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)tok * prm.nheads + h) * kP);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                                pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[bAccE + s]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, K::TMEM_COLS);
  }
}

// 3-D bf16 map, innermost first, box {64, b1, b2}, 128-byte swizzle
bool map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b1, uint32_t b2) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {2 * d0, 2 * d0 * d1};
  const cuuint32_t box[3] = {64, b1, b2};
  const cuuint32_t es[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int R, bool UP, bool GATE>
int launch_k(const ProjArgs& a, cudaStream_t s) {
  using K = PCfg<R, UP>;
  const long long T = a.tokens;
  const int H = a.nheads;
  CUtensorMap tmIn, tmW;
  if (UP) {
    // u [T, H, P]; Wx [H, R P, P]
    if (!map3(&tmIn, a.in, kP, H, T, 1, kRows) || !map3(&tmW, a.weight, kP, R * kP, H, R * kP, 1))
      return MAMBA3_ERR_CUDA;
  } else {
    // y [T, H, R P]; Wy [H, P, R P]
    if (!map3(&tmIn, a.in, R * kP, H, T, 1, kRows) || !map3(&tmW, a.weight, R * kP, kP, H, kP, 1))
      return MAMBA3_ERR_CUDA;
  }
  ProjParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.tokens = T;
  prm.nheads = H;
  prm.tiles = (int)((T + kRows - 1) / kRows);
  // about two CTAs' worth of tiles per SM in total, whole tiles per CTA
  const long long total = (long long)prm.tiles * H;
  long long per = (total + 2 * 148 - 1) / (2 * 148);
  if (per < 1) per = 1;
  if (per > prm.tiles) per = prm.tiles;
  prm.tiles_per_cta = (int)per;
  const int ctas_per_head = (prm.tiles + prm.tiles_per_cta - 1) / prm.tiles_per_cta;
  prm.out = a.out;
  prm.z = a.z;
  prm.w = a.w;
  prm.eps = a.eps;
  prm.wait_limit = a.wait_limit;
  prm.test_withhold = a.test_withhold;
  auto k = mimo_proj_kernel<R, UP, GATE>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, K::SMEM_ALLOC) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  k<<<ctas_per_head * H, kThreads, K::SMEM_ALLOC, s>>>(tmIn, tmW, prm);
  return cudaGetLastError() == cudaSuccess ? MAMBA3_OK : MAMBA3_ERR_CUDA;
}

}  // namespace

int proj_status_read_and_clear(int* code) {
  DeviceStatus st, zero = {0, 0, 0, 0};
  if (cudaMemcpyFromSymbol(&st, g_proj_status, sizeof(st)) != cudaSuccess) return MAMBA3_ERR_CUDA;
  if (st.code != 0 && cudaMemcpyToSymbol(g_proj_status, &zero, sizeof(zero)) != cudaSuccess) return MAMBA3_ERR_CUDA;
  *code = st.code;
  return MAMBA3_OK;
}

int launch_mimo_proj(const ProjArgs& a, cudaStream_t s) {
  if (a.tokens == 0) return MAMBA3_OK;
  if (a.up) {
    if (a.R == 1) return launch_k<1, true, false>(a, s);
    if (a.R == 2) return launch_k<2, true, false>(a, s);
    if (a.R == 4) return launch_k<4, true, false>(a, s);
  } else if (a.z) {
    if (a.R == 1) return launch_k<1, false, true>(a, s);
    if (a.R == 2) return launch_k<2, false, true>(a, s);
    if (a.R == 4) return launch_k<4, false, true>(a, s);
  } else {
    if (a.R == 1) return launch_k<1, false, false>(a, s);
    if (a.R == 2) return launch_k<2, false, false>(a, s);
    if (a.R == 4) return launch_k<4, false, false>(a, s);
  }
  return MAMBA3_ERR_UNSUPPORTED;
}

}  // namespace m3

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
// Persistent CTAs (one or two per SM) each take an even share of the (head,
// 128-token tile) work items in head order.  Warp 4 (one lane) loads each head's
// weight tile as the CTA's items reach that head (two buffers where they fit),
// streams the token tiles (and, with the gate, the z tiles) through 2-stage TMA
// rings and issues one MMA chain per tile into one of two TMEM accumulators;
// warps 0..3 (one TMEM lane quadrant each, thread = token row) drain the other
// accumulator: fp32 -> (norm, gate) -> bf16 into a 128-byte-swizzled staging tile
// per 64 output columns, which one thread writes out with a TMA store (rows past
// the last token are clipped by the tensor map).  The work is HBM-bound (about 50
// FLOP per byte at R = 4, against a ridge near 250).
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
  int nheads, tiles;  // tiles of 128 tokens per head; work item = head * tiles + tile
  long long items;    // nheads * tiles, split evenly over the grid
  const float* w;          // down with the gate: norm weight [H, P] or null (1)
  float eps;
  long long wait_limit;
  int test_withhold;
};

// UP: A = u tile [128 x 64], B = Wx[h] [R P x 64]      -> D [128 x R P]
// DOWN: A = y tile [128 x R P] (R P / 64 blocks), B = Wy[h] [64 x R P] -> D [128 x 64]
template <int R, bool UP, bool GATE>
struct PCfg {
  static constexpr int KB = UP ? 1 : R;                   // 64-wide K blocks
  static constexpr int NOUT = UP ? R * kP : kP;           // accumulator columns
  static constexpr int NB = NOUT / 64;                    // 64-column output blocks
  static constexpr int IN_BYTES = KB * kRows * 128;       // one token tile
  static constexpr int W_BYTES = R * kP * 128;            // (R P rows x 128 B) or (64 rows x R blocks)
  static constexpr int Z_BYTES = GATE ? kRows * 128 : 0;  // one gate tile
  static constexpr int OUT_BYTES = NB * kRows * 128;      // staging of one output tile
  static constexpr int fit(int nwb) { return nwb * W_BYTES + 2 * IN_BYTES + 2 * Z_BYTES + OUT_BYTES + 256 + 1024; }
  static constexpr int NWB = fit(2) <= 232448 ? 2 : 1;   // weight buffers (heads alternate)
  static constexpr int OFF_W = 0;
  static constexpr int OFF_IN = OFF_W + NWB * W_BYTES;
  static constexpr int OFF_Z = OFF_IN + 2 * IN_BYTES;
  static constexpr int OFF_OUT = OFF_Z + 2 * Z_BYTES;
  static constexpr int OFF_BAR = OFF_OUT + OUT_BYTES;     // full, empty, accf, acce, w, zf, ze: [2] each
  static constexpr int OFF_MISC = OFF_BAR + 128;
  static constexpr int SMEM = OFF_MISC + 16;
  static constexpr int SMEM_ALLOC = SMEM + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * NOUT <= 32 ? 32 : (2 * NOUT <= 64 ? 64 : (2 * NOUT <= 128 ? 128 : (2 * NOUT <= 256 ? 256 : 512)));
  static_assert(SMEM_ALLOC <= 232448, "shared memory");
  static_assert(NOUT <= 256, "one MMA per tile");
};

enum { bFull = 0, bEmpty = 2, bAccF = 4, bAccE = 6, bW = 8, bZF = 10, bZE = 12 };

// named barrier over the 128 epilogue threads (id 1) that also ORs a predicate, so
// that every epilogue thread takes the same decision
__device__ __forceinline__ bool epi_sync_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// byte offset of 16-byte chunk `c` (0..7) of row `row` inside a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t swz(int row, int c) { return (uint32_t)(row * 128 + ((c ^ (row & 7)) << 4)); }

// The CTA's work items [i0, i1) of the flattened (head, tile) space; the heads
// they span are its head segments k = 0, 1, ... (head = item / tiles), each using
// weight buffer k % NWB.
struct ItemRange {
  long long i0, i1;
  int h0;
};
__device__ __forceinline__ ItemRange item_range(const ProjParams& p) {
  ItemRange r;
  r.i0 = p.items * blockIdx.x / gridDim.x;
  r.i1 = p.items * (blockIdx.x + 1) / gridDim.x;
  r.h0 = (int)(r.i0 / p.tiles);
  return r;
}

template <int R, bool UP, bool GATE>
__global__ void __launch_bounds__(kThreads) mimo_proj_kernel(const __grid_constant__ CUtensorMap tmIn,
                                                             const __grid_constant__ CUtensorMap tmW,
                                                             const __grid_constant__ CUtensorMap tmOut,
                                                             const __grid_constant__ CUtensorMap tmZ,
                                                             const ProjParams prm) {
  using K = PCfg<R, UP, GATE>;
  constexpr int NWB = K::NWB;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + K::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + K::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 4);
  // items whose MMA is known complete (the epilogue saw their accumulator full);
  // monotone, so the producer can tell when a weight buffer is free
  volatile int* mma_done = reinterpret_cast<volatile int*>(smem + K::OFF_MISC + 8);
  const ItemRange rg = item_range(prm);
  const int n = (int)(rg.i1 - rg.i0);  // items of this CTA
  auto head_of = [&](int j) { return (int)((rg.i0 + j) / prm.tiles); };
  auto tile_of = [&](int j) { return (int)((rg.i0 + j) % prm.tiles); };

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars[bFull + i], 1);
      mbar_init(&bars[bEmpty + i], 1);
      mbar_init(&bars[bAccF + i], 1);
      mbar_init(&bars[bAccE + i], 128);
      mbar_init(&bars[bW + i], 1);
      mbar_init(&bars[bZF + i], 1);
      mbar_init(&bars[bZE + i], 128);
    }
    *abort_flag = 0;
    *mma_done = 0;
    fence_mbar_init();
    prefetch_tmap(&tmIn);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmOut);
    if (GATE) prefetch_tmap(&tmZ);
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
      // ---- producer and MMA issuer: inputs (and gate tiles) through 2-stage rings,
      // the weights of head segment k into buffer k % NWB once segment k - NWB's
      // MMAs are complete ----
      int loaded = 0, done = 0, zl = 0;  // items whose loads / MMAs / gate loads were issued
      int wseg = 0;                      // head segments whose weights were issued
      // the CTA's last item of head segment k
      auto seg_last = [&](int k) {
        const long long e = (long long)(rg.h0 + k + 1) * prm.tiles - rg.i0;
        return (int)(e < n ? e : n) - 1;
      };
      const uint32_t idesc = idesc_bf16(kRows, K::NOUT, 0, 0);
      bool ok = true;
      long long t_last = clock64();
      // (the gate tiles follow the epilogue, so they can still be due after the last MMA)
      while (ok && (done < n || (GATE && zl < n))) {
        bool progress = false;
        // weights of the next head segment, once its buffer is free
        const int seg_needed = head_of(loaded < n ? loaded : n - 1) - rg.h0;
        if (!prm.test_withhold && wseg <= seg_needed && wseg <= head_of(n - 1) - rg.h0) {
          const int slot = wseg % NWB;
          // buffer free once the MMA of segment wseg - NWB's last item has completed
          // (every item of that segment, not only those issued so far)
          if (wseg < NWB || seg_last(wseg - NWB) < *mma_done) {
            const int h = rg.h0 + wseg;
            uint8_t* wb = smem + K::OFF_W + slot * K::W_BYTES;
            mbar_arrive_expect_tx(&bars[bW + slot], K::W_BYTES);
            if (UP) {
              tma_load_3d(wb, &tmW, &bars[bW + slot], 0, 0, h);
            } else {
#pragma unroll
              for (int kb = 0; kb < R; ++kb) tma_load_3d(wb + kb * kP * 128, &tmW, &bars[bW + slot], kb * 64, 0, h);
            }
            ++wseg;
            progress = true;
          }
        }
        // inputs of item `loaded` into stage loaded & 1 once the MMA of item loaded - 2 has read it
        if (!prm.test_withhold && loaded < n && loaded < done + 2 &&
            (loaded < 2 || mbar_test(&bars[bEmpty + (loaded & 1)], ((loaded >> 1) - 1) & 1))) {
          const int s = loaded & 1;
          const int row0 = tile_of(loaded) * kRows;
          mbar_arrive_expect_tx(&bars[bFull + s], K::IN_BYTES);
#pragma unroll
          for (int kb = 0; kb < K::KB; ++kb)
            tma_load_3d(smem + K::OFF_IN + s * K::IN_BYTES + kb * kRows * 128, &tmIn, &bars[bFull + s], kb * 64,
                        head_of(loaded), row0);
          ++loaded;
          progress = true;
        }
        // gate tile of item `zl` into slot zl & 1 once the epilogue of item zl - 2 has read it
        if (GATE && !prm.test_withhold && zl < n &&
            (zl < 2 || mbar_test(&bars[bZE + (zl & 1)], ((zl >> 1) - 1) & 1))) {
          const int s = zl & 1;
          mbar_arrive_expect_tx(&bars[bZF + s], K::Z_BYTES);
          tma_load_3d(smem + K::OFF_Z + s * K::Z_BYTES, &tmZ, &bars[bZF + s], 0, head_of(zl), tile_of(zl) * kRows);
          ++zl;
          progress = true;
        }
        // MMA of item `done`: inputs landed, accumulator free, its head's weights loaded
        if (done < loaded) {
          const int seg = head_of(done) - rg.h0, slot = seg % NWB;
          if (seg < wseg && mbar_test(&bars[bFull + (done & 1)], (done >> 1) & 1) &&
              (done < 2 || mbar_test(&bars[bAccE + (done & 1)], ((done >> 1) - 1) & 1)) &&
              mbar_test(&bars[bW + slot], (seg / NWB) & 1)) {
            tc_fence_after();
            const int s = done & 1;
            const uint32_t cIn = smem_u32(smem + K::OFF_IN + s * K::IN_BYTES);
            const uint32_t cW = smem_u32(smem + K::OFF_W + slot * K::W_BYTES);
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
      for (int k = (wseg >= NWB ? wseg - NWB : 0); k < wseg; ++k)
        if (!mbar_wait_drain(&bars[bW + (k % NWB)], (k / NWB) & 1)) report_timeout(&g_proj_status, 32);
      for (int i = done; i < loaded; ++i)
        if (!mbar_wait_drain(&bars[bFull + (i & 1)], (i >> 1) & 1)) report_timeout(&g_proj_status, 32);
      if (GATE)  // gate tiles not yet waited for by the epilogue (at most the last two)
        for (int i = (zl >= 2 ? zl - 2 : 0); i < zl; ++i)
          if (!mbar_wait_drain(&bars[bZF + (i & 1)], (i >> 1) & 1)) report_timeout(&g_proj_status, 32);
      if (done > 0 && !mbar_wait_drain(&bars[bAccF + ((done - 1) & 1)], ((done - 1) >> 1) & 1))
        report_timeout(&g_proj_status, 32);
    }
  } else {
    // ---- epilogue: warp w reads TMEM lanes 32 w .. 32 w + 31 (thread = token row m) ----
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int m = warp * 32 + lane;
    for (int i = 0; i < n; ++i) {
      const int s = i & 1;
      bool ok = mbar_wait(&bars[bAccF + s], (i >> 1) & 1, abort_flag, &g_proj_status, 33, prm.wait_limit);
      if (GATE && ok) ok = mbar_wait(&bars[bZF + s], (i >> 1) & 1, abort_flag, &g_proj_status, 34, prm.wait_limit);
      if (epi_sync_any(!ok || *abort_flag != 0)) break;  // one decision for all epilogue threads
      tc_fence_after();
      if (tid == 0) *mma_done = i + 1;  // MMA i (and every earlier one) has completed
      const int h = head_of(i), row0 = tile_of(i) * kRows;
      const uint32_t tacc = tmem + lane_base + (uint32_t)(s * K::NOUT);
#pragma unroll 1
      for (int k = 0; k < K::NB; ++k) {
        float v[64];
        tmem_ld32(tacc + 64 * k, v);
        tmem_ld32(tacc + 64 * k + 32, v + 32);
        tmem_ld_wait();
        if (k == K::NB - 1) {  // the accumulator is free for the MMA of item i + 2
          tc_fence_before();
          mbar_arrive(&bars[bAccE + s]);
        }
        if constexpr (GATE) {
          float ms = 0.f;
#pragma unroll
          for (int p = 0; p < 64; ++p) ms += v[p] * v[p];
          const float var = ms * (1.f / kP) + prm.eps;
          const float inv = var > 0.f ? rsqrtf(var) : 0.f;  // an all-zero row with eps = 0 gives 0
          const uint8_t* zt = smem + K::OFF_Z + s * K::Z_BYTES;
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 zq = *reinterpret_cast<const uint4*>(zt + swz(m, q));
            const uint32_t zw[4] = {zq.x, zq.y, zq.z, zq.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const float z0 = __uint_as_float(zw[kk] << 16), z1 = __uint_as_float(zw[kk] & 0xffff0000u);
              const int p = 8 * q + 2 * kk;
              const float w0 = prm.w ? prm.w[h * kP + p] : 1.f, w1 = prm.w ? prm.w[h * kP + p + 1] : 1.f;
              v[p] = v[p] * inv * w0 * __fdividef(z0, 1.f + __expf(-z0));
              v[p + 1] = v[p + 1] * inv * w1 * __fdividef(z1, 1.f + __expf(-z1));
            }
          }
          mbar_arrive(&bars[bZE + s]);  // every value read from the gate tile is consumed above
        }
        // staging block k is free once the store that last read it (item i - 1) has
        uint8_t* stg = smem + K::OFF_OUT + k * kRows * 128;
        if (tid == 0) bulk_wait_read<K::NB - 1>();
        epi_sync();
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + swz(m, q)) =
              make_uint4(pack_bf16(v[8 * q], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
        fence_proxy_async_smem();
        epi_sync();
        if (tid == 0) {
          tma_store_3d(&tmOut, stg, 64 * k, h, row0);
          bulk_commit();
        }
      }
    }
    if (tid == 0) bulk_wait_all();  // the stores have read the staging tiles and completed
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
  using K = PCfg<R, UP, GATE>;
  const long long T = a.tokens;
  const int H = a.nheads;
  CUtensorMap tmIn, tmW, tmOut, tmZ;
  memset(&tmZ, 0, sizeof(tmZ));
  if (UP) {
    // u [T, H, P]; Wx [H, R P, P]; x [T, H, R P]
    if (!map3(&tmIn, a.in, kP, H, T, 1, kRows) || !map3(&tmW, a.weight, kP, R * kP, H, R * kP, 1) ||
        !map3(&tmOut, a.out, R * kP, H, T, 1, kRows))
      return MAMBA3_ERR_CUDA;
  } else {
    // y [T, H, R P]; Wy [H, P, R P]; o [T, H, P] (and z [T, H, P])
    if (!map3(&tmIn, a.in, R * kP, H, T, 1, kRows) || !map3(&tmW, a.weight, R * kP, kP, H, kP, 1) ||
        !map3(&tmOut, a.out, kP, H, T, 1, kRows) || (GATE && !map3(&tmZ, a.z, kP, H, T, 1, kRows)))
      return MAMBA3_ERR_CUDA;
  }
  ProjParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.tokens = T;
  prm.nheads = H;
  prm.tiles = (int)((T + kRows - 1) / kRows);
  prm.items = (long long)prm.tiles * H;
  // persistent: two CTAs per SM where both fit (TMEM and shared memory), else one;
  // a CTA that takes all 512 TMEM columns asks for enough shared memory to keep a
  // second one off the SM
  const int per_sm = (K::TMEM_COLS <= 256 && K::SMEM_ALLOC <= 233472 / 2 - 1024) ? 2 : 1;
  const long long grid = prm.items < (long long)kSMs * per_sm ? prm.items : (long long)kSMs * per_sm;
  const int smem = K::TMEM_COLS >= 512 && K::SMEM_ALLOC < 120 * 1024 ? 120 * 1024 : K::SMEM_ALLOC;
  prm.w = a.w;
  prm.eps = a.eps;
  prm.wait_limit = a.wait_limit;
  prm.test_withhold = a.test_withhold;
  auto k = mimo_proj_kernel<R, UP, GATE>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
      cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return MAMBA3_ERR_CUDA;
  k<<<(int)grid, kThreads, smem, s>>>(tmIn, tmW, tmOut, tmZ, prm);
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

// Factor accumulation H += A^T A on the 5th-generation tensor cores.
//
// KronQ README intro / "WaterKron and FlipFlop Hessian" Table 1 ("Marginal"
// row): H_X = sum_t x_t x_t^T and H_G = sum_t g_t g_t^T.  For row-major
// token data A (T x d) this is the GEMM C = A^T A with M = N = d and K = T;
// both operands are read straight from A, so both are MN-major in shared
// memory (d contiguous), which tcgen05 supports for bf16.
//
// Design (sm_100a):
//  * persistent: one CTA per SM walks 128 x 256 output tiles of the upper
//    triangle (tiles entirely below the diagonal are never computed: ~half
//    of the dense work), tile t = blockIdx.x + i * gridDim.x;
//  * warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner), warps 2-5 =
//    epilogue; 4-stage smem ring of 64-token slices (48 KB per stage) that
//    runs across tile boundaries;
//  * tcgen05.mma kind::f16 (bf16 x bf16 -> fp32), M = 128, N = 256, K = 16,
//    two accumulators of 256 TMEM columns: the epilogue of tile i reads one
//    while the MMAs of tile i + 1 fill the other;
//  * epilogue: tcgen05.ld 32x32b, each element written once: (i, j) for
//    i <= j and its mirror (j, i) for i < j, so H stays fully symmetric.
//    Each output element belongs to exactly one tile: no atomics.
//  * tile order: strips of 16 tile rows, column-major inside a strip, so
//    the ~148 tiles in flight at any time span ~2k rows and ~2.4k columns
//    of H and share their token slices in L2 (all tiles have the same K
//    loop, so the CTAs walk the tokens nearly in step).  A row-major order
//    over a wide H makes every concurrent tile read different columns and
//    the kernel DRAM-bound.
//  * from d = 2048 on, the same on SM pairs (syrk_pair_kernel below):
//    256 x 256 tiles, one tcgen05 instruction for two SMs, a third fewer
//    operand bytes per flop and six stages instead of four.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int BOX_BYTES = 64 * BK * 2;                 // one 64-column x 64-token box
constexpr int A_BYTES = BM * BK * 2;                   // 16 KB
constexpr int B_BYTES = BN * BK * 2;                   // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;         // 48 KB
constexpr int NBARS = 2 * STAGES + 4;                  // full, empty, acc_full[2], acc_empty[2]
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
constexpr int THREADS = 192;
constexpr int EPI_WARPS = 4;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int STRIP = 16;                              // tile rows per raster strip
// From this order on the factor is accumulated on SM pairs (256 x 256 tiles)
constexpr int64_t kSyrkPairMinD = 2048;

struct SyrkArgs {
  float* H;
  int64_t d;
  int nk;       // number of 64-token slices
  int nr, nc;   // row / column tile counts
  int ntiles;   // tiles of the upper triangle
  int accumulate;
};

// Tile t of the raster order -> (tile row, tile column).  Tile (tr, tc) is
// kept when it reaches the upper triangle: tc >= tr * BM / BN = tr / 2, i.e.
// tr < 2 tc + 2.  Strips of STRIP tile rows, column-major inside a strip.
__device__ __forceinline__ void tile_of(int t, int nr, int nc, int& tr, int& tc) {
  for (int s0 = 0; s0 < nr; s0 += STRIP) {
    const int s1 = min(s0 + STRIP, nr);
    int cnt = 0;
    for (int r = s0; r < s1; ++r) cnt += nc - r / 2;
    if (t < cnt) {
      for (int c = s0 / 2; c < nc; ++c) {
        const int rend = min(s1, 2 * c + 2);
        const int k = rend - s0;
        if (t < k) {
          tr = s0 + t;
          tc = c;
          return;
        }
        t -= k;
      }
    }
    t -= cnt;
  }
  tr = nr;  // unreachable for t < ntiles
  tc = nc;
}

__global__ void __launch_bounds__(THREADS, 1)
    syrk_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmap, SyrkArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[STAGES]);
  const uint32_t accfull0 = smem_u32(&bars[2 * STAGES]);
  const uint32_t accempty0 = smem_u32(&bars[2 * STAGES + 2]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8 * b, 1);
      mbar_init(accempty0 + 8 * b, EPI_WARPS);
    }
    *abort_s = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t stage0 = smem_u32(smem);
  const int nk = args.nk;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;   // k slices issued, over all tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.ntiles; t += gridDim.x) {
        int tr, tc;
        tile_of(t, args.nr, args.nc, tr, tc);
        const int r0 = tr * BM, c0 = tc * BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (*abort_s || !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          const uint32_t full = full0 + 8 * s;
          mbar_arrive_expect_tx(full, STAGE_BYTES);
          const uint32_t a = stage0 + s * STAGE_BYTES;
          const uint32_t b = a + A_BYTES;
          const int y = kb * BK;
          tma_load_2d(a, &tmap, full, r0, y);
          tma_load_2d(a + BOX_BYTES, &tmap, full, r0 + 64, y);
#pragma unroll
          for (int h = 0; h < 4; ++h) tma_load_2d(b + h * BOX_BYTES, &tmap, full, c0 + 64 * h, y);
        }
      }
      // Make sure no copy is still landing when the CTA leaves (normally
      // these phases completed long ago and each test returns at once).
      for (uint32_t k = it > STAGES ? it - STAGES : 0; k < it; ++k)
        mbar_wait(full0 + 8 * (k % STAGES), (k / STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, true, true);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.ntiles; t += gridDim.x, ++tl) {
        const int b = tl & 1;
        const uint32_t u = (uint32_t)(tl >> 1);
        // the epilogue of tile tl - 2 has read accumulator b
        if (u > 0 && (*abort_s || !mbar_wait(accempty0 + 8 * b, (u - 1) & 1))) {
          *abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * BN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (*abort_s || !mbar_wait(full0 + 8 * s, ph)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = stage0 + s * STAGE_BYTES;
          const uint32_t bb = a + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // 16 tokens = 16 rows of 128 B inside every box: +2048 B per step.
            const uint64_t ad = smem_desc_sw128(a + kk * 2048, BOX_BYTES, 1024);
            const uint64_t bd = smem_desc_sw128(bb + kk * 2048, BOX_BYTES, 1024);
            mma_bf16(acc, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(empty0 + 8 * s);
        }
        if (ok) mma_commit(accfull0 + 8 * b);
      }
    }
    __syncwarp();
  } else {
    // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 (its sub-partition).
    const int q = warp & 3;
    const int64_t d = args.d;
    float* H = args.H;
    const int accm = args.accumulate;
    int tl = 0;
    for (int t = blockIdx.x; t < args.ntiles; t += gridDim.x, ++tl) {
      const int b = tl & 1;
      const uint32_t u = (uint32_t)(tl >> 1);
      int ok = 1;
      if (lane == 0) ok = (!*abort_s && mbar_wait(accfull0 + 8 * b, u & 1)) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) {
        if (lane == 0) *abort_s = 1;
        break;
      }
      tc_fence_after();
      int tr, tc;
      tile_of(t, args.nr, args.nc, tr, tc);
      const int r0 = tr * BM, c0 = tc * BN;
      const int64_t i = r0 + q * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        const int64_t jb = c0 + cc * 32;
        // Every load of the element pair (i, jb..jb+31) / (jb..jb+31, i) is
        // issued before the accumulator is read and before any store, so the
        // read-modify-write costs one memory round trip per 32 columns
        // instead of one per element.
        const bool dense = (i < d) && (jb >= i) && (jb + 32 <= d) &&
                           ((reinterpret_cast<uintptr_t>(H + i * d + jb) & 15) == 0);
        float old[32], mir[32];
        if (accm) {
          if (dense) {
            const float4* src = reinterpret_cast<const float4*>(H + i * d + jb);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 o = src[e];
              old[4 * e] = o.x; old[4 * e + 1] = o.y; old[4 * e + 2] = o.z; old[4 * e + 3] = o.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int64_t j = jb + e;
              old[e] = (i < d && j < d && i <= j) ? H[i * d + j] : 0.f;
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int64_t j = jb + e;
            mir[e] = (i < d && j < d && i < j) ? H[j * d + i] : 0.f;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) old[e] = mir[e] = 0.f;
        }
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)(b * BN + cc * 32), v);
        tmem_wait_ld();
        if (dense) {
          float4* dst = reinterpret_cast<float4*>(H + i * d + jb);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]) + old[4 * e], __uint_as_float(v[4 * e + 1]) + old[4 * e + 1],
                                 __uint_as_float(v[4 * e + 2]) + old[4 * e + 2],
                                 __uint_as_float(v[4 * e + 3]) + old[4 * e + 3]);
        } else if (i < d) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int64_t j = jb + e;
            if (j < d && i <= j) H[i * d + j] = __uint_as_float(v[e]) + old[e];
          }
        }
        // Mirror (j, i) for i < j: 32 lanes write 32 consecutive floats.
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int64_t j = jb + e;
          if (i < d && j < d && i < j) H[j * d + i] = __uint_as_float(v[e]) + mir[e];
        }
      }
      // accumulator b may be refilled once all four warps have read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty0 + 8 * b);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// The same accumulation on SM pairs (tcgen05 cta_group::2): a cluster of
// two CTAs owns 256 x 256 tiles of H's upper triangle (square tiles, tile
// row <= tile column).  Each CTA loads, per 64-token slice, the 128 token
// columns of its half of the tile's rows (A) and of its half of the
// tile's columns (B): 32 KB per stage instead of 48 KB for a 128 x 256
// tile of one SM, so six stages fit and the operand bytes per flop drop by
// a third.  The even CTA's warp 1 issues one M = 256, N = 256, K = 16 MMA
// per 16 tokens for both; each CTA's TMEM holds its 128 rows x 256
// columns (two accumulators of 256 columns, double-buffered across
// tiles), and each CTA's four epilogue warps write its rows.
// Barriers: full[s] in the even CTA (its producer expects both CTAs'
// bytes; both CTAs' TMA loads complete on it), empty[s] and accfull[b] in
// both CTAs (the MMA commits arrive on both), accempty[b] in the even CTA
// (the eight epilogue warps of the pair arrive on it).
constexpr int PM = 256, PN = 256, PH = 128;         // pair tile, per-CTA half
constexpr int P_STAGES = 6;
constexpr int P_BOX = 64 * BK * 2;                  // 8 KB: 64 columns x 64 tokens
constexpr int P_HALF = PH * BK * 2;                 // 16 KB
constexpr int P_STAGE = 2 * P_HALF;                 // 32 KB: A half + B half
constexpr int P_NBARS = 2 * P_STAGES + 5;           // full, empty, accfull[2], accempty[2], done
constexpr int P_SMEM = P_STAGES * P_STAGE + 1024 + 256;
constexpr uint32_t P_TMEM = 2 * PN;
constexpr int P_STRIP = 8;                          // tile rows (of 256) per raster strip
constexpr int64_t kSyrkSplitMinD = 16384;
constexpr int64_t kSyrkSplitT = 8192;

struct SyrkPairArgs {
  float* H;
  int64_t d;
  int nk;
  int nt;        // 256-tiles per side
  int ntiles;    // upper-triangle tiles
  int accumulate;
};

// Upper-triangle tile t (tr <= tc) in strips of P_STRIP tile rows,
// column-major inside a strip.
__device__ __forceinline__ void pair_tile_of(int t, int nt, int& tr, int& tc) {
  for (int s0 = 0; s0 < nt; s0 += P_STRIP) {
    const int s1 = min(s0 + P_STRIP, nt);
    int cnt = 0;
    for (int r = s0; r < s1; ++r) cnt += nt - r;
    if (t < cnt) {
      for (int c = s0; c < nt; ++c) {
        const int k = min(s1, c + 1) - s0;
        if (t < k) {
          tr = s0 + t;
          tc = c;
          return;
        }
        t -= k;
      }
    }
    t -= cnt;
  }
  tr = tc = nt;  // unreachable for t < ntiles
}

__global__ void __launch_bounds__(THREADS, 1)
    syrk_pair_kernel(const __grid_constant__ CUtensorMap tmap, SyrkPairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + P_NBARS);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[P_STAGES]);
  const uint32_t accfull0 = smem_u32(&bars[2 * P_STAGES]);
  const uint32_t accempty0 = smem_u32(&bars[2 * P_STAGES + 2]);
  const uint32_t done = smem_u32(&bars[2 * P_STAGES + 4]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cl_rank();
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8 * b, 1);
      mbar_init(accempty0 + 8 * b, 2 * EPI_WARPS);
    }
    mbar_init(done, 1);
    *abort_s = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), P_TMEM);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cl_sync();   // both CTAs' barriers initialised, both TMEM allocations made
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t stage0 = smem_u32(smem);
  const int nk = args.nk;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_lead = cl_map(full0, 0);   // the even CTA's full barriers
      uint32_t it = 0;
      bool ok = true;
      for (int t = pair; ok && t < args.ntiles; t += npairs) {
        int tr, tc;
        pair_tile_of(t, args.nt, tr, tc);
        const int ra = tr * PM + PH * (int)rank;   // this CTA's rows of the tile (A)
        const int cb = tc * PN + PH * (int)rank;   // this CTA's columns of the tile (B)
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (*abort_s || !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * P_STAGE);
          const uint32_t a = stage0 + s * P_STAGE;
          const uint32_t b = a + P_HALF;
          const uint32_t fb = full_lead + 8 * s;
          const int y = kb * BK;
          tma_load_2d_pair(a, &tmap, fb, ra, y);
          tma_load_2d_pair(a + P_BOX, &tmap, fb, ra + 64, y);
          tma_load_2d_pair(b, &tmap, fb, cb, y);
          tma_load_2d_pair(b + P_BOX, &tmap, fb, cb + 64, y);
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(PM, PN, true, true);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true;
      bool issued = false;
      for (int t = pair; ok && t < args.ntiles; t += npairs, ++tl) {
        const int b = tl & 1;
        const uint32_t u = (uint32_t)(tl >> 1);
        // both CTAs' epilogues have read accumulator b (tile tl - 2)
        if (u > 0 && (*abort_s || !mbar_wait(accempty0 + 8 * b, (u - 1) & 1))) {
          *abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * PN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % P_STAGES;
          const uint32_t ph = (it / P_STAGES) & 1;
          if (*abort_s || !mbar_wait(full0 + 8 * s, ph)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = stage0 + s * P_STAGE;
          const uint32_t bb = a + P_HALF;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(a + kk * 2048, P_BOX, 1024);
            const uint64_t bd = smem_desc_sw128(bb + kk * 2048, P_BOX, 1024);
            mma_bf16_pair(acc, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit_pair_mc(empty0 + 8 * s, 0x3);
        }
        if (ok) mma_commit_pair_mc(accfull0 + 8 * b, 0x3);
      }
      // every MMA issued has completed (they write both CTAs' TMEM) before
      // the pair frees its TMEM
      if (issued) {
        mma_commit_pair_mc(done, 0x1);
        mbar_wait(done, 0);
      }
    }
    __syncwarp();
  } else {
    // Epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 of this CTA: rows
    // ra + 32 (w % 4) + lane of H, the tile's 256 columns.
    const int q = warp & 3;
    const int64_t d = args.d;
    float* H = args.H;
    const int accm = args.accumulate;
    const uint32_t accempty_lead = cl_map(accempty0, 0);
    int tl = 0;
    for (int t = pair; t < args.ntiles; t += npairs, ++tl) {
      const int b = tl & 1;
      const uint32_t u = (uint32_t)(tl >> 1);
      int ok = 1;
      if (lane == 0) ok = (!*abort_s && mbar_wait(accfull0 + 8 * b, u & 1)) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) {
        if (lane == 0) *abort_s = 1;
        break;
      }
      tc_fence_after();
      int tr, tc;
      pair_tile_of(t, args.nt, tr, tc);
      const int64_t i = (int64_t)tr * PM + PH * rank + q * 32 + lane;
      const int64_t c0 = (int64_t)tc * PN;
#pragma unroll 1
      for (int cc = 0; cc < PN / 32; ++cc) {
        const int64_t jb = c0 + cc * 32;
        // 32 columns left of every row of this warp: nothing of them is kept
        // (uniform over the warp, which loads TMEM collectively)
        if (jb + 31 < (int64_t)tr * PM + PH * rank + q * 32) continue;
        // H is symmetric on input (every call leaves both triangles equal):
        // the upper element is read, and it and its mirror get the sum
        const bool dense = (i < d) && (jb >= i) && (jb + 32 <= d) &&
                           ((reinterpret_cast<uintptr_t>(H + i * d + jb) & 15) == 0);
        float old[32];
        if (accm) {
          if (dense) {
            const float4* src = reinterpret_cast<const float4*>(H + i * d + jb);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 o = src[e];
              old[4 * e] = o.x; old[4 * e + 1] = o.y; old[4 * e + 2] = o.z; old[4 * e + 3] = o.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int64_t j = jb + e;
              old[e] = (i < d && j < d && i <= j) ? H[i * d + j] : 0.f;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) old[e] = 0.f;
        }
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)(b * PN + cc * 32), v);
        tmem_wait_ld();
        float sum[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) sum[e] = __uint_as_float(v[e]) + old[e];
        if (dense) {
          float4* dst = reinterpret_cast<float4*>(H + i * d + jb);
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = make_float4(sum[4 * e], sum[4 * e + 1], sum[4 * e + 2], sum[4 * e + 3]);
        } else if (i < d) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int64_t j = jb + e;
            if (j < d && i <= j) H[i * d + j] = sum[e];
          }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int64_t j = jb + e;
          if (i < d && j < d && i < j) H[j * d + i] = sum[e];
        }
      }
      // accumulator b may be refilled once the pair's eight warps have read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(accempty_lead + 8 * b);
    }
  }
  tc_fence_before();
  __syncthreads();
  cl_sync();   // no pair MMA, TMEM read or remote arrive is left in either CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, P_TMEM);
  }
}

__global__ void fill_kernel(float* p, int64_t count, float v) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    p[i] = v;
}


}  // namespace

cudaError_t fill_f32(float* p, int64_t count, float v, cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = ceil_div(count, threads);
  if (blocks > 4 * 148 * 8) blocks = 4 * 148 * 8;
  fill_kernel<<<(unsigned)blocks, threads, 0, s>>>(p, count, v);
  count_launch();
  return cudaGetLastError();
}

cudaError_t status_fetch_syrk(int* out, cudaStream_t s) {
  int v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return e;
  const int zero = 0;
  e = cudaMemcpyToSymbolAsync(g_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(s);
  *out = v;
  return e;
}

kronq_status syrk_bf16_tc(const void* A, int64_t T, int64_t d, int64_t lda, float* H,
                          bool zero_first, cudaStream_t s) {
  // From d = 16384 on, the tokens go in launches of at most 8192: the 256
  // token columns of the ~18 tile rows and columns that a wave of 74 SM
  // pairs touches then take ~72 MB and stay in L2 while the wave runs (at
  // 16384 tokens, ~144 MB do not, and the chunk is read from DRAM ~35
  // times), for one more read-modify-write of H per 8192 tokens.
  if (d >= kSyrkSplitMinD && T > kSyrkSplitT) {
    for (int64_t t0 = 0; t0 < T; t0 += kSyrkSplitT) {
      const int64_t tn = (T - t0) < kSyrkSplitT ? (T - t0) : kSyrkSplitT;
      kronq_status r = syrk_bf16_tc(static_cast<const __nv_bfloat16*>(A) + t0 * lda, tn, d, lda, H,
                                    zero_first && t0 == 0, s);
      if (r != KRONQ_OK) return r;
    }
    return KRONQ_OK;
  }
  auto encode = tma_encode_fn();
  if (!encode) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)d, (cuuint64_t)T};
  cuuint64_t gstride[1] = {(cuuint64_t)(lda * 2)};
  cuuint32_t box[2] = {64, (cuuint32_t)BK};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), gdim, gstride,
                      box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed");

  SyrkArgs args;
  args.H = H;
  args.d = d;
  args.nk = (int)ceil_div(T, BK);
  args.nr = (int)ceil_div(d, BM);
  args.nc = (int)ceil_div(d, BN);
  args.accumulate = zero_first ? 0 : 1;
  int64_t ntiles = 0;
  for (int tr = 0; tr < args.nr; ++tr) ntiles += args.nc - (tr * BM) / BN;
  args.ntiles = (int)ntiles;

  if (d >= kSyrkPairMinD) {
    // SM pairs: 256 x 256 tiles, as many clusters of two as fit at once
    SyrkPairArgs pa;
    pa.H = H;
    pa.d = d;
    pa.nk = args.nk;
    pa.nt = (int)ceil_div(d, PM);
    pa.ntiles = pa.nt * (pa.nt + 1) / 2;
    pa.accumulate = args.accumulate;
    const void* fn = reinterpret_cast<const void*>(&syrk_pair_kernel);
    cudaError_t e = allow_smem(fn, P_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(syrk pair)");
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)P_SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(2 * (sm_count() / 2)));
    int active = 0;
    e = cudaOccupancyMaxActiveClusters(&active, fn, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(syrk pair)");
    if (active >= 1) {
      const int64_t npairs = pa.ntiles < (int64_t)active ? pa.ntiles : (int64_t)active;
      cfg.gridDim = dim3((unsigned)(2 * npairs));
      e = cudaLaunchKernelEx(&cfg, syrk_pair_kernel, map, pa);
      count_launch();
      if (e != cudaSuccess) return cuda_fail(e, "syrk_pair_kernel");
      return KRONQ_OK;
    }
  }
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&syrk_bf16_tc_kernel), SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(syrk)");
  const int64_t grid = ntiles < (int64_t)sm_count() ? ntiles : (int64_t)sm_count();
  syrk_bf16_tc_kernel<<<(unsigned)grid, THREADS, SMEM_BYTES, s>>>(map, args);
  KQ_LAUNCH_CHECK("syrk_bf16_tc_kernel");
  return KRONQ_OK;
}

}  // namespace kq

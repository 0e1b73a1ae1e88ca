// One 128 x 128 tile of the Schur-complement update of the blocked reverse
// Cholesky, on the tensor cores:
//   A[r0:r0+128, c0:c0+128] -= R_p[r0:] R_p[c0:]^T   (entries i <= j < j0 only)
// where R_p is the current 64-column panel, given as three bf16 splits
// (x = hi + mid + lo, each the bf16 rounding of the remainder) whose six
// products hh + hm + mh + hl + lh + mm keep float32-level accuracy.
//
// Roles inside the CTA: warp 0 lane 0 issues the TMA loads (the fp32 tile
// of A into shared memory when tma_c, and the splits of both panel row
// ranges), warp 1 lane 0 the 24 tcgen05.mma (M 128, N 128, K 16) into 128
// TMEM columns, four or eight epilogue warps subtract the accumulator from
// the staged tile and write it back with TMA stores (or read-modify-write
// global memory directly when the rows are not 16-byte aligned).  Used by
// the per-step Schur kernel and by the persistent factorisation kernel.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace kq {
namespace schur {

constexpr int BM = 128, BN = 128, KP = 64;
constexpr int P_BOX = BM * KP * 2;            // 16 KB: 128 panel rows x 64 k, one split
constexpr int C_BOX = BM * 32 * 4;            // 16 KB: 128 rows x 32 fp32 (128-byte swizzle)
constexpr int C_BYTES = (BN / 32) * C_BOX;    // 64 KB
constexpr int TILE_SMEM = 6 * P_BOX + C_BYTES;  // 160 KB, 1024-byte aligned base
constexpr uint32_t TMEM_COLS = BN;

struct TileMaps {
  const CUtensorMap* pH;
  const CUtensorMap* pM;
  const CUtensorMap* pL;
  const CUtensorMap* mC;
};

// Processes one tile; every thread of the CTA calls it.  Entries i <= j < j0
// with i < rowlim (default j0) are updated (j0 a multiple of 32).  Warp 0 lane 0
// issues the TMA loads, warp 1 lane 0 the MMAs; warps EPI_W0 .. EPI_W0+NW-1
// (NW = 4 or 8; the role warps may be among them) run the epilogue, warp w
// on TMEM lanes 32 (w % 4) and, with eight warps, on half of the columns.
// parity: the phase parity of this CTA's barriers for this tile (the tile
// count modulo 2).  store_done: 1 waits until the TMA store has reached
// global memory, 0 only until it has read shared memory (the issuing thread,
// EPI_W0 * 32, must then wait with tma_store_wait_all before publishing).
// Returns false on a barrier timeout (the device status word is set).  The
// caller puts a CTA barrier between tiles.
template <int EPI_W0, int NW>
__device__ __forceinline__ bool tile(uint8_t* smem, uint32_t full, uint32_t cbar, uint32_t accbar,
                                     uint32_t parity, uint32_t tmem, const TileMaps& mp, float* H,
                                     int64_t n, int64_t j0, int64_t r0, int64_t c0, int tma_c,
                                     int store_done = 1, int64_t rowlim = -1) {
  static_assert(NW == 4 || NW == 8, "four or eight epilogue warps");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base = smem_u32(smem);
  const uint32_t sa[3] = {base, base + P_BOX, base + 2 * P_BOX};
  const uint32_t sb[3] = {base + 3 * P_BOX, base + 4 * P_BOX, base + 5 * P_BOX};
  const uint32_t cs = base + 6 * P_BOX;
  bool ok = true;
  if (warp == 0 && lane == 0) {
    if (tma_c) {
      mbar_arrive_expect_tx(cbar, C_BYTES);
#pragma unroll
      for (int h = 0; h < BN / 32; ++h) tma_load_2d(cs + h * C_BOX, mp.mC, cbar, (int)(c0 + 32 * h), (int)r0);
    }
    mbar_arrive_expect_tx(full, 6 * P_BOX);
    tma_load_2d(sa[0], mp.pH, full, 0, (int)r0);
    tma_load_2d(sa[1], mp.pM, full, 0, (int)r0);
    tma_load_2d(sa[2], mp.pL, full, 0, (int)r0);
    tma_load_2d(sb[0], mp.pH, full, 0, (int)c0);
    tma_load_2d(sb[1], mp.pM, full, 0, (int)c0);
    tma_load_2d(sb[2], mp.pL, full, 0, (int)c0);
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
    ok = mbar_wait(full, parity);
    if (ok) {
      tc_fence_after();
      // split pairs (a, b) with a + b <= 2: hh, hm, mh, hl, lh, mm
      const int pa[6] = {0, 0, 1, 0, 2, 1};
      const int pb[6] = {0, 1, 0, 2, 0, 1};
      uint32_t acc = 0;
#pragma unroll
      for (int kk = 0; kk < KP / 16; ++kk) {
#pragma unroll
        for (int t = 0; t < 6; ++t) {
          const uint64_t da = smem_desc_sw128(sa[pa[t]] + kk * 32, 16, 1024);
          const uint64_t db = smem_desc_sw128(sb[pb[t]] + kk * 32, 16, 1024);
          mma_bf16(tmem, da, db, idesc, acc);
          acc = 1;
        }
      }
    }
    mma_commit(accbar);
  }
  __syncwarp();
  if (warp >= EPI_W0 && warp < EPI_W0 + NW) {
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    constexpr int NCH = (BN / 32) * 4 / NW;        // 32-column chunks per warp
    const int ch0 = (NW == 8) ? ((warp - EPI_W0) >> 2) * NCH : 0;
    int good = 1;
    if (lane == 0) {
      good = mbar_wait(accbar, parity) ? 1 : 0;
      if (good && tma_c) good = mbar_wait(cbar, parity) ? 1 : 0;
    }
    good = __shfl_sync(0xffffffffu, good, 0);
    ok = ok && good != 0;
    __syncwarp();
    if (good) {
      tc_fence_after();
      const int i = (int)(r0 + rl);
      const int j0i = (int)j0;
      const int rlim = (int)(rowlim < 0 ? j0 : rowlim);
      // every entry of a tile strictly above the diagonal, left of j0 and
      // above the row limit is updated
      const bool interior = (r0 + BM <= c0) && (c0 + BN <= j0) && (r0 + BM <= rlim);
#pragma unroll 1
      for (int cc = ch0; cc < ch0 + NCH; ++cc) {
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + cc * 32, v);
        tmem_wait_ld();
        const int jb = (int)c0 + cc * 32;
        if (tma_c) {
          uint8_t* box = smem + 6 * P_BOX + cc * C_BOX;
          if (interior) {
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              float4* p4 = reinterpret_cast<float4*>(box + sw128_f32(rl, 4 * c4));
              float4 w = *p4;
              w.x -= __uint_as_float(v[4 * c4]);
              w.y -= __uint_as_float(v[4 * c4 + 1]);
              w.z -= __uint_as_float(v[4 * c4 + 2]);
              w.w -= __uint_as_float(v[4 * c4 + 3]);
              *p4 = w;
            }
          } else {
            const bool rowok = i < rlim;
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              float4* p4 = reinterpret_cast<float4*>(box + sw128_f32(rl, 4 * c4));
              float4 w = *p4;
              const int j = jb + 4 * c4;
              if (rowok && j + 0 < j0i && j + 0 >= i) w.x -= __uint_as_float(v[4 * c4]);
              if (rowok && j + 1 < j0i && j + 1 >= i) w.y -= __uint_as_float(v[4 * c4 + 1]);
              if (rowok && j + 2 < j0i && j + 2 >= i) w.z -= __uint_as_float(v[4 * c4 + 2]);
              if (rowok && j + 3 < j0i && j + 3 >= i) w.w -= __uint_as_float(v[4 * c4 + 3]);
              *p4 = w;
            }
          }
        } else if (i < rlim && jb < j0i && jb + 31 >= i) {
          float* row = H + (int64_t)i * n + jb;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int j = jb + t;
            if (j < j0i && j >= i) row[t] -= __uint_as_float(v[t]);
          }
        }
      }
      if (tma_c) fence_proxy_async_smem();
    }
    if (tma_c) {
      named_barrier(1, NW * 32);            // the epilogue warps, each exactly once
      if (ok && warp == EPI_W0 && lane == 0) {
        // only the 32-column boxes left of j0: the columns from j0 on may
        // belong to a block that another CTA is writing
#pragma unroll
        for (int h = 0; h < BN / 32; ++h)
          if (c0 + 32 * h < j0) tma_store_2d(mp.mC, cs + h * C_BOX, (int)(c0 + 32 * h), (int)r0);
        tma_store_commit();
        if (store_done) tma_store_wait_all();
        else tma_store_wait_read();
      }
    }
  }
  return ok;
}

}  // namespace schur
}  // namespace kq

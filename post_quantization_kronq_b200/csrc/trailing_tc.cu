// Lazy-batch trailing updates of the column sweep on the tensor cores:
//   W[:, cols] -= E_grp[:, k0 : k0 + K] U_grp[k0 : k0 + K, cols]
// (GPTQ's block error feedback, which KronQ's sweep keeps; KronQ README intro),
// where E_grp / U_grp hold the scaled errors and the rows of U of the blocks of
// the current group (up to eight 128-column blocks, K up to 1024).
//
// To keep float32-level accuracy with bf16 MMAs both operands are split,
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi), and the product is
// E_hi U_hi + E_hi U_lo + E_lo U_hi (the dropped lo*lo term is ~2^-16
// relative), accumulated in fp32 in TMEM.
//
// One CTA per 128 x 128 tile of W[:, cols]: warp 0 lane 0 streams 64-deep k
// chunks (E_hi/E_lo K-major, U_hi/U_lo MN-major) through a two-stage ring and
// the fp32 W tile into shared memory, warp 1 lane 0 issues 12 tcgen05.mma
// (M 128, N 128, K 16) per chunk into 128 TMEM columns, then all eight warps
// subtract the accumulator from the staged tile (128-byte swizzled boxes,
// conflict-free float4 accesses) and one thread writes it back with TMA
// stores.  Each element is owned by one CTA.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BM = 128, BN = 128, KC = 64, NSTAGE = 2;
// The group-end updates (K of a whole group) run on SM pairs
constexpr int64_t kTrailPairMinK = 512;
constexpr int A_BOX = BM * KC * 2;         // 16 KB: 128 rows x 64 k (K-major, 128 B rows)
constexpr int B_BOX = 64 * KC * 2;         // 8 KB: 64 k rows x 64 columns (MN-major)
constexpr int B_SPLIT = (BN / 64) * B_BOX; // 16 KB: one split of the B chunk
constexpr int CHUNK_BYTES = 2 * A_BOX + 2 * B_SPLIT;   // hi+lo of A and B: 64 KB per stage
constexpr int C_BOX = BM * 32 * 4;         // 16 KB: 128 rows x 32 fp32 (128-byte swizzle)
constexpr int C_BYTES = (BN / 32) * C_BOX; // 64 KB
constexpr int SMEM_BYTES = NSTAGE * CHUNK_BYTES + C_BYTES + 1024 + 256;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = BN;

struct TrailArgs {
  float* W;       // full W~ (row stride n)
  int64_t m, n;
  int64_t c_begin;  // first column to update
  int k0;         // first k row of the group buffers
  int nkc;        // 64-deep k chunks
  int tma_c;      // 1: W tile staged through shared memory by TMA
  const int* info;
};

__global__ void __launch_bounds__(THREADS, 1)
    trailing_tc_kernel(const __grid_constant__ CUtensorMap mEh, const __grid_constant__ CUtensorMap mEl,
                       const __grid_constant__ CUtensorMap mUh, const __grid_constant__ CUtensorMap mUl,
                       const __grid_constant__ CUtensorMap mW, TrailArgs args) {
  if (args.info && *args.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTAGE * CHUNK_BYTES + C_BYTES);
  // full[2], free[2], cbar, accbar
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NSTAGE + 2);
  const uint32_t cbar = smem_u32(&bars[2 * NSTAGE]);
  const uint32_t accbar = smem_u32(&bars[2 * NSTAGE + 1]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = (int64_t)blockIdx.y * BM;
  const int64_t c0 = args.c_begin + (int64_t)blockIdx.x * BN;

  if (threadIdx.x == 0) {
    for (int st = 0; st < NSTAGE; ++st) {
      mbar_init(smem_u32(&bars[st]), 1);
      mbar_init(smem_u32(&bars[NSTAGE + st]), 1);
    }
    mbar_init(cbar, 1);
    mbar_init(accbar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t base = smem_u32(smem);
  const uint32_t cs = base + NSTAGE * CHUNK_BYTES;   // staged W tile

  if (warp == 0 && lane == 0) {
    if (args.tma_c) {
      mbar_arrive_expect_tx(cbar, C_BYTES);
#pragma unroll
      for (int h = 0; h < BN / 32; ++h) tma_load_2d(cs + h * C_BOX, &mW, cbar, (int)(c0 + 32 * h), (int)r0);
    }
    for (int c = 0; c < args.nkc; ++c) {
      const int st = c & 1;
      const uint32_t full = smem_u32(&bars[st]);
      // stage st is free once the MMAs of chunk c - 2 have read it
      if (c >= NSTAGE && !mbar_wait(smem_u32(&bars[NSTAGE + st]), (uint32_t)(((c - NSTAGE) >> 1) & 1))) break;
      const uint32_t s = base + st * CHUNK_BYTES;
      const int k = args.k0 + c * KC;
      mbar_arrive_expect_tx(full, CHUNK_BYTES);
      tma_load_2d(s, &mEh, full, k, (int)r0);
      tma_load_2d(s + A_BOX, &mEl, full, k, (int)r0);
#pragma unroll
      for (int h = 0; h < BN / 64; ++h) {
        tma_load_2d(s + 2 * A_BOX + h * B_BOX, &mUh, full, (int)(c0 + 64 * h), k);
        tma_load_2d(s + 2 * A_BOX + B_SPLIT + h * B_BOX, &mUl, full, (int)(c0 + 64 * h), k);
      }
    }
  } else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, true);
    uint32_t acc = 0;
    for (int c = 0; c < args.nkc; ++c) {
      const int st = c & 1;
      if (!mbar_wait(smem_u32(&bars[st]), (uint32_t)((c >> 1) & 1))) break;
      tc_fence_after();
      const uint32_t s = base + st * CHUNK_BYTES;
      const uint32_t ah = s, al = s + A_BOX;
      const uint32_t bh = s + 2 * A_BOX, bl = s + 2 * A_BOX + B_SPLIT;
#pragma unroll
      for (int kk = 0; kk < KC / 16; ++kk) {
        // A K-major: 16 k = 32 bytes along each 128-byte row.  B MN-major:
        // 16 k rows of 128 bytes = 2048 bytes inside every 64-column box.
        const uint64_t dah = smem_desc_sw128(ah + kk * 32, 16, 1024);
        const uint64_t dal = smem_desc_sw128(al + kk * 32, 16, 1024);
        const uint64_t dbh = smem_desc_sw128(bh + kk * 2048, B_BOX, 1024);
        const uint64_t dbl = smem_desc_sw128(bl + kk * 2048, B_BOX, 1024);
        mma_bf16(tmem, dah, dbh, idesc, acc);
        acc = 1;
        mma_bf16(tmem, dah, dbl, idesc, 1u);
        mma_bf16(tmem, dal, dbh, idesc, 1u);
      }
      mma_commit(smem_u32(&bars[NSTAGE + st]));   // stage st may be refilled
    }
    mma_commit(accbar);
  }
  __syncwarp();
  {
    // epilogue, all eight warps: warp w takes TMEM lanes 32 (w % 4) and the
    // columns 64 (w / 4) .. +63 of the tile
    const int q = warp & 3, half = warp >> 2;
    const int rl = q * 32 + lane;          // row of the tile
    int good = 1;
    if (lane == 0) {
      good = mbar_wait(accbar, 0) ? 1 : 0;
      if (good && args.tma_c) good = mbar_wait(cbar, 0) ? 1 : 0;
    }
    good = __shfl_sync(0xffffffffu, good, 0);
    __syncwarp();
    if (good) {
      tc_fence_after();
      const int64_t i = r0 + rl;
      const int64_t n = args.n;
#pragma unroll 1
      for (int cc = 2 * half; cc < 2 * half + 2; ++cc) {
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + cc * 32, v);
        tmem_wait_ld();
        if (args.tma_c) {
          uint8_t* box = smem + NSTAGE * CHUNK_BYTES + cc * C_BOX;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            float4* p4 = reinterpret_cast<float4*>(box + sw128_f32(rl, 4 * ch));
            float4 w = *p4;
            w.x -= __uint_as_float(v[4 * ch]);
            w.y -= __uint_as_float(v[4 * ch + 1]);
            w.z -= __uint_as_float(v[4 * ch + 2]);
            w.w -= __uint_as_float(v[4 * ch + 3]);
            *p4 = w;
          }
        } else {
          const int64_t jb = c0 + cc * 32;
          if (i < args.m && jb < n) {
            float* row = args.W + i * n + jb;
#pragma unroll
            for (int t = 0; t < 32; ++t)
              if (jb + t < n) row[t] -= __uint_as_float(v[t]);
          }
        }
      }
      if (args.tma_c) fence_proxy_async_smem();
    }
    if (args.tma_c) {
      __syncthreads();
      if (good && warp == 0 && lane == 0) {
#pragma unroll
        for (int h = 0; h < BN / 32; ++h) tma_store_2d(&mW, cs + h * C_BOX, (int)(c0 + 32 * h), (int)r0);
        tma_store_commit();
        tma_store_wait_read();  // shared memory read; the writes finish on their own
      }
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
// The same update on SM pairs (tcgen05 cta_group::2), persistent: a cluster
// of two CTAs walks 256 x 256 tiles of W[:, cols] (column-major over the
// tiles, so the pairs in flight share U's columns while E, small, stays in
// L2).  Per 64-deep k chunk each CTA loads its 128 rows of E hi/lo and its
// 128 columns of U hi/lo (64 KB; three stages), the even CTA issues the
// three split products for both (M = 256, N = 256, K = 16, 12 MMAs per
// chunk) into one of two 256-column TMEM accumulators, and each CTA's four
// epilogue warps subtract their 128 rows from W in place (rows of 32
// columns at a time, loads before stores) while the next tile's MMAs run.
// Barriers as in the pair factor accumulation.
constexpr int TP_M = 256, TP_N = 256, TP_H = 128;
constexpr int TP_STAGES = 3;
constexpr int TP_ABOX = TP_H * KC * 2;              // 16 KB: 128 rows x 64 k (K-major)
constexpr int TP_BBOX = 64 * KC * 2;                // 8 KB: 64 columns x 64 k (MN-major)
constexpr int TP_STAGE = 2 * TP_ABOX + 4 * TP_BBOX; // 64 KB: E hi, E lo, U hi (2 boxes), U lo (2 boxes)
constexpr int TP_NBARS = 2 * TP_STAGES + 5;
constexpr int TP_SMEM = TP_STAGES * TP_STAGE + 1024 + 256;
constexpr int TP_THREADS = 192;
constexpr int TP_EPI = 4;
constexpr uint32_t TP_TMEM = 2 * TP_N;

struct TrailPairArgs {
  float* W;
  int64_t m, n;
  int64_t c_begin, c_end;   // the columns updated: [c_begin, c_end)
  int k0;
  int nkc;
  int tiles_m, tiles_n, ntiles;
  const int* info;
};

__global__ void __launch_bounds__(TP_THREADS, 1)
    trailing_pair_kernel(const __grid_constant__ CUtensorMap mEh, const __grid_constant__ CUtensorMap mEl,
                         const __grid_constant__ CUtensorMap mUh, const __grid_constant__ CUtensorMap mUl,
                         TrailPairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TP_STAGES * TP_STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + TP_NBARS);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[TP_STAGES]);
  const uint32_t accfull0 = smem_u32(&bars[2 * TP_STAGES]);
  const uint32_t accempty0 = smem_u32(&bars[2 * TP_STAGES + 2]);
  const uint32_t done = smem_u32(&bars[2 * TP_STAGES + 4]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cl_rank();
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  // a failed factorisation leaves nothing to update (uniform over the grid)
  const bool skip = args.info && *args.info != 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < TP_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8 * b, 1);
      mbar_init(accempty0 + 8 * b, 2 * TP_EPI);
    }
    mbar_init(done, 1);
    *abort_s = skip ? 1 : 0;
    fence_mbar_init();
    prefetch_tmap(&mEh);
    prefetch_tmap(&mEl);
    prefetch_tmap(&mUh);
    prefetch_tmap(&mUl);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TP_TMEM);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cl_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t stage0 = smem_u32(smem);
  const int nkc = args.nkc;
  const int ntiles = skip ? 0 : args.ntiles;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_lead = cl_map(full0, 0);
      uint32_t it = 0;
      bool ok = true;
      for (int t = pair; ok && t < ntiles; t += npairs) {
        const int tm = t % args.tiles_m, tn = t / args.tiles_m;   // column-major over the tiles
        const int ra = tm * TP_M + TP_H * (int)rank;
        const int cb = (int)args.c_begin + tn * TP_N + TP_H * (int)rank;
        for (int c = 0; c < nkc; ++c, ++it) {
          const uint32_t s = it % TP_STAGES;
          const uint32_t ph = (it / TP_STAGES) & 1;
          if (*abort_s || !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full0 + 8 * s, 2 * TP_STAGE);
          const uint32_t st = stage0 + s * TP_STAGE;
          const uint32_t fb = full_lead + 8 * s;
          const int k = args.k0 + c * KC;
          tma_load_2d_pair(st, &mEh, fb, k, ra);
          tma_load_2d_pair(st + TP_ABOX, &mEl, fb, k, ra);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_2d_pair(st + 2 * TP_ABOX + h * TP_BBOX, &mUh, fb, cb + 64 * h, k);
            tma_load_2d_pair(st + 2 * TP_ABOX + 2 * TP_BBOX + h * TP_BBOX, &mUl, fb, cb + 64 * h, k);
          }
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(TP_M, TP_N, false, true);
      uint32_t it = 0;
      int tl = 0;
      bool ok = true, issued = false;
      for (int t = pair; ok && t < ntiles; t += npairs, ++tl) {
        const int b = tl & 1;
        const uint32_t u = (uint32_t)(tl >> 1);
        if (u > 0 && (*abort_s || !mbar_wait(accempty0 + 8 * b, (u - 1) & 1))) {
          *abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(b * TP_N);
        for (int c = 0; c < nkc; ++c, ++it) {
          const uint32_t s = it % TP_STAGES;
          const uint32_t ph = (it / TP_STAGES) & 1;
          if (*abort_s || !mbar_wait(full0 + 8 * s, ph)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = stage0 + s * TP_STAGE;
          const uint32_t ah = st, al = st + TP_ABOX;
          const uint32_t bh = st + 2 * TP_ABOX, bl = st + 2 * TP_ABOX + 2 * TP_BBOX;
#pragma unroll
          for (int kk = 0; kk < KC / 16; ++kk) {
            // A K-major: 16 k = 32 bytes along each 128-byte row.  B MN-major:
            // 16 k rows of 128 bytes = 2048 bytes inside every 64-column box.
            const uint64_t dah = smem_desc_sw128(ah + kk * 32, 16, 1024);
            const uint64_t dal = smem_desc_sw128(al + kk * 32, 16, 1024);
            const uint64_t dbh = smem_desc_sw128(bh + kk * 2048, TP_BBOX, 1024);
            const uint64_t dbl = smem_desc_sw128(bl + kk * 2048, TP_BBOX, 1024);
            mma_bf16_pair(acc, dah, dbh, idesc, (c | kk) != 0 ? 1u : 0u);
            mma_bf16_pair(acc, dah, dbl, idesc, 1u);
            mma_bf16_pair(acc, dal, dbh, idesc, 1u);
          }
          issued = true;
          mma_commit_pair_mc(empty0 + 8 * s, 0x3);
        }
        if (ok) mma_commit_pair_mc(accfull0 + 8 * b, 0x3);
      }
      if (issued) {
        mma_commit_pair_mc(done, 0x1);
        mbar_wait(done, 0);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3;
    const int64_t n = args.n;
    float* W = args.W;
    const uint32_t accempty_lead = cl_map(accempty0, 0);
    int tl = 0;
    for (int t = pair; t < ntiles; t += npairs, ++tl) {
      const int b = tl & 1;
      const uint32_t u = (uint32_t)(tl >> 1);
      int good = 1;
      if (lane == 0) good = (!*abort_s && mbar_wait(accfull0 + 8 * b, u & 1)) ? 1 : 0;
      good = __shfl_sync(0xffffffffu, good, 0);
      __syncwarp();
      if (!good) {
        if (lane == 0) *abort_s = 1;
        break;
      }
      tc_fence_after();
      const int tm = t % args.tiles_m, tn = t / args.tiles_m;
      const int64_t i = (int64_t)tm * TP_M + TP_H * rank + q * 32 + lane;
      const int64_t c0 = args.c_begin + (int64_t)tn * TP_N;
#pragma unroll 1
      for (int cc = 0; cc < TP_N / 32; ++cc) {
        const int64_t jb = c0 + cc * 32;
        if (jb >= args.c_end) break;   // uniform over the warp
        const bool dense = (i < args.m) && (jb + 32 <= args.c_end) &&
                           ((reinterpret_cast<uintptr_t>(W + i * n + jb) & 15) == 0);
        float old[32];
        if (dense) {
          const float4* src = reinterpret_cast<const float4*>(W + i * n + jb);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 o = src[e];
            old[4 * e] = o.x; old[4 * e + 1] = o.y; old[4 * e + 2] = o.z; old[4 * e + 3] = o.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            old[e] = (i < args.m && jb + e < args.c_end) ? W[i * n + jb + e] : 0.f;
        }
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + (uint32_t)(b * TP_N + cc * 32), v);
        tmem_wait_ld();
        if (dense) {
          float4* dst = reinterpret_cast<float4*>(W + i * n + jb);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(old[4 * e] - __uint_as_float(v[4 * e]), old[4 * e + 1] - __uint_as_float(v[4 * e + 1]),
                                 old[4 * e + 2] - __uint_as_float(v[4 * e + 2]),
                                 old[4 * e + 3] - __uint_as_float(v[4 * e + 3]));
        } else if (i < args.m) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (jb + e < args.c_end) W[i * n + jb + e] = old[e] - __uint_as_float(v[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(accempty_lead + 8 * b);
    }
  }
  tc_fence_before();
  __syncthreads();
  cl_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TP_TMEM);
  }
}

}  // namespace

cudaError_t status_fetch_trailing(int* out, cudaStream_t s) {
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

kronq_status trailing_maps(TrailingMaps* tm, const void* Eh, const void* El, int64_t m, int64_t lde,
                           const void* Uh, const void* Ul, int64_t ku, int64_t ldu, float* W, int64_t n) {
  static_assert(sizeof(tm->raw) == 5 * sizeof(CUtensorMap), "map storage");
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(tm->raw);
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  // E hi/lo: m rows x lde k, K-major boxes of 64 k x 128 rows.
  // U hi/lo: ku k rows x n columns (row stride ldu), boxes of 64 columns x 64 k.
  if (!tma_map_2d(&maps[0], bf, 2, Eh, lde, m, lde, 64, BM) || !tma_map_2d(&maps[1], bf, 2, El, lde, m, lde, 64, BM) ||
      !tma_map_2d(&maps[2], bf, 2, Uh, n, ku, ldu, 64, KC) || !tma_map_2d(&maps[3], bf, 2, Ul, n, ku, ldu, 64, KC))
    return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (trailing update)");
  // W tile staging (fp32, 32-column boxes): needs a 16-byte row stride.
  tm->tma_c = ((n % 4) == 0 && aligned(W, 16)) ? 1 : 0;
  if (tm->tma_c && !tma_map_2d(&maps[4], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, W, n, m, n, 32, BM))
    return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (trailing update, W)");
  return KRONQ_OK;
}

kronq_status trailing_update_tc(const TrailingMaps* tm, float* W, int64_t m, int64_t n, int64_t c_begin,
                                int64_t ncols, int64_t k0, int64_t K, const int* info, cudaStream_t s) {
  if (ncols <= 0 || K <= 0) return KRONQ_OK;
  const CUtensorMap* maps = reinterpret_cast<const CUtensorMap*>(tm->raw);
  if (K >= kTrailPairMinK && m >= TP_M) {
    // SM pairs, persistent over 256 x 256 tiles
    TrailPairArgs pa;
    pa.W = W;
    pa.m = m;
    pa.n = n;
    pa.c_begin = c_begin;
    pa.c_end = c_begin + ncols;
    pa.k0 = (int)k0;
    pa.nkc = (int)((K + KC - 1) / KC);
    pa.tiles_m = (int)ceil_div(m, TP_M);
    pa.tiles_n = (int)ceil_div(ncols, TP_N);
    pa.ntiles = pa.tiles_m * pa.tiles_n;
    pa.info = info;
    const void* fn = reinterpret_cast<const void*>(&trailing_pair_kernel);
    cudaError_t e = allow_smem(fn, TP_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(trailing pair)");
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(TP_THREADS);
    cfg.dynamicSmemBytes = (size_t)TP_SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3((unsigned)(2 * (sm_count() / 2)));
    int active = 0;
    e = cudaOccupancyMaxActiveClusters(&active, fn, &cfg);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(trailing pair)");
    if (active >= 1) {
      const int64_t npairs = pa.ntiles < (int64_t)active ? pa.ntiles : (int64_t)active;
      cfg.gridDim = dim3((unsigned)(2 * npairs));
      e = cudaLaunchKernelEx(&cfg, trailing_pair_kernel, maps[0], maps[1], maps[2], maps[3], pa);
      count_launch();
      if (e != cudaSuccess) return cuda_fail(e, "trailing_pair_kernel");
      return KRONQ_OK;
    }
  }
  TrailArgs a;
  a.W = W;
  a.m = m;
  a.n = n;
  a.c_begin = c_begin;
  a.k0 = (int)k0;
  a.nkc = (int)((K + KC - 1) / KC);
  a.tma_c = tm->tma_c;
  a.info = info;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&trailing_tc_kernel), SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(trailing)");
  dim3 grid((unsigned)ceil_div(ncols, BN), (unsigned)ceil_div(m, BM));
  trailing_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], a);
  KQ_LAUNCH_CHECK("trailing_tc_kernel");
  return KRONQ_OK;
}

}  // namespace kq

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

// Schur-complement update of the blocked reverse Cholesky on the tensor
// cores:  A[0:j0, 0:j0] -= R_p R_p^T  (upper triangle only),
// where R_p = R[0:j0, J] is the just-solved 64-column panel.
//
// Float32-level accuracy from bf16 MMAs: the panel is split three ways,
// x = hi + mid + lo (each a bf16 rounding of the remainder), and the product
// keeps the six terms down to 2^-24 relative: hh + hm + mh + hl + lh + mm.
// The panel kernel writes the three splits (j0 x 64, row-major, K-major for
// both operands).  One CTA per 128 x 128 tile of the upper triangle: warp 0
// issues the TMA loads (the fp32 tile of A into shared memory, the splits of
// the two panel row ranges), warp 1 the 24 tcgen05.mma (M 128, N 128, K 16)
// into 128 TMEM columns, warps 2-5 subtract the accumulator from the staged
// tile (i <= j only) and write it back with TMA stores.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BM = 128, BN = 128, KP = 64;
constexpr int P_BOX = BM * KP * 2;           // 16 KB: 128 panel rows x 64 k, one split
constexpr int C_BOX = BM * 32 * 4;           // 16 KB: 128 rows x 32 fp32 (128-byte swizzle)
constexpr int C_BYTES = (BN / 32) * C_BOX;   // 64 KB
constexpr int SMEM_BYTES = 6 * P_BOX + C_BYTES + 1024 + 256;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = BN;

struct SchurArgs {
  float* H;
  int64_t n, j0;
  int nt;         // tiles per side
  int tma_c;      // 1: H tile staged through shared memory by TMA
  const int* info;
};

// t-th tile (row-major over tr <= tc) of the upper triangle of nt x nt tiles.
__device__ __forceinline__ void tile_of(int t, int nt, int& tr, int& tc) {
  for (tr = 0; tr < nt; ++tr) {
    const int cnt = nt - tr;
    if (t < cnt) {
      tc = tr + t;
      return;
    }
    t -= cnt;
  }
  tc = nt;
}

__global__ void __launch_bounds__(THREADS, 1)
    schur_tc_kernel(const __grid_constant__ CUtensorMap pH, const __grid_constant__ CUtensorMap pM,
                    const __grid_constant__ CUtensorMap pL, const __grid_constant__ CUtensorMap mC,
                    SchurArgs args) {
  if (args.info && *args.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * P_BOX + C_BYTES);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  const uint32_t full = smem_u32(&bars[0]);
  const uint32_t cbar = smem_u32(&bars[1]);
  const uint32_t accbar = smem_u32(&bars[2]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int tr, tc;
  tile_of(blockIdx.x, args.nt, tr, tc);
  const int64_t r0 = (int64_t)tr * BM, c0 = (int64_t)tc * BN;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
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
  const uint32_t sa[3] = {base, base + P_BOX, base + 2 * P_BOX};
  const uint32_t sb[3] = {base + 3 * P_BOX, base + 4 * P_BOX, base + 5 * P_BOX};
  const uint32_t cs = base + 6 * P_BOX;

  if (warp == 0) {
    if (lane == 0) {
      if (args.tma_c) {
        mbar_arrive_expect_tx(cbar, C_BYTES);
#pragma unroll
        for (int h = 0; h < BN / 32; ++h) tma_load_2d(cs + h * C_BOX, &mC, cbar, (int)(c0 + 32 * h), (int)r0);
      }
      mbar_arrive_expect_tx(full, 6 * P_BOX);
      tma_load_2d(sa[0], &pH, full, 0, (int)r0);
      tma_load_2d(sa[1], &pM, full, 0, (int)r0);
      tma_load_2d(sa[2], &pL, full, 0, (int)r0);
      tma_load_2d(sb[0], &pH, full, 0, (int)c0);
      tma_load_2d(sb[1], &pM, full, 0, (int)c0);
      tma_load_2d(sb[2], &pL, full, 0, (int)c0);
      mbar_wait(full, 0);
      if (args.tma_c) mbar_wait(cbar, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, false);
      if (mbar_wait(full, 0)) {
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
  } else {
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    bool ok = true;
    if (lane == 0) {
      ok = mbar_wait(accbar, 0);
      if (ok && args.tma_c) ok = mbar_wait(cbar, 0);
    }
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    if (ok) {
      tc_fence_after();
      const int64_t i = r0 + rl;
      const int64_t n = args.n, j0 = args.j0;
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) + cc * 32, v);
        tmem_wait_ld();
        const int64_t jb = c0 + cc * 32;
        if (args.tma_c) {
          uint8_t* box = smem + 6 * P_BOX + cc * C_BOX;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            float4* p4 = reinterpret_cast<float4*>(box + sw128_f32(rl, 4 * ch));
            float4 w = *p4;
            const int64_t j = jb + 4 * ch;
            const bool rowok = i < j0;
            if (rowok && j + 0 < j0 && j + 0 >= i) w.x -= __uint_as_float(v[4 * ch]);
            if (rowok && j + 1 < j0 && j + 1 >= i) w.y -= __uint_as_float(v[4 * ch + 1]);
            if (rowok && j + 2 < j0 && j + 2 >= i) w.z -= __uint_as_float(v[4 * ch + 2]);
            if (rowok && j + 3 < j0 && j + 3 >= i) w.w -= __uint_as_float(v[4 * ch + 3]);
            *p4 = w;
          }
        } else if (i < j0 && jb < j0 && jb + 31 >= i) {
          float* row = args.H + i * n + jb;
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const int64_t j = jb + t;
            if (j < j0 && j >= i) row[t] -= __uint_as_float(v[t]);
          }
        }
      }
      if (args.tma_c) {
        fence_proxy_async_smem();
        named_barrier(1, 128);             // the four epilogue warps
        if (warp == 2 && lane == 0) {
#pragma unroll
          for (int h = 0; h < BN / 32; ++h) tma_store_2d(&mC, cs + h * C_BOX, (int)(c0 + 32 * h), (int)r0);
          tma_store_commit();
          tma_store_wait_all();
        }
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

cudaError_t status_fetch_schur(int* out, cudaStream_t s) {
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

kronq_status schur_maps(SchurMaps* sm, const __nv_bfloat16* splits, float* H, int64_t n) {
  static_assert(sizeof(sm->raw) == 4 * sizeof(CUtensorMap), "map storage");
  CUtensorMap* maps = reinterpret_cast<CUtensorMap*>(sm->raw);
  for (int t = 0; t < 3; ++t) {
    const __nv_bfloat16* p = splits + (int64_t)t * n * KP;
    if (!tma_map_2d(&maps[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p, KP, n, KP, KP, BM))
      return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (Schur update)");
  }
  sm->tma_c = ((n % 4) == 0 && aligned(H, 16)) ? 1 : 0;
  if (sm->tma_c && !tma_map_2d(&maps[3], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, n, n, n, 32, BM))
    return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (Schur update, H)");
  return KRONQ_OK;
}

kronq_status schur_update_tc(const SchurMaps* sm, float* H, int64_t n, int64_t j0, const int* info,
                             cudaStream_t s) {
  if (j0 <= 0) return KRONQ_OK;
  const CUtensorMap* maps = reinterpret_cast<const CUtensorMap*>(sm->raw);
  SchurArgs a;
  a.H = H;
  a.n = n;
  a.j0 = j0;
  a.nt = (int)ceil_div(j0, BM);
  a.tma_c = sm->tma_c;
  a.info = info;
  const int64_t ntiles = (int64_t)a.nt * (a.nt + 1) / 2;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&schur_tc_kernel), SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(schur)");
  schur_tc_kernel<<<(unsigned)ntiles, THREADS, SMEM_BYTES, s>>>(maps[0], maps[1], maps[2], maps[3], a);
  KQ_LAUNCH_CHECK("schur_tc_kernel");
  return KRONQ_OK;
}

}  // namespace kq

// Schur-complement update of the blocked reverse Cholesky on the tensor
// cores:  A[0:j0, 0:j0] -= R_p R_p^T  (upper triangle only),
// where R_p = R[0:j0, J] is the just-solved 64-column panel.
//
// Float32-level accuracy from bf16 MMAs: the panel is split three ways,
// x = hi + mid + lo (each a bf16 rounding of the remainder), and the product
// keeps the six terms down to 2^-24 relative: hh + hm + mh + hl + lh + mm.
// The panel kernel writes the three splits (j0 x 64, row-major, K-major for
// both operands).  One CTA per 128 x 128 tile of the upper triangle; the
// tile itself is schur::tile (warp 0 TMA, warp 1 MMA, warps 2-5 epilogue).
#include "common.cuh"
#include "internal.h"
#include "schur_tile.cuh"

namespace kq {
namespace {

using schur::BM;
using schur::BN;
using schur::KP;
constexpr int SMEM_BYTES = schur::TILE_SMEM + 1024 + 256;
constexpr int THREADS = 192;

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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + schur::TILE_SMEM);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  const uint32_t full = smem_u32(&bars[0]);
  const uint32_t cbar = smem_u32(&bars[1]);
  const uint32_t accbar = smem_u32(&bars[2]);
  const int warp = threadIdx.x >> 5;
  int tr, tc;
  tile_of(blockIdx.x, args.nt, tr, tc);

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(cbar, 1);
    mbar_init(accbar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), schur::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const schur::TileMaps mp{&pH, &pM, &pL, &mC};
  schur::tile<2, 4>(smem, full, cbar, accbar, 0, tmem, mp, args.H, args.n, args.j0, (int64_t)tr * BM,
                 (int64_t)tc * BN, args.tma_c);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, schur::TMEM_COLS);
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

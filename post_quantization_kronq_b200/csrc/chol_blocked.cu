// Two-level blocked reverse Cholesky factorisation of the damped input
// factor, for orders above kOuterBlock (GPTQ's Cholesky factor of the damped
// inverse, which KronQ's sweep keeps; KronQ README intro).
//
// A = H + lambda I is factored as A = R R^T with R upper triangular,
// eliminating from the last index, and U = R^-1 (U^T U = A^-1).  With blocks
// of B = kOuterBlock rows aligned from the top (the last one may be short),
// for each block J from the bottom-right one up:
//
//   1. the diagonal block, already holding every update of the later blocks,
//      is copied to a contiguous B x B buffer and factored and inverted there
//      by the single-level path (chol_core: the persistent kernel with 64-wide
//      diagonal steps, then the recursive inverse), giving U_JJ;
//   2. T = U_JJ A[J, 0:j0] on the tensor cores (fp32-level split products),
//      which is R[0:j0, J]^T since A[0:j0, J] = R[0:j0, J] R_JJ^T;
//   3. R[0:j0, J] = T^T is stored above the diagonal block (for the inverse)
//      and as bf16 hi/mid/lo splits, K-major, for
//   4. the Schur update A[0:j0, 0:j0] -= R[0:j0, J] R[0:j0, J]^T, one K = B
//      tcgen05 product over the upper triangle's 128 x 128 tiles (six split
//      products per k step), both triangles written so that step 2 of the
//      next block can read its rows left of the diagonal.
//
// Finally the off-diagonal blocks of U come from the recursive two-block
// formula level by level, starting from the B x B diagonal blocks.  When R
// itself is wanted (the sweep's R form), step 1 keeps R_JJ in the diagonal
// block (U_JJ, still needed by step 2, is formed in the contiguous copy) and
// the last stage is skipped: the upper triangle then holds R.
//
// Compared with one chain of 64-wide steps over the whole order, each
// element of the trailing matrix goes through HBM once per B columns
// instead of once per 64: at n = 28672 the Schur updates move ~7 GB instead
// of ~490 GB and run tensor-bound.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int SK_BM = 128, SK_BN = 128, SK_BK = 64, SK_STAGES = 2;
constexpr int SK_BOX = SK_BM * SK_BK * 2;       // 16 KB: 128 rows x 64 k (K-major, 128-byte rows)
constexpr int SK_STAGE = 6 * SK_BOX;            // 96 KB: A hi/mid/lo, B hi/mid/lo
constexpr int SK_NBARS = 2 * SK_STAGES + 4;
constexpr int SK_SMEM = SK_STAGES * SK_STAGE + 1024 + 256;
constexpr int SK_EPI_WARPS = 8;
constexpr int SK_THREADS = 64 + 32 * SK_EPI_WARPS;
constexpr uint32_t SK_TMEM = 2 * SK_BN;
constexpr int SK_STRIP = 16;
constexpr int SK_SEG = 1;                        // 64-deep chunks per accumulation segment

struct SkArgs {
  float* H;       // the j0 x j0 block at the top left, row stride ld
  int64_t ld;
  int j0;
  int nk;         // 64-deep k chunks
  int nt;         // tiles per side
  int ntiles;     // upper-triangle tiles
  const int* info;
};

// Upper-triangle tile t (tr <= tc) in strips of SK_STRIP tile rows,
// column-major inside a strip.
__device__ __forceinline__ void sk_tile_of(int t, int nt, int& tr, int& tc) {
  for (int s0 = 0; s0 < nt; s0 += SK_STRIP) {
    const int s1 = min(s0 + SK_STRIP, nt);
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

// A[0:j0, 0:j0] -= R R^T with R (j0 x K) given as three bf16 planes
// (K-major, one 128-row x 64-k box per load).  Persistent; warp 0 = TMA
// producer, warp 1 = MMA issuer and TMEM owner, warps 2-9 = epilogue; two
// 96 KB stages.  Accumulation in segments: the MMAs of SK_SEG k chunks
// (64 k, six split products each) go to one of two 128-column TMEM
// accumulators, and the epilogue adds each finished segment into float32
// registers with round-to-nearest while the next segment runs.  One TMEM
// accumulator over the whole K = 4096 loses ~1e-4 relative (the tensor
// core's accumulation drifts with the number of MMAs summed into it); short
// segments keep the Schur complement near float32 accuracy.
__global__ void __launch_bounds__(SK_THREADS, 1)
    schur_k_kernel(const __grid_constant__ CUtensorMap mH, const __grid_constant__ CUtensorMap mM,
                   const __grid_constant__ CUtensorMap mL, SkArgs args) {
  if (args.info && *args.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SK_STAGES * SK_STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + SK_NBARS);
  volatile int* abort_s = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t full0 = smem_u32(&bars[0]);
  const uint32_t empty0 = smem_u32(&bars[SK_STAGES]);
  const uint32_t accfull0 = smem_u32(&bars[2 * SK_STAGES]);
  const uint32_t accempty0 = smem_u32(&bars[2 * SK_STAGES + 2]);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SK_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull0 + 8 * b, 1);
      mbar_init(accempty0 + 8 * b, SK_EPI_WARPS);
    }
    *abort_s = 0;
    fence_mbar_init();
    prefetch_tmap(&mH);
    prefetch_tmap(&mM);
    prefetch_tmap(&mL);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), SK_TMEM);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t stage0 = smem_u32(smem);
  const int nk = args.nk;
  const int nseg = (nk + SK_SEG - 1) / SK_SEG;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* maps[3] = {&mH, &mM, &mL};
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.ntiles; t += gridDim.x) {
        int tr, tc;
        sk_tile_of(t, args.nt, tr, tc);
        const int r0 = tr * SK_BM, c0 = tc * SK_BN;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % SK_STAGES;
          const uint32_t ph = (it / SK_STAGES) & 1;
          if (*abort_s || !mbar_wait(empty0 + 8 * s, ph ^ 1)) {
            *abort_s = 1;
            ok = false;
            break;
          }
          const uint32_t full = full0 + 8 * s;
          mbar_arrive_expect_tx(full, SK_STAGE);
          const uint32_t st = stage0 + s * SK_STAGE;
#pragma unroll
          for (int p = 0; p < 3; ++p) {
            tma_load_2d(st + p * SK_BOX, maps[p], full, kb * SK_BK, r0);
            tma_load_2d(st + (3 + p) * SK_BOX, maps[p], full, kb * SK_BK, c0);
          }
        }
      }
      for (uint32_t k = it > SK_STAGES ? it - SK_STAGES : 0; k < it; ++k)
        mbar_wait(full0 + 8 * (k % SK_STAGES), (k / SK_STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(SK_BM, SK_BN, false, false);
      // split pairs (a, b) with a + b <= 2: hh, hm, mh, hl, lh, mm
      const int pa[6] = {0, 0, 1, 0, 2, 1};
      const int pb[6] = {0, 1, 0, 2, 0, 1};
      uint32_t it = 0, sg = 0;   // k chunks and segments issued over all tiles
      bool ok = true;
      for (int t = blockIdx.x; ok && t < args.ntiles; t += gridDim.x) {
        for (int g = 0; ok && g < nseg; ++g, ++sg) {
          const int b = sg & 1;
          const uint32_t u = sg >> 1;
          // the epilogue has drained the segment that used accumulator b
          if (u > 0 && (*abort_s || !mbar_wait(accempty0 + 8 * b, (u - 1) & 1))) {
            *abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc = tmem + (uint32_t)(b * SK_BN);
          const int k1 = min(nk, (g + 1) * SK_SEG);
          for (int kb = g * SK_SEG; kb < k1; ++kb, ++it) {
            const uint32_t s = it % SK_STAGES;
            const uint32_t ph = (it / SK_STAGES) & 1;
            if (*abort_s || !mbar_wait(full0 + 8 * s, ph)) {
              *abort_s = 1;
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t st = stage0 + s * SK_STAGE;
#pragma unroll
            for (int kk = 0; kk < SK_BK / 16; ++kk) {
#pragma unroll
              for (int q = 0; q < 6; ++q) {
                // K-major boxes: 16 k = 32 bytes along each 128-byte row
                const uint64_t da = smem_desc_sw128(st + pa[q] * SK_BOX + kk * 32, 16, 1024);
                const uint64_t db = smem_desc_sw128(st + (3 + pb[q]) * SK_BOX + kk * 32, 16, 1024);
                mma_bf16(acc, da, db, idesc, (kb != g * SK_SEG || kk != 0 || q != 0) ? 1u : 0u);
              }
            }
            mma_commit(empty0 + 8 * s);
          }
          if (ok) mma_commit(accfull0 + 8 * b);
        }
      }
    }
    __syncwarp();
  } else {
    // Epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 and the columns
    // 64 hc .. 64 hc + 63 of the tile, hc = (w - 2) / 4.  Each finished
    // segment is added into acc[]; at the tile's end entry (i, j),
    // i <= j < j0, gets A - acc, and so does its mirror (j, i).
    const int q = warp & 3, hc = (warp - 2) >> 2;
    const int64_t ld = args.ld;
    const int j0 = args.j0;
    float* H = args.H;
    uint32_t sg = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < args.ntiles; t += gridDim.x) {
      float acc[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) acc[e] = 0.f;
      for (int g = 0; g < nseg; ++g, ++sg) {
        const int b = sg & 1;
        const uint32_t u = sg >> 1;
        int good = 1;
        if (lane == 0) good = (!*abort_s && mbar_wait(accfull0 + 8 * b, u & 1)) ? 1 : 0;
        good = __shfl_sync(0xffffffffu, good, 0);
        __syncwarp();
        if (!good) {
          if (lane == 0) *abort_s = 1;
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t v[32];
          __syncwarp();  // the TMEM load is warp-collective
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(q * 32) << 16) +
                                 (uint32_t)(b * SK_BN + 64 * hc + 32 * h), v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[32 * h + e] = __fadd_rn(acc[32 * h + e], __uint_as_float(v[e]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty0 + 8 * b);
      }
      if (!ok) break;
      int tr, tc;
      sk_tile_of(t, args.nt, tr, tc);
      const int i = tr * SK_BM + q * 32 + lane;
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const int jb = tc * SK_BN + 64 * hc + 16 * h;
        // every load of these 16 columns first, then the stores
        const bool dense = i < j0 && jb >= i && jb + 16 <= j0 && (ld % 4) == 0 &&
                           ((reinterpret_cast<uintptr_t>(H) & 15) == 0);
        float up[16], mir[16];
        if (dense) {
          const float4* src = reinterpret_cast<const float4*>(H + (int64_t)i * ld + jb);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 o = src[e];
            up[4 * e] = o.x; up[4 * e + 1] = o.y; up[4 * e + 2] = o.z; up[4 * e + 3] = o.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j = jb + e;
            up[e] = (i < j0 && j < j0 && i <= j) ? H[(int64_t)i * ld + j] : 0.f;
          }
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = jb + e;
          mir[e] = (i < j0 && j < j0 && i < j) ? H[(int64_t)j * ld + i] : 0.f;
        }
        const float* a = acc + 16 * h;
        if (dense) {
          float4* dst = reinterpret_cast<float4*>(H + (int64_t)i * ld + jb);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(up[4 * e] - a[4 * e], up[4 * e + 1] - a[4 * e + 1], up[4 * e + 2] - a[4 * e + 2],
                                 up[4 * e + 3] - a[4 * e + 3]);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int j = jb + e;
            if (i < j0 && j < j0 && i <= j) H[(int64_t)i * ld + j] = up[e] - a[e];
          }
        }
        // mirror (j, i), i < j: 32 lanes write 32 consecutive floats
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = jb + e;
          if (i < j0 && j < j0 && i < j) H[(int64_t)j * ld + i] = mir[e] - a[e];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, SK_TMEM);
  }
}

// dst[r, c] = src[r, c] for r < rows, c < cols (upper: only c >= r).
__global__ void copy_block_kernel(float* dst, int64_t ldd, const float* src, int64_t lds, int64_t rows,
                                  int64_t cols, int upper, const int* info) {
  if (info && *info != 0) return;
  const int64_t tot = rows * cols;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < tot; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / cols, c = t - (t / cols) * cols;
    if (!upper || c >= r) dst[r * ldd + c] = src[r * lds + c];
  }
}

// R = T^T for T (K x j0, row stride ldt): R[i][k] into the block above the
// diagonal (row stride ldh) and as three bf16 planes (row stride ldp), the
// hi/mid/lo splits x = hi + mid + lo of each value.  32 x 32 tiles through
// shared memory.
__global__ void __launch_bounds__(256) transpose_split_kernel(const float* T, int64_t ldt, int K, int64_t j0,
                                                              float* Hp, int64_t ldh, __nv_bfloat16* Rh,
                                                              __nv_bfloat16* Rm, __nv_bfloat16* Rl,
                                                              int64_t ldp, const int* info) {
  if (info && *info != 0) return;
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t i0 = (int64_t)blockIdx.x * 32;
  const int64_t k0 = (int64_t)blockIdx.y * 32;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t k = k0 + ty + 8 * r, i = i0 + tx;
    tile[ty + 8 * r][tx] = (k < K && i < j0) ? T[k * ldt + i] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int64_t i = i0 + ty + 8 * r, k = k0 + tx;
    if (i < j0 && k < K) {
      const float x = tile[tx][ty + 8 * r];
      Hp[i * ldh + k] = x;
      const __nv_bfloat16 h = __float2bfloat16_rn(x);
      const float r1 = x - __bfloat162float(h);
      const __nv_bfloat16 m = __float2bfloat16_rn(r1);
      const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
      Rh[i * ldp + k] = h;
      Rm[i * ldp + k] = m;
      Rl[i * ldp + k] = l;
    }
  }
}

// A failing pivot inside block J's factorisation, at local index k, is the
// global index j0 + k (LAPACK convention, 1-based).
__global__ void merge_info_kernel(int* info, const int* local, int64_t j0) {
  if (*info == 0 && *local != 0) *info = (int)(j0 + *local);
}

int64_t plane_ld(int64_t K) { return (K + 7) / 8 * 8; }

}  // namespace

cudaError_t status_fetch_schurk(int* out, cudaStream_t s) {
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

// Workspace: [T / inverse products: chol_tbuf_bytes(n)] [three bf16 planes
// of R, n x B each] [the B x B diagonal block] [chol_core's workspace for
// order B] [the block's info].
static size_t plane_bytes(int64_t n) {
  return (((size_t)n * (size_t)plane_ld(kOuterBlock) * sizeof(__nv_bfloat16)) + 255) & ~size_t(255);
}

size_t chol_blocked_workspace_bytes(int64_t n) {
  const int64_t B = kOuterBlock;
  return chol_tbuf_bytes(n) + 3 * plane_bytes(n) + (size_t)B * B * sizeof(float) +
         chol_core_workspace_bytes(B) + 256;
}

kronq_status chol_blocked(float* H, int64_t n, int* info, void* ws, cudaStream_t s, bool want_u) {
  const int64_t B = kOuterBlock;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* Tbuf = reinterpret_cast<float*>(w);
  w += chol_tbuf_bytes(n);
  __nv_bfloat16* Rp[3];
  for (int p = 0; p < 3; ++p) {
    Rp[p] = reinterpret_cast<__nv_bfloat16*>(w);
    w += plane_bytes(n);
  }
  float* Sbuf = reinterpret_cast<float*>(w);
  w += (size_t)B * B * sizeof(float);
  void* core_ws = w;
  w += chol_core_workspace_bytes(B);
  int* info_local = reinterpret_cast<int*>(w);

  const int64_t nblk = ceil_div(n, B);
  const int copy_grid = 4 * sm_count();
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&schur_k_kernel), SK_SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(schur_k)");
  for (int64_t J = nblk - 1; J >= 0; --J) {
    const int64_t j0 = J * B;
    const int64_t nb = (j0 + B <= n) ? B : n - j0;
    // 1. U_JJ of the diagonal block, in a contiguous copy
    copy_block_kernel<<<copy_grid, 256, 0, s>>>(Sbuf, nb, H + j0 * n + j0, n, nb, nb, 1, info);
    KQ_LAUNCH_CHECK("copy_block_kernel");
    KQ_CUDA(cudaMemsetAsync(info_local, 0, sizeof(int), s));
    // (for R: R_JJ first, copied out, then turned into U_JJ for step 2)
    kronq_status r = chol_core(Sbuf, nb, info_local, core_ws, s, want_u);
    if (r != KRONQ_OK) return r;
    merge_info_kernel<<<1, 1, 0, s>>>(info, info_local, j0);
    KQ_LAUNCH_CHECK("merge_info_kernel");
    copy_block_kernel<<<copy_grid, 256, 0, s>>>(H + j0 * n + j0, n, Sbuf, nb, nb, nb, 1, info);
    KQ_LAUNCH_CHECK("copy_block_kernel");
    if (j0 == 0) break;
    if (!want_u) {
      r = chol_core_finish_u(Sbuf, nb, info_local, core_ws, s);
      if (r != KRONQ_OK) return r;
    }
    // 2. T = U_JJ A[J, 0:j0]  (nb x j0)
    TriGemm t;
    t.M = nb; t.N = j0; t.K = nb;
    t.A = Sbuf; t.lda = nb; t.a_upper = true;
    t.B = H + j0 * n; t.ldb = n;
    t.C = Tbuf; t.ldc = j0;
    t.alpha = 1.f;
    t.info = info;
    t.holdA = Sbuf; t.holdA_rows = nb; t.holdA_cols = nb;
    t.holdB = H; t.holdB_rows = n; t.holdB_cols = n;
    r = trigemm_tc(t, s);
    if (r != KRONQ_OK) return r;
    // 3. R[0:j0, J] = T^T above the diagonal block, and its splits
    const int64_t ldp = plane_ld(nb);
    dim3 tg((unsigned)ceil_div(j0, 32), (unsigned)ceil_div(nb, 32));
    transpose_split_kernel<<<tg, 256, 0, s>>>(Tbuf, j0, (int)nb, j0, H + j0, n, Rp[0], Rp[1], Rp[2], ldp, info);
    KQ_LAUNCH_CHECK("transpose_split_kernel");
    // 4. A[0:j0, 0:j0] -= R R^T
    CUtensorMap maps[3];
    for (int p = 0; p < 3; ++p)
      if (!tma_map_2d(&maps[p], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Rp[p], nb, j0, ldp, SK_BK, SK_BM))
        return fail(KRONQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (blocked Schur update)");
    SkArgs a;
    a.H = H;
    a.ld = n;
    a.j0 = (int)j0;
    a.nk = (int)ceil_div(nb, SK_BK);
    a.nt = (int)ceil_div(j0, SK_BM);
    a.ntiles = a.nt * (a.nt + 1) / 2;
    a.info = info;
    const int grid = a.ntiles < sm_count() ? a.ntiles : sm_count();
    schur_k_kernel<<<(unsigned)grid, SK_THREADS, SK_SMEM, s>>>(maps[0], maps[1], maps[2], a);
    KQ_LAUNCH_CHECK("schur_k_kernel");
  }
  if (!want_u) return KRONQ_OK;   // R: the diagonal blocks R_JJ and R above them
  return chol_inverse_levels(H, n, B, Tbuf, info, s);
}

}  // namespace kq

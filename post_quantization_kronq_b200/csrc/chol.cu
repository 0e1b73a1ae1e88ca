// Damping and the upper Cholesky factor of the damped inverse.
//
// GPTQ (which KronQ extends, KronQ README intro) needs the upper triangular
// U with U^T U = (H + lambda I)^-1.  Instead of inverting and factoring
// again, this library factors A = H + lambda I "in reverse": A = R R^T with
// R upper triangular (eliminating from the last index down), and then
// U = R^-1, since A^-1 = R^-T R^-1 = U^T U.  That is 2 n^3 / 3 flops in total.
//
// Blocked with nb = 64, bottom-right first.  For each diagonal block J:
//   diag_panel_kernel  factor A_JJ = R_JJ R_JJ^T and solve R[0:j0, J] R_JJ^T
//                      = A[0:j0, J] (every CTA factors the small block itself)
//   schur_tc_kernel    A[0:j0, 0:j0] -= R[0:j0, J] R[0:j0, J]^T on the tensor
//                      cores (upper triangle only, fp32-level split products)
// Then every diagonal block is inverted at once (U_JJ = R_JJ^-1), and the
// off-diagonal blocks of U come from the recursive formula
//   inv([[R11, R12], [0, R22]]) = [[U11, -U11 R12 U22], [0, U22]]
// evaluated level by level (block sizes nb, 2 nb, 4 nb, ...), each level one
// batched pair of GEMMs.  A non-positive pivot stops the chain and records
// info = 1 + its index (LAPACK convention); every later kernel then returns.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int NB = 64;

__global__ void __launch_bounds__(1024) damp_kernel(float* H, int64_t n, float damp_rel,
                                                    uint8_t* dead, int* info) {
  __shared__ double red[32];
  if (threadIdx.x == 0) *info = 0;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    float h = H[j * n + j];
    const bool isdead = (h == 0.f);
    if (isdead) {
      h = 1.f;
      H[j * n + j] = 1.f;
    }
    if (dead) dead[j] = isdead ? 1 : 0;
    acc += (double)h;
  }
  acc = warp_sum_d(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    v = warp_sum_d(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float lam = (float)((double)damp_rel * (red[0] / (double)n));
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) H[j * n + j] = H[j * n + j] + lam;
}

__global__ void zero_info_kernel(int* info) { *info = 0; }

// Factor the diagonal block A_JJ = R_JJ R_JJ^T (reverse order) in shared
// memory and solve the panel rows above it, R[i, J] R_JJ^T = A[i, J].
// Every CTA factors the (small) block itself, so no extra launch sits on the
// sequential path; CTA 0 writes R_JJ back.  A short block (nb < 64) is padded
// with the identity.  The panel rows are also written as bf16 hi/mid/lo
// splits for the tensor-core Schur update.
__global__ void __launch_bounds__(256) diag_panel_kernel(float* H, int64_t n, int64_t j0, int nb,
                                                         int* info, __nv_bfloat16* splits) {
  if (*info != 0) return;
  __shared__ float a[NB][NB + 1];
  __shared__ float rdiag[NB], rinv[NB];
  const int tid = threadIdx.x;
  const int tx = tid & 63, ty = tid >> 6;
  {
    float x[NB / 4];
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {  // all sixteen loads in flight
      const int r = 4 * sl + ty;
      x[sl] = (r <= tx && tx < nb) ? H[(j0 + r) * n + j0 + tx] : 0.f;
    }
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {
      const int r = 4 * sl + ty;
      a[r][tx] = (tx < nb) ? x[sl] : (r == tx ? 1.f : 0.f);
    }
  }
  // One barrier per pivot: the update of column c < k uses
  // r_ik r_ck = a_ik a_ck / pivot, so column k itself is left unscaled until
  // the end (it is never written again once its pivot is done).
  for (int k = NB - 1; k >= 0; --k) {
    __syncthreads();
    const float piv = a[k][k];
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (tid == 0 && blockIdx.x == 0) *info = (int)(j0 + k + 1);
      return;  // uniform: every thread read the same pivot
    }
    if (tid == 0) {
      const float rk = sqrtf(piv);
      rdiag[k] = rk;
      rinv[k] = 1.f / rk;
    }
    if (tx < k) {
      // all loads first: stores to column tx cannot be proven not to alias
      // column k, so interleaving would serialise the sixteen updates
      const float act = a[tx][k] * (1.f / piv);
      float ck[NB / 4], ct[NB / 4];
#pragma unroll
      for (int sl = 0; sl < NB / 4; ++sl) {
        ck[sl] = a[4 * sl + ty][k];
        ct[sl] = a[4 * sl + ty][tx];
      }
#pragma unroll
      for (int sl = 0; sl < NB / 4; ++sl) {
        const int i = 4 * sl + ty;
        if (i <= tx) a[i][tx] = ct[sl] - ck[sl] * act;
      }
    }
  }
  __syncthreads();
  // scale every column k of R above the diagonal by 1 / r_kk
#pragma unroll
  for (int sl = 0; sl < NB / 4; ++sl) {
    const int i = 4 * sl + ty;
    if (i < tx) a[i][tx] *= rinv[tx];
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int t = tid; t < nb * NB; t += blockDim.x) {
      const int r = t >> 6, c = t & 63;
      if (c < nb) H[(j0 + r) * n + j0 + c] = (r < c) ? a[r][c] : (r == c ? rdiag[r] : 0.f);
    }
  }
  // Panel rows: x R_JJ^T = a, back substitution from the last column; one
  // warp per row, lane l holds columns l and l + 32.
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t plane = (int64_t)n * NB;
  for (int64_t i = (int64_t)blockIdx.x * 8 + warp; i < j0; i += (int64_t)gridDim.x * 8) {
    float* row = H + i * n + j0;
    float acc0 = (lane < nb) ? row[lane] : 0.f;
    float acc1 = (lane + 32 < nb) ? row[lane + 32] : 0.f;
    float x0 = 0.f, x1 = 0.f;
    for (int k = NB - 1; k >= 0; --k) {
      const bool upper_half = k >= 32;
      const int owner = k & 31;
      float xk = (upper_half ? acc1 : acc0) * rinv[k];
      xk = __shfl_sync(0xffffffffu, xk, owner);
      if (lane == owner) {
        if (upper_half) x1 = xk;
        else x0 = xk;
      }
      if (lane < k) acc0 -= a[lane][k] * xk;
      if (lane + 32 < k) acc1 -= a[lane + 32][k] * xk;
    }
    if (lane < nb) row[lane] = x0;
    if (lane + 32 < nb) row[lane + 32] = x1;
    const float xs[2] = {x0, x1};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float x = xs[h];
      const __nv_bfloat16 bh = __float2bfloat16_rn(x);
      const float r1 = x - __bfloat162float(bh);
      const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
      const __nv_bfloat16 bl = __float2bfloat16_rn(r1 - __bfloat162float(bm));
      const int64_t o = i * NB + lane + 32 * h;
      splits[o] = bh;
      splits[plane + o] = bm;
      splits[2 * plane + o] = bl;
    }
  }
}

// U_JJ = R_JJ^-1 for every diagonal block at once (one CTA per block).
// Entry (i, i + dd) depends only on entries of smaller distance dd, so the
// diagonals are computed one after the other, four adjacent lanes per entry.
__global__ void __launch_bounds__(256) diag_inverse_kernel(float* H, int64_t n, const int* info) {
  if (*info != 0) return;
  __shared__ float a[NB][NB + 1];
  __shared__ float u[NB][NB + 1];
  __shared__ float rinv[NB];
  const int64_t j0 = (int64_t)blockIdx.x * NB;
  const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
  const int tid = threadIdx.x;
  for (int t = tid; t < NB * NB; t += blockDim.x) {
    const int r = t >> 6, c = t & 63;
    float x = 0.f;
    if (r <= c) x = (c < nb) ? H[(j0 + r) * n + j0 + c] : (r == c ? 1.f : 0.f);
    a[r][c] = x;
    u[r][c] = 0.f;
  }
  __syncthreads();
  if (tid < NB) rinv[tid] = 1.f / a[tid][tid];
  __syncthreads();
  const int ii = tid >> 2, part = tid & 3;
  if (part == 0) u[ii][ii] = rinv[ii];
  __syncthreads();
  for (int dd = 1; dd < NB; ++dd) {
    const int jj = ii + dd;
    float acc = 0.f;
    if (jj < NB)
      for (int k = ii + 1 + part; k <= jj; k += 4) acc = fmaf(a[ii][k], u[k][jj], acc);
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (jj < NB && part == 0) u[ii][jj] = -acc * rinv[ii];
    __syncthreads();
  }
  for (int t = tid; t < nb * NB; t += blockDim.x) {
    const int r = t >> 6, c = t & 63;
    if (c < nb) H[(j0 + r) * n + j0 + c] = (r <= c) ? u[r][c] : 0.f;
  }
}

}  // namespace

size_t chol_workspace_bytes(int64_t n) {
  // recursive inverse: products T of the pairs of one level (at most n*n/4
  // floats); bf16 hi/mid/lo splits of the current panel (3 x n x 64)
  const size_t tbytes = (size_t)((n * n) / 4 + n + 64) * sizeof(float);
  const size_t sbytes = (size_t)3 * n * NB * sizeof(__nv_bfloat16);
  return ((tbytes + 255) & ~size_t(255)) + sbytes;
}

kronq_status chol_upper_inverse(float* H, int64_t n, float damp_rel, bool skip_damp,
                                uint8_t* dead, int* info, void* ws, cudaStream_t s) {
  if (!skip_damp) {
    damp_kernel<<<1, 1024, 0, s>>>(H, n, damp_rel, dead, info);
    KQ_LAUNCH_CHECK("damp_kernel");
  } else {
    zero_info_kernel<<<1, 1, 0, s>>>(info);
    KQ_LAUNCH_CHECK("zero_info_kernel");
  }
  if (n <= 0) return KRONQ_OK;
  const size_t tbytes = (size_t)((n * n) / 4 + n + 64) * sizeof(float);
  __nv_bfloat16* splits = reinterpret_cast<__nv_bfloat16*>(
      static_cast<uint8_t*>(ws) + ((tbytes + 255) & ~size_t(255)));
  SchurMaps maps;
  if (n > NB) {
    kronq_status r = schur_maps(&maps, splits, H, n);
    if (r != KRONQ_OK) return r;
  }
  // Blocks are aligned from the top (0, NB, 2 NB, ...); the last may be short.
  const int64_t nblk = ceil_div(n, NB);
  const int64_t pmax = sm_count();
  for (int64_t bj = nblk - 1; bj >= 0; --bj) {
    const int64_t j0 = bj * NB;
    const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
    // One CTA per SM at most (each CTA factors the block itself), at least
    // four panel rows per warp.
    int64_t pg = j0 > 0 ? ceil_div(j0, 32) : 1;
    if (pg > pmax) pg = pmax;
    diag_panel_kernel<<<(unsigned)pg, 256, 0, s>>>(H, n, j0, nb, info, splits);
    KQ_LAUNCH_CHECK("diag_panel_kernel");
    if (j0 == 0) break;
    kronq_status r = schur_update_tc(&maps, H, n, j0, info, s);
    if (r != KRONQ_OK) return r;
  }
  diag_inverse_kernel<<<(unsigned)nblk, 256, 0, s>>>(H, n, info);
  KQ_LAUNCH_CHECK("diag_inverse_kernel");
  // Recursive inverse of the off-diagonal blocks.
  float* Tbuf = reinterpret_cast<float*>(ws);
  for (int64_t S = NB; S < n; S *= 2) {
    const int64_t npairs_full = n / (2 * S);  // pairs whose R22 has full size S
    struct Pair { int64_t p0, cnt, s2; };
    Pair groups[2] = {{0, npairs_full, S}, {npairs_full, 0, 0}};
    const int64_t rem_start = npairs_full * 2 * S + S;  // start of a ragged R22
    if (rem_start < n) groups[1] = {npairs_full, 1, n - rem_start};
    for (const Pair& gp : groups) {
      if (gp.cnt <= 0) continue;
      const int64_t base = gp.p0 * 2 * S;  // R11 origin of the first pair
      const int64_t s2 = gp.s2;
      // T = R12 * U22   (S x s2) = (S x s2)(s2 x s2, upper)
      GemmDesc t;
      t.M = S; t.N = s2; t.K = s2;
      t.A = H + base * n + base + S; t.lda = n;
      t.B = H + (base + S) * n + base + S; t.ldb = n; t.b_upper = true;
      t.C = Tbuf; t.ldc = s2;
      t.alpha = 1.f; t.beta = 0.f;
      t.batch = (int)gp.cnt;
      t.strideA = 2 * S * n + 2 * S; t.strideB = 2 * S * n + 2 * S; t.strideC = S * s2;
      t.info = info;
      cudaError_t e = gemm_f32(t, s);
      if (e != cudaSuccess) return cuda_fail(e, "gemm(inverse T)");
      // U12 = -U11 * T  (S x s2) = (S x S, upper)(S x s2)
      GemmDesc u;
      u.M = S; u.N = s2; u.K = S;
      u.A = H + base * n + base; u.lda = n; u.a_upper = true;
      u.B = Tbuf; u.ldb = s2;
      u.C = H + base * n + base + S; u.ldc = n;
      u.alpha = -1.f; u.beta = 0.f;
      u.batch = (int)gp.cnt;
      u.strideA = 2 * S * n + 2 * S; u.strideB = S * s2; u.strideC = 2 * S * n + 2 * S;
      u.info = info;
      e = gemm_f32(u, s);
      if (e != cudaSuccess) return cuda_fail(e, "gemm(inverse U12)");
    }
  }
  return KRONQ_OK;
}

}  // namespace kq

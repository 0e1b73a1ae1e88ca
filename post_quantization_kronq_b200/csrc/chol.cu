// Damping and the upper Cholesky factor of the damped inverse.
//
// GPTQ (which KronQ extends, KronQ README intro) needs the upper triangular
// U with U^T U = (H + lambda I)^-1.  Instead of inverting and factoring
// again, this library factors A = H + lambda I "in reverse": A = R R^T with
// R upper triangular (eliminating from the last index down), and then
// U = R^-1, since A^-1 = R^-T R^-1 = U^T U.  That is 2 n^3 / 3 flops in total.
//
// Blocked with nb = 64, bottom-right first.  For each diagonal block J:
//   K_A  one CTA factors A_JJ = R_JJ R_JJ^T and writes U_JJ = R_JJ^-1 in place;
//   K_B  R[0:j0, J] = A[0:j0, J] U_JJ^T                 (panel)
//   K_C  A[0:j0, 0:j0] -= R[0:j0, J] R[0:j0, J]^T         (upper triangle only)
// Then the off-diagonal blocks of U come from the recursive formula
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

// Factor the nb x nb diagonal block at j0 (reverse order), then invert R_JJ.
__global__ void __launch_bounds__(256) diag_kernel(float* H, int64_t n, int64_t j0, int nb,
                                                   int* info) {
  if (*info != 0) return;
  __shared__ float a[NB][NB + 1];
  __shared__ float u[NB][NB + 1];
  __shared__ int bad;
  const int tid = threadIdx.x;
  for (int t = tid; t < nb * nb; t += blockDim.x) {
    const int r = t / nb, c = t % nb;
    // upper triangle (symmetric storage may hold only it reliably)
    a[r][c] = (r <= c) ? H[(j0 + r) * n + j0 + c] : H[(j0 + c) * n + j0 + r];
    u[r][c] = 0.f;
  }
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int k = nb - 1; k >= 0; --k) {
    const float piv = a[k][k];
    if (!(piv > 0.f) || !isfinite(piv)) {
      if (tid == 0) {
        *info = (int)(j0 + k + 1);
        bad = 1;
      }
      __syncthreads();
      return;
    }
    const float rk = sqrtf(piv);
    __syncthreads();
    for (int i = tid; i < k; i += blockDim.x) a[i][k] = a[i][k] / rk;
    if (tid == 0) a[k][k] = rk;
    __syncthreads();
    // Schur complement on the leading k x k upper triangle
    for (int t = tid; t < k * k; t += blockDim.x) {
      const int i = t / k, j = t % k;
      if (i <= j) a[i][j] = a[i][j] - a[i][k] * a[j][k];
    }
    __syncthreads();
  }
  // U_JJ = R_JJ^-1, column c by back substitution (one thread per column)
  if (tid < nb) {
    const int c = tid;
    u[c][c] = 1.f / a[c][c];
    for (int i = c - 1; i >= 0; --i) {
      float acc = 0.f;
      for (int k = i + 1; k <= c; ++k) acc = fmaf(a[i][k], u[k][c], acc);
      u[i][c] = -acc / a[i][i];
    }
  }
  __syncthreads();
  for (int t = tid; t < nb * nb; t += blockDim.x) {
    const int r = t / nb, c = t % nb;
    H[(j0 + r) * n + j0 + c] = (r <= c) ? u[r][c] : 0.f;
  }
}

// R[0:j0, J] = A[0:j0, J] * U_JJ^T, rows in place.  One warp per row.
__global__ void __launch_bounds__(256) panel_kernel(float* H, int64_t n, int64_t j0, int nb,
                                                    const int* info) {
  if (*info != 0) return;
  __shared__ float u[NB][NB + 1];
  __shared__ float rowbuf[8][NB];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int t = tid; t < nb * nb; t += blockDim.x) {
    const int r = t / nb, c = t % nb;
    u[r][c] = (r <= c) ? H[(j0 + r) * n + j0 + c] : 0.f;
  }
  __syncthreads();
  for (int64_t i = (int64_t)blockIdx.x * 8 + warp; i < j0; i += (int64_t)gridDim.x * 8) {
    float* row = H + i * n + j0;
    for (int k = lane; k < nb; k += 32) rowbuf[warp][k] = row[k];
    __syncwarp();
    float out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = lane + 32 * h;
      float acc = 0.f;
      if (c < nb)
        for (int k = c; k < nb; ++k) acc = fmaf(rowbuf[warp][k], u[c][k], acc);
      out[h] = acc;
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = lane + 32 * h;
      if (c < nb) row[c] = out[h];
    }
    __syncwarp();
  }
}

}  // namespace

size_t chol_workspace_bytes(int64_t n) {
  // recursive inverse: products T of the pairs of one level, at most n*n/4
  return (size_t)((n * n) / 4 + n + 64) * sizeof(float);
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
  // Blocks are aligned from the top (0, NB, 2 NB, ...); the last may be short.
  const int64_t nblk = ceil_div(n, NB);
  for (int64_t bj = nblk - 1; bj >= 0; --bj) {
    const int64_t j0 = bj * NB;
    const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
    diag_kernel<<<1, 256, 0, s>>>(H, n, j0, nb, info);
    KQ_LAUNCH_CHECK("diag_kernel");
    if (j0 == 0) break;
    int64_t pg = ceil_div(j0, 8);
    if (pg > 148 * 16) pg = 148 * 16;
    panel_kernel<<<(unsigned)pg, 256, 0, s>>>(H, n, j0, nb, info);
    KQ_LAUNCH_CHECK("panel_kernel");
    GemmDesc g;
    g.M = j0; g.N = j0; g.K = nb;
    g.A = H + j0; g.lda = n; g.transA = false;
    g.B = H + j0; g.ldb = n; g.transB = true;
    g.C = H; g.ldc = n;
    g.alpha = -1.f; g.beta = 1.f;
    g.c_mode = 1;
    g.info = info;
    cudaError_t e = gemm_f32(g, s);
    if (e != cudaSuccess) return cuda_fail(e, "gemm(schur)");
  }
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

// Float32 SIMT GEMM with triangular operand/output masks and an exactly
// ordered mode.  Used by the factorisation (Schur updates, the recursive
// triangular inverse), the float32 factor path, the ordered trailing update
// of the column sweep and the loss diagnostic.
//
// 128 x 128 output tile per CTA, 8-deep k slices double-buffered in shared
// memory, 256 threads each owning an 8 x 8 register block split in two 4-row
// and two 4-column halves (conflict-free float4 shared-memory reads).
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int TM = 128, TN = 128, TK = 8, NT = 256;

template <bool ORDERED>
__global__ void __launch_bounds__(NT) gemm_kernel(GemmDesc g) {
  if (g.info && *g.info != 0) return;
  const int64_t i0 = (int64_t)blockIdx.y * TM;
  const int64_t j0 = (int64_t)blockIdx.x * TN;
  if (i0 >= g.M || j0 >= g.N) return;
  if (g.c_mode != 0 && i0 > j0 + TN - 1) return;  // tile entirely below the diagonal

  const float* A = g.A + (int64_t)blockIdx.z * g.strideA;
  const float* B = g.B + (int64_t)blockIdx.z * g.strideB;
  float* C = g.C + (int64_t)blockIdx.z * g.strideC;

  int64_t kbeg = 0, kend = g.K;
  if (g.a_upper) kbeg = i0;                                  // rows i >= i0 need k >= i
  if (g.b_upper) kend = (j0 + TN < kend) ? j0 + TN : kend;   // cols j < j0+TN need k <= j
  kbeg = (kbeg / TK) * TK;

  __shared__ __align__(16) float As[2][TK][TM];
  __shared__ __align__(16) float Bs[2][TK][TN];

  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;

  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

  float ra[4], rb[4];
  auto load_regs = [&](int64_t k0) {
    // A slice: 128 rows x 8 k -> As[k][row]
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      int row, kk;
      if (g.transA) { kk = tid >> 5; row = ((tid & 31) << 2) + t; }
      else          { row = tid >> 1; kk = ((tid & 1) << 2) + t; }
      const int64_t i = i0 + row, k = k0 + kk;
      float v = 0.f;
      if (i < g.M && k < kend && k >= 0 && !(g.a_upper && k < i))
        v = g.transA ? __ldg(A + k * g.lda + i) : __ldg(A + i * g.lda + k);
      ra[t] = v;
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      int col, kk;
      if (!g.transB) { kk = tid >> 5; col = ((tid & 31) << 2) + t; }
      else           { col = tid >> 1; kk = ((tid & 1) << 2) + t; }
      const int64_t j = j0 + col, k = k0 + kk;
      float v = 0.f;
      if (j < g.N && k < kend && k >= 0 && !(g.b_upper && k > j))
        v = g.transB ? __ldg(B + j * g.ldb + k) : __ldg(B + k * g.ldb + j);
      rb[t] = v;
    }
  };
  auto store_regs = [&](int buf) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (g.transA) As[buf][tid >> 5][((tid & 31) << 2) + t] = ra[t];
      else          As[buf][((tid & 1) << 2) + t][tid >> 1] = ra[t];
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      if (!g.transB) Bs[buf][tid >> 5][((tid & 31) << 2) + t] = rb[t];
      else           Bs[buf][((tid & 1) << 2) + t][tid >> 1] = rb[t];
    }
  };

  if (kbeg < kend) {
    load_regs(kbeg);
    store_regs(0);
    __syncthreads();
    int buf = 0;
    for (int64_t k0 = kbeg; k0 < kend; k0 += TK) {
      const bool more = k0 + TK < kend;
      if (more) load_regs(k0 + TK);
#pragma unroll
      for (int kk = 0; kk < TK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
        const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            if (ORDERED) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(av[a], bv[b]));
            else acc[a][b] = fmaf(av[a], bv[b], acc[a][b]);
          }
      }
      if (more) {
        store_regs(buf ^ 1);
        __syncthreads();
        buf ^= 1;
      }
    }
  }

#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int64_t i = i0 + (a < 4 ? ty * 4 + a : 64 + ty * 4 + (a - 4));
    if (i >= g.M) continue;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int64_t j = j0 + (b < 4 ? tx * 4 + b : 64 + tx * 4 + (b - 4));
      if (j >= g.N) continue;
      if (g.c_mode != 0 && i > j) continue;
      float* p = C + i * g.ldc + j;
      float v;
      if (ORDERED) v = __fsub_rn(*p, acc[a][b]);
      else v = (g.beta == 0.f) ? g.alpha * acc[a][b] : fmaf(g.alpha, acc[a][b], g.beta * *p);
      *p = v;
      if (g.c_mode == 2 && i < j) C[j * g.ldc + i] = v;
    }
  }
}

}  // namespace

cudaError_t gemm_f32(const GemmDesc& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return cudaSuccess;
  dim3 grid((unsigned)ceil_div(g.N, TN), (unsigned)ceil_div(g.M, TM), (unsigned)g.batch);
  if (g.ordered) gemm_kernel<true><<<grid, NT, 0, s>>>(g);
  else gemm_kernel<false><<<grid, NT, 0, s>>>(g);
  count_launch();
  return cudaGetLastError();
}

}  // namespace kq

// Small reductions: the trace sensitivity (KronQ abstract point (2); README
// bullet "Inter-layer mixed precision": tr(H_G) * tr(H_X)) and the float64
// dot product behind the K-FAC loss diagnostic.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

__device__ double block_sum(double v) {
  __shared__ double red[32];
  v = warp_sum_d(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x < 32) {
    double x = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    x = warp_sum_d(x);
    if (threadIdx.x == 0) red[0] = x;
  }
  __syncthreads();
  const double r = red[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) diag_sum_kernel(const float* HX, int64_t n, const float* HG,
                                                        int64_t m, double* out2) {
  const float* H = blockIdx.x == 0 ? HX : HG;
  const int64_t d = blockIdx.x == 0 ? n : m;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < d; j += blockDim.x) acc += (double)H[j * d + j];
  acc = block_sum(acc);
  if (threadIdx.x == 0) out2[blockIdx.x] = acc;
}

constexpr int DOT_BLOCKS = 592;

__global__ void __launch_bounds__(1024) dot_partial_kernel(const float* a, const float* b,
                                                           int64_t count, double* partial) {
  double acc = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count;
       i += (int64_t)gridDim.x * blockDim.x)
    acc += (double)a[i] * (double)b[i];
  acc = block_sum(acc);
  if (threadIdx.x == 0) partial[blockIdx.x] = acc;
}

__global__ void __launch_bounds__(1024) dot_final_kernel(const double* partial, int cnt, double* out) {
  double acc = 0.0;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) acc += partial[i];
  acc = block_sum(acc);
  if (threadIdx.x == 0) *out = acc;
}

// Sum of squares of a token matrix (T x d, row stride lda), read once:
// tr(A^T A) = sum_t |a_t|^2 without forming A^T A.  Each block reduces a
// contiguous range of rows in float64 into partial[blockIdx.x]; 16-byte
// loads when the rows allow them.
template <bool BF16>
__global__ void __launch_bounds__(512) token_sqsum_kernel(const void* A, int64_t T, int64_t d, int64_t lda,
                                                          int vec, double* partial) {
  double acc = 0.0;
  const int64_t rows_per = (T + gridDim.x - 1) / gridDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * rows_per;
  const int64_t t1 = (t0 + rows_per < T) ? t0 + rows_per : T;
  if (vec) {
    constexpr int E = BF16 ? 8 : 4;               // elements per 16-byte load
    const int64_t dv = d / E;
    for (int64_t t = t0; t < t1; ++t) {
      const uint4* row = reinterpret_cast<const uint4*>(static_cast<const char*>(A) + t * lda * (BF16 ? 2 : 4));
      for (int64_t c = threadIdx.x; c < dv; c += blockDim.x) {
        const uint4 w = row[c];
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (BF16) {
            const double lo = (double)__uint_as_float(u[q] << 16), hi = (double)__uint_as_float(u[q] & 0xFFFF0000u);
            acc += lo * lo + hi * hi;
          } else {
            const double x = (double)__uint_as_float(u[q]);
            acc += x * x;
          }
        }
      }
    }
  } else {
    for (int64_t t = t0; t < t1; ++t)
      for (int64_t c = threadIdx.x; c < d; c += blockDim.x) {
        const double x = BF16 ? (double)__bfloat162float(static_cast<const __nv_bfloat16*>(A)[t * lda + c])
                              : (double)static_cast<const float*>(A)[t * lda + c];
        acc += x * x;
      }
  }
  acc = block_sum(acc);
  if (threadIdx.x == 0) partial[blockIdx.x] = acc;
}

// out (+)= sum of the partials, in a fixed order (deterministic).
__global__ void __launch_bounds__(1024) sum_into_kernel(const double* partial, int cnt, double* out, int zero_first) {
  double acc = 0.0;
  for (int i = threadIdx.x; i < cnt; i += blockDim.x) acc += partial[i];
  acc = block_sum(acc);
  if (threadIdx.x == 0) *out = zero_first ? acc : *out + acc;
}

}  // namespace

size_t token_sqsum_partials() { return DOT_BLOCKS; }

kronq_status token_sqsum(const void* A, bool bf16, int64_t T, int64_t d, int64_t lda, double* out,
                         int zero_first, double* partial, cudaStream_t s) {
  const int E = bf16 ? 8 : 4;
  const int vec = (aligned(A, 16) && (d % E) == 0 && (lda % E) == 0) ? 1 : 0;
  if (bf16) token_sqsum_kernel<true><<<DOT_BLOCKS, 512, 0, s>>>(A, T, d, lda, vec, partial);
  else token_sqsum_kernel<false><<<DOT_BLOCKS, 512, 0, s>>>(A, T, d, lda, vec, partial);
  KQ_LAUNCH_CHECK("token_sqsum_kernel");
  sum_into_kernel<<<1, 1024, 0, s>>>(partial, DOT_BLOCKS, out, zero_first);
  KQ_LAUNCH_CHECK("sum_into_kernel");
  return KRONQ_OK;
}

kronq_status diag_sums(const float* HX, int64_t n, const float* HG, int64_t m, double* dev2,
                       cudaStream_t s) {
  diag_sum_kernel<<<2, 1024, 0, s>>>(HX, n, HG, m, dev2);
  KQ_LAUNCH_CHECK("diag_sum_kernel");
  return KRONQ_OK;
}

kronq_status dot_sum(const float* a, const float* b, int64_t count, double* dev1, double* partial,
                     cudaStream_t s) {
  dot_partial_kernel<<<DOT_BLOCKS, 1024, 0, s>>>(a, b, count, partial);
  KQ_LAUNCH_CHECK("dot_partial_kernel");
  dot_final_kernel<<<1, 1024, 0, s>>>(partial, DOT_BLOCKS, dev1);
  KQ_LAUNCH_CHECK("dot_final_kernel");
  return KRONQ_OK;
}

}  // namespace kq

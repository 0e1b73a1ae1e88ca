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

}  // namespace

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

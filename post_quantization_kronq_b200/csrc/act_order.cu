// The recipe's act-order option on the GPU (KronQ README, "Reproduce from
// scratch": --act_order; the pages do not define it, the reading taken is
// GPTQ's published heuristic):
//
//   after the dead-column rule, the columns are swept in order of
//   decreasing diagonal of H~_X (ties keep the column order); groups are
//   consecutive columns of that order; codes, the dequantised W~ and the
//   scaled errors come back in the original column order, and column j
//   uses the scale and zero of group g_idx[j] = rank(j) / group.
//
// Steps: the rank of every column from the diagonal (a comparison count,
// one thread per column), the dead-column rule and damping in place, the
// symmetric permutation of H~_X and the column permutation of W~ into the
// workspace, the plain pass (factorisation and sweep) on the permuted
// problem, and the scatter of its outputs back to the original order.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

// rank[j] = #{i : d_i > d_j} + #{i < j : d_i == d_j} with d the diagonal
// after the dead-column rule (a zero diagonal counts as 1); perm[rank[j]] = j;
// g_idx[j] = rank[j] / group (0 for one group per row).
__global__ void __launch_bounds__(256) act_rank_kernel(const float* H, int64_t n, int group, int* rank,
                                                       int* perm, int* g_idx) {
  __shared__ float dsh[1024];
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  float dj = 0.f;
  if (j < n) {
    dj = H[j * n + j];
    if (dj == 0.f) dj = 1.f;
  }
  int r = 0;
  for (int64_t i0 = 0; i0 < n; i0 += 1024) {
    __syncthreads();
    for (int t = threadIdx.x; t < 1024; t += blockDim.x) {
      const int64_t i = i0 + t;
      float di = 0.f;
      if (i < n) {
        di = H[i * n + i];
        if (di == 0.f) di = 1.f;
      }
      dsh[t] = di;
    }
    __syncthreads();
    const int cnt = (int)((n - i0) < 1024 ? (n - i0) : 1024);
    if (j < n)
      for (int t = 0; t < cnt; ++t) {
        const float di = dsh[t];
        r += (di > dj || (di == dj && i0 + t < j)) ? 1 : 0;
      }
  }
  if (j < n) {
    rank[j] = r;
    perm[r] = (int)j;
    g_idx[j] = group > 0 ? r / group : 0;
  }
}

// P[r][c] = H[perm[r]][perm[c]] (one CTA per row, grid-stride).
__global__ void __launch_bounds__(256) permute_sym_kernel(const float* H, int64_t n, const int* perm, float* P) {
  for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
    const float* src = H + (int64_t)perm[r] * n;
    float* dst = P + r * n;
    for (int64_t c = threadIdx.x; c < n; c += blockDim.x) dst[c] = src[perm[c]];
  }
}

// Wp[i][k] = dead[perm[k]] ? 0 : W[i][perm[k]].
__global__ void __launch_bounds__(256) permute_cols_kernel(const float* W, int64_t m, int64_t n, const int* perm,
                                                           const uint8_t* dead, float* Wp) {
  for (int64_t i = blockIdx.x; i < m; i += gridDim.x)
    for (int64_t k = threadIdx.x; k < n; k += blockDim.x) {
      const int j = perm[k];
      Wp[i * n + k] = dead[j] ? 0.f : W[i * n + j];
    }
}

// out[i][perm[k]] = in[i][k] for float and byte matrices.
template <typename T>
__global__ void __launch_bounds__(256) unpermute_cols_kernel(const T* in, int64_t m, int64_t n, const int* perm,
                                                             T* out) {
  for (int64_t i = blockIdx.x; i < m; i += gridDim.x)
    for (int64_t k = threadIdx.x; k < n; k += blockDim.x) out[i * n + perm[k]] = in[i * n + k];
}

__global__ void copy_f32_kernel(float* dst, const float* src, int64_t count) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < count; t += (int64_t)gridDim.x * blockDim.x)
    dst[t] = src[t];
}

struct ActCarve {
  float* P;
  float* Wp;
  float* Ep;
  uint8_t* codes_p;
  int* rank;
  int* perm;
  uint8_t* dead;
  void* inner;
  size_t total;
};

ActCarve act_carve(void* base, int64_t m, int64_t n, bool with_e, bool rform) {
  ActCarve c;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    off = (off + 255) & ~size_t(255);
    void* p = base ? static_cast<uint8_t*>(base) + off : nullptr;
    off += bytes;
    return p;
  };
  c.P = static_cast<float*>(take((size_t)n * n * sizeof(float)));
  c.Wp = static_cast<float*>(take((size_t)m * n * sizeof(float)));
  c.Ep = with_e ? static_cast<float*>(take((size_t)m * n * sizeof(float))) : nullptr;
  c.codes_p = static_cast<uint8_t*>(take((size_t)m * n));
  c.rank = static_cast<int*>(take((size_t)n * sizeof(int)));
  c.perm = static_cast<int*>(take((size_t)n * sizeof(int)));
  c.dead = static_cast<uint8_t*>(take((size_t)n));
  c.inner = take(quantize_core_workspace_bytes(m, n, rform));
  c.total = (off + 255) & ~size_t(255);
  return c;
}

}  // namespace
}  // namespace kq

using namespace kq;

extern "C" {

size_t kronq_quantize_act_order_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p) {
  if (m <= 0 || n <= 0) return 0;
  const bool with_e = p && (p->flags & KRONQ_WRITE_E);
  return act_carve(nullptr, m, n, with_e, p && (p->flags & KRONQ_R_FORM)).total;
}

kronq_status kronq_quantize_layer_act_order(float* Wt, float* HX, int64_t m, int64_t n,
                                            const kronq_quant_params* p, uint8_t* codes, float* scales,
                                            float* zeros, float* E, int* g_idx, int* perm, int* info,
                                            void* workspace, size_t ws_bytes, kronq_stream_t s) {
  kronq_status v = check_quant_args(Wt, HX, m, n, p, codes, scales, zeros, E, info, "quantize_layer_act_order");
  if (v != KRONQ_OK) return v;
  if (p->flags & KRONQ_U_GIVEN)
    return fail(KRONQ_ERR_INVALID_ARG, "quantize_layer_act_order: the sweep order comes from H~_X, not from U");
  if (!g_idx) return fail(KRONQ_ERR_INVALID_ARG, "quantize_layer_act_order: g_idx is NULL");
  const bool with_e = (p->flags & KRONQ_WRITE_E) != 0;
  ActCarve c = act_carve(workspace, m, n, with_e, (p->flags & KRONQ_R_FORM) != 0);
  if (!workspace || ws_bytes < c.total || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "quantize_layer_act_order: workspace too small or not 256-byte aligned");
  cudaStream_t st = as_stream(s);
  // 1. the sweep order from the diagonal (dead columns count as 1)
  act_rank_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, st>>>(HX, n, p->group, c.rank, c.perm, g_idx);
  KQ_LAUNCH_CHECK("act_rank_kernel");
  // 2. dead columns and damping in the original order (the mean diagonal
  //    does not depend on the order), then the permuted copies
  kronq_status r = damp_factor(HX, n, p->damp_rel, c.dead, info, st);
  if (r != KRONQ_OK) return r;
  const int grid = 4 * sm_count();
  permute_sym_kernel<<<grid, 256, 0, st>>>(HX, n, c.perm, c.P);
  KQ_LAUNCH_CHECK("permute_sym_kernel");
  permute_cols_kernel<<<grid, 256, 0, st>>>(Wt, m, n, c.perm, c.dead, c.Wp);
  KQ_LAUNCH_CHECK("permute_cols_kernel");
  // 3. the plain pass on the permuted problem (already damped)
  r = quantize_core(c.Wp, c.P, m, n, p, c.codes_p, scales, zeros, c.Ep, info, c.inner, st, 2);
  if (r != KRONQ_OK) return r;
  // 4. outputs back to the original column order; U or R (of the sweep
  //    order) to HX
  unpermute_cols_kernel<float><<<grid, 256, 0, st>>>(c.Wp, m, n, c.perm, Wt);
  KQ_LAUNCH_CHECK("unpermute_cols_kernel");
  unpermute_cols_kernel<uint8_t><<<grid, 256, 0, st>>>(c.codes_p, m, n, c.perm, codes);
  KQ_LAUNCH_CHECK("unpermute_cols_kernel");
  if (with_e) {
    unpermute_cols_kernel<float><<<grid, 256, 0, st>>>(c.Ep, m, n, c.perm, E);
    KQ_LAUNCH_CHECK("unpermute_cols_kernel");
  }
  copy_f32_kernel<<<grid, 256, 0, st>>>(HX, c.P, n * n);
  KQ_LAUNCH_CHECK("copy_f32_kernel");
  if (perm) {
    cudaError_t e = cudaMemcpyAsync(perm, c.perm, (size_t)n * sizeof(int), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(perm)");
  }
  return KRONQ_OK;
}

}  // extern "C"

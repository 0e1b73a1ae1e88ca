// Kronecker factor estimators A (x) B ~ H = E[x x^T (x) g g^T]: the input,
// marginal, Frobenius and FlipFlop rows of Table 1 of the "WaterKron and
// FlipFlop Hessian" page, Frobenius and FlipFlop by the alternating
// fixed-point iteration from the identity (the table's caption), each update
// the exact minimiser of the row's target over one factor.
//
// One update, say A from B, is a weighted second moment of the tokens x with
// per-token weights w_t = g_t^T M g_t:
//   Frobenius  M = B,      A = E[w x x^T] / ||B||_F^2
//   FlipFlop   M = B^-1,   A = E[w x x^T] / m,  w_t = |U g_t|^2, U^T U = B^-1
// Per chunk of tokens:
//   1. Y = -G_chunk Op on the tensor cores (the trailing-update kernel of the
//      sweep: Op is split into bf16 hi/lo, the tokens are exact in bf16;
//      passing the tokens as both splits and hi/2 as the high split gives
//      G hi/2 + G lo + G hi/2 = G (hi + lo) with the kernel's three products).
//      Op = U^T (FlipFlop, U from the reverse Cholesky factorisation and
//      triangular inverse of B) or B (Frobenius).
//   2. w_t = c sum_i Y_ti^2 (FlipFlop) or c sum_i (-Y_ti) G_ti (Frobenius),
//      with the constant c of the row folded in.
//   3. The tokens scaled by sqrt(w_t), rounded to bf16, accumulate into A by
//      the tensor-core SYRK of the factor accumulation.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int64_t EST_CHUNK = 16384;   // tokens per chunk of the weighted moment

__global__ void eye_kernel(float* M, int64_t d) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < d * d; i += (int64_t)gridDim.x * blockDim.x)
    M[i] = (i / d == i % d) ? 1.f : 0.f;
}

__global__ void scale_kernel(float* M, int64_t count, float c) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    M[i] *= c;
}

// out = sum of squares of M (one CTA; double accumulation).
__global__ void __launch_bounds__(1024) sumsq_kernel(const float* M, int64_t count, float* out) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < count; i += blockDim.x) {
    const double v = M[i];
    s += v * v;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) *out = (float)s;
  }
}

// Operand of the weight product, K x N = d x d (row j, column i), as bf16
// splits: hi/2 and lo of Op[j][i] = F[i][j] for j >= i, else 0 (upper_t: F
// holds U in its upper triangle, scratch below) or Op[j][i] = F[j][i].
__global__ void op_split_kernel(const float* F, int64_t d, int upper_t, __nv_bfloat16* Oh,
                                __nv_bfloat16* Ol) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < d * d; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = t / d, i = t - j * d;
    const float v = upper_t ? (j >= i ? F[i * d + j] : 0.f) : F[t];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const float hf = __bfloat162float(h);
    Oh[t] = __float2bfloat16_rn(0.5f * hf);
    Ol[t] = __float2bfloat16_rn(v - hf);
  }
}

// Per-token weight from Y = -G Op: one warp per token.
// square: w = c sum Y^2; else w = c sum (-Y) g (clamped at 0).  c = c_host,
// divided by *c_div when c_div is not null.
__global__ void weights_kernel(const float* Y, const __nv_bfloat16* Gc, int64_t rows, int64_t d, int square,
                               float c_host, const float* c_div, float* w) {
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= rows) return;
  const float* y = Y + t * d;
  const __nv_bfloat16* g = Gc + t * d;
  float s = 0.f;
  for (int64_t i = lane; i < d; i += 32) s += square ? y[i] * y[i] : -y[i] * __bfloat162float(g[i]);
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    float c = c_host;
    if (c_div) c = c / *c_div;
    w[t] = fmaxf(s, 0.f) * c;
  }
}

// Zs[t][:] = bf16(sqrt(w_t) Z[t][:]).
__global__ void scale_rows_kernel(const __nv_bfloat16* Z, int64_t rows, int64_t d, const float* w,
                                  __nv_bfloat16* Zs) {
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < rows * d; t += (int64_t)gridDim.x * blockDim.x) {
    const float s = sqrtf(w[t / d]);
    Zs[t] = __float2bfloat16_rn(s * __bfloat162float(Z[t]));
  }
}

// info |= the factorisation's status (the first failure is kept).
__global__ void merge_info_kernel(int* info, const int* step_info) {
  if (*info == 0 && *step_info != 0) *info = *step_info;
}

inline unsigned grid_for(int64_t count) {
  const int64_t g = ceil_div(count, 256);
  return (unsigned)(g < 4 * (int64_t)sm_count() ? (g > 0 ? g : 1) : 4 * (int64_t)sm_count());
}

struct EstWs {
  float* Y;              // chunk x d
  __nv_bfloat16* Zs;     // chunk x d
  __nv_bfloat16* Oh;     // d x d
  __nv_bfloat16* Ol;     // d x d
  float* F;              // d x d (factor copy for the Cholesky path)
  float* w;              // chunk
  float* nrm;            // 1
  int* step_info;        // 1
  void* chol;            // chol_workspace_bytes(d)
};

size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

size_t est_layout(int64_t T, int64_t n, int64_t m, uint8_t* base, EstWs* ws) {
  const int64_t d = n > m ? n : m;
  const int64_t chunk = T < EST_CHUNK ? (T > 0 ? T : 1) : EST_CHUNK;
  const size_t sizes[9] = {align256(chunk * d * 4), align256(chunk * d * 2), align256(d * d * 2),
                           align256(d * d * 2),     align256(d * d * 4),     align256(chunk * 4),
                           256, 256, align256(chol_workspace_bytes(d))};
  size_t off = 0;
  void* p[9];
  for (int i = 0; i < 9; ++i) {
    p[i] = base ? base + off : nullptr;
    off += sizes[i];
  }
  if (ws) {
    ws->Y = static_cast<float*>(p[0]);
    ws->Zs = static_cast<__nv_bfloat16*>(p[1]);
    ws->Oh = static_cast<__nv_bfloat16*>(p[2]);
    ws->Ol = static_cast<__nv_bfloat16*>(p[3]);
    ws->F = static_cast<float*>(p[4]);
    ws->w = static_cast<float*>(p[5]);
    ws->nrm = static_cast<float*>(p[6]);
    ws->step_info = static_cast<int*>(p[7]);
    ws->chol = p[8];
  }
  return off;
}

// out (dz x dz) = E[w z z^T] with w_t = weight of token t from the other
// side's tokens Gs (T x dg) and factor Fo (dg x dg).
kronq_status weighted_moment(const __nv_bfloat16* Z, int64_t dz, const __nv_bfloat16* Gs, int64_t dg,
                             int64_t T, const float* Fo, bool flipflop, float* out, int* info,
                             const EstWs& ws, cudaStream_t s) {
  if (flipflop) {
    KQ_CUDA(cudaMemcpyAsync(ws.F, Fo, dg * dg * sizeof(float), cudaMemcpyDeviceToDevice, s));
    kronq_status r = chol_upper_inverse(ws.F, dg, 0.f, true, nullptr, ws.step_info, ws.chol, s);
    if (r != KRONQ_OK) return r;
    merge_info_kernel<<<1, 1, 0, s>>>(info, ws.step_info);
    KQ_LAUNCH_CHECK("merge_info_kernel");
    op_split_kernel<<<grid_for(dg * dg), 256, 0, s>>>(ws.F, dg, 1, ws.Oh, ws.Ol);
    KQ_LAUNCH_CHECK("op_split_kernel");
  } else {
    sumsq_kernel<<<1, 1024, 0, s>>>(Fo, dg * dg, ws.nrm);
    KQ_LAUNCH_CHECK("sumsq_kernel");
    op_split_kernel<<<grid_for(dg * dg), 256, 0, s>>>(Fo, dg, 0, ws.Oh, ws.Ol);
    KQ_LAUNCH_CHECK("op_split_kernel");
  }
  const float c_host = flipflop ? (float)(1.0 / ((double)T * (double)dg)) : (float)(1.0 / (double)T);
  for (int64_t t0 = 0; t0 < T; t0 += EST_CHUNK) {
    const int64_t rows = (T - t0) < EST_CHUNK ? (T - t0) : EST_CHUNK;
    const __nv_bfloat16* gc = Gs + t0 * dg;
    TrailingMaps maps;
    kronq_status r = trailing_maps(&maps, gc, gc, rows, dg, ws.Oh, ws.Ol, dg, dg, ws.Y, dg);
    if (r != KRONQ_OK) return r;
    KQ_CUDA(cudaMemsetAsync(ws.Y, 0, rows * dg * sizeof(float), s));
    r = trailing_update_tc(&maps, ws.Y, rows, dg, 0, dg, 0, dg, info, s);
    if (r != KRONQ_OK) return r;
    weights_kernel<<<(unsigned)ceil_div(rows, 8), 256, 0, s>>>(ws.Y, gc, rows, dg, flipflop ? 1 : 0, c_host,
                                                               flipflop ? nullptr : ws.nrm, ws.w);
    KQ_LAUNCH_CHECK("weights_kernel");
    scale_rows_kernel<<<grid_for(rows * dz), 256, 0, s>>>(Z + t0 * dz, rows, dz, ws.w, ws.Zs);
    KQ_LAUNCH_CHECK("scale_rows_kernel");
    r = kronq_accumulate_factors(ws.Zs, KRONQ_BF16, rows, dz, dz, out, t0 == 0 ? 1 : 0,
                                 reinterpret_cast<kronq_stream_t>(s));
    if (r != KRONQ_OK) return r;
  }
  return KRONQ_OK;
}

}  // namespace
}  // namespace kq

using namespace kq;

extern "C" {

size_t kronq_kron_factors_workspace_bytes(int64_t T, int64_t n, int64_t m) {
  if (T < 0 || n <= 0 || m <= 0) return 0;
  return est_layout(T, n, m, nullptr, nullptr);
}

kronq_status kronq_kron_factors(const void* X, const void* G, int64_t T, int64_t n, int64_t m,
                                kronq_estimator est, int iters, float* A, float* B, int* info,
                                void* workspace, size_t ws_bytes, kronq_stream_t s) {
  if (est < KRONQ_EST_INPUT || est > KRONQ_EST_FLIPFLOP)
    return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: unknown estimator");
  if (T <= 0 || n < 64 || m < 64 || (n % 8) != 0 || (m % 8) != 0 || n > 65536 || m > 65536 ||
      T > ((int64_t)1 << 31) - 64)
    return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: need T > 0 and 64 <= n, m <= 65536, multiples of 8");
  if (!X || !G || !A || !B || !info) return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: NULL pointer");
  if (!aligned(X, 16) || !aligned(G, 16)) return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: X, G not 16-byte aligned");
  if (iters < 0) return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: iters < 0");
  const size_t need = kronq_kron_factors_workspace_bytes(T, n, m);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "kron_factors: workspace too small or not 256-byte aligned");
  cudaStream_t st = as_stream(s);
  EstWs ws;
  est_layout(T, n, m, static_cast<uint8_t*>(workspace), &ws);
  KQ_CUDA(cudaMemsetAsync(info, 0, sizeof(int), st));
  const auto* Xb = static_cast<const __nv_bfloat16*>(X);
  const auto* Gb = static_cast<const __nv_bfloat16*>(G);
  const float inv_t = (float)(1.0 / (double)T);
  if (est == KRONQ_EST_INPUT || est == KRONQ_EST_MARGINAL) {
    kronq_status r = kronq_accumulate_factors(X, KRONQ_BF16, T, n, n, A, 1, s);
    if (r != KRONQ_OK) return r;
    scale_kernel<<<grid_for(n * n), 256, 0, st>>>(A, n * n, inv_t);
    KQ_LAUNCH_CHECK("scale_kernel");
    if (est == KRONQ_EST_INPUT) {
      eye_kernel<<<grid_for(m * m), 256, 0, st>>>(B, m);
      KQ_LAUNCH_CHECK("eye_kernel");
      return KRONQ_OK;
    }
    r = kronq_accumulate_factors(G, KRONQ_BF16, T, m, m, B, 1, s);
    if (r != KRONQ_OK) return r;
    scale_kernel<<<grid_for(m * m), 256, 0, st>>>(B, m * m, inv_t);
    KQ_LAUNCH_CHECK("scale_kernel");
    return KRONQ_OK;
  }
  const bool ff = est == KRONQ_EST_FLIPFLOP;
  eye_kernel<<<grid_for(m * m), 256, 0, st>>>(B, m);
  KQ_LAUNCH_CHECK("eye_kernel");
  if (iters == 0) {
    eye_kernel<<<grid_for(n * n), 256, 0, st>>>(A, n);
    KQ_LAUNCH_CHECK("eye_kernel");
    return KRONQ_OK;
  }
  for (int it = 0; it < iters; ++it) {
    kronq_status r = weighted_moment(Xb, n, Gb, m, T, B, ff, A, info, ws, st);
    if (r != KRONQ_OK) return r;
    r = weighted_moment(Gb, m, Xb, n, T, A, ff, B, info, ws, st);
    if (r != KRONQ_OK) return r;
  }
  return KRONQ_OK;
}

}  // extern "C"

// extern "C" surface of libkronq: argument validation on the host, then
// dispatch to the kernels of the other translation units.  Nothing here
// computes on the host except the bit allocation (a host-only call).
#include <math.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace kq {

static thread_local std::string g_last_error;
static std::atomic<unsigned long long> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void set_error(const std::string& msg) { g_last_error = msg; }

kronq_status fail(kronq_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}

kronq_status cuda_fail(cudaError_t e, const char* what) {
  g_last_error = std::string(what) + ": " + cudaGetErrorString(e);
  return KRONQ_ERR_CUDA;
}

int sm_count() {
  int dev = 0, v = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
  return v;
}

cudaError_t allow_smem(const void* func, int bytes) {
  return cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

namespace {

// Workspace carving: 256-byte aligned slices.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
  size_t size() const { return (off + 255) & ~size_t(255); }
};

// Small-shape bf16 factor kernel (one thread per upper entry).
__global__ void syrk_small_bf16_kernel(const __nv_bfloat16* A, int64_t T, int64_t d, int64_t lda,
                                       float* H, int zero_first) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t tot = d * d;
  if (t >= tot) return;
  const int64_t i = t / d, j = t - i * d;
  if (i > j) return;
  float acc = 0.f;
  for (int64_t k = 0; k < T; ++k)
    acc = fmaf(__bfloat162float(A[k * lda + i]), __bfloat162float(A[k * lda + j]), acc);
  float v = zero_first ? acc : H[i * d + j] + acc;
  H[i * d + j] = v;
  if (i != j) H[j * d + i] = v;
}

bool valid_mode(int mode) { return mode >= 0 && mode <= 3; }

int64_t odd_part(int64_t L) {
  while (L % 2 == 0) L /= 2;
  return L;
}

size_t biip_ws(int64_t m, int64_t n) {
  Carver c(nullptr);
  int64_t big = m * n;
  if (n * n > big) big = n * n;
  if (m * m > big) big = m * m;
  c.take<float>((size_t)big);
  c.take<float>((size_t)n);
  c.take<float>((size_t)m);
  c.take<float>(wnorms_partial_floats(m, n));
  c.take<float>((size_t)(m > n ? m : n));   // column factors of one row pass
  return c.size();
}

int64_t quant_ldu(int64_t n) { return (n + 7) / 8 * 8; }

// Blocks per group of the two-level trailing update: up to eight (K = 1024).
int64_t quant_gblocks(int64_t n) {
  const int64_t nblk = ceil_div(n, 128);
  return nblk < 8 ? (nblk < 1 ? 1 : nblk) : 8;
}

size_t quant_ws(int64_t m, int64_t n, bool rform) {
  Carver c(nullptr);
  c.take<uint8_t>(chol_workspace_bytes(n));
  c.take<uint8_t>((size_t)n);
  c.take<float>((size_t)(m * 128));
  const int64_t kg = 128 * quant_gblocks(n);
  c.take<__nv_bfloat16>((size_t)(m * kg));
  c.take<__nv_bfloat16>((size_t)(m * kg));
  c.take<__nv_bfloat16>((size_t)(kg * quant_ldu(n)));
  c.take<__nv_bfloat16>((size_t)(kg * quant_ldu(n)));
  if (rform) {
    c.take<float>((size_t)(m * n));                        // W~ before the sweep
    c.take<float>((size_t)(128 * 128 * ceil_div(n, 128)));  // diagonal blocks of U
  }
  return c.size();
}

bool wants_rform(const kronq_quant_params* p) { return p && (p->flags & KRONQ_R_FORM) != 0; }

}  // namespace
}  // namespace kq

using namespace kq;

extern "C" {

const char* kronq_last_error(void) { return g_last_error.c_str(); }

const char* kronq_version(void) { return "kronq-b200 0.1 (sm_100a)"; }

uint64_t kronq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

kronq_status kronq_accumulate_factors(const void* A, kronq_dtype dt, int64_t T, int64_t d,
                                      int64_t lda, float* H, int zero_first, kronq_stream_t s) {
  if (dt != KRONQ_BF16 && dt != KRONQ_F32) return fail(KRONQ_ERR_INVALID_ARG, "accumulate_factors: bad dtype");
  if (d <= 0 || T < 0 || lda < d) return fail(KRONQ_ERR_INVALID_ARG, "accumulate_factors: need d > 0, T >= 0, lda >= d");
  if (!H) return fail(KRONQ_ERR_INVALID_ARG, "accumulate_factors: H is NULL");
  if (T > 0 && !A) return fail(KRONQ_ERR_INVALID_ARG, "accumulate_factors: A is NULL");
  if (d > (int64_t)1 << 20 || T > ((int64_t)1 << 31) - 64)
    return fail(KRONQ_ERR_INVALID_ARG, "accumulate_factors: size out of range");
  cudaStream_t st = as_stream(s);
  if (T == 0) {
    if (zero_first) {
      cudaError_t e = fill_f32(H, d * d, 0.f, st);
      if (e != cudaSuccess) return cuda_fail(e, "fill");
    }
    return KRONQ_OK;
  }
  if (dt == KRONQ_F32) {
    GemmDesc g;
    g.M = d; g.N = d; g.K = T;
    g.A = static_cast<const float*>(A); g.lda = lda; g.transA = true;
    g.B = static_cast<const float*>(A); g.ldb = lda; g.transB = false;
    g.C = H; g.ldc = d;
    g.alpha = 1.f; g.beta = zero_first ? 0.f : 1.f;
    g.c_mode = 2;
    cudaError_t e = gemm_f32(g, st);
    if (e != cudaSuccess) return cuda_fail(e, "gemm(factor f32)");
    return KRONQ_OK;
  }
  const bool tc_ok = d >= 128 && T >= 64 && aligned(A, 16) && (lda % 8) == 0;
  if (tc_ok) return syrk_bf16_tc(A, T, d, lda, H, zero_first != 0, st);
  const int64_t tot = d * d;
  syrk_small_bf16_kernel<<<(unsigned)ceil_div(tot, 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(A), T, d, lda, H, zero_first);
  KQ_LAUNCH_CHECK("syrk_small_bf16_kernel");
  return KRONQ_OK;
}

kronq_status kronq_sensitivity(const float* HX, int64_t n, const float* HG, int64_t m, double* out3,
                               void* workspace, size_t ws_bytes, kronq_stream_t s) {
  if (!HX || !HG || !out3 || n <= 0 || m <= 0)
    return fail(KRONQ_ERR_INVALID_ARG, "sensitivity: NULL pointer or non-positive size");
  if (!workspace || ws_bytes < 16 || !aligned(workspace, 8))
    return fail(KRONQ_ERR_INVALID_ARG, "sensitivity: workspace must hold 16 bytes, 8-byte aligned");
  cudaStream_t st = as_stream(s);
  double* dev2 = static_cast<double*>(workspace);
  kronq_status r = diag_sums(HX, n, HG, m, dev2, st);
  if (r != KRONQ_OK) return r;
  double h[2];
  KQ_CUDA(cudaMemcpyAsync(h, dev2, sizeof(h), cudaMemcpyDeviceToHost, st));
  KQ_CUDA(cudaStreamSynchronize(st));
  out3[0] = h[0];
  out3[1] = h[1];
  out3[2] = h[1] * h[0];
  return KRONQ_OK;
}

size_t kronq_trace_tokens_workspace_bytes(void) {
  return ((token_sqsum_partials() * sizeof(double)) + 255) & ~size_t(255);
}

kronq_status kronq_trace_tokens(const void* A, kronq_dtype dt, int64_t T, int64_t d, int64_t lda,
                                double* trace, int zero_first, void* workspace, size_t ws_bytes,
                                kronq_stream_t s) {
  if (dt != KRONQ_BF16 && dt != KRONQ_F32) return fail(KRONQ_ERR_INVALID_ARG, "trace_tokens: bad dtype");
  if (d <= 0 || T < 0 || lda < d) return fail(KRONQ_ERR_INVALID_ARG, "trace_tokens: need d > 0, T >= 0, lda >= d");
  if (!trace || (T > 0 && !A)) return fail(KRONQ_ERR_INVALID_ARG, "trace_tokens: NULL pointer");
  if (!aligned(trace, 8)) return fail(KRONQ_ERR_INVALID_ARG, "trace_tokens: trace must be 8-byte aligned");
  if (!workspace || ws_bytes < kronq_trace_tokens_workspace_bytes() || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "trace_tokens: workspace too small or not 256-byte aligned");
  return token_sqsum(A, dt == KRONQ_BF16, T, d, lda, trace, zero_first, static_cast<double*>(workspace),
                     as_stream(s));
}

kronq_status kronq_sensitivity_from_traces(const double* traces, double* out3, kronq_stream_t s) {
  if (!traces || !out3) return fail(KRONQ_ERR_INVALID_ARG, "sensitivity_from_traces: NULL pointer");
  cudaStream_t st = as_stream(s);
  double h[2];
  KQ_CUDA(cudaMemcpyAsync(h, traces, sizeof(h), cudaMemcpyDeviceToHost, st));
  KQ_CUDA(cudaStreamSynchronize(st));
  out3[0] = h[0];
  out3[1] = h[1];
  out3[2] = h[1] * h[0];
  return KRONQ_OK;
}

kronq_status kronq_allocate_bits(const double* sens, const int64_t* sizes, int L, double avg_bits,
                                 int bmin, int bmax, int* bits_out) {
  if (L < 0 || (L > 0 && (!sens || !sizes || !bits_out)))
    return fail(KRONQ_ERR_INVALID_ARG, "allocate_bits: bad arrays");
  if (bmin < 1 || bmax < bmin || bmax > 8 || !(avg_bits >= bmin))
    return fail(KRONQ_ERR_INVALID_ARG, "allocate_bits: need 1 <= bmin <= bmax <= 8 and avg_bits >= bmin");
  double total = 0.0;
  for (int i = 0; i < L; ++i) {
    if (sizes[i] <= 0 || !(sens[i] >= 0.0)) return fail(KRONQ_ERR_INVALID_ARG, "allocate_bits: bad size or sensitivity");
    total += (double)sizes[i];
  }
  const double budget = avg_bits * total;
  double used = (double)bmin * total;
  for (int i = 0; i < L; ++i) bits_out[i] = bmin;
  for (;;) {
    int best = -1;
    double best_gain = 0.0;
    for (int i = 0; i < L; ++i) {
      if (bits_out[i] >= bmax || used + (double)sizes[i] > budget) continue;
      const double gain = sens[i] * (ldexp(1.0, -2 * bits_out[i]) - ldexp(1.0, -2 * (bits_out[i] + 1))) /
                          (double)sizes[i];
      if (best < 0 || gain > best_gain) {
        best = i;
        best_gain = gain;
      }
    }
    if (best < 0) break;
    bits_out[best] += 1;
    used += (double)sizes[best];
  }
  return KRONQ_OK;
}

kronq_status kronq_allocate_topn_types(const double* sens, const int* type_ids, int L, int n_types,
                                       int base_bits, int N, int* bits_out) {
  if (L < 0 || n_types <= 0 || N < 0 || (L > 0 && (!sens || !type_ids || !bits_out)))
    return fail(KRONQ_ERR_INVALID_ARG, "allocate_topn_types: bad arguments");
  if (base_bits < 1 || base_bits > 7) return fail(KRONQ_ERR_INVALID_ARG, "allocate_topn_types: bad base_bits");
  std::vector<double> tot((size_t)n_types, 0.0);
  for (int i = 0; i < L; ++i) {
    if (type_ids[i] < 0 || type_ids[i] >= n_types) return fail(KRONQ_ERR_INVALID_ARG, "allocate_topn_types: bad type id");
    tot[(size_t)type_ids[i]] += sens[i];
  }
  std::vector<char> top((size_t)n_types, 0);
  for (int k = 0; k < N && k < n_types; ++k) {
    int best = -1;
    for (int t = 0; t < n_types; ++t)
      if (!top[(size_t)t] && (best < 0 || tot[(size_t)t] > tot[(size_t)best])) best = t;
    top[(size_t)best] = 1;
  }
  for (int i = 0; i < L; ++i) bits_out[i] = base_bits + (top[(size_t)type_ids[i]] ? 1 : 0);
  return KRONQ_OK;
}

size_t kronq_biip_workspace_bytes(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  return biip_ws(m, n);
}

kronq_status kronq_biip_forward(const void* W, kronq_dtype wdt, float* Wt, int64_t m, int64_t n,
                                float* HX, float* HG, uint64_t seed, float alpha,
                                kronq_biip_mode mode, float* d_in, float* d_out, void* workspace,
                                size_t ws_bytes, kronq_stream_t s) {
  if (!W || !Wt || !HX || !d_in || !d_out || m <= 0 || n <= 0)
    return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: NULL pointer or non-positive size");
  if (wdt != KRONQ_BF16 && wdt != KRONQ_F32) return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: bad dtype");
  if (!valid_mode(mode)) return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: bad mode");
  if (!isfinite(alpha)) return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: alpha not finite");
  if (W == static_cast<const void*>(Wt)) return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: W and Wt alias");
  const bool use_in = mode != KRONQ_BIIP_SU_ONLY;
  const bool use_out = mode != KRONQ_BIIP_SV_ONLY;
  const bool rescale = mode != KRONQ_BIIP_NO_RESCALE;
  if (!HG && (mode == KRONQ_BIIP_FULL || mode == KRONQ_BIIP_SU_ONLY))
    return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: H_G is required for the output-side rescale");
  if ((use_in && odd_part(n) > 255) || (use_out && odd_part(m) > 255))
    return fail(KRONQ_ERR_UNSUPPORTED, "biip_forward: odd factor of a rotated dimension exceeds 255");
  if (!workspace || ws_bytes < biip_ws(m, n) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "biip_forward: workspace too small or not 256-byte aligned");
  cudaStream_t st = as_stream(s);
  Carver c(workspace);
  int64_t big = m * n;
  if (n * n > big) big = n * n;
  if (m * m > big) big = m * m;
  float* T = c.take<float>((size_t)big);
  float* colsq = c.take<float>((size_t)n);
  float* rowsq = c.take<float>((size_t)m);
  float* part = c.take<float>(wnorms_partial_floats(m, n));
  float* cfbuf = c.take<float>((size_t)(m > n ? m : n));
  const bool bf16 = wdt == KRONQ_BF16;
  kronq_status r;
  const bool need_in = rescale && use_in, need_out = rescale && use_out;
  if (need_in || need_out) {
    r = wnorms(W, bf16, m, n, need_in ? colsq : nullptr, need_out ? rowsq : nullptr, part, st);
    if (r != KRONQ_OK) return r;
  }
  if (need_in) r = rescale_vector(HX, n, colsq, n, alpha, d_in, st);
  else { cudaError_t e = fill_f32(d_in, n, 1.f, st); r = e == cudaSuccess ? KRONQ_OK : cuda_fail(e, "fill"); }
  if (r != KRONQ_OK) return r;
  if (need_out) r = rescale_vector(HG, m, rowsq, m, alpha, d_out, st);
  else { cudaError_t e = fill_f32(d_out, m, 1.f, st); r = e == cudaSuccess ? KRONQ_OK : cuda_fail(e, "fill"); }
  if (r != KRONQ_OK) return r;

  const uint64_t s_in = 2ull * seed + 0ull, s_out = 2ull * seed + 1ull;
  // W~ = U D_out W D_in V^T: rows of W (input side), then rows of the transpose.
  RowPass p1;
  p1.in = W; p1.in_bf16 = bf16; p1.ld_in = n;
  p1.out = T; p1.ld_out = m;
  p1.rows = m; p1.L = n;
  p1.scale = d_in; p1.scale_mode = need_in ? 1 : 0;
  p1.rotate = use_in; p1.inverse = false; p1.sign_state = s_in; p1.cf = cfbuf;
  p1.tmp = Wt; p1.ld_tmp = n;   // scratch for a row-wise pass + transpose (Wt is written by p2)
  if ((r = rowpass(p1, st)) != KRONQ_OK) return r;
  RowPass p2;
  p2.in = T; p2.ld_in = m;
  p2.out = Wt; p2.ld_out = n;
  p2.rows = n; p2.L = m;
  p2.scale = d_out; p2.scale_mode = need_out ? 1 : 0;
  p2.rotate = use_out; p2.inverse = false; p2.sign_state = s_out; p2.cf = cfbuf;
  p2.tmp = T; p2.ld_tmp = m;    // in place
  if ((r = rowpass(p2, st)) != KRONQ_OK) return r;
  // H~_X = V D_in^-1 H_X D_in^-1 V^T
  if (use_in) {
    RowPass h1;
    h1.in = HX; h1.ld_in = n; h1.out = T; h1.ld_out = n; h1.rows = n; h1.L = n;
    h1.scale = d_in; h1.scale_mode = need_in ? 2 : 0; h1.rotate = true; h1.sign_state = s_in; h1.cf = cfbuf;
    h1.tmp = HX; h1.ld_tmp = n;   // in place
    if ((r = rowpass(h1, st)) != KRONQ_OK) return r;
    RowPass h2 = h1;
    h2.tmp = nullptr;
    h2.in = T; h2.out = HX;
    h2.rowwise = true;   // V F H F V^T is symmetric: no transposed store
    if ((r = rowpass(h2, st)) != KRONQ_OK) return r;
  }
  // H~_G = U D_out^-1 H_G D_out^-1 U^T
  if (use_out && HG) {
    RowPass g1;
    g1.in = HG; g1.ld_in = m; g1.out = T; g1.ld_out = m; g1.rows = m; g1.L = m;
    g1.scale = d_out; g1.scale_mode = need_out ? 2 : 0; g1.rotate = true; g1.sign_state = s_out; g1.cf = cfbuf;
    g1.tmp = HG; g1.ld_tmp = m;   // in place
    if ((r = rowpass(g1, st)) != KRONQ_OK) return r;
    RowPass g2 = g1;
    g2.tmp = nullptr;
    g2.in = T; g2.out = HG;
    g2.rowwise = true;
    if ((r = rowpass(g2, st)) != KRONQ_OK) return r;
  }
  return KRONQ_OK;
}

kronq_status kronq_biip_inverse(float* W, int64_t m, int64_t n, uint64_t seed, kronq_biip_mode mode,
                                const float* d_in, const float* d_out, void* workspace,
                                size_t ws_bytes, kronq_stream_t s) {
  if (!W || !d_in || !d_out || m <= 0 || n <= 0)
    return fail(KRONQ_ERR_INVALID_ARG, "biip_inverse: NULL pointer or non-positive size");
  if (!valid_mode(mode)) return fail(KRONQ_ERR_INVALID_ARG, "biip_inverse: bad mode");
  const bool use_in = mode != KRONQ_BIIP_SU_ONLY;
  const bool use_out = mode != KRONQ_BIIP_SV_ONLY;
  if ((use_in && odd_part(n) > 255) || (use_out && odd_part(m) > 255))
    return fail(KRONQ_ERR_UNSUPPORTED, "biip_inverse: odd factor of a rotated dimension exceeds 255");
  if (!workspace || ws_bytes < biip_ws(m, n) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "biip_inverse: workspace too small or not 256-byte aligned");
  cudaStream_t st = as_stream(s);
  Carver c(workspace);
  int64_t big = m * n;
  if (n * n > big) big = n * n;
  if (m * m > big) big = m * m;
  float* T = c.take<float>((size_t)big);
  c.take<float>((size_t)n);
  c.take<float>((size_t)m);
  c.take<float>(wnorms_partial_floats(m, n));
  float* cfbuf = c.take<float>((size_t)(m > n ? m : n));
  kronq_status r;
  RowPass p1;
  p1.in = W; p1.ld_in = n; p1.out = T; p1.ld_out = m; p1.rows = m; p1.L = n;
  p1.scale = d_in; p1.scale_mode = 2; p1.rotate = use_in; p1.inverse = true;
  p1.sign_state = 2ull * seed; p1.cf = cfbuf;
  if ((r = rowpass(p1, st)) != KRONQ_OK) return r;
  RowPass p2;
  p2.in = T; p2.ld_in = m; p2.out = W; p2.ld_out = n; p2.rows = n; p2.L = m;
  p2.scale = d_out; p2.scale_mode = 2; p2.rotate = use_out; p2.inverse = true;
  p2.sign_state = 2ull * seed + 1ull; p2.cf = cfbuf;
  return rowpass(p2, st);
}

size_t kronq_quantize_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p) {
  if (m <= 0 || n <= 0) return 0;
  return quant_ws(m, n, wants_rform(p));
}

kronq_status kronq_quantize_layer(float* Wt, float* HX, int64_t m, int64_t n,
                                  const kronq_quant_params* p, uint8_t* codes, float* scales,
                                  float* zeros, float* E, int* info, void* workspace,
                                  size_t ws_bytes, kronq_stream_t s) {
  kronq_status v = check_quant_args(Wt, HX, m, n, p, codes, scales, zeros, E, info, "quantize_layer");
  if (v != KRONQ_OK) return v;
  if (!workspace || ws_bytes < quant_ws(m, n, wants_rform(p)) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "quantize_layer: workspace too small or not 256-byte aligned");
  const int mode = (p->flags & KRONQ_U_GIVEN) ? 1 : 0;
  return quantize_core(Wt, HX, m, n, p, codes, scales, zeros, E, info, workspace, as_stream(s), mode);
}

}  // extern "C"

namespace kq {

kronq_status check_quant_args(float* Wt, float* HX, int64_t m, int64_t n, const kronq_quant_params* p,
                              uint8_t* codes, float* scales, float* zeros, float* E, int* info,
                              const char* who) {
  const std::string w(who);
  if (!p) return fail(KRONQ_ERR_INVALID_ARG, w + ": params is NULL");
  if (!Wt || !HX || !codes || !scales || !zeros || !info || m <= 0 || n <= 0)
    return fail(KRONQ_ERR_INVALID_ARG, w + ": NULL pointer or non-positive size");
  if (p->bits < 2 || p->bits > 4) return fail(KRONQ_ERR_INVALID_ARG, w + ": bits must be 2, 3 or 4");
  if (p->asym != 0 && p->asym != 1) return fail(KRONQ_ERR_INVALID_ARG, w + ": asym must be 0 or 1");
  if (p->block != 128) return fail(KRONQ_ERR_UNSUPPORTED, w + ": only block = 128 is implemented");
  if (!(p->group == -1 || (p->group > 0 && (128 % p->group == 0 || p->group % 128 == 0))))
    return fail(KRONQ_ERR_INVALID_ARG, w + ": group must be -1, a divisor of 128 or a multiple of 128");
  if (!(p->damp_rel >= 0.f) || !isfinite(p->damp_rel))
    return fail(KRONQ_ERR_INVALID_ARG, w + ": damp_rel must be finite and >= 0");
  if (p->flags & ~(KRONQ_U_GIVEN | KRONQ_ORDERED_FP32 | KRONQ_WRITE_E | KRONQ_R_FORM))
    return fail(KRONQ_ERR_INVALID_ARG, w + ": unknown flag");
  if ((p->flags & KRONQ_R_FORM) && (p->flags & (KRONQ_U_GIVEN | KRONQ_ORDERED_FP32)))
    return fail(KRONQ_ERR_INVALID_ARG, w + ": KRONQ_R_FORM excludes KRONQ_U_GIVEN and KRONQ_ORDERED_FP32");
  if ((p->flags & KRONQ_R_FORM) && p->group > 128)
    return fail(KRONQ_ERR_UNSUPPORTED, w + ": KRONQ_R_FORM takes groups of at most 128 columns (or -1)");
  if ((p->flags & KRONQ_WRITE_E) && !E) return fail(KRONQ_ERR_INVALID_ARG, w + ": KRONQ_WRITE_E needs E");
  if (m > ((int64_t)1 << 31) / 16 || n > ((int64_t)1 << 20))
    return fail(KRONQ_ERR_INVALID_ARG, w + ": size out of range");
  return KRONQ_OK;
}

size_t quantize_core_workspace_bytes(int64_t m, int64_t n, bool rform) { return quant_ws(m, n, rform); }

kronq_status quantize_core(float* Wt, float* HX, int64_t m, int64_t n, const kronq_quant_params* p,
                           uint8_t* codes, float* scales, float* zeros, float* E, int* info,
                           void* workspace, cudaStream_t st, int mode) {
  Carver c(workspace);
  void* cws = c.take<uint8_t>(chol_workspace_bytes(n));
  uint8_t* dead = c.take<uint8_t>((size_t)n);
  float* Eblk = c.take<float>((size_t)(m * 128));
  const int64_t kg = 128 * quant_gblocks(n);
  __nv_bfloat16* Eh = c.take<__nv_bfloat16>((size_t)(m * kg));
  __nv_bfloat16* El = c.take<__nv_bfloat16>((size_t)(m * kg));
  __nv_bfloat16* Uh = c.take<__nv_bfloat16>((size_t)(kg * quant_ldu(n)));
  __nv_bfloat16* Ul = c.take<__nv_bfloat16>((size_t)(kg * quant_ldu(n)));
  const bool u_given = mode == 1;
  const bool rform = !u_given && wants_rform(p);
  float* W0 = rform ? c.take<float>((size_t)(m * n)) : nullptr;
  float* Ublk = rform ? c.take<float>((size_t)(128 * 128 * ceil_div(n, 128))) : nullptr;
  kronq_status r;
  if (u_given) {
    r = chol_upper_inverse(HX, 0, 0.f, true, nullptr, info, cws, st);  // resets info only
  } else if (mode == 2) {
    r = chol_upper_inverse(HX, n, 0.f, true, nullptr, info, cws, st, !rform);  // already damped
  } else {
    r = chol_upper_inverse(HX, n, p->damp_rel, false, dead, info, cws, st, !rform);
  }
  if (r != KRONQ_OK) return r;
  if (rform) {
    // W0 = W~, W~ := 0 (it accumulates the feedback F), U's diagonal blocks
    r = diag_block_inverse(HX, n, Ublk, info, st);
    if (r != KRONQ_OK) return r;
    KQ_CUDA(cudaMemcpyAsync(W0, Wt, (size_t)(m * n) * sizeof(float), cudaMemcpyDeviceToDevice, st));
    KQ_CUDA(cudaMemsetAsync(Wt, 0, (size_t)(m * n) * sizeof(float), st));
  }
  SweepDesc d;
  d.W = Wt; d.U = HX; d.m = m; d.n = n;
  d.bits = p->bits; d.group = p->group; d.asym = p->asym != 0;
  d.codes = codes; d.scales = scales; d.zeros = zeros;
  d.ngroups = (p->group == -1) ? 1 : ceil_div(n, p->group);
  d.E = (p->flags & KRONQ_WRITE_E) ? E : nullptr;
  d.Eblk = Eblk;
  d.dead = mode == 0 ? dead : nullptr;
  d.info = info;
  d.ordered = (p->flags & KRONQ_ORDERED_FP32) != 0;
  d.Eh = Eh; d.El = El; d.Uh = Uh; d.Ul = Ul; d.ldu = quant_ldu(n);
  d.lde = kg;
  d.gblocks = (int)quant_gblocks(n);
  d.W0 = W0;
  d.Ublk = Ublk;
  return gptq_sweep(d, st);
}

}  // namespace kq

extern "C" {

kronq_status kronq_pack(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* out,
                        kronq_stream_t s) {
  if (bits != 2 && bits != 4) return fail(KRONQ_ERR_INVALID_ARG, "pack: bits must be 2 or 4 (3-bit codes are not packable)");
  if (m < 0 || n < 0) return fail(KRONQ_ERR_INVALID_ARG, "pack: negative size");
  if (m * n > 0 && (!codes || !out)) return fail(KRONQ_ERR_INVALID_ARG, "pack: NULL pointer");
  return pack_codes(codes, m, n, bits, out, as_stream(s));
}

kronq_status kronq_unpack(const uint32_t* in, int64_t m, int64_t n, int bits, uint8_t* codes,
                          kronq_stream_t s) {
  if (bits != 2 && bits != 4) return fail(KRONQ_ERR_INVALID_ARG, "unpack: bits must be 2 or 4");
  if (m < 0 || n < 0) return fail(KRONQ_ERR_INVALID_ARG, "unpack: negative size");
  if (m * n > 0 && (!in || !codes)) return fail(KRONQ_ERR_INVALID_ARG, "unpack: NULL pointer");
  return unpack_codes(in, m, n, bits, codes, as_stream(s));
}

kronq_status kronq_device_status(int* out, kronq_stream_t s) {
  if (!out) return fail(KRONQ_ERR_INVALID_ARG, "device_status: out is NULL");
  int v[6] = {0, 0, 0, 0, 0, 0};
  cudaError_t e = status_fetch_syrk(&v[0], as_stream(s));
  if (e == cudaSuccess) e = status_fetch_trailing(&v[1], as_stream(s));
  if (e == cudaSuccess) e = status_fetch_schur(&v[2], as_stream(s));
  if (e == cudaSuccess) e = status_fetch_trigemm(&v[3], as_stream(s));
  if (e == cudaSuccess) e = status_fetch_chol(&v[4], as_stream(s));
  if (e == cudaSuccess) e = status_fetch_schurk(&v[5], as_stream(s));
  if (e != cudaSuccess) return cuda_fail(e, "device_status");
  *out = 0;
  for (int i = 0; i < 6 && *out == 0; ++i) *out = v[i];
  return KRONQ_OK;
}

kronq_status kronq_wait_selftest(int which, uint64_t limit_ns, void* workspace, size_t ws_bytes,
                                 kronq_stream_t s) {
  if (which != 0 && which != 1) return fail(KRONQ_ERR_INVALID_ARG, "wait_selftest: which must be 0 or 1");
  if (limit_ns == 0 || limit_ns > 1000000000ull)
    return fail(KRONQ_ERR_INVALID_ARG, "wait_selftest: limit_ns must be in (0, 1e9]");
  if (!workspace || ws_bytes < 3 * sizeof(int) || !aligned(workspace, 4))
    return fail(KRONQ_ERR_INVALID_ARG, "wait_selftest: workspace must hold 3 ints, 4-byte aligned");
  return wait_selftest(which, (unsigned long long)limit_ns, static_cast<int*>(workspace), as_stream(s));
}

size_t kronq_kfac_loss_workspace_bytes(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  Carver c(nullptr);
  c.take<float>((size_t)(m * n));
  c.take<double>(1024);
  return c.size();
}

kronq_status kronq_kfac_loss(const float* E, const float* HG, int64_t m, int64_t n, double* out,
                             void* workspace, size_t ws_bytes, kronq_stream_t s) {
  if (!E || !HG || !out || m <= 0 || n <= 0) return fail(KRONQ_ERR_INVALID_ARG, "kfac_loss: bad arguments");
  if (!workspace || ws_bytes < kronq_kfac_loss_workspace_bytes(m, n) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "kfac_loss: workspace too small or not 256-byte aligned");
  cudaStream_t st = as_stream(s);
  Carver c(workspace);
  float* F = c.take<float>((size_t)(m * n));
  double* part = c.take<double>(1024);
  GemmDesc g;  // F = HG * E
  g.M = m; g.N = n; g.K = m;
  g.A = HG; g.lda = m; g.B = E; g.ldb = n;
  g.C = F; g.ldc = n; g.alpha = 1.f; g.beta = 0.f;
  cudaError_t e = gemm_f32(g, st);
  if (e != cudaSuccess) return cuda_fail(e, "gemm(loss)");
  kronq_status r = dot_sum(E, F, m * n, part + 1000, part, st);
  if (r != KRONQ_OK) return r;
  KQ_CUDA(cudaMemcpyAsync(out, part + 1000, sizeof(double), cudaMemcpyDeviceToHost, st));
  KQ_CUDA(cudaStreamSynchronize(st));
  return KRONQ_OK;
}

}  // extern "C"

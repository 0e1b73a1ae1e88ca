// Two-sided adaptive rounding on the GPU: GPTQ's error feedback applied to
// vec(W) under the Kronecker-factored Hessian H_X (x) H_G, after the BaKron
// abstract ("BaKron: Efficient Quantization with Kronecker-Factored
// Hessians" page: anti-diagonal parallelism, O(m + n) sequential steps,
// O(mn(m + n)) work).  The abstract gives no algorithm; the definition
// followed is GPTQ on vec(W) with the upper factor U = U_X (x) U_G of the
// damped inverse Hessian: element (i, j) is rounded on its row's static
// group grid (taken from W~ before the sweep), and its scaled error
//     e_ij = (w~_ij - q_ij) / (U_X[j, j] U_G[i, i])
// is subtracted as e_ij U_G[i, i'] U_X[j, j'] from every later element
// (i' >= i, j' >= j, not (i, j) itself).
//
// Blocked form.  W is cut into tiles of TR = 32 rows by TC = 32 columns.
// A tile depends only on the tiles above and to the left of it, so the
// tiles of one anti-diagonal I + J = s run at once (one CTA each), and
// there are ceil(m / 32) + ceil(n / 32) - 1 such steps.  With
// P[I, J] = sum_{J'' <= J} E[I, J''] U_X[J'', J] (E U_X, block row by block
// row), tile (I, J) starts from
//     S = W~[I, J] - sum_{I'' < I} U_G[I'', I]^T P[I'', J] - U_G[I, I]^T P-[I, J]
// where P- leaves out the tile's own column block.  The first sum is
// applied to W~ after each step (the column-direction update), P- is
// accumulated in P after each step (the row-direction update); both are
// fp32 tile products over the tiles of the step that just finished.
//
// Inside a tile, row r is a one-sided GPTQ sweep on U_X[J, J] started from
// S[r] minus the contributions of the tile's earlier rows,
//     cross_r(c) = sum_{r'' < r} U_G[r'', r] P_loc[r''](c),
//     P_loc[r''](c) = (S[r''](c) - cross_r''(c) - deq[r''](c)) / U_G[r'', r'']
// (P_loc is the tile's own E U_X), so row r can take column c as soon as
// the rows above it have taken column c: warp r handles column t - r at
// step t, and a tile takes TR + TC - 1 steps.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int TR = 32;            // tile rows: one warp each
constexpr int TC = 32;            // tile columns: one per lane
constexpr int LD = 33;            // odd stride of the 32 x 32 shared arrays

constexpr int UB = 128;           // update blocks: 32 x 128 (row direction) or 128 x 32 (column direction)
constexpr int UPD_SMEM = (UB * LD + 32 * UB) * (int)sizeof(float);

struct TsArgs {
  float* W;            // m x n: W~ with the column-direction updates; Q on return
  const float* UX;     // n x n, upper triangle
  const float* UG;     // m x m, upper triangle
  float* P;            // m x n: E U_X block row by block row
  float* E;            // m x n scaled errors
  uint8_t* codes;      // m x n
  const float* scales; // m x ngroups
  const float* zeros;
  const int* info;     // two ints: the factorisations of H_X and H_G
  int64_t m, n;
  int ngroups, group, bits;
  int s;               // anti-diagonal I + J
  int I0;              // first tile row on it
  int NI, NJ;          // tile rows and columns
};

// Static grid of every (row, group) from W~ before the sweep: one warp per
// pair; x_min = min(0, min w), x_max = max(0, max w), equal -> (-1, 1),
// scale = (x_max - x_min) / (2^b - 1), zero = rint(-x_min / scale) (or
// 2^(b-1) symmetric).
__global__ void __launch_bounds__(256) ts_grid_kernel(const float* W, int64_t m, int64_t n, int group,
                                                      int ngroups, int bits, int asym, float* scales,
                                                      float* zeros) {
  const int64_t p = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (p >= m * ngroups) return;
  const int64_t i = p / ngroups, g = p - i * ngroups;
  const int64_t j0 = group == -1 ? 0 : g * group;
  const int64_t j1 = group == -1 ? n : (j0 + group < n ? j0 + group : n);
  float lo = INFINITY, hi = -INFINITY;
  for (int64_t j = j0 + lane; j < j1; j += 32) {
    const float x = W[i * n + j];
    lo = fminf(lo, x);
    hi = fmaxf(hi, x);
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    const float maxq = (float)((1 << bits) - 1);
    float xmin = fminf(lo, 0.f), xmax = fmaxf(hi, 0.f);
    if (!asym) {
      xmax = fmaxf(fabsf(xmin), xmax);
      xmin = -xmax;
    }
    if (xmin == xmax) {
      xmin = -1.f;
      xmax = 1.f;
    }
    const float sc = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
    scales[p] = sc;
    zeros[p] = asym ? rintf(__fdiv_rn(-xmin, sc)) : (float)(1 << (bits - 1));
  }
}

// One tile of the anti-diagonal per CTA: warp r is row r, lane l column l.
// Per step, warp r's dependent chain is one shared-memory load (row r - 1's
// P_loc at column c, written the step before), the rounding on lane c and
// one shuffle of e; the sum over the rows above r - 1 for column c + 1 is
// formed in the same step, off that chain.  The quantizer multiplies by
// 1 / scale and the errors by 1 / U_X[c, c] and 1 / U_G[r, r], as the
// one-sided sweep does.
__global__ void __launch_bounds__(TR * 32) ts_tile_kernel(TsArgs a) {
  if (a.info[0] != 0 || a.info[1] != 0) return;
  __shared__ float X[TC * LD];     // U_X[J, J] (zero outside the tile)
  __shared__ float G[TR * LD];     // U_G[I, I]
  __shared__ float PL[TR * LD];    // P- of the tile, then P_loc
  __shared__ float XI[TC];         // 1 / U_X[c, c]
  const int I = a.I0 + (int)blockIdx.x;
  const int J = a.s - I;
  const int64_t r0 = (int64_t)I * TR, c0 = (int64_t)J * TC;
  const int rows = (int)((a.m - r0) < TR ? (a.m - r0) : TR);
  const int cols = (int)((a.n - c0) < TC ? (a.n - c0) : TC);
  const int r = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool live = r < rows, in = live && lane < cols;
  const int64_t row = r0 + r;

  X[r * LD + lane] = (r < cols && lane < cols) ? a.UX[(c0 + r) * a.n + c0 + lane] : 0.f;
  G[r * LD + lane] = (live && lane < rows) ? a.UG[row * a.m + r0 + lane] : 0.f;
  PL[r * LD + lane] = in ? a.P[row * a.n + c0 + lane] : 0.f;
  if (r == 0) XI[lane] = lane < cols ? __frcp_rn(a.UX[(c0 + lane) * a.n + c0 + lane]) : 1.f;
  const float w0 = in ? a.W[row * a.n + c0 + lane] : 0.f;
  const int64_t g = a.group == -1 ? 0 : (c0 + lane) / a.group;
  const float sc = in ? a.scales[row * a.ngroups + g] : 1.f;
  const float zp = in ? a.zeros[row * a.ngroups + g] : 0.f;
  const float isc = __frcp_rn(sc);
  __syncthreads();

  // Row r's start S = W~ - (U_G[I, I]^T P-)[r]; w = S minus the row's own
  // feedback so far; pm = P-[r].
  const float pm = PL[r * LD + lane];
  float S = w0;
  for (int q = 0; q <= r; ++q) S = fmaf(-G[q * LD + r], PL[q * LD + lane], S);
  float w = S;
  const float invg = live ? __frcp_rn(G[r * LD + r]) : 1.f;
  const float gl = (lane < r - 1) ? G[lane * LD + r] : 0.f;   // rows above r - 1
  const float gp = (r >= 1) ? G[(r - 1) * LD + r] : 0.f;       // row r - 1
  const float maxq = (float)((1 << a.bits) - 1);
  __syncthreads();   // PL now holds P_loc, written before it is read

  float xp = 0.f;    // sum over the rows above r - 1 for the current column
  for (int t = 0; t < TR + TC - 1; ++t) {
    const int c = t - r;
    float xpn = 0.f;
    if (live && r >= 2 && c + 1 >= 0 && c + 1 < cols) {
      // rows l < r - 1 took column c + 1 at step l + c + 1 < t
      const float v = PL[lane * LD + c + 1];
      xpn = warp_sum((lane < r - 1) ? gl * v : 0.f);
    }
    if (live && c >= 0 && c < cols) {
      const float x = (r >= 1) ? fmaf(gp, PL[(r - 1) * LD + c], xp) : 0.f;
      const float wt = w - x;             // w~ at (row, c) on lane c
      float q = rintf(wt * isc) + zp;
      q = fminf(fmaxf(q, 0.f), maxq);
      const float deq = sc * (q - zp);
      const float e1 = __shfl_sync(0xffffffffu, (wt - deq) * XI[c], c);
      if (lane == c) {
        const int64_t gi = row * a.n + c0 + c;
        a.W[gi] = deq;
        a.codes[gi] = (uint8_t)q;
        a.E[gi] = e1 * invg;
        PL[r * LD + c] = (S - x - deq) * invg;
      }
      if (lane > c) w = fmaf(-e1, X[c * LD + lane], w);
    }
    xp = xpn;
    __syncthreads();
  }

  // P[I, J] = P- + P_loc
  if (in) a.P[row * a.n + c0 + lane] = pm + PL[r * LD + lane];
}

struct UpdArgs {
  float* W;
  float* P;
  const float* E;
  const float* UX;
  const float* UG;
  const int* info;
  int64_t m, n;
  int s, I0, NI, NJ;
};

// After anti-diagonal s: for each of its tiles (I, J) (blockIdx.y), item
// blockIdx.x is either a row-direction block P[I, cols] += E[I, J] U_X[J, cols]
// (32 x 128, over the columns past the tile) or a column-direction block
// W~[rows, J] -= U_G[I, rows]^T P[I, J] (128 x 32, over the rows below it);
// K = 32.  256 threads own 4 x 4 outputs each.
__global__ void __launch_bounds__(256) ts_update_kernel(UpdArgs a) {
  if (a.info[0] != 0 || a.info[1] != 0) return;
  extern __shared__ float smem[];
  float* As = smem;               // BM x LD: As[i][k]
  float* Bs = As + UB * LD;       // 32 x BN: Bs[k][j]
  const int I = a.I0 + (int)blockIdx.y;
  const int J = a.s - I;
  const int64_t r0 = (int64_t)I * TR, c0 = (int64_t)J * TC;
  const int trows = (int)((a.m - r0) < TR ? (a.m - r0) : TR);
  const int tcols = (int)((a.n - c0) < TC ? (a.n - c0) : TC);
  const int64_t cpast = c0 + TC, rpast = r0 + TR;
  const int na = cpast < a.n ? (int)((a.n - cpast + UB - 1) / UB) : 0;
  const int nb = rpast < a.m ? (int)((a.m - rpast + UB - 1) / UB) : 0;
  const int it = (int)blockIdx.x;
  if (it >= na + nb) return;
  const int tid = threadIdx.x;
  float* C;
  int crows, ccols, K, BN, ti, tj;
  float sign;
  if (it < na) {
    // row direction: C = P[r0 .. +32, cc0 .. +128]
    const int64_t cc0 = cpast + (int64_t)it * UB;
    K = tcols;
    crows = trows;
    ccols = (int)((a.n - cc0) < UB ? (a.n - cc0) : UB);
    BN = UB;
    for (int t = tid; t < 32 * 32; t += 256) {
      const int i = t >> 5, k = t & 31;
      As[i * LD + k] = (i < crows && k < K) ? a.E[(r0 + i) * a.n + c0 + k] : 0.f;
    }
    for (int t = tid; t < 32 * UB; t += 256) {
      const int k = t / UB, j = t - k * UB;
      Bs[t] = (k < K && j < ccols) ? a.UX[(c0 + k) * a.n + cc0 + j] : 0.f;
    }
    C = a.P + r0 * a.n + cc0;
    sign = 1.f;
    ti = tid >> 5;   // rows 4 ti .. 4 ti + 3 of 32
    tj = tid & 31;   // columns 4 tj .. 4 tj + 3 of 128
  } else {
    // column direction: C = W~[rr0 .. +128, c0 .. +32]
    const int64_t rr0 = rpast + (int64_t)(it - na) * UB;
    K = trows;
    crows = (int)((a.m - rr0) < UB ? (a.m - rr0) : UB);
    ccols = tcols;
    BN = 32;
    for (int t = tid; t < 32 * UB; t += 256) {
      const int k = t / UB, i = t - k * UB;
      As[i * LD + k] = (i < crows && k < K) ? a.UG[(r0 + k) * a.m + rr0 + i] : 0.f;
    }
    for (int t = tid; t < 32 * 32; t += 256) {
      const int k = t >> 5, j = t & 31;
      Bs[t] = (k < K && j < ccols) ? a.P[(r0 + k) * a.n + c0 + j] : 0.f;
    }
    C = a.W + rr0 * a.n + c0;
    sign = -1.f;
    ti = tid >> 3;   // rows 4 ti .. 4 ti + 3 of 128
    tj = tid & 7;    // columns 4 tj .. 4 tj + 3 of 32
  }
  __syncthreads();
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k = 0; k < K; ++k) {
    const float4 b = *reinterpret_cast<const float4*>(Bs + k * BN + 4 * tj);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float av = As[(4 * ti + i) * LD + k];
      acc[i][0] = fmaf(av, b.x, acc[i][0]);
      acc[i][1] = fmaf(av, b.y, acc[i][1]);
      acc[i][2] = fmaf(av, b.z, acc[i][2]);
      acc[i][3] = fmaf(av, b.w, acc[i][3]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ri = 4 * ti + i;
    if (ri >= crows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int cj = 4 * tj + j;
      if (cj < ccols) C[ri * a.n + cj] = fmaf(sign, acc[i][j], C[ri * a.n + cj]);
    }
  }
}

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

size_t two_sided_workspace_bytes(int64_t m, int64_t n) {
  const size_t cws = chol_workspace_bytes(n) > chol_workspace_bytes(m) ? chol_workspace_bytes(n)
                                                                        : chol_workspace_bytes(m);
  return align256(cws) + 2 * align256((size_t)(m * n) * sizeof(float));
}

kronq_status two_sided_core(float* Wt, float* HX, float* HG, int64_t m, int64_t n, const kronq_quant_params* p,
                            uint8_t* codes, float* scales, float* zeros, float* E, int* info, void* workspace,
                            cudaStream_t st) {
  uint8_t* base = static_cast<uint8_t*>(workspace);
  const size_t cws = align256(two_sided_workspace_bytes(m, n) - 2 * align256((size_t)(m * n) * sizeof(float)));
  void* chol_ws = base;
  float* P = reinterpret_cast<float*>(base + cws);
  float* Escr = reinterpret_cast<float*>(base + cws + align256((size_t)(m * n) * sizeof(float)));
  float* Eout = (p->flags & KRONQ_WRITE_E) ? E : Escr;
  const bool u_given = (p->flags & KRONQ_U_GIVEN) != 0;
  kronq_status r;
  if (u_given) {
    r = chol_upper_inverse(HX, 0, 0.f, true, nullptr, info, chol_ws, st);        // info[0] := 0
    if (r == KRONQ_OK) r = chol_upper_inverse(HG, 0, 0.f, true, nullptr, info + 1, chol_ws, st);
  } else {
    r = damp_only(HX, n, p->damp_rel, info, st);
    if (r == KRONQ_OK) r = chol_upper_inverse(HX, n, 0.f, true, nullptr, info, chol_ws, st, true);
    if (r == KRONQ_OK) r = damp_only(HG, m, p->damp_rel, info + 1, st);
    if (r == KRONQ_OK) r = chol_upper_inverse(HG, m, 0.f, true, nullptr, info + 1, chol_ws, st, true);
  }
  if (r != KRONQ_OK) return r;
  const int ngroups = p->group == -1 ? 1 : (int)ceil_div(n, p->group);
  ts_grid_kernel<<<(unsigned)ceil_div(m * ngroups, 8), 256, 0, st>>>(Wt, m, n, p->group, ngroups, p->bits,
                                                                     p->asym, scales, zeros);
  KQ_LAUNCH_CHECK("ts_grid_kernel");
  KQ_CUDA(cudaMemsetAsync(P, 0, (size_t)(m * n) * sizeof(float), st));
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&ts_update_kernel), UPD_SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(ts_update_kernel)");
  const int NI = (int)ceil_div(m, TR), NJ = (int)ceil_div(n, TC);
  TsArgs a;
  a.W = Wt; a.UX = HX; a.UG = HG; a.P = P; a.E = Eout; a.codes = codes;
  a.scales = scales; a.zeros = zeros; a.info = info;
  a.m = m; a.n = n; a.ngroups = ngroups; a.group = p->group; a.bits = p->bits;
  a.NI = NI; a.NJ = NJ;
  UpdArgs u;
  u.W = Wt; u.P = P; u.E = Eout; u.UX = HX; u.UG = HG; u.info = info;
  u.m = m; u.n = n; u.NI = NI; u.NJ = NJ;
  for (int s = 0; s <= NI + NJ - 2; ++s) {
    const int i0 = s - (NJ - 1) > 0 ? s - (NJ - 1) : 0;
    const int i1 = s < NI - 1 ? s : NI - 1;
    a.s = s;
    a.I0 = i0;
    ts_tile_kernel<<<(unsigned)(i1 - i0 + 1), TR * 32, 0, st>>>(a);
    KQ_LAUNCH_CHECK("ts_tile_kernel");
    // update blocks of the step's tiles: at most the row-direction blocks of
    // its leftmost tile plus the column-direction blocks of its topmost one
    const int items = (int)(ceil_div(n - (int64_t)(s - i1 + 1) * TC, UB) + ceil_div(m - (int64_t)(i0 + 1) * TR, UB));
    if (items > 0) {
      u.s = s;
      u.I0 = i0;
      ts_update_kernel<<<dim3((unsigned)items, (unsigned)(i1 - i0 + 1)), 256, UPD_SMEM, st>>>(u);
      KQ_LAUNCH_CHECK("ts_update_kernel");
    }
  }
  return KRONQ_OK;
}

}  // namespace kq

extern "C" {

size_t kronq_quantize_two_sided_workspace_bytes(int64_t m, int64_t n, const kronq_quant_params* p) {
  (void)p;
  if (m <= 0 || n <= 0) return 0;
  return kq::two_sided_workspace_bytes(m, n);
}

kronq_status kronq_quantize_two_sided(float* Wt, float* HX, float* HG, int64_t m, int64_t n,
                                      const kronq_quant_params* p, uint8_t* codes, float* scales,
                                      float* zeros, float* E, int* info, void* workspace, size_t ws_bytes,
                                      kronq_stream_t s) {
  using namespace kq;
  kronq_status v = check_quant_args(Wt, HX, m, n, p, codes, scales, zeros, E, info, "quantize_two_sided");
  if (v != KRONQ_OK) return v;
  if (!HG) return fail(KRONQ_ERR_INVALID_ARG, "quantize_two_sided: HG is NULL");
  if (p->flags & (KRONQ_R_FORM | KRONQ_ORDERED_FP32))
    return fail(KRONQ_ERR_INVALID_ARG, "quantize_two_sided: takes KRONQ_U_GIVEN and KRONQ_WRITE_E only");
  if (m > ((int64_t)1 << 20)) return fail(KRONQ_ERR_INVALID_ARG, "quantize_two_sided: m out of range");
  if (!workspace || ws_bytes < two_sided_workspace_bytes(m, n) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "quantize_two_sided: workspace too small or not 256-byte aligned");
  return two_sided_core(Wt, HX, HG, m, n, p, codes, scales, zeros, E, info, workspace, as_stream(s));
}

}  // extern "C"

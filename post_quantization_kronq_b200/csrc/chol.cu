// Damping and the upper Cholesky factor of the damped inverse.
//
// GPTQ (which KronQ extends, KronQ README intro) needs the upper triangular
// U with U^T U = (H + lambda I)^-1.  Instead of inverting and factoring
// again, this library factors A = H + lambda I "in reverse": A = R R^T with
// R upper triangular (eliminating from the last index down), and then
// U = R^-1, since A^-1 = R^-T R^-1 = U^T U.  That is 2 n^3 / 3 flops in total.
//
// Blocked with nb = 64, bottom-right first.  For n > 256 with 16-byte rows
// the whole chain is one persistent kernel (chol_persistent_kernel below,
// with a one-step look-ahead); otherwise, for each diagonal block J:
//   diag_panel_kernel  factor A_JJ = R_JJ R_JJ^T (itself blocked by 16),
//                      invert it, U_JJ = R_JJ^-1, and form the panel
//                      R[0:j0, J] = A[0:j0, J] U_JJ^T (every CTA factors the
//                      small block itself)
//   schur_tc_kernel    A[0:j0, 0:j0] -= R[0:j0, J] R[0:j0, J]^T on the tensor
//                      cores (upper triangle only, fp32-level split products)
// Then the diagonal blocks U_JJ are stored, and the
// off-diagonal blocks of U come from the recursive formula
//   inv([[R11, R12], [0, R22]]) = [[U11, -U11 R12 U22], [0, U22]]
// evaluated level by level (block sizes nb, 2 nb, 4 nb, ...), each level one
// batched pair of tensor-core products with a triangular factor.  A non-positive pivot stops the chain and records
// info = 1 + its index (LAPACK convention); every later kernel then returns.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "schur_tile.cuh"

namespace kq {
namespace {

constexpr int NB = 64;

// fix_zero: a zero diagonal entry becomes 1 before the mean is taken (the
// one-sided pass's dead-column rule); without it the diagonal is damped as is.
__global__ void __launch_bounds__(1024) damp_kernel(float* H, int64_t n, float damp_rel,
                                                    uint8_t* dead, int* info, bool fix_zero) {
  __shared__ double red[32];
  if (threadIdx.x == 0) *info = 0;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    float h = H[j * n + j];
    const bool isdead = fix_zero && (h == 0.f);
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

// ---------------------------------------------------------------------------
// Diagonal step of the blocked factorisation: one 64 x 64 block A_JJ,
// factored and inverted in shared memory by 256 threads, then the panel
// rows above it.  The block is handled as four 16 x 16 leaves (bottom-right
// first); each leaf is factored in the registers of one thread, the rows
// above the leaf are solved against R_leaf, and a rank-16 update follows.
// Then four threads invert the leaves at once and U_JJ is assembled from
// them with the recursive two-block formula.

constexpr int LF = 16;                       // leaf width
constexpr int PR = 32;                       // panel rows per chunk

struct alignas(16) DiagSmem {
  union {
    float a[NB][NB + 1];      // A_JJ (upper) -> R_JJ
    float ut[NB][NB + 4];     // afterwards: U_JJ^T (16-byte aligned rows)
  } x;
  float u[NB][NB + 1];        // U_JJ (upper, zero below)
  union {
    float tb[32][33];         // products R12 U22 while U_JJ is assembled
    float ach[PR][NB + 1];    // a chunk of panel rows
  } y;
  float rinv[NB];
  int bad;
};

// Factor the leaf at offset o in the registers of one thread (its upper
// triangle, 136 values; the last pivot first, each pivot scaled by rsqrt).
// Writes R_leaf into a and 1 / R_kk into rinv; records the first
// non-positive pivot in S.bad.  One thread keeps the whole dependency chain
// in registers, which is several times faster than sharing it across a warp.
template <class SM>
__device__ __forceinline__ void leaf_factor(SM& S, int o) {
  float r[LF][LF];
#pragma unroll
  for (int i = 0; i < LF; ++i)
#pragma unroll
    for (int j = i; j < LF; ++j) r[i][j] = S.x.a[o + i][o + j];
  int badk = -1;
#pragma unroll
  for (int K = LF - 1; K >= 0; --K) {
    const float piv = r[K][K];
    if ((!(piv > 0.f) || !isfinite(piv)) && badk < 0) badk = K;
    const float rs = rsqrtf(piv);
    S.rinv[o + K] = rs;
    r[K][K] = piv * rs;
#pragma unroll
    for (int i = 0; i < K; ++i) r[i][K] *= rs;
#pragma unroll
    for (int j = 0; j < K; ++j)
#pragma unroll
      for (int i = 0; i <= j; ++i) r[i][j] = fmaf(-r[i][K], r[j][K], r[i][j]);
  }
  if (badk >= 0 && S.bad == 0) S.bad = o + badk + 1;
#pragma unroll
  for (int i = 0; i < LF; ++i)
#pragma unroll
    for (int j = i; j < LF; ++j) S.x.a[o + i][o + j] = r[i][j];
}

// U_leaf = R_leaf^-1 for the leaf at offset o, in place in the registers of
// one thread: column j of U is -U[0:j, 0:j] R[0:j, j] / R_jj, the leading
// block already inverted.  Reads R from a and 1 / R_kk from rinv, writes u.
template <class SM>
__device__ __forceinline__ void leaf_invert(SM& S, int o) {
  float r[LF][LF];
#pragma unroll
  for (int i = 0; i < LF; ++i)
#pragma unroll
    for (int j = i; j < LF; ++j) r[i][j] = S.x.a[o + i][o + j];
#pragma unroll
  for (int j = 0; j < LF; ++j) {
    const float ujj = S.rinv[o + j];
    float t[LF];
#pragma unroll
    for (int i = 0; i < j; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int k = i; k < j; ++k) acc = fmaf(r[i][k], r[k][j], acc);
      t[i] = acc;
    }
#pragma unroll
    for (int i = 0; i < j; ++i) r[i][j] = -t[i] * ujj;
    r[j][j] = ujj;
  }
#pragma unroll
  for (int i = 0; i < LF; ++i)
#pragma unroll
    for (int j = i; j < LF; ++j) S.u[o + i][o + j] = r[i][j];
}

// Factors the 64 x 64 block in S.x.a (upper triangle; S.u zero, S.bad zero)
// into R_JJ (in S.x.a) and U_JJ = R_JJ^-1 (in S.u).  Returns false
// (uniformly) at a non-positive pivot, S.bad = its index + 1.  256 threads.
template <class SM>
__device__ bool factor_invert_block(SM& S) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int o = NB - LF; o >= 0; o -= LF) {
    if (tid == 0) leaf_factor(S, o);
    __syncthreads();
    if (S.bad) return false;  // uniform: read after the barrier
    if (o == 0) break;
    // rows i < o of the leaf's columns: solve x R_leaf^T = A[i, leaf], last
    // column first (one thread per row)
    if (tid < o) {
      const int i = tid;
      float x[LF];
#pragma unroll
      for (int k = 0; k < LF; ++k) x[k] = S.x.a[i][o + k];
#pragma unroll
      for (int k = LF - 1; k >= 0; --k) {
        float s0 = x[k], s1 = 0.f;
#pragma unroll
        for (int l = k + 1; l < LF; ++l) {
          if ((l - k) & 1) s0 = fmaf(-S.x.a[o + k][o + l], x[l], s0);
          else s1 = fmaf(-S.x.a[o + k][o + l], x[l], s1);
        }
        x[k] = (s0 + s1) * S.rinv[o + k];
      }
#pragma unroll
      for (int k = 0; k < LF; ++k) S.x.a[i][o + k] = x[k];
    }
    __syncthreads();
    // rank-16 update of the leading o x o upper triangle
    {
      const int cc = tid & 63, ty = tid >> 6;
      if (cc < o) {
        float rc[LF];
#pragma unroll
        for (int k = 0; k < LF; ++k) rc[k] = S.x.a[cc][o + k];
        for (int i = ty; i <= cc; i += 4) {
          float acc = 0.f;
#pragma unroll
          for (int k = 0; k < LF; ++k) acc = fmaf(S.x.a[i][o + k], rc[k], acc);
          S.x.a[i][cc] -= acc;
        }
      }
    }
    __syncthreads();
  }

  if (lane == 0 && warp < NB / LF) leaf_invert(S, warp * LF);
  __syncthreads();
  // U_JJ from the leaf inverses: for pairs of diagonal blocks of size s,
  // U12 = -U11 (R12 U22).  s = 16: two pairs, two outputs per thread.
  {
    const int p = tid >> 7, r = (tid >> 3) & 15, c = (tid & 7) * 2;
    const int b0 = 32 * p;
    float t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float rk = S.x.a[b0 + r][b0 + 16 + k];
      t0 = fmaf(rk, S.u[b0 + 16 + k][b0 + 16 + c], t0);
      t1 = fmaf(rk, S.u[b0 + 16 + k][b0 + 16 + c + 1], t1);
    }
    S.y.tb[16 * p + r][c] = t0;
    S.y.tb[16 * p + r][c + 1] = t1;
    __syncthreads();
    float v0 = 0.f, v1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float uk = S.u[b0 + r][b0 + k];
      v0 = fmaf(uk, S.y.tb[16 * p + k][c], v0);
      v1 = fmaf(uk, S.y.tb[16 * p + k][c + 1], v1);
    }
    S.u[b0 + r][b0 + 16 + c] = -v0;
    S.u[b0 + r][b0 + 16 + c + 1] = -v1;
    __syncthreads();
  }
  // s = 32: one pair, four outputs per thread.
  {
    const int r = tid >> 3, c = (tid & 7) * 4;
    float t[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float rk = S.x.a[r][32 + k];
#pragma unroll
      for (int q = 0; q < 4; ++q) t[q] = fmaf(rk, S.u[32 + k][32 + c + q], t[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) S.y.tb[r][c + q] = t[q];
    __syncthreads();
    float v[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float uk = S.u[r][k];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = fmaf(uk, S.y.tb[k][c + q], v[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) S.u[r][32 + c + q] = -v[q];
    __syncthreads();
  }
  return true;
}

// Loads PR panel rows [r0, r0 + PR) of columns J into registers (8 per thread).
__device__ __forceinline__ void load_chunk(const float* H, int64_t n, int64_t j0, int nb,
                                           int64_t r0, bool vec4, float (&v)[8]) {
  const int t = threadIdx.x;
  const int r = t >> 3, seg = (t & 7) * 8;
  const int64_t i = r0 + r;
  const float* src = H + i * n + j0 + seg;
  if (i < j0 && vec4 && seg + 8 <= nb) {
    const float4 p = *reinterpret_cast<const float4*>(src);
    const float4 q = *reinterpret_cast<const float4*>(src + 4);
    v[0] = p.x; v[1] = p.y; v[2] = p.z; v[3] = p.w;
    v[4] = q.x; v[5] = q.y; v[6] = q.z; v[7] = q.w;
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = (i < j0 && seg + q < nb) ? src[q] : 0.f;
  }
}

// Factor the diagonal block A_JJ = R_JJ R_JJ^T (reverse order), invert it,
// and form the panel above it, R[i, J] = A[i, J] U_JJ^T.  Every CTA factors
// the (small) block itself, so no extra launch sits on the sequential path;
// CTA 0 stages U_JJ (64 x 64, row-major) at stage[j0 * 64].  A short block
// (nb < 64) is padded with the identity.  The panel rows are also written
// as bf16 hi/mid/lo splits for the tensor-core Schur update.
// The diagonal step of block J (rows/columns j0 .. j0 + nb) by CTA cta of
// ncta: returns false (uniformly over the CTA) when a pivot is not
// positive, after CTA 0 has recorded info.  256 threads.
__device__ bool diag_step(DiagSmem& S, float* H, int64_t n, int64_t j0, int nb, int* info,
                          __nv_bfloat16* splits, float* stage, float* stage_r, int vec4, int cta,
                          int ncta) {
  const int tid = threadIdx.x;
  {
    const int tx = tid & 63, ty = tid >> 6;
    float x[NB / 4];
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {  // all sixteen loads in flight
      const int r = 4 * sl + ty;
      x[sl] = (r <= tx && tx < nb) ? H[(j0 + r) * n + j0 + tx] : 0.f;
    }
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {
      const int r = 4 * sl + ty;
      S.x.a[r][tx] = (tx < nb) ? x[sl] : (r == tx ? 1.f : 0.f);
      S.u[r][tx] = 0.f;
    }
  }
  // the first chunk of panel rows is fetched while the block is factored
  float pv[8];
  const int64_t chunk0 = (int64_t)cta * PR;
  load_chunk(H, n, j0, nb, chunk0, vec4 != 0, pv);
  if (tid == 0) S.bad = 0;
  __syncthreads();
  if (!factor_invert_block(S)) {
    if (tid == 0 && cta == 0) *info = (int)(j0 + S.bad);
    return false;  // uniform: read after the barrier
  }
  // CTA 0 stages R_JJ when the factor itself is kept (before U_JJ^T
  // overwrites it)
  if (stage_r && cta == 0) {
    float* dst = stage_r + j0 * NB;
    for (int t = tid; t < nb * NB; t += blockDim.x) {
      const int r = t >> 6, c = t & 63;
      dst[t] = (c >= r) ? S.x.a[r][c] : 0.f;
    }
    __syncthreads();
  }
  // U_JJ^T (over R_JJ, no longer needed); CTA 0 stages U_JJ.
  for (int t = tid; t < NB * NB; t += blockDim.x) {
    const int r = t >> 6, c = t & 63;
    S.x.ut[c][r] = S.u[r][c];
  }
  if (cta == 0) {
    float* dst = stage + j0 * NB;
    for (int t = tid; t < nb * NB; t += blockDim.x) dst[t] = S.u[t >> 6][t & 63];
  }
  // Panel rows, chunks of PR rows: R[i][c] = sum_k A[i][k] U[c][k].
  const int64_t plane = (int64_t)n * NB;
  const int rp = tid >> 4, c0 = (tid & 15) * 4;
  for (int64_t r0 = chunk0; r0 < j0; r0 += (int64_t)ncta * PR) {
    {
      const int r = tid >> 3, seg = (tid & 7) * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) S.y.ach[r][seg + q] = pv[q];
    }
    __syncthreads();
    // the next chunk of this CTA is fetched while this one is multiplied
    if (r0 + (int64_t)ncta * PR < j0) load_chunk(H, n, j0, nb, r0 + (int64_t)ncta * PR, vec4 != 0, pv);
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 16
    for (int k = 0; k < NB; ++k) {
      const float a0 = S.y.ach[2 * rp][k], a1 = S.y.ach[2 * rp + 1][k];
      const float4 w = *reinterpret_cast<const float4*>(&S.x.ut[k][c0]);
      acc[0][0] = fmaf(a0, w.x, acc[0][0]);
      acc[0][1] = fmaf(a0, w.y, acc[0][1]);
      acc[0][2] = fmaf(a0, w.z, acc[0][2]);
      acc[0][3] = fmaf(a0, w.w, acc[0][3]);
      acc[1][0] = fmaf(a1, w.x, acc[1][0]);
      acc[1][1] = fmaf(a1, w.y, acc[1][1]);
      acc[1][2] = fmaf(a1, w.z, acc[1][2]);
      acc[1][3] = fmaf(a1, w.w, acc[1][3]);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t i = r0 + 2 * rp + h;
      if (i >= j0) continue;
      float* row = H + i * n + j0 + c0;
      if (vec4 && c0 + 4 <= nb) {
        *reinterpret_cast<float4*>(row) = make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]);
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (c0 + q < nb) row[q] = acc[h][q];
      }
      uint32_t wh[2] = {0u, 0u}, wm[2] = {0u, 0u}, wl[2] = {0u, 0u};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float x = acc[h][q];
        const __nv_bfloat16 bh = __float2bfloat16_rn(x);
        const float r1 = x - __bfloat162float(bh);
        const __nv_bfloat16 bm = __float2bfloat16_rn(r1);
        const __nv_bfloat16 bl = __float2bfloat16_rn(r1 - __bfloat162float(bm));
        const int sh = 16 * (q & 1);
        wh[q >> 1] |= (uint32_t)__bfloat16_as_ushort(bh) << sh;
        wm[q >> 1] |= (uint32_t)__bfloat16_as_ushort(bm) << sh;
        wl[q >> 1] |= (uint32_t)__bfloat16_as_ushort(bl) << sh;
      }
      const int64_t off = i * NB + c0;
      *reinterpret_cast<uint2*>(splits + off) = make_uint2(wh[0], wh[1]);
      *reinterpret_cast<uint2*>(splits + plane + off) = make_uint2(wm[0], wm[1]);
      *reinterpret_cast<uint2*>(splits + 2 * plane + off) = make_uint2(wl[0], wl[1]);
    }
    __syncthreads();  // ach is rewritten by the next chunk
  }
  return true;
}

__global__ void __launch_bounds__(256) diag_panel_kernel(float* H, int64_t n, int64_t j0, int nb,
                                                         int* info, __nv_bfloat16* splits,
                                                         float* stage, float* stage_r, int vec4) {
  if (*info != 0) return;
  __shared__ DiagSmem S;
  diag_step(S, H, n, j0, nb, info, splits, stage, stage_r, vec4, blockIdx.x, gridDim.x);
}

// ---------------------------------------------------------------------------
// The diagonal step of the persistent kernel: as diag_step, but each
// diagonal CTA handles its panel rows in chunks of 128 that arrive by
// cp.async while the block is factored, and multiplies them by U_JJ^T with
// 4 x 8 register tiles.
constexpr int PRF = 128;   // panel rows per chunk

struct alignas(16) DiagSmemP {
  union {
    float a[NB][NB + 1];      // A_JJ (upper) -> R_JJ
  } x;
  float u[NB][NB + 1];        // U_JJ (upper, zero below)
  union {
    float tb[32][33];         // products R12 U22 while U_JJ is assembled
    float wk[NB][NB + 4];     // then U_JJ^T
  } y;
  float ach[PRF][NB + 4];     // panel rows A[i, J]
  float rinv[NB];
  int bad;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Starts the copies of A[i, J] (columns j0 .. j0 + nb) of rows r0 .. r0 + PRF - 1
// (zero beyond nb and in the rows from rend on).
__device__ __forceinline__ void fetch_rows(DiagSmemP& S, const float* H, int64_t n, int64_t j0, int nb,
                                           int64_t r0, int64_t rend) {
  const int tid = threadIdx.x;
#pragma unroll 4
  for (int q = 0; q < PRF * 16 / 256; ++q) {
    const int t = tid + 256 * q;
    const int row = t >> 4, seg = t & 15;
    const int64_t i = r0 + row;
    const int c = 4 * seg;
    int valid = nb - c;
    valid = valid < 0 ? 0 : (valid > 4 ? 4 : valid);
    if (i >= rend) valid = 0;
    const float* src = (valid > 0) ? H + i * n + j0 + c : H;
    cp_async16(&S.ach[row][c], src, 4 * valid);
  }
  cp_async_commit();
}

// acc[j][q] = sum_k ach[rg + 32 j][k] wk[k][8 cg + q] for the first NSL
// 32-row slices.
template <int NSL>
__device__ __forceinline__ void panel_product(const DiagSmemP& S, int rg, int cg, float (&acc)[4][8]) {
#pragma unroll 4
  for (int k = 0; k < NB; ++k) {
    const float4 w0 = *reinterpret_cast<const float4*>(&S.y.wk[k][8 * cg]);
    const float4 w1 = *reinterpret_cast<const float4*>(&S.y.wk[k][8 * cg + 4]);
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int j = 0; j < NSL; ++j) {
      const float av = S.ach[rg + 32 * j][k];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[j][q] = fmaf(av, wv[q], acc[j][q]);
    }
  }
}

// ---- leader CTA: the chain of diagonal blocks -----------------------------
// On entry S.x.a holds the diagonal block (upper triangle; identity beyond
// nb), S.u is zero and S.bad is zero.  Factors and inverts it, stages U_JJ
// (64 x 64 row-major at stage[j0 * 64]) and, when stage_r is given, R_JJ
// (at stage_r[j0 * 64]), and leaves U_JJ^T in S.y.wk.
__device__ bool leader_factor(DiagSmemP& S, int64_t j0, int* info, float* stage, float* stage_r) {
  const int tid = threadIdx.x;
  if (!factor_invert_block(S)) {
    if (tid == 0) *info = (int)(j0 + S.bad);
    return false;  // uniform: read after the barrier
  }
  // all 64 x 64 (a short block's identity padding too: the panel CTAs
  // multiply by the whole U_JJ; the staging area has room for it)
  float* dst = stage + j0 * NB;
  float* dstr = stage_r ? stage_r + j0 * NB : nullptr;
  for (int t = tid; t < NB * NB; t += blockDim.x) {
    const int k = t >> 6, c = t & 63;
    S.y.wk[k][c] = S.u[c][k];
    dst[t] = S.u[k][c];
    if (dstr) dstr[t] = (c >= k) ? S.x.a[k][c] : 0.f;
  }
  return true;
}

// The next diagonal block with this step's update folded in:
//   P = A[j0 - 64 : j0, J] U_JJ^T   (those 64 rows of the panel; nb = width of J)
//   S.x.a = A[J-1, J-1] - P P^T      (upper triangle)
// A[J-1, J-1] must hold every update of the later steps (the Schur CTAs
// leave this block out of step J's update).  The 64 rows of A are read by
// leader_rows before the panel CTAs overwrite them with R.
__device__ void leader_rows(DiagSmemP& S, const float* H, int64_t n, int64_t j0, int nb) {
  const int tid = threadIdx.x;
  const int64_t jp = j0 - NB;
  const int r = tid >> 2, c0 = (tid & 3) * 16;
  const float* src = H + (jp + r) * n + j0 + c0;
  float v[16];
#pragma unroll
  for (int q = 0; q < 16; q += 4) {
    if (c0 + q + 4 <= nb) {
      const float4 x = *reinterpret_cast<const float4*>(src + q);
      v[q] = x.x; v[q + 1] = x.y; v[q + 2] = x.z; v[q + 3] = x.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[q + e] = (c0 + q + e < nb) ? src[q + e] : 0.f;
    }
  }
#pragma unroll
  for (int q = 0; q < 16; ++q) S.ach[r][c0 + q] = v[q];
  __syncthreads();
}

// Tensor-core form of the two 64^3 products of the leader (P = A_rows U^T,
// then S.x.a -= P P^T): operands split into bf16 hi/mid/lo in the UMMA
// 128-byte-swizzled K-major layout (rows of 128 bytes), six split products
// per 16-deep k step, M = 128 (rows 64 .. 127 of the A operand stay zero),
// N = 64, accumulators in TMEM columns 0 .. 63 (P) and 64 .. 127 (P P^T).
constexpr int LSPLIT_A = 128 * 128;            // 16 KB: 128 rows x 64 k bf16
constexpr int LSPLIT_B = 64 * 128;             // 8 KB: 64 rows x 64 k bf16
constexpr int LEAD_SPLIT_BYTES = 3 * LSPLIT_A + 3 * LSPLIT_B;   // 72 KB

__device__ __forceinline__ uint32_t kmaj_off(int r, int k) {
  return (uint32_t)(r * 128 + ((((k >> 3) ^ (r & 7))) << 4) + (k & 7) * 2);
}

// Splits four consecutive-k floats of row r into three bf16 planes.
__device__ __forceinline__ void lsplit4(uint8_t* base, uint32_t plane, int r, int k, float4 v) {
  const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
  const float r0 = v.x - __low2float(h01), r1 = v.y - __high2float(h01);
  const float r2 = v.z - __low2float(h23), r3 = v.w - __high2float(h23);
  const __nv_bfloat162 m01 = __floats2bfloat162_rn(r0, r1);
  const __nv_bfloat162 m23 = __floats2bfloat162_rn(r2, r3);
  const __nv_bfloat162 l01 = __floats2bfloat162_rn(r0 - __low2float(m01), r1 - __high2float(m01));
  const __nv_bfloat162 l23 = __floats2bfloat162_rn(r2 - __low2float(m23), r3 - __high2float(m23));
  auto bits = [](__nv_bfloat162 x) { return *reinterpret_cast<const uint32_t*>(&x); };
  const uint32_t off = kmaj_off(r, k);
  *reinterpret_cast<uint2*>(base + off) = make_uint2(bits(h01), bits(h23));
  *reinterpret_cast<uint2*>(base + plane + off) = make_uint2(bits(m01), bits(m23));
  *reinterpret_cast<uint2*>(base + 2 * plane + off) = make_uint2(bits(l01), bits(l23));
}

// One thread: the 24 MMAs of a 64-deep product, D[tmem_col ..] = A B^T.
__device__ __forceinline__ void lead_mma(uint32_t tmem_d, uint32_t sa, uint32_t sb, uint32_t pb) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 64, false, false);
  const int pa_[6] = {0, 0, 1, 0, 2, 1};
  const int pb_[6] = {0, 1, 0, 2, 0, 1};
  uint32_t acc = 0;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int t = 0; t < 6; ++t) {
      const uint64_t da = smem_desc_sw128(sa + pa_[t] * LSPLIT_A + kk * 32, 16, 1024);
      const uint64_t db = smem_desc_sw128(sb + pb_[t] * pb + kk * 32, 16, 1024);
      mma_bf16(tmem_d, da, db, idesc, acc);
      acc = 1;
    }
  }
}

// The next diagonal block: P = A[j0 - 64 : j0, J] U_JJ^T (rows in S.ach,
// U_JJ in S.u), then S.x.a = A[J-1, J-1] - P P^T (upper triangle).  sp: the
// 1024-aligned split area (its A rows 64 .. 127 are zero); bar: an mbarrier
// of this CTA, par its next phase parity.  256 threads.
__device__ bool leader_next(DiagSmemP& S, uint8_t* sp, uint32_t tmem, uint32_t bar, uint32_t& par,
                            const float* H, int64_t n, int64_t j0) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t jp = j0 - NB;
  uint8_t* SA = sp;
  uint8_t* SB = sp + 3 * LSPLIT_A;
  const uint32_t sa = smem_u32(SA), sb = smem_u32(SB);
  {
    // splits of the 64 A rows and of U's rows (U[c][k]: B K-major)
    const int r = tid >> 2, k0 = (tid & 3) * 16;
#pragma unroll
    for (int q = 0; q < 16; q += 4) {
      const float4 v = *reinterpret_cast<const float4*>(&S.ach[r][k0 + q]);
      lsplit4(SA, LSPLIT_A, r, k0 + q, v);
      const float4 w = make_float4(S.u[r][k0 + q], S.u[r][k0 + q + 1], S.u[r][k0 + q + 2], S.u[r][k0 + q + 3]);
      lsplit4(SB, LSPLIT_B, r, k0 + q, w);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    lead_mma(tmem, sa, sb, LSPLIT_B);
    mma_commit(bar);
  }
  // meanwhile: the diagonal block J - 1 from H, S.u cleared
  {
    const int tx = tid & 63, ty = tid >> 6;
    float x[NB / 4];
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {
      const int r = 4 * sl + ty;
      x[sl] = (r <= tx) ? H[(jp + r) * n + jp + tx] : 0.f;
    }
#pragma unroll
    for (int sl = 0; sl < NB / 4; ++sl) {
      S.x.a[4 * sl + ty][tx] = x[sl];
      S.u[4 * sl + ty][tx] = 0.f;
    }
  }
  if (tid == 0) S.bad = 0;
  int good = 1;
  if (warp < 2) {
    if (lane == 0) good = mbar_wait(bar, par) ? 1 : 0;
    good = __shfl_sync(0xffffffffu, good, 0);
    __syncwarp();
    if (good) {
      tc_fence_after();
      // P rows 32 warp + lane: two loads of 32 columns, then the splits of
      // the row into SA (rows 0 .. 63; A and B of the second product)
      const int r = 32 * warp + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 32 * h, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; q += 4)
          lsplit4(SA, LSPLIT_A, r, 32 * h + q,
                  make_float4(__uint_as_float(v[q]), __uint_as_float(v[q + 1]), __uint_as_float(v[q + 2]),
                              __uint_as_float(v[q + 3])));
      }
    }
  }
  par ^= 1u;
  fence_proxy_async_smem();
  tc_fence_before();
  good = __syncthreads_and(good);
  if (!good) return false;
  if (tid == 0) {
    tc_fence_after();
    lead_mma(tmem + 64, sa, sa, LSPLIT_A);   // P P^T: B = the first 64 rows of P's splits
    mma_commit(bar);
  }
  if (warp < 2) {
    if (lane == 0) good = mbar_wait(bar, par) ? 1 : 0;
    good = __shfl_sync(0xffffffffu, good, 0);
    __syncwarp();
    if (good) {
      tc_fence_after();
      const int r = 32 * warp + lane;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64 + 32 * h, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          const int c = 32 * h + q;
          if (c >= r) S.x.a[r][c] -= __uint_as_float(v[q]);
        }
      }
    }
  }
  par ^= 1u;
  tc_fence_before();
  good = __syncthreads_and(good);
  return good != 0;
}

// ---- panel CTAs: R[i, J] = A[i, J] U_JJ^T for a share of the rows i < j0 ----
// U_JJ comes from the leader's staging.  Rows arrive by cp.async in chunks
// of 128 and are multiplied with 4 x 8 register tiles; the result goes to H
// and, as bf16 hi/mid/lo splits, to the Schur tiles.
__device__ void panel_rows(DiagSmemP& S, float* H, int64_t n, int64_t j0, int nb,
                           __nv_bfloat16* splits, const float* stage, int pcta, int npan) {
  const int tid = threadIdx.x;
  // this CTA's rows: an even share of 0 .. j0, in multiples of 32
  const int64_t per = (((j0 + npan - 1) / npan + 31) / 32) * 32;
  const int64_t rbeg = (int64_t)pcta * per;
  const int64_t rend = (rbeg + per < j0) ? rbeg + per : j0;
  if (rbeg >= rend) return;
  fetch_rows(S, H, n, j0, nb, rbeg, rend);
  const float* src = stage + j0 * NB;
  for (int t = tid; t < NB * NB; t += blockDim.x) {
    const int c = t >> 6, k = t & 63;
    S.y.wk[k][c] = src[t];  // U[c][k]
  }
  const int64_t plane = (int64_t)n * NB;
  const int rg = tid >> 3, cg = tid & 7;
  for (int64_t r0 = rbeg; r0 < rend; r0 += PRF) {
    cp_async_wait_all();
    __syncthreads();
    float acc[4][8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[j][q] = 0.f;
    const int rows = (int)((rend - r0 < PRF) ? (rend - r0) : PRF);
    // only the 32-row slices that hold rows of the panel (uniform branch)
    const int nsl = (rows + 31) >> 5;
    if (nsl == 4) panel_product<4>(S, rg, cg, acc);
    else if (nsl == 3) panel_product<3>(S, rg, cg, acc);
    else if (nsl == 2) panel_product<2>(S, rg, cg, acc);
    else panel_product<1>(S, rg, cg, acc);
    __syncthreads();                          // the rows are consumed
    if (r0 + PRF < rend) fetch_rows(S, H, n, j0, nb, r0 + PRF, rend);
    auto bits = [](__nv_bfloat162 v) { return *reinterpret_cast<const uint32_t*>(&v); };
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t i = r0 + rg + 32 * j;
      if (i >= rend) continue;
      float* row = H + i * n + j0 + 8 * cg;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c0 = 8 * cg + 4 * h;
        const float* v = &acc[j][4 * h];
        if (c0 + 4 <= nb) {
          *reinterpret_cast<float4*>(row + 4 * h) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (c0 + q < nb) row[4 * h + q] = v[q];
        }
        const __nv_bfloat162 h01 = __floats2bfloat162_rn(v[0], v[1]);
        const __nv_bfloat162 h23 = __floats2bfloat162_rn(v[2], v[3]);
        const float e0 = v[0] - __low2float(h01), e1 = v[1] - __high2float(h01);
        const float e2 = v[2] - __low2float(h23), e3 = v[3] - __high2float(h23);
        const __nv_bfloat162 m01 = __floats2bfloat162_rn(e0, e1);
        const __nv_bfloat162 m23 = __floats2bfloat162_rn(e2, e3);
        const __nv_bfloat162 l01 = __floats2bfloat162_rn(e0 - __low2float(m01), e1 - __high2float(m01));
        const __nv_bfloat162 l23 = __floats2bfloat162_rn(e2 - __low2float(m23), e3 - __high2float(m23));
        const int64_t off = i * NB + c0;
        *reinterpret_cast<uint2*>(splits + off) = make_uint2(bits(h01), bits(h23));
        *reinterpret_cast<uint2*>(splits + plane + off) = make_uint2(bits(m01), bits(m23));
        *reinterpret_cast<uint2*>(splits + 2 * plane + off) = make_uint2(bits(l01), bits(l23));
      }
    }
  }
  cp_async_wait_all();
}

// Copy the staged diagonal blocks U_JJ into H (one CTA per block).  They are
// staged because other CTAs of a diag_panel launch still read A_JJ from H.
__global__ void __launch_bounds__(256) diag_store_kernel(float* H, int64_t n, const float* stage,
                                                         const int* info) {
  if (*info != 0) return;
  const int64_t j0 = (int64_t)blockIdx.x * NB;
  const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
  const float* src = stage + j0 * NB;
  for (int t = threadIdx.x; t < nb * NB; t += blockDim.x) {
    const int r = t >> 6, c = t & 63;
    if (c < nb) H[(j0 + r) * n + j0 + c] = src[t];
  }
}

// ---------------------------------------------------------------------------
// The whole blocked factorisation as one persistent kernel: one CTA per SM
// (cooperative launch, so every CTA is resident and CTAs may wait for one
// another), no launch per step.  The first nd CTAs run the diagonal steps
// (diag_step_p: each factors the block, they share the panel rows), the
// others the tensor-core Schur tiles, the last tile column of each step
// first: it holds the next diagonal block, so the next diagonal step starts
// while the rest of the update is still running (a one-step look-ahead).
// Tile (r, c) always belongs to the Schur CTA (c (c+1)/2 + r) mod ns, so the
// updates of one tile follow each other in that CTA's program order.
// Cross-CTA order goes through counters in global memory:
//   panel_done[J]  diagonal CTAs that finished D(J)        (step J waits for all)
//   colready[J-1]  finished last-column tiles of step J    (D(J-1) waits for all)
//   schur_done[J]  finished tiles of step J                (D(J-2) waits: it reuses
//                                                           the split buffer of J)
// Every wait is bounded; a timeout sets the device status and an abort flag
// that ends every CTA's loop.
constexpr int PERSIST_THREADS = 256;
// the leader's split area sits after its DiagSmemP, 1024-aligned
constexpr int LEAD_SPLIT_OFF = (int)((sizeof(DiagSmemP) + 1023) & ~(size_t)1023);
constexpr int LEAD_BODY = LEAD_SPLIT_OFF + LEAD_SPLIT_BYTES;
constexpr int PERSIST_BODY = (schur::TILE_SMEM > LEAD_BODY) ? schur::TILE_SMEM : LEAD_BODY;
constexpr int PERSIST_SMEM = PERSIST_BODY + 1024 + 256;
static_assert(sizeof(DiagSmemP) + 2048 + 256 <= 227 * 1024, "diagonal step fits one CTA's shared memory");

struct PersistArgs {
  float* H;
  int64_t n;
  int nblk;
  __nv_bfloat16* splits[2];
  float* stage;
  float* stage_r;   // R_JJ staging (nullptr: only U_JJ)
  int* info;
  int* ctr;     // panel_done, colready, schur_done, uready, diagready (nblk each), abort
  int vec4;
  int npanel;   // CTAs that form the panel rows
};

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Thread 0 waits until *p >= target (bounded, and ended by the abort flag);
// the result is shared with the whole CTA.  Orders the CTA's later reads
// (generic and TMA) after the other CTAs' published writes.
__device__ __forceinline__ bool cta_wait(const int* p, int target, int* abortf,
                                         unsigned long long limit_ns = kWaitLimitNs) {
  int ok = 1;
  if (threadIdx.x == 0 && ld_acquire_gpu(p) < target) {
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (ld_acquire_gpu(p) >= target) break;
      if (ld_acquire_gpu(abortf) != 0) {
        ok = 0;
        break;
      }
      if ((it & 63u) == 0 && global_ns() - t0 > limit_ns) {
        record_timeout();
        atomicExch(abortf, 1);
        ok = 0;
        break;
      }
      __nanosleep(100);
    }
  }
  ok = __syncthreads_and(ok);
  fence_proxy_async_global();
  return ok != 0;
}

// Publishes this CTA's global writes (generic and TMA) and adds 1 to each
// counter given.
__device__ __forceinline__ void cta_publish(int* p0, int* p1) {
  fence_proxy_async_global();
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    red_release_gpu_add(p0, 1);
    if (p1) red_release_gpu_add(p1, 1);
  }
}

__device__ __forceinline__ int tri_count(int nt) { return nt * (nt + 1) / 2; }

// Column-major index of the upper triangle -> (r, c), r <= c.
__device__ __forceinline__ void tri_rc(int idx, int& r, int& c) {
  c = (int)((sqrtf(8.f * (float)idx + 1.f) - 1.f) * 0.5f);
  while (tri_count(c) > idx) --c;
  while (tri_count(c + 1) <= idx) ++c;
  r = idx - tri_count(c);
}

__global__ void __launch_bounds__(PERSIST_THREADS, 1)
    chol_persistent_kernel(const __grid_constant__ CUtensorMap p0h, const __grid_constant__ CUtensorMap p0m,
                           const __grid_constant__ CUtensorMap p0l, const __grid_constant__ CUtensorMap p1h,
                           const __grid_constant__ CUtensorMap p1m, const __grid_constant__ CUtensorMap p1l,
                           const __grid_constant__ CUtensorMap mC, PersistArgs a) {
  if (*a.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PERSIST_BODY);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3);
  const uint32_t full = smem_u32(&bars[0]);
  const uint32_t cbar = smem_u32(&bars[1]);
  const uint32_t accbar = smem_u32(&bars[2]);
  const int warp = threadIdx.x >> 5;
  const int cta = blockIdx.x, ncta = gridDim.x;
  const int nblk = a.nblk;
  const int64_t n = a.n;
  int* panel_done = a.ctr;
  int* colready = a.ctr + nblk;
  int* schur_done = a.ctr + 2 * nblk;
  int* uready = a.ctr + 3 * nblk;
  int* diagready = a.ctr + 4 * nblk;
  int* abortf = a.ctr + 5 * nblk;

  if (threadIdx.x == 0) {
    mbar_init(full, 1);
    mbar_init(cbar, 1);
    mbar_init(accbar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), schur::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const schur::TileMaps maps[2] = {{&p0h, &p0m, &p0l, &mC}, {&p1h, &p1m, &p1l, &mC}};
  uint32_t tcount = 0;
  // Roles: CTA 0 leads the chain of diagonal blocks, CTAs 1 .. npan form the
  // panel rows, the rest run the Schur tiles.
  const int npan = a.npanel, ns = ncta - 1 - npan;

  // nt(J): tiles per side of the update of step J (the upper triangle of j0 x j0)
  auto nt_of = [](int J) { return (J * NB + 127) / 128; };

  if (cta == 0) {
    // ---- leader
    DiagSmemP& F = *reinterpret_cast<DiagSmemP*>(smem);
    uint8_t* sp = smem + LEAD_SPLIT_OFF;
    uint32_t par = 0;
    for (int t = threadIdx.x; t < LEAD_SPLIT_BYTES / 16; t += blockDim.x)
      reinterpret_cast<uint4*>(sp)[t] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    {
      const int64_t j0 = (int64_t)(nblk - 1) * NB;
      const int nb = (int)(n - j0);
      const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
      for (int sl = 0; sl < NB / 4; ++sl) {
        const int r = 4 * sl + ty;
        F.x.a[r][tx] = (tx < nb) ? ((r <= tx) ? a.H[(j0 + r) * n + j0 + tx] : 0.f) : (r == tx ? 1.f : 0.f);
        F.u[r][tx] = 0.f;
      }
      if (threadIdx.x == 0) F.bad = 0;
      __syncthreads();
    }
    for (int J = nblk - 1; J >= 0; --J) {
      const int64_t j0 = (int64_t)J * NB;
      const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
      if (!leader_factor(F, j0, a.info, a.stage, a.stage_r)) {
        if (threadIdx.x == 0) atomicExch(abortf, 2);  // stop every other CTA
        break;
      }
      if (J > 0) {
        // the 64 panel rows of block J - 1 need step J + 1's last tile
        // column; they are read before the panel CTAs may overwrite them
        if (J + 1 <= nblk - 1 && !cta_wait(&colready[J], nt_of(J + 1), abortf)) break;
        leader_rows(F, a.H, n, j0, nb);
      }
      cta_publish(&uready[J], nullptr);
      if (J == 0) break;
      // block J - 1's diagonal needs step J + 1's tile holding it
      if (J + 1 <= nblk - 1 && !cta_wait(&diagready[J - 1], 1, abortf)) break;
      if (!leader_next(F, sp, tmem, accbar, par, a.H, n, j0)) {
        if (threadIdx.x == 0) atomicExch(abortf, 1);
        break;
      }
    }
  } else if (cta <= npan) {
    // ---- panel rows
    DiagSmemP& F = *reinterpret_cast<DiagSmemP*>(smem);
    const int pc = cta - 1;
    for (int J = nblk - 1; J >= 1; --J) {
      if (!cta_wait(&uready[J], 1, abortf)) break;
      if (J + 1 <= nblk - 1 && !cta_wait(&colready[J], nt_of(J + 1), abortf)) break;
      if (J + 2 <= nblk - 1 && !cta_wait(&schur_done[J + 2], tri_count(nt_of(J + 2)), abortf)) break;
      const int64_t j0 = (int64_t)J * NB;
      const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
      panel_rows(F, a.H, n, j0, nb, a.splits[J & 1], a.stage, pc, npan);
      cta_publish(&panel_done[J], nullptr);
    }
  } else {
    // ---- Schur tiles
    const int sc = cta - 1 - npan;
    // One tile of step J; the last-column tiles and the tile holding block
    // J - 2's diagonal are published at once (the panel CTAs and the leader
    // wait for them), the bulk tiles of a step together at its end.
    auto run_tile = [&](int J, int idx, bool last, bool diag) -> bool {
      int r, c;
      tri_rc(idx, r, c);
      const bool urgent = last || diag;
      const bool ok = schur::tile<0, 8>(smem, full, cbar, accbar, tcount & 1u, tmem, maps[J & 1], a.H,
                                        n, (int64_t)J * NB, (int64_t)r * 128, (int64_t)c * 128, 1,
                                        urgent ? 1 : 0, (int64_t)(J - 1) * NB);
      ++tcount;
      tc_fence_before();
      if (urgent) {
        cta_publish(&schur_done[J], last ? &colready[J - 1] : nullptr);
        if (diag) cta_publish(&diagready[J - 2], nullptr);
      }
      const int all = __syncthreads_and(ok ? 1 : 0);
      tc_fence_after();
      if (!all) {
        if (threadIdx.x == 0) atomicExch(abortf, 1);
        return false;
      }
      return true;
    };
    bool ok = true;
    for (int J = nblk - 1; ok && J >= 1; --J) {
      const int nt = nt_of(J);
      const int lo = tri_count(nt - 1), hi = tri_count(nt);
      // the tile holding block J - 2's diagonal (the leader needs it next)
      int idx_d = -1;
      if (J >= 2) {
        const int d = ((J - 2) * NB) / 128;
        idx_d = tri_count(d) + d;
      }
      if (!cta_wait(&panel_done[J], npan, abortf)) break;
      // the last tile column (block J - 1's panel rows) first
      for (int idx = lo + ((sc - lo % ns) % ns + ns) % ns; ok && idx < hi; idx += ns)
        ok = run_tile(J, idx, true, idx == idx_d);
      if (ok && idx_d >= 0 && idx_d < lo && idx_d % ns == sc) ok = run_tile(J, idx_d, false, true);
      // the rest from the right
      const int top = lo - 1 - ((((lo - 1) - sc) % ns) + ns) % ns;   // largest idx < lo owned by sc
      int nbulk = 0;
      for (int idx = top; ok && idx >= 0; idx -= ns) {
        if (idx == idx_d) continue;
        ok = run_tile(J, idx, false, false);
        ++nbulk;
      }
      if (!ok) break;
      if (nbulk > 0) {
        if (threadIdx.x == 0) tma_store_wait_all();   // the bulk tiles' stores reached memory
        fence_proxy_async_global();
        __syncthreads();
        if (threadIdx.x == 0) {
          __threadfence();
          red_release_gpu_add(&schur_done[J], nbulk);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, schur::TMEM_COLS);
  }
}

// Self-test of the two bounded waits above: one CTA waits on a condition
// that nothing satisfies, with a short bound.  which 0: an mbarrier phase
// that no thread or copy completes (mbar_wait, as every tensor-core kernel
// uses it); which 1: a step counter that no CTA increments (cta_wait, as the
// persistent factorisation uses it), which also raises the abort flag.
// w[0] = counter, w[1] = abort flag, w[2] = 1 when the wait gave up.
__global__ void __launch_bounds__(32) wait_selftest_kernel(int which, unsigned long long limit_ns, int* w) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    w[0] = 0;
    w[1] = 0;
    w[2] = 0;
    __threadfence();
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  bool gave_up;
  if (which == 0) {
    int ok = 1;
    if (threadIdx.x == 0) ok = mbar_wait(smem_u32(&bar), 0u, limit_ns) ? 1 : 0;
    gave_up = __syncthreads_and(ok) == 0;
  } else {
    gave_up = !cta_wait(&w[0], 1, &w[1], limit_ns);
  }
  if (threadIdx.x == 0) w[2] = gave_up ? 1 : 0;
}

}  // namespace

kronq_status wait_selftest(int which, unsigned long long limit_ns, int* w, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(which, limit_ns, w);
  KQ_LAUNCH_CHECK("wait_selftest_kernel");
  return KRONQ_OK;
}

cudaError_t status_fetch_chol(int* out, cudaStream_t s) {
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

static size_t tbuf_bytes(int64_t n) {
  // recursive inverse: products T of the pairs of one level (at most n*n/4
  // floats); before it, the staged diagonal blocks U_JJ and R_JJ (n x 64
  // floats each)
  int64_t f = (n * n) / 4 + n + 64;
  if (f < 2 * n * NB + NB * NB) f = 2 * n * NB + NB * NB;
  return (((size_t)f * sizeof(float)) + 255) & ~size_t(255);
}

static size_t splits_bytes(int64_t n) {
  return (((size_t)3 * n * NB * sizeof(__nv_bfloat16)) + 255) & ~size_t(255);
}

size_t chol_core_workspace_bytes(int64_t n) {
  // T / staging buffer, two buffers of bf16 hi/mid/lo panel splits
  // (3 x n x 64 each), the step counters of the persistent kernel
  const int64_t nblk = ceil_div(n, NB);
  return tbuf_bytes(n) + 2 * splits_bytes(n) + (size_t)(5 * nblk + 4) * sizeof(int);
}

size_t chol_workspace_bytes(int64_t n) {
  return n > kOuterBlock ? chol_blocked_workspace_bytes(n) : chol_core_workspace_bytes(n);
}

size_t chol_tbuf_bytes(int64_t n) { return tbuf_bytes(n); }

kronq_status damp_only(float* H, int64_t n, float damp_rel, int* info, cudaStream_t s) {
  damp_kernel<<<1, 1024, 0, s>>>(H, n, damp_rel, nullptr, info, false);
  KQ_LAUNCH_CHECK("damp_kernel");
  return KRONQ_OK;
}

kronq_status damp_factor(float* H, int64_t n, float damp_rel, uint8_t* dead, int* info, cudaStream_t s) {
  damp_kernel<<<1, 1024, 0, s>>>(H, n, damp_rel, dead, info, true);
  KQ_LAUNCH_CHECK("damp_kernel");
  return KRONQ_OK;
}

kronq_status chol_upper_inverse(float* H, int64_t n, float damp_rel, bool skip_damp,
                                uint8_t* dead, int* info, void* ws, cudaStream_t s, bool want_u) {
  if (!skip_damp) {
    damp_kernel<<<1, 1024, 0, s>>>(H, n, damp_rel, dead, info, true);
    KQ_LAUNCH_CHECK("damp_kernel");
  } else {
    zero_info_kernel<<<1, 1, 0, s>>>(info);
    KQ_LAUNCH_CHECK("zero_info_kernel");
  }
  if (n <= 0) return KRONQ_OK;
  if (n > kOuterBlock) return chol_blocked(H, n, info, ws, s, want_u);
  return chol_core(H, n, info, ws, s, want_u);
}

kronq_status chol_core(float* H, int64_t n, int* info, void* ws, cudaStream_t s, bool want_u) {
  float* Tbuf = reinterpret_cast<float*>(ws);
  float* stage_r = want_u ? nullptr : Tbuf + n * NB;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  __nv_bfloat16* splits = reinterpret_cast<__nv_bfloat16*>(wsb + tbuf_bytes(n));
  __nv_bfloat16* splits1 = reinterpret_cast<__nv_bfloat16*>(wsb + tbuf_bytes(n) + splits_bytes(n));
  int* ctr = reinterpret_cast<int*>(wsb + tbuf_bytes(n) + 2 * splits_bytes(n));
  SchurMaps maps;
  if (n > NB) {
    kronq_status r = schur_maps(&maps, splits, H, n);
    if (r != KRONQ_OK) return r;
  }
  // Blocks are aligned from the top (0, NB, 2 NB, ...); the last may be short.
  const int64_t nblk = ceil_div(n, NB);
  const int64_t pmax = sm_count();
  const int vec4 = ((n % 4) == 0 && aligned(H, 16)) ? 1 : 0;
  // The persistent kernel (one launch for the whole chain) when the tile of
  // A can be staged by TMA and every CTA can be resident at once.
  bool persist = n > 4 * NB && maps.tma_c && nblk < (1 << 20);
  int coop = 0, per_sm = 0;
  if (persist) {
    int dev = 0;
    KQ_CUDA(cudaGetDevice(&dev));
    KQ_CUDA(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(&chol_persistent_kernel), PERSIST_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(persistent factorisation)");
    KQ_CUDA(cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, reinterpret_cast<const void*>(&chol_persistent_kernel), PERSIST_THREADS, PERSIST_SMEM));
    persist = coop != 0 && per_sm >= 1;
  }
  if (persist) {
    SchurMaps maps1;
    kronq_status r = schur_maps(&maps1, splits1, H, n);
    if (r != KRONQ_OK) return r;
    KQ_CUDA(cudaMemsetAsync(ctr, 0, (size_t)(5 * nblk + 4) * sizeof(int), s));
    const CUtensorMap* m0 = reinterpret_cast<const CUtensorMap*>(maps.raw);
    const CUtensorMap* m1 = reinterpret_cast<const CUtensorMap*>(maps1.raw);
    CUtensorMap a0 = m0[0], a1 = m0[1], a2 = m0[2], b0 = m1[0], b1 = m1[1], b2 = m1[2], c = m0[3];
    PersistArgs pa;
    pa.H = H;
    pa.n = n;
    pa.nblk = (int)nblk;
    pa.splits[0] = splits;
    pa.splits[1] = splits1;
    pa.stage = Tbuf;
    pa.stage_r = stage_r;
    pa.info = info;
    pa.ctr = ctr;
    pa.vec4 = vec4;
    pa.npanel = (int)(pmax >= 64 ? 31 : pmax / 2);
    void* args[] = {&a0, &a1, &a2, &b0, &b1, &b2, &c, &pa};
    KQ_CUDA(cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(&chol_persistent_kernel),
                                        dim3((unsigned)pmax), dim3(PERSIST_THREADS), args,
                                        (size_t)PERSIST_SMEM, s));
    count_launch();
  }
  for (int64_t bj = persist ? -1 : nblk - 1; bj >= 0; --bj) {
    const int64_t j0 = bj * NB;
    const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
    // One CTA per SM at most (each CTA factors the block itself), one chunk
    // of panel rows per CTA where that suffices.
    int64_t pg = j0 > 0 ? ceil_div(j0, PR) : 1;
    if (pg > pmax) pg = pmax;
    diag_panel_kernel<<<(unsigned)pg, 256, 0, s>>>(H, n, j0, nb, info, splits, Tbuf, stage_r, vec4);
    KQ_LAUNCH_CHECK("diag_panel_kernel");
    if (j0 == 0) break;
    kronq_status r = schur_update_tc(&maps, H, n, j0, info, s);
    if (r != KRONQ_OK) return r;
  }
  if (!want_u) {
    // R: its diagonal blocks R_JJ from the staging, the blocks above them
    // already hold R.  The staged U_JJ stay for chol_core_finish_u.
    diag_store_kernel<<<(unsigned)nblk, 256, 0, s>>>(H, n, stage_r, info);
    KQ_LAUNCH_CHECK("diag_store_kernel");
    return KRONQ_OK;
  }
  return chol_core_finish_u(H, n, info, ws, s);
}

kronq_status chol_core_finish_u(float* H, int64_t n, int* info, void* ws, cudaStream_t s) {
  float* Tbuf = reinterpret_cast<float*>(ws);
  diag_store_kernel<<<(unsigned)ceil_div(n, NB), 256, 0, s>>>(H, n, Tbuf, info);
  KQ_LAUNCH_CHECK("diag_store_kernel");
  return chol_inverse_levels(H, n, NB, Tbuf, info, s);
}

kronq_status chol_inverse_levels(float* H, int64_t n, int64_t S0, float* Tbuf, const int* info,
                                 cudaStream_t s) {
  // Recursive inverse of the off-diagonal blocks: the diagonal blocks of
  // size S0 (aligned from the top, the last one possibly short) hold U_JJ,
  // the blocks above them R.
  for (int64_t S = S0; S < n; S *= 2) {
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
      TriGemm t;
      t.M = S; t.N = s2; t.K = s2;
      t.A = H + base * n + base + S; t.lda = n;
      t.B = H + (base + S) * n + base + S; t.ldb = n; t.b_upper = true;
      t.C = Tbuf; t.ldc = s2;
      t.alpha = 1.f;
      t.batch = (int)gp.cnt;
      t.strideA = 2 * S * n + 2 * S; t.strideB = 2 * S * n + 2 * S; t.strideC = S * s2;
      t.info = info;
      t.holdA = H; t.holdA_rows = n; t.holdA_cols = n;
      t.holdB = H; t.holdB_rows = n; t.holdB_cols = n;
      kronq_status r = trigemm_tc(t, s);
      if (r != KRONQ_OK) return r;
      // U12 = -U11 * T  (S x s2) = (S x S, upper)(S x s2)
      TriGemm u;
      u.M = S; u.N = s2; u.K = S;
      u.A = H + base * n + base; u.lda = n; u.a_upper = true;
      u.B = Tbuf; u.ldb = s2;
      u.C = H + base * n + base + S; u.ldc = n;
      u.alpha = -1.f;
      u.batch = (int)gp.cnt;
      u.strideA = 2 * S * n + 2 * S; u.strideB = S * s2; u.strideC = 2 * S * n + 2 * S;
      u.info = info;
      u.holdA = H; u.holdA_rows = n; u.holdA_cols = n;
      u.holdB = Tbuf; u.holdB_rows = gp.cnt * S; u.holdB_cols = s2;
      r = trigemm_tc(u, s);
      if (r != KRONQ_OK) return r;
    }
  }
  return KRONQ_OK;
}

}  // namespace kq

// Damping and the upper Cholesky factor of the damped inverse.
//
// GPTQ (which KronQ extends, KronQ README intro) needs the upper triangular
// U with U^T U = (H + lambda I)^-1.  Instead of inverting and factoring
// again, this library factors A = H + lambda I "in reverse": A = R R^T with
// R upper triangular (eliminating from the last index down), and then
// U = R^-1, since A^-1 = R^-T R^-1 = U^T U.  That is 2 n^3 / 3 flops in total.
//
// Blocked with nb = 64, bottom-right first.  For each diagonal block J:
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
__device__ __forceinline__ void leaf_factor(DiagSmem& S, int o) {
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
__device__ __forceinline__ void leaf_invert(DiagSmem& S, int o) {
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
__global__ void __launch_bounds__(256) diag_panel_kernel(float* H, int64_t n, int64_t j0, int nb,
                                                         int* info, __nv_bfloat16* splits,
                                                         float* stage, int vec4) {
  if (*info != 0) return;
  __shared__ DiagSmem S;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
  const int64_t chunk0 = (int64_t)blockIdx.x * PR;
  load_chunk(H, n, j0, nb, chunk0, vec4 != 0, pv);
  if (tid == 0) S.bad = 0;
  __syncthreads();

  for (int o = NB - LF; o >= 0; o -= LF) {
    if (tid == 0) leaf_factor(S, o);
    __syncthreads();
    if (S.bad) {
      if (tid == 0 && blockIdx.x == 0) *info = (int)(j0 + S.bad);
      return;  // uniform: read after the barrier
    }
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
  // U_JJ^T (over R_JJ, no longer needed); CTA 0 stages U_JJ.
  for (int t = tid; t < NB * NB; t += blockDim.x) {
    const int r = t >> 6, c = t & 63;
    S.x.ut[c][r] = S.u[r][c];
  }
  if (blockIdx.x == 0) {
    float* dst = stage + j0 * NB;
    for (int t = tid; t < nb * NB; t += blockDim.x) dst[t] = S.u[t >> 6][t & 63];
  }
  // Panel rows, chunks of PR rows: R[i][c] = sum_k A[i][k] U[c][k].
  const int64_t plane = (int64_t)n * NB;
  const int rp = tid >> 4, c0 = (tid & 15) * 4;
  for (int64_t r0 = chunk0; r0 < j0; r0 += (int64_t)gridDim.x * PR) {
    if (r0 != chunk0) load_chunk(H, n, j0, nb, r0, vec4 != 0, pv);
    {
      const int r = tid >> 3, seg = (tid & 7) * 8;
#pragma unroll
      for (int q = 0; q < 8; ++q) S.y.ach[r][seg + q] = pv[q];
    }
    __syncthreads();
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

}  // namespace

static size_t tbuf_bytes(int64_t n) {
  // recursive inverse: products T of the pairs of one level (at most n*n/4
  // floats); before it, the staged diagonal blocks U_JJ (n x 64 floats)
  int64_t f = (n * n) / 4 + n + 64;
  if (f < n * NB + NB * NB) f = n * NB + NB * NB;
  return (((size_t)f * sizeof(float)) + 255) & ~size_t(255);
}

size_t chol_workspace_bytes(int64_t n) {
  // T / staging buffer, then the bf16 hi/mid/lo splits of the current panel
  // (3 x n x 64)
  const size_t tbytes = tbuf_bytes(n);
  const size_t sbytes = (size_t)3 * n * NB * sizeof(__nv_bfloat16);
  return tbytes + sbytes;
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
  float* Tbuf = reinterpret_cast<float*>(ws);
  __nv_bfloat16* splits =
      reinterpret_cast<__nv_bfloat16*>(static_cast<uint8_t*>(ws) + tbuf_bytes(n));
  SchurMaps maps;
  if (n > NB) {
    kronq_status r = schur_maps(&maps, splits, H, n);
    if (r != KRONQ_OK) return r;
  }
  // Blocks are aligned from the top (0, NB, 2 NB, ...); the last may be short.
  const int64_t nblk = ceil_div(n, NB);
  const int64_t pmax = sm_count();
  const int vec4 = ((n % 4) == 0 && aligned(H, 16)) ? 1 : 0;
  for (int64_t bj = nblk - 1; bj >= 0; --bj) {
    const int64_t j0 = bj * NB;
    const int nb = (int)((j0 + NB <= n) ? NB : n - j0);
    // One CTA per SM at most (each CTA factors the block itself), one chunk
    // of panel rows per CTA where that suffices.
    int64_t pg = j0 > 0 ? ceil_div(j0, PR) : 1;
    if (pg > pmax) pg = pmax;
    diag_panel_kernel<<<(unsigned)pg, 256, 0, s>>>(H, n, j0, nb, info, splits, Tbuf, vec4);
    KQ_LAUNCH_CHECK("diag_panel_kernel");
    if (j0 == 0) break;
    kronq_status r = schur_update_tc(&maps, H, n, j0, info, s);
    if (r != KRONQ_OK) return r;
  }
  diag_store_kernel<<<(unsigned)nblk, 256, 0, s>>>(H, n, Tbuf, info);
  KQ_LAUNCH_CHECK("diag_store_kernel");
  // Recursive inverse of the off-diagonal blocks.
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

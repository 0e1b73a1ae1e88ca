// GPTQ-style blocked column sweep under the K-FAC loss.
//
// KronQ README intro (extends GPTQ/GPTAQ) and "Reproduce from scratch"
// (--w_bits --w_groupsize --w_asym).  Rows of W~ are independent once U is
// known, so the in-block sweep needs no block-wide synchronisation.  Sixteen
// lanes share a pair of rows: lane q holds, for both rows, the columns q,
// q + 16, ..., q + 112 of the 128-column block in registers, so every lane
// has later columns to update at every step and each value of U read from
// shared memory serves two rows.
//
// Every lane also holds a window of each row's next two columns c and
// c + 1, so the sixteen lanes evaluate the quantizer of column c on the same
// value and get the same scaled error e = (w - deq) / U_cc without a
// cross-lane step in the column chain.  After column c the window's column
// c + 1 takes its update, and the owner of column c + 2 (whose register now
// has every update up to column c) hands its value over with one shuffle,
// needed only after column c + 1's quantizer.  Window and owner register
// receive the same updates in the same order, so they hold the same value.
// The block runs in four rounds of 32 columns; after a round the two retired
// registers of each row are stored and the registers shift down by two, so
// one round's code serves all four with static register indices.
//
// Arithmetic: the quantizer and the error are single float32 operations
// (divisions by the group scale and by U_cc are multiplications by their
// correctly rounded reciprocals).  In the ordered test mode each update is a
// product then a difference (one rounding each), in ascending column order
// per element: bit for bit the float32 mirror.  Otherwise each update is one
// fused multiply-add, two columns at a time as packed float32x2 (sm_100).
//
// After each block the later columns get W[:, later] -= E_blk U[blk, later]
// (the lazy-batch update), either as a fast GEMM or, in the ordered test mode,
// with one rounding per product and per sum in ascending k.
//
// R form (SweepDesc::W0 set): the factor is R (H~ = R R^T) and only the
// diagonal blocks U_GG = (R_GG)^-1 of U = R^-1 are formed.  For the swept
// columns S and the rest T, GPTQ's partial state W_T - E_S U_ST equals
// W_T + F U_TT with F = (W0 - Q)_S R_ST, since E_S = (W0 - Q)_S R_SS and
// R_SS U_ST = -R_ST U_TT.  W then holds F; a block G starts from
// W0_G + F_G U_GG (its columns' partial state, from which GPTQ grids the
// group), is swept on U_GG exactly as in the U form, and hands
// D = deq - W0 of its columns to the trailing update with R's rows:
// F_later -= D_G R_G,later.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BW = 128;        // block width (columns)
constexpr int LPR = 16;        // lanes per pair of rows
constexpr int NREG = BW / LPR; // registers per row and lane: register k holds column 16k + q
constexpr int NP = NREG / 2;   // register pairs per row
constexpr int RC = 32;         // columns per round
constexpr int NROUND = BW / RC;
constexpr int RET = RC / LPR;  // registers retired per round (one pair)
constexpr int WARPS = 8;       // warps per CTA
constexpr int ROWS_PER_CTA = WARPS * 32 / LPR * 2;   // 32
// U block in shared memory, permuted: Up[c][q][k] = U[c][16k + q] for
// 16k + q > c (zero on and below the diagonal and past the block), k < 8,
// and zero for 8 <= k < 14 (round R reads k = 2R .. 2R + 7).  A stride of 18
// floats puts the sixteen lanes of a half warp on distinct bank pairs for
// the 8-byte reads of one column.
constexpr int UP_LD = 18;
constexpr int UP_ROW = LPR * UP_LD;
constexpr int SWEEP_SMEM = (BW * UP_ROW + BW) * (int)sizeof(float);
// R form: the CTA's rows of W0 for the block (odd stride: the four rows a
// warp reads at once sit in distinct banks) and the diagonal of U_GG
constexpr int W0_LD = BW + 1;
constexpr int RF_SMEM = SWEEP_SMEM + (ROWS_PER_CTA * W0_LD + BW) * (int)sizeof(float);
constexpr int UB_PER_THREAD = (BW * BW / 4) / (WARPS * 32);   // float4 loads of the U block

struct BlockArgs {
  SweepDesc d;
  int64_t j0;
  int bw;         // columns in this block
  int wide;       // 1: the grid of this block's first column was computed beforehand
  float* Eb;      // scaled-error output of this block (fp32) or nullptr
  int64_t lde;
  int slot;       // position of the block in its group (split buffers)
};

__device__ __forceinline__ void grid_from_range(float lo, float hi, int bits, bool asym, float& scale,
                                                float& zero) {
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
  scale = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
  zero = asym ? rintf(__fdiv_rn(-xmin, scale)) : (float)(1 << (bits - 1));
}

// Quantizer state of the current group.  The clamp of rint(w / scale) + zero
// to [0, maxq] is applied as the clamp of rint(w / scale) to [-zero,
// maxq - zero]: zero is an integer below 2^8, so both forms give the same
// deq = scale (q - zero) and the same code q.
struct Grid {
  float sc, zp, isc, lo, hi;
  float zp2;   // zero + 2^23: the code q = rr + zero is the low byte of rr + zp2
};

__device__ __forceinline__ Grid make_grid(float sc, float zp, float maxq) {
  Grid g;
  g.sc = sc;
  g.zp = zp;
  g.isc = __frcp_rn(sc);
  g.lo = __fsub_rn(0.f, zp);
  g.hi = __fsub_rn(maxq, zp);
  g.zp2 = __fadd_rn(zp, 8388608.f);
  return g;
}

__device__ __forceinline__ float reg_of(const float2 (&v)[NP], int k) {
  return (k & 1) ? v[k >> 1].y : v[k >> 1].x;
}

// Grid of the group that starts at block column cs, for one row: the
// sixteen lanes reduce over their registers in [cs, min(cs + group, bw)).
// Register k holds column 32 R + 16 k + q in round R.
__device__ __forceinline__ Grid group_start(const float2 (&v)[NP], int cs, int R, int q, int bw,
                                            const SweepDesc& d, bool live, int64_t r, int64_t gi,
                                            float maxq) {
  const int ce = min(cs + d.group, bw);
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int k = 0; k < NREG; ++k) {
    const int col = RC * R + LPR * k + q;
    const float x = reg_of(v, k);
    if (col >= cs && col < ce) {
      lo = fminf(lo, x);
      hi = fmaxf(hi, x);
    }
  }
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  float sc, zp;
  grid_from_range(lo, hi, d.bits, d.asym, sc, zp);
  if (q == 0 && live) {
    d.scales[r * d.ngroups + gi] = sc;
    d.zeros[r * d.ngroups + gi] = zp;
  }
  return make_grid(sc, zp, maxq);
}

// v -= e u on a pair of columns, with ne = -e in both halves.  Ordered
// mode: product then sum, each rounded (-(e u) rounds like e u), as scalar
// operations that are never fused; otherwise one packed fused multiply-add.
template <bool ORD>
__device__ __forceinline__ void upd2(float2& v, float2 ne, float2 u) {
  if (ORD) {
    v.x = __fadd_rn(v.x, __fmul_rn(ne.x, u.x));
    v.y = __fadd_rn(v.y, __fmul_rn(ne.y, u.y));
  } else {
    v = __ffma2_rn(ne, u, v);
  }
}

template <bool ORD>
__device__ __forceinline__ float upd1(float v, float ne, float u) {
  return ORD ? __fadd_rn(v, __fmul_rn(ne, u)) : fmaf(ne, u, v);
}

// rint for the quantizer: adding and removing 1.5 * 2^23 rounds to the
// nearest integer, ties to even, for |x| < 2^22 (two adds on the FMA pipe).
// Larger |x| give values beyond any grid, which the clamp that follows maps
// to the same end point as rint would.
__device__ __forceinline__ float rint_grid(float x) {
  return __fsub_rn(__fadd_rn(x, 12582912.f), 12582912.f);
}

// bf16 hi/lo split of one float4 into 4 + 4 bf16.
__device__ __forceinline__ void split4(float4 x, __nv_bfloat16* dh, __nv_bfloat16* dl) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x.x), h1 = __float2bfloat16_rn(x.y);
  const __nv_bfloat16 h2 = __float2bfloat16_rn(x.z), h3 = __float2bfloat16_rn(x.w);
  __nv_bfloat162 hh[2] = {__halves2bfloat162(h0, h1), __halves2bfloat162(h2, h3)};
  __nv_bfloat162 ll[2] = {
      __halves2bfloat162(__float2bfloat16_rn(x.x - __bfloat162float(h0)),
                         __float2bfloat16_rn(x.y - __bfloat162float(h1))),
      __halves2bfloat162(__float2bfloat16_rn(x.z - __bfloat162float(h2)),
                         __float2bfloat16_rn(x.w - __bfloat162float(h3)))};
  *reinterpret_cast<uint2*>(dh) = *reinterpret_cast<uint2*>(hh);
  *reinterpret_cast<uint2*>(dl) = *reinterpret_cast<uint2*>(ll);
}

// One block of up to 128 columns.  GM: group - 1 for in-block groups of 16
// to 128 columns (group starts known at compile time), -2 for in-block
// groups of 1 to 8 columns (tested per column), -1 when the block's grid was
// computed beforehand (one group per row, or groups wider than a block).
// With groups of 32 columns or more the grid is fixed within a round: the
// owner keeps the rounded quotient and the error and the outputs are formed
// when the round retires; otherwise the owner keeps deq and the code.
template <bool ORD, int GM, bool RF>
__global__ void __launch_bounds__(WARPS * 32, 1) sweep_block_kernel(BlockArgs a) {
  static_assert(!(ORD && RF), "the ordered mode takes U");
  constexpr bool PERCOL = (GM == 15 || GM == -2);
  const SweepDesc& d = a.d;
  extern __shared__ __align__(16) float smem[];
  float* Up = smem;
  float* iu = smem + BW * UP_ROW;
  float* w0s = iu + BW;                 // R form only
  float* ud = w0s + ROWS_PER_CTA * W0_LD;
  // the in-block factor: U's rows j0 .. (U form) or the diagonal block U_GG
  const float* ublk = RF ? d.Ublk + a.j0 * BW : d.U + a.j0 * d.n + a.j0;
  const int64_t ldub = RF ? BW : d.n;
  const int tid = threadIdx.x, lane = tid & 31;
  const int q = lane & (LPR - 1);
  const int64_t n = d.n, j0 = a.j0;
  const int bw = a.bw;
  const int64_t r0 = (int64_t)blockIdx.x * ROWS_PER_CTA + (tid >> 4) * 2;   // rows r0, r0 + 1
  const bool live[2] = {r0 < d.m, r0 + 1 < d.m};
  const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(d.U) & 15) == 0);
  const bool uvec = RF || vec;
  const int64_t j1 = j0 + bw;

  // Issue every load of the block's inputs first: the U block (16-byte
  // loads when rows are aligned; bw is then a multiple of 4, so a load never
  // passes the block's last column), U's diagonal, the rows' columns q,
  // q + 16, ... (zero past bw and for rows past m), and the row of U whose
  // bf16 split this CTA writes.
  float4 ub[UB_PER_THREAD];
#pragma unroll
  for (int it = 0; it < UB_PER_THREAD; ++it) {
    const int idx = it * (WARPS * 32) + tid;
    const int k = idx >> 5, c = (idx & 31) * 4;
    ub[it] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (k < bw && c < bw) {
      const float* src = ublk + k * ldub + c;
      if (uvec) {
        ub[it] = *reinterpret_cast<const float4*>(src);
      } else {
        ub[it].x = src[0];
        ub[it].y = (c + 1 < bw) ? src[1] : 0.f;
        ub[it].z = (c + 2 < bw) ? src[2] : 0.f;
        ub[it].w = (c + 3 < bw) ? src[3] : 0.f;
      }
    }
  }
  const float udiag = (tid < bw) ? ublk[tid * ldub + tid] : 1.f;
  float2 v[2][NP];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float* wrow = d.W + (r0 + h) * n + j0;
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int c0 = 32 * p + q, c1 = c0 + 16;
      v[h][p] = make_float2((live[h] && c0 < bw) ? wrow[c0] : 0.f, (live[h] && c1 < bw) ? wrow[c1] : 0.f);
    }
  }
  float2 w0v[2][NP];   // R form: the weights before the sweep
  if (RF) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float* wrow = d.W0 + (r0 + h) * n + j0;
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const int c0 = 32 * p + q, c1 = c0 + 16;
        w0v[h][p] = make_float2((live[h] && c0 < bw) ? wrow[c0] : 0.f, (live[h] && c1 < bw) ? wrow[c1] : 0.f);
      }
    }
  }
  // The tensor-core trailing update reads bf16 hi/lo copies of this block's
  // rows of U, columns j1..; each CTA writes rows blockIdx.x, + gridDim.x, ...
  // The first row's loads are issued here (up to 4096 - 128 columns).
  const bool split = !ORD && j1 < n;
  const bool split_fast = split && vec && (int)gridDim.x >= bw && (int)blockIdx.x < bw &&
                          (n - j1) <= 4 * 4 * WARPS * 32;
  float4 sv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t c = j1 + 4 * tid + (int64_t)i * 4 * WARPS * 32;
    sv[i] = (split_fast && c < n) ? *reinterpret_cast<const float4*>(d.U + (j0 + blockIdx.x) * n + c)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if (d.info && *d.info != 0) return;
  if (d.dead) {
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const int c0 = 32 * p + q, c1 = c0 + 16;
      const bool z0 = c0 < bw && d.dead[j0 + c0], z1 = c1 < bw && d.dead[j0 + c1];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (z0) v[h][p].x = 0.f;
        if (z1) v[h][p].y = 0.f;
        if (RF && z0) w0v[h][p].x = 0.f;
        if (RF && z1) w0v[h][p].y = 0.f;
      }
    }
  }

  // U block into the permuted layout (strictly upper part), zero pads, and
  // the correctly rounded reciprocals of the diagonal (0 past bw).
#pragma unroll
  for (int it = 0; it < UB_PER_THREAD; ++it) {
    const int idx = it * (WARPS * 32) + tid;
    const int k = idx >> 5, c = (idx & 31) * 4;
    const float x[4] = {ub[it].x, ub[it].y, ub[it].z, ub[it].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int cc = c + i;
      Up[(k * LPR + (cc & (LPR - 1))) * UP_LD + (cc >> 4)] = (cc > k && cc < bw) ? x[i] : 0.f;
    }
  }
  for (int t = tid; t < BW * LPR * 3; t += WARPS * 32) {
    const int row = t / 3, p = t - 3 * (t / 3);
    *reinterpret_cast<float2*>(Up + row * UP_LD + NREG + 2 * p) = make_float2(0.f, 0.f);
  }
  if (tid < BW) iu[tid] = (tid < bw) ? __frcp_rn(udiag) : 0.f;
  if (RF) {
    if (tid < BW) ud[tid] = (tid < bw) ? udiag : 0.f;
    const int rl0 = (tid >> 4) * 2;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        w0s[(rl0 + h) * W0_LD + 32 * p + q] = w0v[h][p].x;
        w0s[(rl0 + h) * W0_LD + 32 * p + q + 16] = w0v[h][p].y;
      }
  }

  if (split_fast) {
    const int64_t k = blockIdx.x;
    __nv_bfloat16* dh = d.Uh + ((int64_t)a.slot * BW + k) * d.ldu;
    __nv_bfloat16* dl = d.Ul + ((int64_t)a.slot * BW + k) * d.ldu;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t c = j1 + 4 * tid + (int64_t)i * 4 * WARPS * 32;
      if (c < n) split4(sv[i], dh + c, dl + c);
    }
  } else if (split) {
    for (int64_t k = blockIdx.x; k < bw; k += gridDim.x) {
      const float* src = d.U + (j0 + k) * n;
      __nv_bfloat16* dh = d.Uh + ((int64_t)a.slot * BW + k) * d.ldu;
      __nv_bfloat16* dl = d.Ul + ((int64_t)a.slot * BW + k) * d.ldu;
      if (vec) {
        for (int64_t c = j1 + 4 * tid; c < n; c += 4 * blockDim.x)
          split4(*reinterpret_cast<const float4*>(src + c), dh + c, dl + c);
      } else {
        for (int64_t c = j1 + tid; c < n; c += blockDim.x) {
          const float x = src[c];
          const __nv_bfloat16 hb = __float2bfloat16_rn(x);
          dh[c] = hb;
          dl[c] = __float2bfloat16_rn(x - __bfloat162float(hb));
        }
      }
    }
  }

  const float maxq = (float)((1 << d.bits) - 1);
  Grid g[2] = {make_grid(1.f, 0.f, maxq), make_grid(1.f, 0.f, maxq)};
  if (GM == -1) {
    const int64_t gi = (d.group == -1) ? 0 : j0 / d.group;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (live[h]) g[h] = make_grid(d.scales[(r0 + h) * d.ngroups + gi], d.zeros[(r0 + h) * d.ngroups + gi], maxq);
  }
  int gshift = 0;
  while (GM != -1 && (1 << gshift) < d.group) ++gshift;
  const int gmask = (GM == -1) ? 0 : d.group - 1;
  const int64_t g0 = j0 >> gshift;
  __syncthreads();

  const int src_base = lane & ~(LPR - 1);
  if (RF) {
    // the block's partial state: W0_G + F_G U_GG (F in v): the diagonal
    // term, then every row t of U_GG's strictly upper part
    float2 acc[2][NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
      const float2 dg = make_float2(ud[32 * p + q], ud[32 * p + q + 16]);
#pragma unroll
      for (int h = 0; h < 2; ++h) acc[h][p] = __ffma2_rn(v[h][p], dg, w0v[h][p]);
    }
#pragma unroll
    for (int kk = 0; kk < NREG; ++kk) {          // row t = 16 kk + o of U_GG, F_t from lane o
#pragma unroll 4
      for (int o = 0; o < LPR; ++o) {
        const int t = LPR * kk + o;
        const float2* u2 = reinterpret_cast<const float2*>(Up + (t * LPR + q) * UP_LD);
        float ft[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) ft[h] = __shfl_sync(0xffffffffu, reg_of(v[h], kk), src_base + o);
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const float2 u = u2[p];
#pragma unroll
          for (int h = 0; h < 2; ++h) acc[h][p] = __ffma2_rn(make_float2(ft[h], ft[h]), u, acc[h][p]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int p = 0; p < NP; ++p) v[h][p] = acc[h][p];
  }
  // the windows: columns 0 and 1 (register 0 of lanes 0 and 1)
  float win[2][2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    win[h][0] = __shfl_sync(0xffffffffu, v[h][0].x, src_base + 0);
    win[h][1] = __shfl_sync(0xffffffffu, v[h][0].x, src_base + 1);
  }
#pragma unroll 1
  for (int R = 0; R < NROUND; ++R) {
    const float* up = Up + (RC * R) * UP_ROW + q * UP_LD + 2 * R;
    const float* upw = Up + (RC * R) * UP_ROW + 2 * R;
    const float* iur = iu + RC * R;
    float ke[2][RET];      // the owner's -e of its retired columns
    uint32_t code2[2] = {0u, 0u};
#pragma unroll
    for (int t = 0; t < RC; ++t) {
      const int kt = t >> 4, o = t & (LPR - 1);
      bool gs = false;
      if (GM >= 0) {
        gs = (t & (GM & (RC - 1))) == 0 && ((RC * R) & GM) == 0 && RC * R + t < bw;
      } else if (GM == -2) {
        gs = ((RC * R + t) & gmask) == 0 && RC * R + t < bw;
      }
      if (gs) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          g[h] = group_start(v[h], RC * R + t, R, q, bw, d, live[h], r0 + h, g0 + ((RC * R + t) >> gshift), maxq);
      }
      const float ivu = iur[t];
      const float uw = upw[t * UP_ROW + ((t + 1) & (LPR - 1)) * UP_LD + ((t + 1) >> 4)];
      float ne[2], rr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        // the quantizer of column c on the window (the same value in the
        // sixteen lanes of the row)
        const float w = win[h][t & 1];
        rr[h] = fminf(fmaxf(rint_grid(__fmul_rn(w, g[h].isc)), g[h].lo), g[h].hi);
        ne[h] = ORD ? __fmul_rn(__fsub_rn(__fmul_rn(g[h].sc, rr[h]), w), ivu)   // -e, exactly
                    : __fmul_rn(fmaf(g[h].sc, rr[h], -w), ivu);
        // column c + 1 in the window: U[c][c + 1]
        win[h][(t + 1) & 1] = upd1<ORD>(win[h][(t + 1) & 1], ne[h], uw);
      }
      // the owner lane keeps its column's result
      if (q == o) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          ke[h][kt] = ne[h];
          if (PERCOL) {
            const float deq = __fmul_rn(g[h].sc, rr[h]);
            if (kt) v[h][0].y = deq;
            else v[h][0].x = deq;
            code2[h] |= (__float_as_uint(__fadd_rn(rr[h], g[h].zp2)) & 0xFFu) << (8 * kt);
          } else {
            if (kt) v[h][0].y = rr[h];
            else v[h][0].x = rr[h];
          }
        }
      }
      // later columns in the registers: every pair (U is zero on and below
      // the diagonal, so the retired and current columns stay unchanged)
      const float2* u2 = reinterpret_cast<const float2*>(up + t * UP_ROW);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        const float2 u = u2[p];
#pragma unroll
        for (int h = 0; h < 2; ++h) upd2<ORD>(v[h][p], make_float2(ne[h], ne[h]), u);
      }
      // column c + 2 (updated up to column c) from its owner into the slot
      // column c leaves
      const int k2 = (t + 2) >> 4, o2 = (t + 2) & (LPR - 1);
#pragma unroll
      for (int h = 0; h < 2; ++h)
        win[h][t & 1] = __shfl_sync(0xffffffffu, reg_of(v[h], k2), src_base + o2);
    }
    // retire registers 0 and 1: columns 32 R + q and 32 R + 16 + q
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (!live[h]) continue;
      const int64_t r = r0 + h;
#pragma unroll
      for (int k = 0; k < RET; ++k) {
        const int col = RC * R + LPR * k + q;
        if (col >= bw) continue;
        const float x = reg_of(v[h], k);
        const float deq = PERCOL ? x : __fmul_rn(g[h].sc, x);
        const uint32_t code = PERCOL ? ((code2[h] >> (8 * k)) & 0xFFu)
                                     : (__float_as_uint(__fadd_rn(x, g[h].zp2)) & 0xFFu);
        const float e = -ke[h][k];
        d.W[r * n + j0 + col] = deq;
        d.codes[r * n + j0 + col] = (uint8_t)code;
        if (a.Eb) a.Eb[r * a.lde + col] = e;
        if (!ORD) {
          // the trailing update's left operand: e (U form) or deq - w0
          const float et = RF ? __fsub_rn(deq, w0s[((tid >> 4) * 2 + h) * W0_LD + col]) : e;
          const __nv_bfloat16 hb = __float2bfloat16_rn(et);
          const int64_t eo = r * d.lde + (int64_t)a.slot * BW + col;
          d.Eh[eo] = hb;
          d.El[eo] = __float2bfloat16_rn(et - __bfloat162float(hb));
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int p = 0; p < NP - 1; ++p) v[h][p] = v[h][p + 1];
      v[h][NP - 1] = make_float2(0.f, 0.f);
    }
  }
}

// Grid of a group that starts at column j0 and reaches past this block:
// one warp per row, min/max over the current values of the group's columns.
__global__ void group_params_kernel(SweepDesc d, int64_t j0, int64_t gw, int64_t gi) {
  if (d.info && *d.info != 0) return;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= d.m) return;
  float lo = INFINITY, hi = -INFINITY;
  const int64_t j1 = (j0 + gw < d.n) ? j0 + gw : d.n;
  const float* src = d.W0 ? d.W0 : d.W;   // R form: only at column 0, where F = 0
  for (int64_t j = j0 + lane; j < j1; j += 32) {
    float x = src[r * d.n + j];
    if (d.dead && d.dead[j]) x = 0.f;
    lo = fminf(lo, x);
    hi = fmaxf(hi, x);
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    float sc, zp;
    grid_from_range(lo, hi, d.bits, d.asym, sc, zp);
    d.scales[r * d.ngroups + gi] = sc;
    d.zeros[r * d.ngroups + gi] = zp;
  }
}

template <bool ORD, int GM, bool RF>
cudaError_t launch_gm(const BlockArgs& a, unsigned grid, cudaStream_t s) {
  const void* fn = reinterpret_cast<const void*>(&sweep_block_kernel<ORD, GM, RF>);
  const int smem = RF ? RF_SMEM : SWEEP_SMEM;
  cudaError_t e = allow_smem(fn, smem);
  if (e != cudaSuccess) return e;
  sweep_block_kernel<ORD, GM, RF><<<grid, WARPS * 32, smem, s>>>(a);
  count_launch();
  return cudaGetLastError();
}

// Picks the instance for the block's group layout.
template <bool ORD, bool RF>
cudaError_t launch_block(const BlockArgs& a, unsigned grid, cudaStream_t s) {
  if (a.wide) return launch_gm<ORD, -1, RF>(a, grid, s);
  switch (a.d.group) {
    case 128: return launch_gm<ORD, 127, RF>(a, grid, s);
    case 64: return launch_gm<ORD, 63, RF>(a, grid, s);
    case 32: return launch_gm<ORD, 31, RF>(a, grid, s);
    case 16: return launch_gm<ORD, 15, RF>(a, grid, s);
    default: return launch_gm<ORD, -2, RF>(a, grid, s);
  }
}

// U_GG = (R_GG)^-1 for the 128 x 128 diagonal blocks of R (one CTA of 128
// threads per block; the last block padded with the identity): thread c
// forms column c by back substitution in float64, u_cc = 1 / R_cc and
// u_ic = -(sum_{k = i+1 .. c} R_ik u_kc) / R_ii for i = c - 1 .. 0, and
// rounds it to float once.  Out: Ublk[(128 b + i) * 128 + c], zero below the
// diagonal.
constexpr int DBI_LD = BW + 1;
constexpr int DBI_SMEM = BW * DBI_LD * (int)(sizeof(float) + sizeof(double));

__global__ void __launch_bounds__(BW) diag_block_inverse_kernel(const float* R, int64_t n, float* Ublk,
                                                                const int* info) {
  if (info && *info != 0) return;
  extern __shared__ __align__(16) unsigned char dbi_raw[];
  double* sU = reinterpret_cast<double*>(dbi_raw);
  float* sR = reinterpret_cast<float*>(sU + BW * DBI_LD);
  const int64_t j0 = (int64_t)blockIdx.x * BW;
  const int bw = (int)((n - j0) < BW ? (n - j0) : BW);
  const int c = threadIdx.x;
  for (int r = 0; r < BW; ++r) {
    float x = (r == c) ? 1.f : 0.f;
    if (r < bw && c < bw) x = (c >= r) ? R[(j0 + r) * n + j0 + c] : 0.f;
    sR[r * DBI_LD + c] = x;
  }
  __syncthreads();
  sU[c * DBI_LD + c] = 1.0 / (double)sR[c * DBI_LD + c];
  for (int i = c - 1; i >= 0; --i) {
    double acc = 0.0;
    for (int k = i + 1; k <= c; ++k) acc = fma((double)sR[i * DBI_LD + k], sU[k * DBI_LD + c], acc);
    sU[i * DBI_LD + c] = -acc / (double)sR[i * DBI_LD + i];
  }
  for (int r = 0; r < BW; ++r) Ublk[(j0 + r) * BW + c] = (r <= c) ? (float)sU[r * DBI_LD + c] : 0.f;
}

}  // namespace

kronq_status diag_block_inverse(const float* R, int64_t n, float* Ublk, const int* info, cudaStream_t s) {
  if (n <= 0) return KRONQ_OK;
  const void* fn = reinterpret_cast<const void*>(&diag_block_inverse_kernel);
  cudaError_t e = allow_smem(fn, DBI_SMEM);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(diag_block_inverse)");
  diag_block_inverse_kernel<<<(unsigned)ceil_div(n, BW), BW, DBI_SMEM, s>>>(R, n, Ublk, info);
  KQ_LAUNCH_CHECK("diag_block_inverse_kernel");
  return KRONQ_OK;
}

kronq_status gptq_sweep(const SweepDesc& d, cudaStream_t s) {
  const int64_t n = d.n, m = d.m;
  if (d.W0 && (d.ordered || !d.Ublk || d.group > BW))
    return fail(KRONQ_ERR_INVALID_ARG, "sweep: the R form takes groups of at most 128 columns, no ordered mode");
  const unsigned grid = (unsigned)ceil_div(m, ROWS_PER_CTA);
  TrailingMaps maps;
  if (!d.ordered && n > BW) {
    kronq_status r = trailing_maps(&maps, d.Eh, d.El, m, d.lde, d.Uh, d.Ul, (int64_t)d.gblocks * BW,
                                   d.ldu, d.W, n);
    if (r != KRONQ_OK) return r;
  }
  int64_t blk = 0;
  for (int64_t j0 = 0; j0 < n; j0 += BW, ++blk) {
    const int bw = (int)((j0 + BW <= n) ? BW : n - j0);
    BlockArgs a;
    a.d = d;
    a.j0 = j0;
    a.bw = bw;
    a.slot = (int)(blk % d.gblocks);
    a.wide = 0;
    if (d.group == -1 && j0 == 0) a.wide = 1;
    if (d.group > BW && (j0 % d.group) == 0) a.wide = 1;
    if (d.group > BW && (j0 % d.group) != 0) a.wide = 1;  // grid carried from the group start
    if (a.wide && (d.group == -1 ? j0 == 0 : (j0 % d.group) == 0)) {
      const int64_t gw = (d.group == -1) ? n : d.group;
      const int64_t gi = (d.group == -1) ? 0 : j0 / d.group;
      group_params_kernel<<<(unsigned)ceil_div(m, 8), 256, 0, s>>>(d, j0, gw, gi);
      KQ_LAUNCH_CHECK("group_params_kernel");
    }
    if (d.group == -1 && j0 > 0) a.wide = 1;  // single group per row: grid from column 0
    if (d.E) {
      a.Eb = d.E + j0;
      a.lde = n;
    } else if (d.ordered) {
      a.Eb = d.Eblk;
      a.lde = BW;
    } else {
      a.Eb = nullptr;   // the tensor-core update reads the bf16 hi/lo copies
      a.lde = BW;
    }
    cudaError_t el = d.ordered ? launch_block<true, false>(a, grid, s)
                               : (d.W0 ? launch_block<false, true>(a, grid, s)
                                       : launch_block<false, false>(a, grid, s));
    if (el != cudaSuccess) return cuda_fail(el, "sweep_block_kernel");
    const int64_t j1 = j0 + bw;
    if (j1 < n && !d.ordered) {
      // Inside a group: this block's errors (K = 128) to the group's later
      // columns.  At the group's end: the whole group (K = 128 gblocks) to
      // every column past it.  (A block followed by columns is a full block.)
      const bool group_end = (a.slot == d.gblocks - 1);
      const int64_t gend = j0 + (int64_t)(d.gblocks - a.slot) * BW;
      const int64_t k0 = group_end ? 0 : (int64_t)a.slot * BW;
      const int64_t K = group_end ? (int64_t)d.gblocks * BW : BW;
      const int64_t ncols = group_end ? n - j1 : ((gend < n ? gend : n) - j1);
      kronq_status r = trailing_update_tc(&maps, d.W, m, n, j1, ncols, k0, K, d.info, s);
      if (r != KRONQ_OK) return r;
    } else if (j1 < n) {
      GemmDesc g;
      g.M = m; g.N = n - j1; g.K = bw;
      g.A = a.Eb; g.lda = a.lde;
      g.B = d.U + j0 * n + j1; g.ldb = n;
      g.C = d.W + j1; g.ldc = n;
      g.alpha = -1.f; g.beta = 1.f;
      g.ordered = d.ordered;
      g.info = d.info;
      cudaError_t e = gemm_f32(g, s);
      if (e != cudaSuccess) return cuda_fail(e, "gemm(trailing)");
    }
  }
  return KRONQ_OK;
}

}  // namespace kq

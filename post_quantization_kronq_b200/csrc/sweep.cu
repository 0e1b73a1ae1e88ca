// GPTQ-style blocked column sweep under the K-FAC loss.
//
// KronQ README intro (extends GPTQ/GPTAQ) and "Reproduce from scratch"
// (--w_bits --w_groupsize --w_asym).  Rows of W~ are independent once U is
// known, so the in-block sweep runs one warp per pair of rows with no
// block-wide synchronisation: lane l holds columns 4l..4l+3 of the 128-column
// block, the owner lane of column j quantizes it, forms the scaled error
// e = (w - deq) / U_jj, broadcasts e with a shuffle and every lane applies the
// rank-1 update to its later columns.  All arithmetic of the sweep is single
// float32 operations (division correctly rounded, multiply and subtract not
// fused), so the result is reproducible bit for bit.
//
// After each block the later columns get W[:, later] -= E_blk U[blk, later]
// (the lazy-batch update), either as a fast GEMM or, in the ordered test mode,
// with one rounding per product and per sum in ascending k.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BW = 128;        // block width (columns)
constexpr int RPW = 2;         // rows per warp
constexpr int WARPS = 8;       // warps per CTA
constexpr int ROWS_PER_CTA = RPW * WARPS;

struct BlockArgs {
  SweepDesc d;
  int64_t j0;
  int bw;         // columns in this block
  int wide;       // 1: the grid of this block's first column was computed beforehand
  float* Eb;      // scaled-error output of this block
  int64_t lde;
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

__global__ void __launch_bounds__(WARPS * 32) sweep_block_kernel(BlockArgs a) {
  const SweepDesc& d = a.d;
  if (d.info && *d.info != 0) return;
  extern __shared__ __align__(16) float us_raw[];
  float (*Us)[BW] = reinterpret_cast<float (*)[BW]>(us_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n = d.n, j0 = a.j0;
  const int bw = a.bw;

  for (int t = tid; t < BW * BW; t += blockDim.x) {
    const int r = t / BW, c = t % BW;
    Us[r][c] = (r < bw && c < bw && c >= r) ? d.U[(j0 + r) * n + j0 + c] : 0.f;
  }
  __syncthreads();

  const float maxq = (float)((1 << d.bits) - 1);
  const int64_t rbase = ((int64_t)blockIdx.x * WARPS + warp) * RPW;

  float v[RPW][4], ev[RPW][4];
  uint32_t code[RPW];
  float sc[RPW], zp[RPW];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int64_t r = rbase + rr;
    code[rr] = 0;
    sc[rr] = 1.f;
    zp[rr] = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int c = 4 * lane + s;
      float x = 0.f;
      if (r < d.m && c < bw) {
        x = d.W[r * n + j0 + c];
        if (d.dead && d.dead[j0 + c]) x = 0.f;
      }
      v[rr][s] = x;
      ev[rr][s] = 0.f;
    }
    if (a.wide && r < d.m) {
      const int64_t gi = (d.group == -1) ? 0 : j0 / d.group;
      sc[rr] = d.scales[r * d.ngroups + gi];
      zp[rr] = d.zeros[r * d.ngroups + gi];
    }
  }

  for (int j = 0; j < bw; ++j) {
    const int64_t gc = j0 + j;
    if (d.group > 0 && d.group <= BW && (gc % d.group) == 0) {
      const int gend = (j + d.group < bw) ? j + d.group : bw;
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        float lo = INFINITY, hi = -INFINITY;
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int c = 4 * lane + s;
          if (c >= j && c < gend) {
            lo = fminf(lo, v[rr][s]);
            hi = fmaxf(hi, v[rr][s]);
          }
        }
        for (int o = 16; o > 0; o >>= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
        }
        grid_from_range(lo, hi, d.bits, d.asym, sc[rr], zp[rr]);
        const int64_t r = rbase + rr;
        if (lane == 0 && r < d.m) {
          d.scales[r * d.ngroups + gc / d.group] = sc[rr];
          d.zeros[r * d.ngroups + gc / d.group] = zp[rr];
        }
      }
    }
    const int owner = j >> 2, slot = j & 3;
    const float ujj = Us[j][j];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      float e = 0.f;
      if (lane == owner) {
        float w = v[rr][0];
#pragma unroll
        for (int s = 1; s < 4; ++s)
          if (s == slot) w = v[rr][s];
        float q = __fadd_rn(rintf(__fdiv_rn(w, sc[rr])), zp[rr]);
        q = fminf(fmaxf(q, 0.f), maxq);
        const float deq = __fmul_rn(sc[rr], __fsub_rn(q, zp[rr]));
        e = __fdiv_rn(__fsub_rn(w, deq), ujj);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          if (s == slot) {
            v[rr][s] = deq;
            ev[rr][s] = e;
          }
        code[rr] |= ((uint32_t)q & 0xFFu) << (8 * slot);
      }
      e = __shfl_sync(0xffffffffu, e, owner);
      const float4 u4 = *reinterpret_cast<const float4*>(&Us[j][4 * lane]);
      const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
      for (int s = 0; s < 4; ++s)
        if (4 * lane + s > j) v[rr][s] = __fsub_rn(v[rr][s], __fmul_rn(e, uu[s]));
    }
  }

#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int64_t r = rbase + rr;
    if (r >= d.m) continue;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int c = 4 * lane + s;
      if (c < bw) {
        d.W[r * n + j0 + c] = v[rr][s];
        d.codes[r * n + j0 + c] = (uint8_t)((code[rr] >> (8 * s)) & 0xFFu);
        a.Eb[r * a.lde + c] = ev[rr][s];
      }
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
  for (int64_t j = j0 + lane; j < j1; j += 32) {
    float x = d.W[r * d.n + j];
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

}  // namespace

kronq_status gptq_sweep(const SweepDesc& d, cudaStream_t s) {
  const int64_t n = d.n, m = d.m;
  constexpr int SWEEP_SMEM = BW * BW * sizeof(float);
  cudaError_t ea = allow_smem(reinterpret_cast<const void*>(&sweep_block_kernel), SWEEP_SMEM);
  if (ea != cudaSuccess) return cuda_fail(ea, "cudaFuncSetAttribute(sweep)");
  const unsigned grid = (unsigned)ceil_div(m, ROWS_PER_CTA);
  for (int64_t j0 = 0; j0 < n; j0 += BW) {
    const int bw = (int)((j0 + BW <= n) ? BW : n - j0);
    BlockArgs a;
    a.d = d;
    a.j0 = j0;
    a.bw = bw;
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
    } else {
      a.Eb = d.Eblk;
      a.lde = BW;
    }
    sweep_block_kernel<<<grid, WARPS * 32, SWEEP_SMEM, s>>>(a);
    KQ_LAUNCH_CHECK("sweep_block_kernel");
    const int64_t j1 = j0 + bw;
    if (j1 < n) {
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

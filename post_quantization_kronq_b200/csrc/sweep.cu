// GPTQ-style blocked column sweep under the K-FAC loss.
//
// KronQ README intro (extends GPTQ/GPTAQ) and "Reproduce from scratch"
// (--w_bits --w_groupsize --w_asym).  Rows of W~ are independent once U is
// known, so the in-block sweep runs one warp per pair of rows with no
// block-wide synchronisation: eight lanes per row, lane q holds columns
// 16q..16q+15 of the 128-column block.  The owner lane of a 16-column quarter
// quantizes its columns one after the other, forming the scaled errors
// e = (w - deq) / U_jj and updating its own later columns; then the sixteen
// errors are shuffled to the row's other lanes, which apply them to their
// (later) columns in column order.  All arithmetic of the sweep is single
// float32 operations (multiply and subtract not fused; the per-column
// divisions by the group scale and by U_jj are multiplications by their
// correctly rounded reciprocals), so the result is reproducible bit for bit.
//
// After each block the later columns get W[:, later] -= E_blk U[blk, later]
// (the lazy-batch update), either as a fast GEMM or, in the ordered test mode,
// with one rounding per product and per sum in ascending k.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BW = 128;        // block width (columns)
constexpr int QW = 16;         // columns held by one lane
constexpr int LPR = BW / QW;   // lanes per row (8)
constexpr int WARPS = 8;       // warps per CTA
constexpr int ROWS_PER_CTA = WARPS * 32 / LPR;   // 32
constexpr int US_LD = BW + 4 * (BW / QW);        // padded row of the U block (160 floats)
constexpr int SWEEP_SMEM = BW * US_LD * sizeof(float) + BW * sizeof(float);  // + 1/U_jj

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

// Grid of the group starting at column j of this block: the eight lanes of
// the row reduce over their columns in [j, j + group).
__device__ __forceinline__ void group_start(const float (&v)[QW], int j, int bw, int q,
                                            const SweepDesc& d, bool live, int64_t r, int64_t gi,
                                            float& sc, float& zp, float& isc) {
  const int gend = (j + d.group < bw) ? j + d.group : bw;
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int cc = 0; cc < QW; ++cc) {
    const int col = q * QW + cc;
    if (col >= j && col < gend) {
      lo = fminf(lo, v[cc]);
      hi = fmaxf(hi, v[cc]);
    }
  }
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  grid_from_range(lo, hi, d.bits, d.asym, sc, zp);
  isc = __frcp_rn(sc);
  if (q == 0 && live) {
    d.scales[r * d.ngroups + gi] = sc;
    d.zeros[r * d.ngroups + gi] = zp;
  }
}

// Column c of the block lives at Us[k * US_LD + ucol(c)]: 4 floats of padding
// per 16 columns put the eight lanes of a row on different banks for the
// float4 reads of one U row.
__device__ __forceinline__ int ucol(int c) { return c + 4 * (c >> 4); }

// One block of 128 columns.  Eight lanes per row: lane q holds the row's
// columns 16q .. 16q+15 in registers (v[]), so every step of the sequential
// column loop is register arithmetic with static indices (the unrolled
// 16-step body stays small enough for the instruction cache).  For each
// quarter, the lane holding it quantizes its columns in order (forming
// e = (w - deq) / U_jj and applying v[c] -= e * U[j][c] to its own later
// columns), with no shuffle inside that dependency chain; the sixteen
// errors are then shuffled to the later lanes at once.  Every update is a
// multiply followed by a subtract, in ascending j per element: the
// operation order of the float32 reference.
template <bool SMALLG>
__global__ void __launch_bounds__(WARPS * 32) sweep_block_kernel(BlockArgs a) {
  const SweepDesc& d = a.d;
  if (d.info && *d.info != 0) return;
  extern __shared__ __align__(16) float Us[];
  const int tid = threadIdx.x, lane = tid & 31;
  const int q = lane & (LPR - 1);
  const int64_t n = d.n, j0 = a.j0;
  const int bw = a.bw;
  const int64_t r = (int64_t)blockIdx.x * ROWS_PER_CTA + (tid >> 3);
  const bool live = r < d.m;

  // U block (rows j0.., columns j0..j0+127, upper part) into shared memory.
  // float4 loads, eight in flight per thread.
  const bool vec = ((n & 3) == 0) && ((reinterpret_cast<uintptr_t>(d.U) & 15) == 0);
  if (vec) {
#pragma unroll 8
    for (int it = 0; it < (BW * BW / 4) / (WARPS * 32); ++it) {
      const int idx = it * (WARPS * 32) + tid;
      const int k = idx >> 5, c = (idx & 31) * 4;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < bw) x = *reinterpret_cast<const float4*>(d.U + (j0 + k) * n + j0 + c);
      x.x = (c + 0 >= k && c + 0 < bw) ? x.x : 0.f;
      x.y = (c + 1 >= k && c + 1 < bw) ? x.y : 0.f;
      x.z = (c + 2 >= k && c + 2 < bw) ? x.z : 0.f;
      x.w = (c + 3 >= k && c + 3 < bw) ? x.w : 0.f;
      *reinterpret_cast<float4*>(Us + k * US_LD + ucol(c)) = x;
    }
  } else {
    for (int t = tid; t < BW * BW; t += blockDim.x) {
      const int k = t >> 7, c = t & (BW - 1);
      Us[k * US_LD + ucol(c)] = (k < bw && c < bw && c >= k) ? d.U[(j0 + k) * n + j0 + c] : 0.f;
    }
  }

  // bf16 hi/lo copy of this block's rows of U, columns j1.. (operand B of
  // the tensor-core trailing update); rows are spread over the CTAs.
  const int64_t j1 = j0 + bw;
  if (!d.ordered && j1 < n) {
    for (int64_t k = blockIdx.x; k < bw; k += gridDim.x) {
      const float* src = d.U + (j0 + k) * n;
      __nv_bfloat16* dh = d.Uh + ((int64_t)a.slot * BW + k) * d.ldu;
      __nv_bfloat16* dl = d.Ul + ((int64_t)a.slot * BW + k) * d.ldu;
      if (vec) {
#pragma unroll 4
        for (int64_t c = j1 + 4 * tid; c < n; c += 4 * blockDim.x) {
          const float4 x = *reinterpret_cast<const float4*>(src + c);
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x.x), h1 = __float2bfloat16_rn(x.y);
          const __nv_bfloat16 h2 = __float2bfloat16_rn(x.z), h3 = __float2bfloat16_rn(x.w);
          __nv_bfloat162 hh[2] = {__halves2bfloat162(h0, h1), __halves2bfloat162(h2, h3)};
          __nv_bfloat162 ll[2] = {
              __halves2bfloat162(__float2bfloat16_rn(x.x - __bfloat162float(h0)),
                                 __float2bfloat16_rn(x.y - __bfloat162float(h1))),
              __halves2bfloat162(__float2bfloat16_rn(x.z - __bfloat162float(h2)),
                                 __float2bfloat16_rn(x.w - __bfloat162float(h3)))};
          *reinterpret_cast<uint2*>(dh + c) = *reinterpret_cast<uint2*>(hh);
          *reinterpret_cast<uint2*>(dl + c) = *reinterpret_cast<uint2*>(ll);
        }
      } else {
        for (int64_t c = j1 + tid; c < n; c += blockDim.x) {
          const float x = src[c];
          const __nv_bfloat16 h = __float2bfloat16_rn(x);
          dh[c] = h;
          dl[c] = __float2bfloat16_rn(x - __bfloat162float(h));
        }
      }
    }
  }

  float v[QW], ev[QW];
  uint32_t code[QW / 4];
  const float* wrow = d.W + r * n + j0 + q * QW;
  if (live && q * QW + QW <= bw && vec) {
#pragma unroll
    for (int c = 0; c < QW; c += 4) {
      const float4 x = *reinterpret_cast<const float4*>(wrow + c);
      v[c] = x.x; v[c + 1] = x.y; v[c + 2] = x.z; v[c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < QW; ++c) v[c] = (live && q * QW + c < bw) ? wrow[c] : 0.f;
  }
#pragma unroll
  for (int c = 0; c < QW; ++c) {
    if (d.dead && live && q * QW + c < bw && d.dead[j0 + q * QW + c]) v[c] = 0.f;
    ev[c] = 0.f;
  }
#pragma unroll
  for (int c = 0; c < QW / 4; ++c) code[c] = 0;
  float sc = 1.f, zp = 0.f;
  if (a.wide && live) {
    const int64_t gi = (d.group == -1) ? 0 : j0 / d.group;
    sc = d.scales[r * d.ngroups + gi];
    zp = d.zeros[r * d.ngroups + gi];
  }
  float isc = __frcp_rn(sc);
  // correctly rounded reciprocals of the block's diagonal of U
  float* iu = Us + BW * US_LD;
  if (tid < bw) iu[tid] = __frcp_rn(d.U[(j0 + tid) * n + j0 + tid]);
  __syncthreads();

  const float maxq = (float)((1 << d.bits) - 1);
  const int src_base = lane & ~(LPR - 1);
  // In-block groups divide 128, so they are powers of two starting at j0.
  const bool inblock_groups = d.group > 0 && d.group <= BW;
  const int gmask = inblock_groups ? d.group - 1 : 0;
  int gshift = 0;
  while (inblock_groups && (1 << gshift) < d.group) ++gshift;
  const int64_t g0 = inblock_groups ? j0 >> gshift : 0;
  for (int qo = 0; qo < LPR; ++qo) {
    const bool all_later = q > qo;     // every column of this lane comes after the current quarter
    const bool mine = q == qo;
    // Groups of 16 or more columns can only start at a lane boundary.
    if (!SMALLG && inblock_groups && qo * QW < bw && ((qo * QW) & gmask) == 0)
      group_start(v, qo * QW, bw, q, d, live, r, g0 + ((qo * QW) >> gshift), sc, zp, isc);
    // The owner lane sweeps its sixteen columns alone (no cross-lane step
    // inside the sequential chain) ...
    if (mine) {
      const float* urow0 = Us + q * (QW + 4);
#pragma unroll
      for (int c = 0; c < QW; ++c) {
        const int j = qo * QW + c;
        if (j >= bw) break;
        if (SMALLG && (j & gmask) == 0) {
          // a group of fewer than 16 columns lies inside this lane
          float lo = INFINITY, hi = -INFINITY;
#pragma unroll
          for (int cc = c; cc < QW; ++cc)
            if (cc < c + d.group && qo * QW + cc < bw) {
              lo = fminf(lo, v[cc]);
              hi = fmaxf(hi, v[cc]);
            }
          grid_from_range(lo, hi, d.bits, d.asym, sc, zp);
          isc = __frcp_rn(sc);
          if (live) {
            const int64_t gi = g0 + (j >> gshift);
            d.scales[r * d.ngroups + gi] = sc;
            d.zeros[r * d.ngroups + gi] = zp;
          }
        }
        const float w = v[c];
        // division by scale and by U_jj as multiplication by the correctly
        // rounded reciprocals (the float32 schedule of this library)
        float qv = __fadd_rn(rintf(__fmul_rn(w, isc)), zp);
        qv = fminf(fmaxf(qv, 0.f), maxq);
        const float deq = __fmul_rn(sc, __fsub_rn(qv, zp));
        const float e = __fmul_rn(__fsub_rn(w, deq), iu[j]);
        v[c] = deq;
        ev[c] = e;
        code[c >> 2] |= ((uint32_t)qv & 0xFFu) << (8 * (c & 3));
        const float* urow = urow0 + j * US_LD;
#pragma unroll
        for (int c4 = 0; c4 < QW; c4 += 4) {
          if (c4 + 3 <= c) continue;
          const float4 u4 = *reinterpret_cast<const float4*>(urow + c4);
          const float uu[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
          for (int t = 0; t < 4; ++t)
            if (c4 + t > c) v[c4 + t] = __fsub_rn(v[c4 + t], __fmul_rn(e, uu[t]));
        }
      }
    }
    // ... then its sixteen errors go to the other lanes of the row, which
    // apply them to their columns in ascending column order (the same
    // operation sequence per element as a column-by-column update).
    float eq[QW];
#pragma unroll
    for (int c = 0; c < QW; ++c) eq[c] = __shfl_sync(0xffffffffu, ev[c], src_base + qo);
    if (all_later) {
      const float* urow0 = Us + q * (QW + 4);
#pragma unroll
      for (int c = 0; c < QW; ++c) {
        const int j = qo * QW + c;
        if (j >= bw) break;
        const float* urow = urow0 + j * US_LD;
#pragma unroll
        for (int c4 = 0; c4 < QW; c4 += 4) {
          const float4 u4 = *reinterpret_cast<const float4*>(urow + c4);
          v[c4 + 0] = __fsub_rn(v[c4 + 0], __fmul_rn(eq[c], u4.x));
          v[c4 + 1] = __fsub_rn(v[c4 + 1], __fmul_rn(eq[c], u4.y));
          v[c4 + 2] = __fsub_rn(v[c4 + 2], __fmul_rn(eq[c], u4.z));
          v[c4 + 3] = __fsub_rn(v[c4 + 3], __fmul_rn(eq[c], u4.w));
        }
      }
    }
  }

  if (!live) return;
  const int64_t base = r * n + j0 + q * QW;
  const bool full = (q * QW + QW <= bw);
  if (full && ((reinterpret_cast<uintptr_t>(d.W + base) & 15) == 0)) {
    float4* w4 = reinterpret_cast<float4*>(d.W + base);
#pragma unroll
    for (int c = 0; c < QW; c += 4) w4[c >> 2] = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < QW; ++c)
      if (q * QW + c < bw) d.W[base + c] = v[c];
  }
  if (full && ((reinterpret_cast<uintptr_t>(d.codes + base) & 15) == 0)) {
    uint4* c4 = reinterpret_cast<uint4*>(d.codes + base);
#pragma unroll
    for (int t = 0; t < QW / 16; ++t)
      c4[t] = make_uint4(code[4 * t], code[4 * t + 1], code[4 * t + 2], code[4 * t + 3]);
  } else {
#pragma unroll
    for (int c = 0; c < QW; ++c)
      if (q * QW + c < bw) d.codes[base + c] = (uint8_t)((code[c >> 2] >> (8 * (c & 3))) & 0xFFu);
  }
  if (a.Eb) {
#pragma unroll
    for (int c = 0; c < QW; ++c)
      if (q * QW + c < bw) a.Eb[r * a.lde + q * QW + c] = ev[c];
  }
  if (!d.ordered) {
    __nv_bfloat16* eh = d.Eh + r * d.lde + (int64_t)a.slot * BW + q * QW;
    __nv_bfloat16* el = d.El + r * d.lde + (int64_t)a.slot * BW + q * QW;
#pragma unroll
    for (int c = 0; c < QW; c += 2) {
      const __nv_bfloat16 h0 = __float2bfloat16_rn(ev[c]), h1 = __float2bfloat16_rn(ev[c + 1]);
      const __nv_bfloat16 l0 = __float2bfloat16_rn(ev[c] - __bfloat162float(h0));
      const __nv_bfloat16 l1 = __float2bfloat16_rn(ev[c + 1] - __bfloat162float(h1));
      *reinterpret_cast<__nv_bfloat162*>(eh + c) = __halves2bfloat162(h0, h1);
      *reinterpret_cast<__nv_bfloat162*>(el + c) = __halves2bfloat162(l0, l1);
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
  cudaError_t ea = allow_smem(reinterpret_cast<const void*>(&sweep_block_kernel<false>), SWEEP_SMEM);
  if (ea == cudaSuccess) ea = allow_smem(reinterpret_cast<const void*>(&sweep_block_kernel<true>), SWEEP_SMEM);
  if (ea != cudaSuccess) return cuda_fail(ea, "cudaFuncSetAttribute(sweep)");
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
    if (d.group > 0 && d.group < QW)
      sweep_block_kernel<true><<<grid, WARPS * 32, SWEEP_SMEM, s>>>(a);
    else
      sweep_block_kernel<false><<<grid, WARPS * 32, SWEEP_SMEM, s>>>(a);
    KQ_LAUNCH_CHECK("sweep_block_kernel");
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

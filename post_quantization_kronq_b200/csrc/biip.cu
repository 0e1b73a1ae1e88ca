// Bidirectional incoherence processing (BiIP) kernels.
//
// KronQ abstract point (1) and README bullet "Bidirectional incoherence
// processing (BiIP)": rotation + rescale on the input and the output side;
// README flags --incoh_kernel had --alpha.  The rotation of a length
// L = P K vector (P = 2^k, K odd) is (Had_P / sqrt(P) (x) C_K) diag(s): view
// the vector as a P x K matrix Y (index a K + b), apply the orthonormal
// DCT-II C_K along b and the Walsh-Hadamard transform along a.  Signs come
// from SplitMix64 (no table).
//
// One CTA holds R whole rows in shared memory, applies the DCT (K > 1) and
// the FWHT in radix-16 register passes, and stores the result transposed
// (R consecutive floats per output row), so two launches make the two-sided
// transform U M V^T at two HBM round trips.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int RP_THREADS = 512;
constexpr int KREG = 16;     // odd factors up to this size are transformed in registers
constexpr int KMAX = 255;    // largest odd factor supported

__device__ __forceinline__ int padx(int x) { return x + (x >> 5); }

__device__ __forceinline__ float sign_of(uint64_t state, int j) {
  return (splitmix64(state, (uint64_t)j) >> 63) ? -1.f : 1.f;
}

struct RPArgs {
  RowPass p;
  int R, logR;  // rows per CTA (a power of two)
  int P, K, logP;
  int RS;       // padded row stride in shared memory (floats, odd)
  float norm;   // 1 / sqrt(P)
  int two_buf;  // K > KREG: the DCT writes to a second buffer
};

// Per-column factor of the forward pre-scale or the inverse post-scale:
// the sign of column j times d[j] (scale_mode 1) or 1/d[j] (scale_mode 2).
__device__ __forceinline__ float col_factor(const RowPass& p, int j) {
  float f = p.rotate ? sign_of(p.sign_state, j) : 1.f;
  if (p.scale_mode == 1) f = f * p.scale[j];
  else if (p.scale_mode == 2) f = f / p.scale[j];
  return f;
}

// One radix-16 pass of the FWHT over bits LO .. LO+3 of a 4096-long row
// (rows of stride RS, padded by padx).  Item t of a row: a0 has bits LO ..
// LO+3 clear; its sixteen elements a0 + (u << LO) sit at padx(a0) + off(u)
// with off(u) known at compile time (the padding adds one word per 32, and
// a0 never carries into it: a0 mod 32 is 0 or 16 for LO = 0, below 16 for
// LO = 4).
template <int LO>
__device__ __forceinline__ void radix16_pass(float* cur, int RS, int logR) {
  constexpr int PER_ROW = 4096 / 16;
  const int items = PER_ROW << logR;
  for (int t = threadIdx.x; t < items; t += RP_THREADS) {
    const int rr = t >> 8;
    const int rem = t & (PER_ROW - 1);
    int hi = rem >> LO;
    if (LO == 4) {
      // the two 16-item halves of a warp take groups two apart (bank offset
      // 16 instead of 8), so the warp's loads and stores hit 32 distinct banks
      hi = (hi & ~3) | ((hi & 1) << 1) | ((hi >> 1) & 1);
    }
    const int a0 = (hi << (LO + 4)) | (rem & ((1 << LO) - 1));
    float* base = cur + rr * RS + padx(a0);
    float x[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int off = (LO == 0) ? u : (LO == 4 ? 16 * u + (u >> 1) : (u << LO) + (u << (LO - 5)));
      x[u] = base[off];
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if ((u & h) == 0) {
          const float s0 = x[u], s1 = x[u | h];
          x[u] = s0 + s1;
          x[u | h] = s0 - s1;
        }
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int off = (LO == 0) ? u : (LO == 4 ? 16 * u + (u >> 1) : (u << LO) + (u << (LO - 5)));
      base[off] = x[u];
    }
  }
  __syncthreads();
}

// Loads of one group of R <= 8 rows for rows up to 8 x RP_THREADS long:
// thread t takes columns t, t + RP_THREADS, ... of every row, all loads
// issued before any is used.
template <bool BF16>
__device__ __forceinline__ void load_group(const RowPass& p, int L, int64_t r0, int rows_here,
                                           float (&v)[8][8]) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int rr = 0; rr < 8; ++rr) {
    const int64_t row = (r0 + rr) * p.ld_in + tid;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int j = tid + c * RP_THREADS;
      v[c][rr] = 0.f;
      if (j < L && rr < rows_here) {
        if (BF16) v[c][rr] = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.in)[row + c * RP_THREADS]);
        else v[c][rr] = reinterpret_cast<const float*>(p.in)[row + c * RP_THREADS];
      }
    }
  }
}

// Persistent: CTA b transforms the row groups b, b + gridDim.x, ... (R
// rows each).  F4096 (rows of 4096 = 2^12, three radix-16 passes): the next
// group's loads are issued into registers right after the current group
// reaches shared memory, so they overlap its transform and its transposed
// store.  Other lengths load each group when it starts.
template <bool BF16, bool F4096>
__global__ void __launch_bounds__(RP_THREADS) rowpass_kernel(RPArgs A) {
  extern __shared__ __align__(16) float sm[];
  const RowPass& p = A.p;
  const int R = A.R, P = A.P, K = A.K;
  const int L = (int)p.L, RS = A.RS;
  float* buf0 = sm;
  float* buf1 = sm + R * RS;
  float* Cm = sm + R * RS * (A.two_buf ? 2 : 1);
  float* cfs = Cm + ((p.rotate && K > 1) ? K * K : 0);   // F4096: column factors
  const int tid = threadIdx.x;
  const int64_t ngroups = (p.rows + R - 1) / R;
  if (F4096) {
    // every group uses the same column factors: computed once per CTA
    for (int j = tid; j < L; j += RP_THREADS) cfs[j] = col_factor(p, j);
    __syncthreads();
  }

  if (p.rotate && K > 1) {
    for (int t = tid; t < K * K; t += RP_THREADS) {
      const int i = t / K, j = t - (t / K) * K;
      const double ci = (i == 0) ? sqrt(0.5) : 1.0;
      Cm[t] = (float)(sqrt(2.0 / K) * ci * cospi((double)((2 * j + 1) * i) / (2.0 * K)));
    }
  }

  const bool reg_load = L <= 8 * RP_THREADS;
  float v[8][8];
  int64_t grp = blockIdx.x;
  if (F4096 && grp < ngroups) {
    const int64_t r0 = grp * R;
    load_group<BF16>(p, L, r0, (int)((p.rows - r0) < R ? (p.rows - r0) : R), v);
  }
  for (; grp < ngroups; grp += gridDim.x) {
    const int64_t r0 = grp * R;
    const int rows_here = (int)((p.rows - r0) < R ? (p.rows - r0) : R);

    // 1. rows into shared memory (forward: times sign and scale of the
    //    column); the column factor is computed once per column and reused
    //    for the R rows.
    if (reg_load) {
      if (!F4096) load_group<BF16>(p, L, r0, rows_here, v);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int j = tid + c * RP_THREADS;
        if (j < L) {
          const float f = p.inverse ? 1.f : (F4096 ? cfs[j] : col_factor(p, j));
          const int pj = padx(j);
#pragma unroll
          for (int rr = 0; rr < 8; ++rr)
            if (rr < R) buf0[rr * RS + pj] = v[c][rr] * f;
        }
      }
    } else for (int j = tid; j < L; j += RP_THREADS) {
      const float f = p.inverse ? 1.f : col_factor(p, j);
      const int pj = padx(j);
      float w[8];
#pragma unroll
      for (int rr = 0; rr < 8; ++rr) {
        w[rr] = 0.f;
        if (rr < rows_here) {
          const int64_t idx = (r0 + rr) * p.ld_in + j;
          w[rr] = BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.in)[idx])
                       : reinterpret_cast<const float*>(p.in)[idx];
        }
      }
#pragma unroll
      for (int rr = 0; rr < 8; ++rr)
        if (rr < R) buf0[rr * RS + pj] = w[rr] * f;
    }
    __syncthreads();
    // the next group's loads, in flight during this group's transform
    const int64_t nxt = grp + gridDim.x;
    if (F4096 && nxt < ngroups) {
      const int64_t n0 = nxt * R;
      load_group<BF16>(p, L, n0, (int)((p.rows - n0) < R ? (p.rows - n0) : R), v);
    }

    float* cur = buf0;
    if (F4096) {
      // length 4096: three radix-16 passes with compile-time offsets
      if (p.rotate) {
        radix16_pass<0>(cur, RS, A.logR);
        radix16_pass<4>(cur, RS, A.logR);
        radix16_pass<8>(cur, RS, A.logR);
      }
    } else if (p.rotate) {
      // 2. DCT along b (odd factor)
      if (K > 1) {
        const int items = R * P;
        for (int t = tid; t < items; t += RP_THREADS) {
          const int rr = t / P;
          const int a = t - rr * P;
          float* row = buf0 + rr * RS;
          const int base = a * K;
          if (!A.two_buf) {
            float y[KREG];
#pragma unroll
            for (int b = 0; b < KREG; ++b) y[b] = (b < K) ? row[padx(base + b)] : 0.f;
#pragma unroll
            for (int o = 0; o < KREG; ++o) {
              if (o < K) {
                float acc = 0.f;
#pragma unroll
                for (int b = 0; b < KREG; ++b)
                  if (b < K) acc = fmaf(p.inverse ? Cm[b * K + o] : Cm[o * K + b], y[b], acc);
                row[padx(base + o)] = acc;
              }
            }
          } else {
            float* orow = buf1 + rr * RS;
            for (int o = 0; o < K; ++o) {
              float acc = 0.f;
              for (int b = 0; b < K; ++b)
                acc = fmaf(p.inverse ? Cm[b * K + o] : Cm[o * K + b], row[padx(base + b)], acc);
              orow[padx(base + o)] = acc;
            }
          }
        }
        if (A.two_buf) cur = buf1;
        __syncthreads();
      }
      // 3. FWHT along a: radix-16 register passes over 4-bit groups of a.
      //    Item order (b fastest, then the low bits of a, then the high bits)
      //    keeps neighbouring threads on neighbouring shared-memory words.
      if (K == 1 && A.logP == 12) {
        // length 4096: three radix-16 passes with compile-time offsets
        radix16_pass<0>(cur, RS, A.logR);
        radix16_pass<4>(cur, RS, A.logR);
        radix16_pass<8>(cur, RS, A.logR);
      } else for (int lo = 0; lo < A.logP; lo += 4) {
        const int nb = (A.logP - lo) < 4 ? (A.logP - lo) : 4;
        const int G = 1 << nb;
        const int per_row = L >> nb;
        const int items = per_row << A.logR;
        const int lo_mask = (1 << lo) - 1;
        if (K == 1 && G == 16) {
          // power-of-two length, full radix-16 pass: shifts and masks only
          int lpr = 0;
          while ((1 << lpr) < per_row) ++lpr;
          for (int t = tid; t < items; t += RP_THREADS) {
            const int rr = t >> lpr;
            const int rem = t & (per_row - 1);
            const int a0 = ((rem >> lo) << (lo + 4)) | (rem & lo_mask);
            float* row = cur + rr * RS;
            float x[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) x[u] = row[padx(a0 + (u << lo))];
#pragma unroll
            for (int h = 1; h < 16; h <<= 1)
#pragma unroll
              for (int u = 0; u < 16; ++u)
                if ((u & h) == 0) {
                  const float s0 = x[u], s1 = x[u | h];
                  x[u] = s0 + s1;
                  x[u | h] = s0 - s1;
                }
#pragma unroll
            for (int u = 0; u < 16; ++u) row[padx(a0 + (u << lo))] = x[u];
          }
          __syncthreads();
          continue;
        }
        for (int t = tid; t < items; t += RP_THREADS) {
          const int rr = t / per_row;
          int rem = t - rr * per_row;
          int b = 0;
          if (K > 1) {
            const int q = rem / K;
            b = rem - q * K;
            rem = q;
          }
          const int a0 = ((rem >> lo) << (lo + nb)) | (rem & lo_mask);
          float* row = cur + rr * RS;
          float x[16];
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (u < G) x[u] = row[padx((a0 + (u << lo)) * K + b)];
#pragma unroll
          for (int h = 1; h < 16; h <<= 1) {
            if (h < G) {
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                if (u < G && (u & h) == 0) {
                  const float s0 = x[u], s1 = x[u | h];
                  x[u] = s0 + s1;
                  x[u | h] = s0 - s1;
                }
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 16; ++u)
            if (u < G) row[padx((a0 + (u << lo)) * K + b)] = x[u];
        }
        __syncthreads();
      }
    }

    // 4. transposed store: consecutive threads take consecutive rows of one
    //    column, so every warp writes R-float runs of the output rows (or,
    //    row-wise, consecutive threads take consecutive columns of a row).
    const float nrm = p.rotate ? A.norm : 1.f;
    const int tot = L << A.logR;
    const int rr = tid & (R - 1);
    const int jstep = RP_THREADS >> A.logR;
    if (p.rowwise) {
      for (int q = 0; q < rows_here; ++q) {
        const float* src = cur + q * RS;
        float* o = p.out + (r0 + q) * p.ld_out;
        for (int j = tid; j < L; j += RP_THREADS) {
          float x = src[padx(j)] * nrm;
          if (p.inverse) x = x * (F4096 ? cfs[j] : col_factor(p, j));
          o[j] = x;
        }
      }
    } else if (rr < rows_here) {
      float* o = p.out + (int64_t)(tid >> A.logR) * p.ld_out + r0 + rr;
      const int64_t ostep = (int64_t)jstep * p.ld_out;
      const float* src = cur + rr * RS;
      for (int t = tid, j = tid >> A.logR; t < tot; t += RP_THREADS, j += jstep, o += ostep) {
        float x = src[padx(j)] * nrm;
        if (p.inverse) x = x * (F4096 ? cfs[j] : col_factor(p, j));
        *o = x;
      }
    }
    // shared memory is refilled by the next group
    __syncthreads();
  }
}

// ------------------------------------------------------------ compile-time row transform
// The same pass for the lengths of the Llama sublayers, L = K 2^LOGP with K
// and LOGP known at compile time, so that every index of the DCT and the
// radix-16 Walsh-Hadamard passes is a shift or a multiply by a constant:
// R rows per CTA group (a power of two), 512 threads, the next group's
// loads held in registers while the current group is transformed and
// stored, the column factors (sign and rescale) read from a table computed
// once per launch.  Arithmetic per element is that of rowpass_kernel.
template <int K, int LOGP, int R>
struct FastShape {
  static constexpr int P = 1 << LOGP;
  static constexpr int L = K * P;
  static constexpr int CPT = (L + RP_THREADS - 1) / RP_THREADS;   // columns per thread and row
  static constexpr int RS = (L + (L >> 5)) | 1;                   // padded row stride
  static constexpr int LOGR = (R == 1) ? 0 : (R == 2) ? 1 : (R == 4) ? 2 : 3;
};

// One radix-2^NB pass over bits LO .. LO+NB-1 of a (index a K + b) of R rows.
template <int K, int LOGP, int R, int LO, int NB>
__device__ __forceinline__ void fwht_pass(float* buf) {
  using S = FastShape<K, LOGP, R>;
  constexpr int G = 1 << NB;
  constexpr int IPR = (S::P / G) * K;          // items per row
  constexpr int LOMASK = (1 << LO) - 1;
  for (int t = threadIdx.x; t < IPR * R; t += RP_THREADS) {
    const int rr = t / IPR;
    const int rem = t - rr * IPR;
    const int b = rem % K;
    const int qv = rem / K;
    const int a0 = ((qv >> LO) << (LO + NB)) | (qv & LOMASK);
    float* row = buf + rr * S::RS;
    float x[G];
#pragma unroll
    for (int u = 0; u < G; ++u) x[u] = row[padx((a0 + (u << LO)) * K + b)];
#pragma unroll
    for (int h = 1; h < G; h <<= 1)
#pragma unroll
      for (int u = 0; u < G; ++u)
        if ((u & h) == 0) {
          const float s0 = x[u], s1 = x[u | h];
          x[u] = s0 + s1;
          x[u | h] = s0 - s1;
        }
#pragma unroll
    for (int u = 0; u < G; ++u) row[padx((a0 + (u << LO)) * K + b)] = x[u];
  }
  __syncthreads();
}

template <int K, int LOGP, int R, int LO>
__device__ __forceinline__ void fwht_all(float* buf) {
  if constexpr (LO < LOGP) {
    constexpr int NB = (LOGP - LO) < 4 ? (LOGP - LO) : 4;
    fwht_pass<K, LOGP, R, LO, NB>(buf);
    fwht_all<K, LOGP, R, LO + NB>(buf);
  }
}

template <bool BF16, int K, int LOGP, int R>
__global__ void __launch_bounds__(RP_THREADS, 1) rowpass_fast_kernel(RowPass p, const float* cf) {
  using S = FastShape<K, LOGP, R>;
  extern __shared__ __align__(16) float sm[];
  float* buf = sm;
  float* Cm = sm + R * S::RS;   // K x K DCT matrix (K > 1)
  const int tid = threadIdx.x;
  const int64_t ngroups = (p.rows + R - 1) / R;
  if (K > 1) {
    for (int t = tid; t < K * K; t += RP_THREADS) {
      const int i = t / K, j = t - (t / K) * K;
      const double ci = (i == 0) ? sqrt(0.5) : 1.0;
      Cm[t] = (float)(sqrt(2.0 / K) * ci * cospi((double)((2 * j + 1) * i) / (2.0 * K)));
    }
  }
  float v[R][S::CPT];
  auto load = [&](int64_t g) {
    const int64_t r0 = g * R;
#pragma unroll
    for (int rr = 0; rr < R; ++rr) {
      const bool live = r0 + rr < p.rows;
      const int64_t base = (r0 + rr) * p.ld_in;
#pragma unroll
      for (int c = 0; c < S::CPT; ++c) {
        const int j = tid + c * RP_THREADS;
        float x = 0.f;
        if (live && j < S::L) {
          if (BF16) x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.in)[base + j]);
          else x = reinterpret_cast<const float*>(p.in)[base + j];
        }
        v[rr][c] = x;
      }
    }
  };
  int64_t grp = blockIdx.x;
  if (grp < ngroups) load(grp);
  for (; grp < ngroups; grp += gridDim.x) {
    const int64_t r0 = grp * R;
    const int rows_here = (int)((p.rows - r0) < R ? (p.rows - r0) : R);
    // 1. rows into shared memory, times the column factors (forward)
#pragma unroll
    for (int c = 0; c < S::CPT; ++c) {
      const int j = tid + c * RP_THREADS;
      if (j < S::L) {
        const float f = p.inverse ? 1.f : (cf ? cf[j] : col_factor(p, j));
#pragma unroll
        for (int rr = 0; rr < R; ++rr) buf[rr * S::RS + padx(j)] = v[rr][c] * f;
      }
    }
    __syncthreads();
    if (grp + gridDim.x < ngroups) load(grp + gridDim.x);   // in flight during the transform
    if (p.rotate) {
      // 2. DCT along b: one thread per (row, a), all K inputs in registers,
      //    each output written as soon as it is formed
      if (K > 1) {
        for (int t = tid; t < R * S::P; t += RP_THREADS) {
          const int rr = t >> LOGP;
          const int a = t & (S::P - 1);
          float* row = buf + rr * S::RS;
          float y[K];
#pragma unroll
          for (int bb = 0; bb < K; ++bb) y[bb] = row[padx(a * K + bb)];
#pragma unroll
          for (int o = 0; o < K; ++o) {
            float acc = 0.f;
#pragma unroll
            for (int bb = 0; bb < K; ++bb) acc = fmaf(p.inverse ? Cm[bb * K + o] : Cm[o * K + bb], y[bb], acc);
            row[padx(a * K + o)] = acc;
          }
        }
        __syncthreads();
      }
      // 3. Walsh-Hadamard along a, radix-16 passes (a shorter last one)
      fwht_all<K, LOGP, R, 0>(buf);
    }
    // 4. transposed store: consecutive threads take consecutive rows of one
    //    column (R-float runs of the output rows); row-wise: four
    //    consecutive columns of a row per thread (16-byte stores)
    const float nrm = p.rotate ? (float)(1.0 / sqrt((double)S::P)) : 1.f;
    const int rr = tid & (R - 1);
    constexpr int JSTEP = RP_THREADS >> S::LOGR;
    if (p.rowwise) {
      static_assert(S::L % 4 == 0, "row-wise stores take four columns at a time");
      const bool v4 = (p.ld_out % 4) == 0 && ((reinterpret_cast<uintptr_t>(p.out) & 15) == 0);
      for (int q = 0; q < rows_here; ++q) {
        const float* src = buf + q * S::RS;
        float* o = p.out + (r0 + q) * p.ld_out;
        for (int j = 4 * tid; j < S::L; j += 4 * RP_THREADS) {
          // j .. j + 3 sit in one 32-float run of the padded row
          float4 x = make_float4(src[padx(j)] * nrm, src[padx(j) + 1] * nrm, src[padx(j) + 2] * nrm,
                                 src[padx(j) + 3] * nrm);
          if (p.inverse) {
            x.x *= cf ? cf[j] : col_factor(p, j);
            x.y *= cf ? cf[j + 1] : col_factor(p, j + 1);
            x.z *= cf ? cf[j + 2] : col_factor(p, j + 2);
            x.w *= cf ? cf[j + 3] : col_factor(p, j + 3);
          }
          if (v4) {
            *reinterpret_cast<float4*>(o + j) = x;
          } else {
            o[j] = x.x;
            o[j + 1] = x.y;
            o[j + 2] = x.z;
            o[j + 3] = x.w;
          }
        }
      }
    } else if (rr < rows_here) {
      const float* src = buf + rr * S::RS;
      for (int j = tid >> S::LOGR; j < S::L; j += JSTEP) {
        float x = src[padx(j)] * nrm;
        if (p.inverse) x = x * (cf ? cf[j] : col_factor(p, j));
        p.out[(int64_t)j * p.ld_out + r0 + rr] = x;
      }
    }
    __syncthreads();
  }
}

// Rows too long for more than one per CTA (L = 28672: 118 KB of shared
// memory each) would leave the transposed store one float wide.  A cluster
// of CL CTAs transforms CL consecutive rows, one per CTA, and then stores
// together: CTA c writes the output rows j of its slice [c L / CL,
// (c + 1) L / CL) with the CL values of each j gathered from the cluster's
// shared memory (distributed shared memory), CL consecutive floats per
// output row.  Cluster barriers separate the transform, the store and the
// next group.
constexpr int CL = 8;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

template <bool BF16, int K, int LOGP>
__global__ void __launch_bounds__(RP_THREADS, 1) rowpass_cluster_kernel(RowPass p, const float* cf) {
  using S = FastShape<K, LOGP, 1>;
  extern __shared__ __align__(16) float sm[];
  float* buf = sm;
  float* Cm = sm + S::RS;
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank();
  const int64_t cid = blockIdx.x / CL, ncl = gridDim.x / CL;
  const int64_t ngroups = (p.rows + CL - 1) / CL;
  if (K > 1) {
    for (int t = tid; t < K * K; t += RP_THREADS) {
      const int i = t / K, j = t - (t / K) * K;
      const double ci = (i == 0) ? sqrt(0.5) : 1.0;
      Cm[t] = (float)(sqrt(2.0 / K) * ci * cospi((double)((2 * j + 1) * i) / (2.0 * K)));
    }
  }
  // the shared-memory address of buf in every CTA of the cluster
  uint32_t peer[CL];
#pragma unroll
  for (int q = 0; q < CL; ++q) peer[q] = map_to_rank(smem_u32(buf), (uint32_t)q);
  const float nrm = p.rotate ? (float)(1.0 / sqrt((double)S::P)) : 1.f;
  float v[S::CPT];
  auto load = [&](int64_t g) {
    const int64_t row = g * CL + rank;
    const bool live = row < p.rows;
#pragma unroll
    for (int c = 0; c < S::CPT; ++c) {
      const int j = tid + c * RP_THREADS;
      float x = 0.f;
      if (live && j < S::L) {
        if (BF16) x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.in)[row * p.ld_in + j]);
        else x = reinterpret_cast<const float*>(p.in)[row * p.ld_in + j];
      }
      v[c] = x;
    }
  };
  int64_t grp = cid;
  if (grp < ngroups) load(grp);
  for (; grp < ngroups; grp += ncl) {
    const int64_t r0 = grp * CL;
    const int rows_here = (int)((p.rows - r0) < CL ? (p.rows - r0) : CL);
#pragma unroll
    for (int c = 0; c < S::CPT; ++c) {
      const int j = tid + c * RP_THREADS;
      if (j < S::L) buf[padx(j)] = v[c] * (p.inverse ? 1.f : (cf ? cf[j] : col_factor(p, j)));
    }
    __syncthreads();
    if (grp + ncl < ngroups) load(grp + ncl);
    if (p.rotate) {
      if (K > 1) {
        for (int a = tid; a < S::P; a += RP_THREADS) {
          float y[K];
#pragma unroll
          for (int bb = 0; bb < K; ++bb) y[bb] = buf[padx(a * K + bb)];
#pragma unroll
          for (int o = 0; o < K; ++o) {
            float acc = 0.f;
#pragma unroll
            for (int bb = 0; bb < K; ++bb) acc = fmaf(p.inverse ? Cm[bb * K + o] : Cm[o * K + bb], y[bb], acc);
            buf[padx(a * K + o)] = acc;
          }
        }
        __syncthreads();
      }
      fwht_all<K, LOGP, 1, 0>(buf);
    }
    cluster_sync_all();   // every row of the group is transformed
    constexpr int SLICE = S::L / CL;
    const int j0 = (int)rank * SLICE;
    const bool vec = rows_here == CL && (p.ld_out % 4) == 0 && (r0 % 4) == 0 &&
                     ((reinterpret_cast<uintptr_t>(p.out) & 15) == 0);
    for (int jj = tid; jj < SLICE; jj += RP_THREADS) {
      const int j = j0 + jj;
      const uint32_t off = (uint32_t)padx(j) * 4u;
      float x[CL];
#pragma unroll
      for (int q = 0; q < CL; ++q) x[q] = ld_cluster_f32(peer[q] + off) * nrm;
      if (p.inverse) {
        const float f = cf ? cf[j] : col_factor(p, j);
#pragma unroll
        for (int q = 0; q < CL; ++q) x[q] *= f;
      }
      float* o = p.out + (int64_t)j * p.ld_out + r0;
      if (vec) {
        reinterpret_cast<float4*>(o)[0] = make_float4(x[0], x[1], x[2], x[3]);
        reinterpret_cast<float4*>(o)[1] = make_float4(x[4], x[5], x[6], x[7]);
      } else {
#pragma unroll
        for (int q = 0; q < CL; ++q)
          if (q < rows_here) o[q] = x[q];
      }
    }
    cluster_sync_all();   // the peers have read this CTA's row
  }
}

__global__ void colfactor_kernel(RowPass p, float* cf) {
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < (int)p.L; j += gridDim.x * blockDim.x)
    cf[j] = col_factor(p, j);
}

template <bool BF16, int K, int LOGP>
kronq_status launch_cluster(const RowPass& p, cudaStream_t s) {
  using S = FastShape<K, LOGP, 1>;
  static_assert(S::L % CL == 0, "the row splits into CL slices");
  const float* cf = nullptr;
  if (p.cf) {
    colfactor_kernel<<<(unsigned)ceil_div(S::L, 256), 256, 0, s>>>(p, p.cf);
    KQ_LAUNCH_CHECK("colfactor_kernel");
    cf = p.cf;
  }
  const int smem = (S::RS + (K > 1 ? K * K : 0)) * (int)sizeof(float);
  const void* fn = reinterpret_cast<const void*>(&rowpass_cluster_kernel<BF16, K, LOGP>);
  cudaError_t e = allow_smem(fn, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rowpass_cluster)");
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(RP_THREADS);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // persistent: as many clusters as fit at once, each looping over groups
  int active = 0;
  cfg.gridDim = dim3((unsigned)(CL * 16));
  e = cudaOccupancyMaxActiveClusters(&active, fn, &cfg);
  if (e != cudaSuccess || active < 1) return e != cudaSuccess ? cuda_fail(e, "cudaOccupancyMaxActiveClusters")
                                                              : fail(KRONQ_ERR_CUDA, "rowpass: no cluster fits");
  const int64_t groups = ceil_div(p.rows, CL);
  const int64_t ncl = groups < (int64_t)active ? groups : (int64_t)active;
  cfg.gridDim = dim3((unsigned)(CL * ncl));
  e = cudaLaunchKernelEx(&cfg, rowpass_cluster_kernel<BF16, K, LOGP>, p, cf);
  count_launch();
  if (e != cudaSuccess) return cuda_fail(e, "rowpass_cluster_kernel");
  return KRONQ_OK;
}

template <bool BF16, int K, int LOGP, int R>
kronq_status launch_fast(const RowPass& p, cudaStream_t s) {
  using S = FastShape<K, LOGP, R>;
  const float* cf = nullptr;
  if (p.cf) {
    colfactor_kernel<<<(unsigned)ceil_div(S::L, 256), 256, 0, s>>>(p, p.cf);
    KQ_LAUNCH_CHECK("colfactor_kernel");
    cf = p.cf;
  }
  const int smem = (R * S::RS + (K > 1 ? K * K : 0)) * (int)sizeof(float);
  const void* fn = reinterpret_cast<const void*>(&rowpass_fast_kernel<BF16, K, LOGP, R>);
  cudaError_t e = allow_smem(fn, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rowpass_fast)");
  const int64_t groups = ceil_div(p.rows, R);
  const int64_t grid = groups < (int64_t)sm_count() ? groups : (int64_t)sm_count();
  rowpass_fast_kernel<BF16, K, LOGP, R><<<(unsigned)grid, RP_THREADS, (size_t)smem, s>>>(p, cf);
  KQ_LAUNCH_CHECK("rowpass_fast_kernel");
  return KRONQ_OK;
}

// ------------------------------------------------------------ register-resident rows of 7 x 4096
// Forward rows of L = 28672 = 7 x 4096 (the Llama-3-70B MLP length), stored
// by rows.  One CTA of 256 threads per SM.  A row passes through shared
// memory only to arrive (one bulk copy; the CTA's next row is copied into the
// second buffer while this one is transformed), for two exchanges, and to
// leave (one bulk copy).  Thread (w, l) holds 16 values of the Hadamard index
// a times the 7 values of the DCT index b in registers; the twelve bits of a
// are transformed four at a time, always in registers:
//   phase 1: a = 256 u + 32 w + l          (registers: bits 8-11)
//            column factors, the DCT along b, radix 16
//   phase 2: a = u + 16 l + 512 w          (bits 0-3), radix 16
//   phase 3: a = (l & 15) + 16 u + 256 (l >> 4) + 512 w   (bits 4-7), radix 16
// The exchanges use the layout 7 a + b + (a >> 4) (one word of padding per
// 16 a), on which the phase-2 and phase-3 accesses of a warp hit 32 distinct
// banks; the arriving and the departing row use 7 a + b.  Per element the
// arithmetic is that of rowpass_kernel (column factor, DCT, unnormalised
// butterflies, 1 / sqrt(P)); the butterflies over the bits of a run in
// another order, which changes only rounding.
constexpr int R7_THREADS = 256;
constexpr int R7_K = 7;
constexpr int R7_P = 4096;
constexpr int R7_L = R7_K * R7_P;
constexpr int R7_BUF = R7_L + R7_P / 16;                     // floats per buffer
constexpr int R7_SMEM = 2 * R7_BUF * (int)sizeof(float) + 16;  // two buffers, two mbarriers

struct Dct7 {
  float c[R7_K * R7_K];   // orthonormal DCT-II, c[o * 7 + b]; a kernel parameter, read from the constant bank
};

__device__ __forceinline__ void radix16_regs(float (&x)[16][R7_K]) {
#pragma unroll
  for (int b = 0; b < R7_K; ++b)
#pragma unroll
    for (int h = 1; h < 16; h <<= 1)
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if ((u & h) == 0) {
          const float s0 = x[u][b], s1 = x[u | h][b];
          x[u][b] = s0 + s1;
          x[u | h][b] = s0 - s1;
        }
}

__device__ __forceinline__ int r7_pad(int a) { return 7 * a + (a >> 4); }

template <bool BF16>
__global__ void __launch_bounds__(R7_THREADS, 1) rowpass_r7_kernel(const void* in, int64_t ld_in, float* out,
                                                                   int64_t ld_out, int64_t rows, const float* cf,
                                                                   Dct7 C) {
  extern __shared__ __align__(16) float sm[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 2 * R7_BUF);
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const uint32_t bar0 = smem_u32(&bars[0]);
  constexpr uint32_t esz = BF16 ? 2u : 4u;
  constexpr uint32_t in_bytes = R7_L * esz;
  constexpr uint32_t out_bytes = R7_L * 4u;
  const char* inb = static_cast<const char*>(in);
  if (tid == 0) {
    mbar_init(bar0, 1);
    mbar_init(bar0 + 8, 1);
    fence_mbar_init();
  }
  __syncthreads();
  int64_t row = blockIdx.x;
  // loads issued and not yet waited for, bit k for buffer k (thread 0 only)
  uint32_t pending = 0;
  if (tid == 0 && row < rows) {
    mbar_arrive_expect_tx(bar0, in_bytes);
    bulk_load(smem_u32(sm), inb + row * ld_in * esz, in_bytes, bar0);
    pending = 1u;
  }
  for (int i = 0; row < rows; ++i, row += gridDim.x) {
    const int b = i & 1;
    float* buf = sm + b * R7_BUF;
    const int64_t nrow = row + gridDim.x;
    if (tid == 0 && nrow < rows) {
      tma_store_wait_read();   // the row stored from the other buffer has been read out
      mbar_arrive_expect_tx(bar0 + 8 * (b ^ 1), in_bytes);
      bulk_load(smem_u32(sm + (b ^ 1) * R7_BUF), inb + nrow * ld_in * esz, in_bytes, bar0 + 8 * (b ^ 1));
      pending |= 1u << (b ^ 1);
    }
    const bool arrived = mbar_wait(bar0 + 8 * b, (uint32_t)(i >> 1) & 1u);
    if (tid == 0 && arrived) pending &= ~(1u << b);
    if (!__syncthreads_and(arrived)) break;   // timed out (recorded): stop the whole CTA

    // phase 1: the arrived row (7 a + b), column factors, DCT along b
    float x[16][R7_K];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int a = 256 * u + 32 * w + l;
      float v[R7_K];
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) {
        const int j = 7 * a + bb;
        const float e = BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(buf)[j]) : buf[j];
        v[bb] = e * __ldg(cf + j);
      }
#pragma unroll
      for (int o = 0; o < R7_K; ++o) {
        float acc = 0.f;
#pragma unroll
        for (int bb = 0; bb < R7_K; ++bb) acc = fmaf(C.c[o * R7_K + bb], v[bb], acc);
        x[u][o] = acc;
      }
    }
    radix16_regs(x);
    __syncthreads();   // every thread has read the arrived row
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int pa = r7_pad(256 * u + 32 * w + l);
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) buf[pa + bb] = x[u][bb];
    }
    __syncthreads();
    // phase 2: bits 0-3 in registers (each thread writes back what it read)
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int pa = r7_pad(u + 16 * l + 512 * w);
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) x[u][bb] = buf[pa + bb];
    }
    radix16_regs(x);
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int pa = r7_pad(u + 16 * l + 512 * w);
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) buf[pa + bb] = x[u][bb];
    }
    __syncthreads();
    // phase 3: bits 4-7 in registers
    const int a3 = (l & 15) + 256 * (l >> 4) + 512 * w;
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int pa = r7_pad(a3 + 16 * u);
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) x[u][bb] = buf[pa + bb];
    }
    radix16_regs(x);
    __syncthreads();   // every phase-3 read is done: the row layout overwrites
    const float nrm = 1.f / 64.f;   // 1 / sqrt(4096), exact
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int j = 7 * (a3 + 16 * u);
#pragma unroll
      for (int bb = 0; bb < R7_K; ++bb) buf[j + bb] = x[u][bb] * nrm;
    }
    fence_proxy_async_smem();   // the row's writes, before the bulk copy reads them
    __syncthreads();
    if (tid == 0) {
      bulk_store(out + row * ld_out, smem_u32(buf), out_bytes);
      tma_store_commit();
    }
  }
  if (tid == 0) {
    // a load left in flight only after a timeout: wait for it (bounded)
    for (int k = 0; k < 2; ++k)
      if (pending & (1u << k)) (void)mbar_wait(bar0 + 8 * k, 0u);
    tma_store_wait_all();
  }
}

// out[j * ldo + r] = in[r * ldi + j] for r < rows, j < cols: 64 x 64 tiles.
__global__ void __launch_bounds__(256) transpose_f32_kernel(const float* in, int64_t ldi, float* out, int64_t ldo,
                                                            int64_t rows, int64_t cols) {
  __shared__ float t[64][65];
  const int64_t r0 = (int64_t)blockIdx.y * 64, c0 = (int64_t)blockIdx.x * 64;
  const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int64_t r = r0 + ty + 4 * k, c = c0 + tx;
    if (r < rows && c < cols) t[ty + 4 * k][tx] = in[r * ldi + c];
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int64_t j = c0 + ty + 4 * k, r = r0 + tx;
    if (j < cols && r < rows) out[j * ldo + r] = t[tx][ty + 4 * k];
  }
}

// The register-resident pass for rows of 28672 when its operands allow the
// bulk copies; a transposed pass runs as a row-wise pass into p.tmp and a
// transpose.  Returns false when it does not apply.
#define KQ_LAUNCH_CHECK_R(r, name)                       \
  do {                                                   \
    ::kq::count_launch();                                \
    cudaError_t e__ = cudaGetLastError();                \
    if (e__ != cudaSuccess) {                            \
      (r) = ::kq::cuda_fail(e__, name);                  \
      return true;                                       \
    }                                                    \
  } while (0)

bool try_r7(const RowPass& p, cudaStream_t s, kronq_status& r) {
  if (!(p.L == R7_L && p.rotate && !p.inverse && p.cf && p.rows > 0)) return false;
  const size_t esz = p.in_bf16 ? 2 : 4;
  float* dst = p.rowwise ? p.out : p.tmp;
  const int64_t ldd = p.rowwise ? p.ld_out : p.ld_tmp;
  if (!dst || !aligned(p.in, 16) || (p.ld_in * esz) % 16 != 0 || !aligned(dst, 16) || (ldd * 4) % 16 != 0)
    return false;
  if (!p.rowwise && p.in_bf16 && static_cast<const void*>(dst) == p.in) return false;
  colfactor_kernel<<<(unsigned)ceil_div(R7_L, 256), 256, 0, s>>>(p, p.cf);
  KQ_LAUNCH_CHECK_R(r, "colfactor_kernel");
  Dct7 C;
  for (int o = 0; o < R7_K; ++o)
    for (int b = 0; b < R7_K; ++b) {
      const double co = (o == 0) ? sqrt(0.5) : 1.0;
      C.c[o * R7_K + b] = (float)(sqrt(2.0 / R7_K) * co * cos(acos(-1.0) * (double)((2 * b + 1) * o) / (2.0 * R7_K)));
    }
  const void* fn = p.in_bf16 ? reinterpret_cast<const void*>(&rowpass_r7_kernel<true>)
                             : reinterpret_cast<const void*>(&rowpass_r7_kernel<false>);
  cudaError_t e = allow_smem(fn, R7_SMEM);
  if (e != cudaSuccess) {
    r = cuda_fail(e, "cudaFuncSetAttribute(rowpass_r7)");
    return true;
  }
  const int64_t grid = p.rows < (int64_t)sm_count() ? p.rows : (int64_t)sm_count();
  if (p.in_bf16)
    rowpass_r7_kernel<true><<<(unsigned)grid, R7_THREADS, R7_SMEM, s>>>(p.in, p.ld_in, dst, ldd, p.rows, p.cf, C);
  else
    rowpass_r7_kernel<false><<<(unsigned)grid, R7_THREADS, R7_SMEM, s>>>(p.in, p.ld_in, dst, ldd, p.rows, p.cf, C);
  KQ_LAUNCH_CHECK_R(r, "rowpass_r7_kernel");
  if (!p.rowwise) {
    dim3 g((unsigned)ceil_div(R7_L, 64), (unsigned)ceil_div(p.rows, 64));
    transpose_f32_kernel<<<g, 256, 0, s>>>(dst, ldd, p.out, p.ld_out, p.rows, R7_L);
    KQ_LAUNCH_CHECK_R(r, "transpose_f32_kernel");
  }
  r = KRONQ_OK;
  return true;
}

// The compile-time variants: (odd factor, log2 of the power of two, rows
// per group).  Returns false when the length has none.
template <bool BF16>
bool try_fast(const RowPass& p, cudaStream_t s, kronq_status& r) {
  switch (p.L) {
    case 28672:                                                        // Llama-3-70B MLP
      r = p.rowwise ? launch_fast<BF16, 7, 12, 1>(p, s) : launch_cluster<BF16, 7, 12>(p, s);
      return true;
    case 14336: r = launch_fast<BF16, 7, 11, 2>(p, s); return true;   // Llama-3-8B MLP
    case 11008: r = launch_fast<BF16, 43, 8, 2>(p, s); return true;   // Llama-2-7B MLP
    case 8192: r = launch_fast<BF16, 1, 13, 4>(p, s); return true;    // Llama-3-70B hidden
    case 1024: r = launch_fast<BF16, 1, 10, 8>(p, s); return true;    // Llama-3-8B k/v
    default: return false;
  }
}

// ------------------------------------------------------------ norms
template <typename T>
__device__ __forceinline__ float ld_val(const void* W, int64_t idx) {
  if constexpr (sizeof(T) == 2)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[idx]);
  else
    return reinterpret_cast<const float*>(W)[idx];
}

template <typename T>
__global__ void rownorm_kernel(const void* W, int64_t m, int64_t n, float* rowsq) {
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (r >= m) return;
  double acc = 0.0;
  for (int64_t j = lane; j < n; j += 32) {
    const double v = ld_val<T>(W, r * n + j);
    acc += v * v;
  }
  acc = warp_sum_d(acc);
  if (lane == 0) rowsq[r] = (float)acc;
}

constexpr int COL_CHUNK = 256;

template <typename T>
__global__ void colnorm_partial_kernel(const void* W, int64_t m, int64_t n, double* partial) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t i0 = (int64_t)blockIdx.y * COL_CHUNK;
  if (j >= n) return;
  double acc = 0.0;
  const int64_t i1 = (i0 + COL_CHUNK < m) ? i0 + COL_CHUNK : m;
  for (int64_t i = i0; i < i1; ++i) {
    const double v = ld_val<T>(W, i * n + j);
    acc += v * v;
  }
  partial[(int64_t)blockIdx.y * n + j] = acc;
}

__global__ void colnorm_final_kernel(const double* partial, int64_t chunks, int64_t n, float* colsq) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  double acc = 0.0;
  for (int64_t c = 0; c < chunks; ++c) acc += partial[c * n + j];
  colsq[j] = (float)acc;
}

__global__ void __launch_bounds__(1024) rescale_kernel(const float* H, int64_t ldh, const float* nrm,
                                                       int64_t len, float alpha, float* d) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < len; j += blockDim.x) {
    const double h = H[j * ldh + j], w = nrm[j];
    const double raw = (h > 0.0 && w > 0.0) ? pow(h / w, (double)alpha) : 1.0;
    acc += log(raw);
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
  const double inv_gm = exp(-red[0] / (double)len);
  for (int64_t j = threadIdx.x; j < len; j += blockDim.x) {
    const double h = H[j * ldh + j], w = nrm[j];
    const double raw = (h > 0.0 && w > 0.0) ? pow(h / w, (double)alpha) : 1.0;
    d[j] = (float)(raw * inv_gm);
  }
}

}  // namespace

kronq_status rowpass(const RowPass& p, cudaStream_t s) {
  if (p.rows <= 0 || p.L <= 0) return KRONQ_OK;
  if (p.L > (1 << 24)) return fail(KRONQ_ERR_UNSUPPORTED, "BiIP rotation: row too long");
  RPArgs A;
  A.p = p;
  int P = 1;
  while (p.L % (2 * (int64_t)P) == 0) P *= 2;
  const int64_t K = p.L / P;
  if (p.rotate && K > KMAX)
    return fail(KRONQ_ERR_UNSUPPORTED, "BiIP rotation: odd factor of the length exceeds 255");
  A.P = P;
  A.K = (int)K;
  A.logP = 0;
  while ((1 << A.logP) < P) ++A.logP;
  A.norm = (float)(1.0 / sqrt((double)P));
  A.two_buf = (p.rotate && K > KREG) ? 1 : 0;
  const int64_t base = p.L + (p.L >> 5);
  A.RS = (int)(base | 1);
  const int64_t bytes_per_row = (int64_t)A.RS * 4 * (A.two_buf ? 2 : 1);
  const int64_t cbytes = (p.rotate && K > 1) ? K * K * 4 : 0;
  const int64_t budget = 200 * 1024;
  int R = 8;
  while (R > 1 && R * bytes_per_row + cbytes > budget) R >>= 1;
  if (R * bytes_per_row + cbytes > budget)
    return fail(KRONQ_ERR_UNSUPPORTED, "BiIP rotation: row does not fit in shared memory");
  A.R = R;
  A.logR = 0;
  while ((1 << A.logR) < R) ++A.logR;
  if (p.rotate) {
    kronq_status r = KRONQ_OK;
    if (try_r7(p, s, r)) return r;
    if (p.in_bf16 ? try_fast<true>(p, s, r) : try_fast<false>(p, s, r)) return r;
  }
  const bool f4096 = (p.L == 4096 && K == 1);
  const int64_t smem = R * bytes_per_row + cbytes + (f4096 ? p.L * 4 : 0);
  const void* fn = f4096 ? (p.in_bf16 ? reinterpret_cast<const void*>(&rowpass_kernel<true, true>)
                                      : reinterpret_cast<const void*>(&rowpass_kernel<false, true>))
                         : (p.in_bf16 ? reinterpret_cast<const void*>(&rowpass_kernel<true, false>)
                                      : reinterpret_cast<const void*>(&rowpass_kernel<false, false>));
  cudaError_t e = allow_smem(fn, (int)smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(rowpass)");
  // one CTA per SM (the row buffers take most of shared memory), each
  // looping over row groups
  const int64_t groups = ceil_div(p.rows, R);
  const int64_t grid = groups < (int64_t)sm_count() ? groups : (int64_t)sm_count();
  if (f4096) {
    if (p.in_bf16) rowpass_kernel<true, true><<<(unsigned)grid, RP_THREADS, (size_t)smem, s>>>(A);
    else rowpass_kernel<false, true><<<(unsigned)grid, RP_THREADS, (size_t)smem, s>>>(A);
  } else {
    if (p.in_bf16) rowpass_kernel<true, false><<<(unsigned)grid, RP_THREADS, (size_t)smem, s>>>(A);
    else rowpass_kernel<false, false><<<(unsigned)grid, RP_THREADS, (size_t)smem, s>>>(A);
  }
  KQ_LAUNCH_CHECK("rowpass_kernel");
  return KRONQ_OK;
}

size_t wnorms_partial_floats(int64_t m, int64_t n) {
  return (size_t)(ceil_div(m, COL_CHUNK) * n * 2);  // doubles, counted in floats
}

kronq_status wnorms(const void* W, bool bf16, int64_t m, int64_t n, float* colsq, float* rowsq,
                    float* partial, cudaStream_t s) {
  double* part = reinterpret_cast<double*>(partial);
  const int64_t chunks = ceil_div(m, COL_CHUNK);
  if (rowsq) {
    const int64_t grid = ceil_div(m, 8);
    if (bf16) rownorm_kernel<__nv_bfloat16><<<(unsigned)grid, 256, 0, s>>>(W, m, n, rowsq);
    else rownorm_kernel<float><<<(unsigned)grid, 256, 0, s>>>(W, m, n, rowsq);
    KQ_LAUNCH_CHECK("rownorm_kernel");
  }
  if (colsq) {
    dim3 g1((unsigned)ceil_div(n, 256), (unsigned)chunks);
    if (bf16) colnorm_partial_kernel<__nv_bfloat16><<<g1, 256, 0, s>>>(W, m, n, part);
    else colnorm_partial_kernel<float><<<g1, 256, 0, s>>>(W, m, n, part);
    KQ_LAUNCH_CHECK("colnorm_partial_kernel");
    colnorm_final_kernel<<<(unsigned)ceil_div(n, 256), 256, 0, s>>>(part, chunks, n, colsq);
    KQ_LAUNCH_CHECK("colnorm_final_kernel");
  }
  return KRONQ_OK;
}

kronq_status rescale_vector(const float* H, int64_t ldh, const float* nrm, int64_t len, float alpha,
                            float* d, cudaStream_t s) {
  rescale_kernel<<<1, 1024, 0, s>>>(H, ldh, nrm, len, alpha, d);
  KQ_LAUNCH_CHECK("rescale_kernel");
  return KRONQ_OK;
}

}  // namespace kq

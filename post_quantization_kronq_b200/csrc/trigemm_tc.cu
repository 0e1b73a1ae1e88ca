// Float32 products with a triangular factor, on the tensor cores:
//   C = alpha * A B,  A (M x K) row-major, B (K x N) row-major, C row-major,
// with A upper triangular (A[i][k] = 0 for k < i) or B upper triangular
// (B[k][j] = 0 for k > j) as the recursive triangular inverse needs them
// (T = R12 U22, then U12 = -U11 T).  The triangle is masked on the fly, so
// the other triangle of the storage may hold anything; a tile only walks
// the k range its triangle leaves non-zero.
//
// Float32-level accuracy from bf16 MMAs: every operand element is split as
// x = hi + mid + lo (bf16 roundings of the remainders) and the six products
// hh + hm + mh + hl + lh + mm are accumulated in fp32 in TMEM (the dropped
// terms are below 2^-24 relative).  There is no pre-pass and no workspace:
// eight warps load the fp32 operands from global memory (one chunk ahead, in
// registers), write the splits into shared memory in the UMMA 128-byte
// swizzled layouts (A K-major, B MN-major), and arrive on the stage's
// barrier; thread 0 then issues the chunk's tcgen05.mma (M 128, N 128,
// K 16; 24 per 64-deep chunk) and commits the stage back.  Two stages of 96 KB.  The
// epilogue stages the accumulator through shared memory and writes C with
// coalesced stores.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int BM = 128, BN = 128, BK = 64;
constexpr int A_SPLIT = BM * BK * 2;            // 16 KB: 128 rows x 64 k, K-major
constexpr int B_BOX = 64 * BK * 2;              // 8 KB: 64 k rows x 64 columns, MN-major
constexpr int B_SPLIT = (BN / 64) * B_BOX;      // 16 KB
constexpr int STAGE = 3 * A_SPLIT + 3 * B_SPLIT;  // 96 KB
constexpr int NSTAGE = 2;
constexpr int CV_THREADS = 256;                 // warps 0-7: convert, MMA issue, epilogue
constexpr int THREADS = CV_THREADS;
constexpr int SMEM_BYTES = NSTAGE * STAGE + 1024 + 256;
constexpr int C_LD = BN + 4;                    // staged C row stride (floats)
constexpr uint32_t TMEM_COLS = 2 * BN;           // two segment accumulators
constexpr int SEG = 2;                            // 64-deep chunks per accumulation segment (128 k)
static_assert(BM * C_LD * 4 <= NSTAGE * STAGE, "C staging fits the stages");

struct TriArgs {
  const float* A;
  const float* B;
  float* C;
  int64_t lda, ldb, ldc, strideA, strideB, strideC;
  int M, N, K;
  float alpha;
  int a_upper, b_upper;
  int tiles_m, tiles_n;
  int vecA, vecB, vecC;   // float4 access allowed
  const int* info;
};

// Up to four consecutive floats p[0..valid-1], zero beyond.
__device__ __forceinline__ float4 ld4(const float* p, int valid, bool vec) {
  if (valid >= 4 && vec) return __ldg(reinterpret_cast<const float4*>(p));
  float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
  if (valid > 0) r.x = __ldg(p);
  if (valid > 1) r.y = __ldg(p + 1);
  if (valid > 2) r.z = __ldg(p + 2);
  if (valid > 3) r.w = __ldg(p + 3);
  return r;
}

// Splits four floats into hi / mid / lo bf16 (each the bf16 rounding of the
// remainder so far) and stores each split as 8 bytes.
__device__ __forceinline__ void split_store4(uint8_t* smem, uint32_t off, uint32_t split_bytes,
                                             float4 v) {
  const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y);
  const __nv_bfloat162 h23 = __floats2bfloat162_rn(v.z, v.w);
  const float r0 = v.x - __low2float(h01), r1 = v.y - __high2float(h01);
  const float r2 = v.z - __low2float(h23), r3 = v.w - __high2float(h23);
  const __nv_bfloat162 m01 = __floats2bfloat162_rn(r0, r1);
  const __nv_bfloat162 m23 = __floats2bfloat162_rn(r2, r3);
  const __nv_bfloat162 l01 = __floats2bfloat162_rn(r0 - __low2float(m01), r1 - __high2float(m01));
  const __nv_bfloat162 l23 = __floats2bfloat162_rn(r2 - __low2float(m23), r3 - __high2float(m23));
  auto bits = [](__nv_bfloat162 x) { return *reinterpret_cast<const uint32_t*>(&x); };
  *reinterpret_cast<uint2*>(smem + off) = make_uint2(bits(h01), bits(h23));
  *reinterpret_cast<uint2*>(smem + off + split_bytes) = make_uint2(bits(m01), bits(m23));
  *reinterpret_cast<uint2*>(smem + off + 2 * split_bytes) = make_uint2(bits(l01), bits(l23));
}

struct Chunk {
  float4 a[8];
  float4 b[8];
};

// Loads chunk kc (64 k) of A's tile rows and B's tile columns.
//   A: load j covers rows 16 j + 2 w + (lane / 16), k = kc + 4 (lane % 16) .. +3
//   B: load j covers k row kc + 8 j + w, columns 4 lane .. +3
__device__ __forceinline__ void load_chunk(const TriArgs& g, const float* A, const float* B,
                                           int m0, int n0, int kc, int warp, int lane, Chunk& c) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = 16 * j + 2 * warp + (lane >> 4);
    const int row = m0 + r;
    const int k = kc + 4 * (lane & 15);
    int valid = (row < g.M) ? g.K - k : 0;
    valid = valid < 0 ? 0 : valid;
    float4 v = ld4(A + (int64_t)row * g.lda + k, valid, g.vecA != 0);
    if (g.a_upper) {  // A[row][k] = 0 for k < row
      if (k + 0 < row) v.x = 0.f;
      if (k + 1 < row) v.y = 0.f;
      if (k + 2 < row) v.z = 0.f;
      if (k + 3 < row) v.w = 0.f;
    }
    c.a[j] = v;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int k = kc + 8 * j + warp;
    const int col = n0 + 4 * lane;
    int valid = (k < g.K) ? g.N - col : 0;
    valid = valid < 0 ? 0 : valid;
    float4 v = ld4(B + (int64_t)k * g.ldb + col, valid, g.vecB != 0);
    if (g.b_upper) {  // B[k][col] = 0 for k > col
      if (k > col + 0) v.x = 0.f;
      if (k > col + 1) v.y = 0.f;
      if (k > col + 2) v.z = 0.f;
      if (k > col + 3) v.w = 0.f;
    }
    c.b[j] = v;
  }
}

// Writes the splits of a loaded chunk into stage memory st.
__device__ __forceinline__ void store_chunk(uint8_t* st, int warp, int lane, const Chunk& c) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = 16 * j + 2 * warp + (lane >> 4);
    const int k = 4 * (lane & 15);
    const uint32_t off = r * 128 + ((((k >> 3) ^ (r & 7))) << 4) + (k & 7) * 2;
    split_store4(st, off, A_SPLIT, c.a[j]);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int k = 8 * j + warp;
    const int nn = 4 * lane;
    const uint32_t off = 3 * A_SPLIT + (nn >> 6) * B_BOX + k * 128 +
                         (((((nn & 63) >> 3) ^ (k & 7))) << 4) + (nn & 7) * 2;
    split_store4(st, off, B_SPLIT, c.b[j]);
  }
}

__global__ void __launch_bounds__(THREADS, 1) trigemm_tc_kernel(TriArgs g) {
  if (g.info && *g.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + NSTAGE * STAGE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * NSTAGE + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile order: the tiles with the longest k range first.
  const int bid = blockIdx.x;
  int tm, tn;
  if (g.b_upper) {
    tn = g.tiles_n - 1 - bid / g.tiles_m;
    tm = bid % g.tiles_m;
  } else {
    tm = bid / g.tiles_n;
    tn = bid % g.tiles_n;
  }
  const int m0 = tm * BM, n0 = tn * BN;
  int kbeg = g.a_upper ? m0 : 0;
  int kend = g.K;
  if (g.b_upper && n0 + BN < kend) kend = n0 + BN;
  const int nchunks = kend > kbeg ? (kend - kbeg + BK - 1) / BK : 0;
  const float* A = g.A + (int64_t)blockIdx.y * g.strideA;
  const float* B = g.B + (int64_t)blockIdx.y * g.strideB;
  float* C = g.C + (int64_t)blockIdx.y * g.strideC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(smem_u32(&bars[s]), CV_THREADS);         // full: every converter thread
      mbar_init(smem_u32(&bars[NSTAGE + s]), 1);         // empty: tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars[2 * NSTAGE + b]), 1);     // accfull[b]: tcgen05.commit
      mbar_init(smem_u32(&bars[2 * NSTAGE + 2 + b]), 8); // accempty[b]: every warp
    }
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t base = smem_u32(smem);
  auto accfull = [&](int b) { return smem_u32(&bars[2 * NSTAGE + b]); };
  auto accempty = [&](int b) { return smem_u32(&bars[2 * NSTAGE + 2 + b]); };

  // Thread 0 also issues the MMAs of a chunk once every thread has stored
  // its part (the instructions run asynchronously; issuing takes little).
  // Accumulation in segments of SEG chunks: the MMAs of segment sg go to
  // TMEM accumulator sg & 1, and every warp adds each finished segment into
  // float32 registers with round-to-nearest (one accumulator over a long K
  // drifts by ~1e-5 relative per 2k of K).
  auto issue = [&](int s) -> bool {
    const int st = s & 1, use = s >> 1;
    const int sg = s / SEG, b = sg & 1;
    const bool first = (s % SEG) == 0;
    // the accumulator is free once the warps have added segment sg - 2
    if (first && sg >= 2 && !mbar_wait(accempty(b), (uint32_t)((sg >> 1) - 1) & 1u)) return false;
    if (!mbar_wait(smem_u32(&bars[st]), use & 1)) return false;
    tc_fence_after();
    const uint32_t acc = tmem + (uint32_t)(b * BN);
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, false, true);
    const uint32_t sa = base + st * STAGE, sb = sa + 3 * A_SPLIT;
#pragma unroll
    for (int kk = 0; kk < BK / 16; ++kk) {
#pragma unroll
      for (int t = 0; t < 6; ++t) {
        // split pairs (a, b) with a + b <= 2: hh, hm, mh, hl, lh, mm
        const int pa = (t == 2 || t == 5) ? 1 : (t == 4 ? 2 : 0);
        const int pb = (t == 1 || t == 5) ? 1 : (t == 3 ? 2 : 0);
        const uint64_t da = smem_desc_sw128(sa + pa * A_SPLIT + kk * 32, 16, 1024);
        const uint64_t db = smem_desc_sw128(sb + pb * B_SPLIT + kk * 2048, B_BOX, 1024);
        mma_bf16(acc, da, db, idesc, (!first || kk > 0 || t > 0) ? 1u : 0u);
      }
    }
    mma_commit(smem_u32(&bars[NSTAGE + st]));
    if (s % SEG == SEG - 1 || s == nchunks - 1) mma_commit(accfull(b));
    return true;
  };

  // Warp w owns TMEM lanes 32 (w % 4) .. +31 and columns 64 (w / 4) .. +63.
  const int q = warp & 3, hc = warp >> 2;
  float sum[64];
#pragma unroll
  for (int e = 0; e < 64; ++e) sum[e] = 0.f;
  auto drain = [&](int sgi) -> bool {
    const int b = sgi & 1;
    int got = 1;
    if (lane == 0) got = mbar_wait(accfull(b), (uint32_t)(sgi >> 1) & 1u) ? 1 : 0;
    got = __shfl_sync(0xffffffffu, got, 0);
    __syncwarp();
    if (!got) return false;
    tc_fence_after();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t v[32];
      __syncwarp();  // the TMEM load is warp-collective
      tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + (uint32_t)(b * BN + 64 * hc + 32 * h), v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) sum[32 * h + e] = __fadd_rn(sum[32 * h + e], __uint_as_float(v[e]));
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(accempty(b));
    return true;
  };
  const int nseg = (nchunks + SEG - 1) / SEG;

  {
    bool ok = true;
    Chunk c0, c1;
    if (nchunks > 0) load_chunk(g, A, B, m0, n0, kbeg, warp, lane, c0);
    for (int s = 0; s < nchunks && ok; s += 2) {
      // chunk s from c0 (prefetch s + 1 into c1), then chunk s + 1 from c1
      if (s + 1 < nchunks) load_chunk(g, A, B, m0, n0, kbeg + (s + 1) * BK, warp, lane, c1);
      {
        const int st = s & 1, use = s >> 1;
        if (use > 0) ok = mbar_wait(smem_u32(&bars[NSTAGE + st]), (use - 1) & 1);
        if (!ok) break;
        store_chunk(smem + st * STAGE, warp, lane, c0);
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&bars[st]));
        if (threadIdx.x == 0) ok = issue(s);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        // the last chunk of segment sg is stored: add segment sg - 1
        if ((s % SEG == SEG - 1 || s == nchunks - 1) && s / SEG >= 1) ok = drain(s / SEG - 1);
        if (!ok) break;
      }
      if (s + 1 >= nchunks) break;
      if (s + 2 < nchunks) load_chunk(g, A, B, m0, n0, kbeg + (s + 2) * BK, warp, lane, c0);
      {
        const int st = (s + 1) & 1, use = (s + 1) >> 1;
        if (use > 0) ok = mbar_wait(smem_u32(&bars[NSTAGE + st]), (use - 1) & 1);
        if (!ok) break;
        store_chunk(smem + st * STAGE, warp, lane, c1);
        fence_proxy_async_smem();
        mbar_arrive(smem_u32(&bars[st]));
        if (threadIdx.x == 0) ok = issue(s + 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
        if (((s + 1) % SEG == SEG - 1 || s + 1 == nchunks - 1) && (s + 1) / SEG >= 1) ok = drain((s + 1) / SEG - 1);
        if (!ok) break;
      }
    }
    // the last segment (every MMA of the tile has completed after it)
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nseg > 0) ok = __all_sync(0xffffffffu, drain(nseg - 1));
    const int r = 32 * q + lane;
    float* cst = reinterpret_cast<float*>(smem);
    if (ok) {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float* dst = cst + r * C_LD + 64 * hc + 32 * cc;
#pragma unroll
        for (int t = 0; t < 32; t += 4)
          *reinterpret_cast<float4*>(dst + t) =
              make_float4(g.alpha * sum[32 * cc + t], g.alpha * sum[32 * cc + t + 1],
                          g.alpha * sum[32 * cc + t + 2], g.alpha * sum[32 * cc + t + 3]);
      }
    }
    named_barrier(1, CV_THREADS);
    if (ok) {
      // rows warp, warp + 8, ...: lane covers columns 4 lane .. +3
      const int col = n0 + 4 * lane;
      const int valid = g.N - col;
#pragma unroll 4
      for (int rr = warp; rr < BM; rr += 8) {
        const int row = m0 + rr;
        if (row >= g.M || valid <= 0) continue;
        const float4 x = *reinterpret_cast<const float4*>(cst + rr * C_LD + 4 * lane);
        float* out = C + (int64_t)row * g.ldc + col;
        if (valid >= 4 && g.vecC) {
          *reinterpret_cast<float4*>(out) = x;
        } else {
          out[0] = x.x;
          if (valid > 1) out[1] = x.y;
          if (valid > 2) out[2] = x.z;
          if (valid > 3) out[3] = x.w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// TMA variant (16-byte aligned rows and origins): the fp32 operand tiles
// arrive by TMA in a three-deep ring of 32-deep chunks; eight warps convert
// each chunk into the bf16 splits (both operands MN-major, 128-byte
// swizzle) in a two-deep ring; warp 8 lane 0 issues the TMA loads, warp 9
// lane 0 the 12 MMAs per chunk.
constexpr int TBK = 32;
constexpr int TF_A = BM * TBK * 4;                // 16 KB: fp32 A box, 32 k x 128 m
constexpr int TF_BBOX = TBK * 32 * 4;             // 4 KB: fp32 B box, 32 n x 32 k
constexpr int TF_STAGE = TF_A + (BN / 32) * TF_BBOX;  // 32 KB
constexpr int TNF = 3;
constexpr int TS_BOX = 64 * TBK * 2;              // 4 KB: 64 m (or n) x 32 k, MN-major
constexpr int TS_SPLIT = 2 * TS_BOX;              // 8 KB
constexpr int TS_STAGE = 6 * TS_SPLIT;            // 48 KB: A hi/mid/lo, B hi/mid/lo
constexpr int TNS = 2;
constexpr int T_THREADS = CV_THREADS + 64;        // + producer warp + MMA warp
constexpr int T_SEG = 4;                          // 32-deep chunks per accumulation segment
constexpr uint32_t T_TMEM_COLS = 2 * BN;          // two segment accumulators
constexpr int T_SMEM = TNF * TF_STAGE + TNS * TS_STAGE + 1024 + 256;
static_assert(BM * C_LD * 4 <= TNF * TF_STAGE + TNS * TS_STAGE, "C staging fits");

struct TriTma {
  int ax0, ay0, adx, ady;   // map coordinates of A(0, 0) of batch 0, and the batch step
  int bx0, by0, bdx, bdy;   // the same for B(0, 0)
};

// MN-major 128-byte-swizzled offset of (mn, k) in one split (64-wide boxes).
__device__ __forceinline__ uint32_t mn_off(int mn, int k) {
  return (uint32_t)((mn >> 6) * TS_BOX + (k >> 3) * 1024 + (k & 7) * 128 +
                    ((((mn & 63) >> 3) ^ (k & 7)) << 4) + (mn & 7) * 2);
}

__global__ void __launch_bounds__(T_THREADS, 1)
    trigemm_tma_kernel(const __grid_constant__ CUtensorMap mapA,
                       const __grid_constant__ CUtensorMap mapB, TriArgs g, TriTma tt) {
  if (g.info && *g.info != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* fst = smem;                              // fp32 ring
  uint8_t* bst = smem + TNF * TF_STAGE;             // bf16 ring
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + TNF * TF_STAGE + TNS * TS_STAGE);
  // ffull[3] fempty[3] bfull[2] bempty[2] accfull[2] accempty[2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * TNF + 2 * TNS + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto ffull = [&](int i) { return smem_u32(&bars[i]); };
  auto fempty = [&](int i) { return smem_u32(&bars[TNF + i]); };
  auto bfull = [&](int i) { return smem_u32(&bars[2 * TNF + i]); };
  auto bempty = [&](int i) { return smem_u32(&bars[2 * TNF + TNS + i]); };
  auto accfull = [&](int i) { return smem_u32(&bars[2 * TNF + 2 * TNS + i]); };
  auto accempty = [&](int i) { return smem_u32(&bars[2 * TNF + 2 * TNS + 2 + i]); };

  const int bid = blockIdx.x;
  int tm, tn;
  if (g.b_upper) {
    tn = g.tiles_n - 1 - bid / g.tiles_m;
    tm = bid % g.tiles_m;
  } else {
    tm = bid / g.tiles_n;
    tn = bid % g.tiles_n;
  }
  const int m0 = tm * BM, n0 = tn * BN;
  const int kbeg = g.a_upper ? m0 : 0;
  int kend = g.K;
  if (g.b_upper && n0 + BN < kend) kend = n0 + BN;
  const int nchunks = kend > kbeg ? (kend - kbeg + TBK - 1) / TBK : 0;
  const int pair = blockIdx.y;
  float* C = g.C + (int64_t)pair * g.strideC;

  if (threadIdx.x == 0) {
    for (int i = 0; i < TNF; ++i) {
      mbar_init(ffull(i), 1);
      mbar_init(fempty(i), 8);
    }
    for (int i = 0; i < TNS; ++i) {
      mbar_init(bfull(i), 8);
      mbar_init(bempty(i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(accfull(i), 1);
      mbar_init(accempty(i), 8);
    }
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(smem_u32(tmem_slot), T_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nseg = (nchunks + T_SEG - 1) / T_SEG;

  if (warp < 8) {
    bool ok = true;
    // Accumulation in segments of T_SEG chunks (128 k): the MMAs of a
    // segment go to one of two TMEM accumulators, and these warps add each
    // finished segment into float32 registers with round-to-nearest (a
    // single accumulator over a long K drifts by ~1e-5 relative per 2k of
    // K).  Warp w owns TMEM lanes 32 (w % 4) and columns 64 (w / 4) .. +63.
    const int q = warp & 3, hc = warp >> 2;
    float acc[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) acc[e] = 0.f;
    auto drain = [&](int sgi) -> bool {
      const int b = sgi & 1;
      int got = 1;
      if (lane == 0) got = mbar_wait(accfull(b), (uint32_t)(sgi >> 1) & 1u) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      __syncwarp();
      if (!got) return false;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[32];
        __syncwarp();  // the TMEM load is warp-collective
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + (uint32_t)(b * BN + 64 * hc + 32 * h), v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) acc[32 * h + e] = __fadd_rn(acc[32 * h + e], __uint_as_float(v[e]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty(b));
      return true;
    };
    for (int s = 0; s < nchunks; ++s) {
      const int fs = s % TNF, fu = s / TNF, bs = s & 1, bu = s >> 1;
      const int kc = kbeg + s * TBK;
      if (!mbar_wait(ffull(fs), fu & 1)) { ok = false; break; }
      const uint8_t* F = fst + fs * TF_STAGE;
      // A: m groups 4 (4 warp + t), k = lane
      float av[4][4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i)
          av[t][i] = *reinterpret_cast<const float*>(F + sw128_f32(16 * warp + 4 * t + i, lane));
      // B: k rows warp + 8 t, n = 4 lane .. +3
      float4 bv[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int k = warp + 8 * t, nn = 4 * lane;
        bv[t] = *reinterpret_cast<const float4*>(F + TF_A + (nn >> 5) * TF_BBOX + sw128_f32(k, nn & 31));
      }
      if (bu > 0 && !mbar_wait(bempty(bs), (bu - 1) & 1)) { ok = false; break; }
      uint8_t* Sb = bst + bs * TS_STAGE;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int mm = 16 * warp + 4 * t;           // tile-local m of av[t][0]
        const int k = kc + lane;                     // global k
        float4 v = make_float4(av[t][0], av[t][1], av[t][2], av[t][3]);
        const int row = m0 + mm;
        const bool kin = k < g.K;
        if (!(kin && row + 0 < g.M && (!g.a_upper || k >= row + 0))) v.x = 0.f;
        if (!(kin && row + 1 < g.M && (!g.a_upper || k >= row + 1))) v.y = 0.f;
        if (!(kin && row + 2 < g.M && (!g.a_upper || k >= row + 2))) v.z = 0.f;
        if (!(kin && row + 3 < g.M && (!g.a_upper || k >= row + 3))) v.w = 0.f;
        split_store4(Sb, mn_off(mm, lane), TS_SPLIT, v);
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int kl = warp + 8 * t, nn = 4 * lane;
        const int k = kc + kl, col = n0 + nn;
        float4 v = bv[t];
        const bool kin = k < g.K;
        if (!(kin && col + 0 < g.N && (!g.b_upper || k <= col + 0))) v.x = 0.f;
        if (!(kin && col + 1 < g.N && (!g.b_upper || k <= col + 1))) v.y = 0.f;
        if (!(kin && col + 2 < g.N && (!g.b_upper || k <= col + 2))) v.z = 0.f;
        if (!(kin && col + 3 < g.N && (!g.b_upper || k <= col + 3))) v.w = 0.f;
        split_store4(Sb + 3 * TS_SPLIT, mn_off(nn, kl), TS_SPLIT, v);
      }
      // The fp32 stage is released only now: its values were consumed by the
      // splits above, and the fence orders these generic reads before the
      // TMA (async-proxy) write of the chunk that refills the stage.  An
      // arrive right after the loads let that write overtake loads still in
      // flight, so that a few percent of calls used a later chunk's values.
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(fempty(fs));
        mbar_arrive(bfull(bs));
      }
      // the last chunk of segment sg is converted: the segment before it is
      // (or soon will be) complete in its accumulator
      const int sg = s / T_SEG;
      if ((s % T_SEG == T_SEG - 1 || s == nchunks - 1) && sg >= 1 && !drain(sg - 1)) { ok = false; break; }
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nseg > 0) ok = __all_sync(0xffffffffu, drain(nseg - 1));
    // epilogue (as in the generic kernel), from the register sums
    const int r = 32 * q + lane;
    float* cst = reinterpret_cast<float*>(smem);
    if (ok) {
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t v[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = __float_as_uint(acc[32 * cc + t]);
        float* dst = cst + r * C_LD + 64 * hc + 32 * cc;
#pragma unroll
        for (int t = 0; t < 32; t += 4)
          *reinterpret_cast<float4*>(dst + t) =
              make_float4(g.alpha * __uint_as_float(v[t]), g.alpha * __uint_as_float(v[t + 1]),
                          g.alpha * __uint_as_float(v[t + 2]), g.alpha * __uint_as_float(v[t + 3]));
      }
    }
    named_barrier(1, CV_THREADS);
    if (ok) {
      const int col = n0 + 4 * lane;
      const int valid = g.N - col;
#pragma unroll 4
      for (int rr = warp; rr < BM; rr += 8) {
        const int row = m0 + rr;
        if (row >= g.M || valid <= 0) continue;
        const float4 x = *reinterpret_cast<const float4*>(cst + rr * C_LD + 4 * lane);
        float* out = C + (int64_t)row * g.ldc + col;
        if (valid >= 4 && g.vecC) {
          *reinterpret_cast<float4*>(out) = x;
        } else {
          out[0] = x.x;
          if (valid > 1) out[1] = x.y;
          if (valid > 2) out[2] = x.z;
          if (valid > 3) out[3] = x.w;
        }
      }
    }
  } else if (warp == 8) {
    if (lane == 0) {
      const int ax = tt.ax0 + pair * tt.adx, ay = tt.ay0 + pair * tt.ady;
      const int bx = tt.bx0 + pair * tt.bdx, by = tt.by0 + pair * tt.bdy;
      for (int s = 0; s < nchunks; ++s) {
        const int fs = s % TNF, fu = s / TNF;
        if (fu > 0 && !mbar_wait(fempty(fs), (fu - 1) & 1)) break;
        const int kc = kbeg + s * TBK;
        const uint32_t F = smem_u32(fst + fs * TF_STAGE);
        mbar_arrive_expect_tx(ffull(fs), TF_STAGE);
        tma_load_2d(F, &mapA, ffull(fs), ax + kc, ay + m0);
#pragma unroll
        for (int j = 0; j < BN / 32; ++j)
          tma_load_2d(F + TF_A + j * TF_BBOX, &mapB, ffull(fs), bx + n0 + 32 * j, by + kc);
      }
    }
    __syncwarp();
  } else {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, true, true);
      for (int s = 0; s < nchunks; ++s) {
        const int bs = s & 1, bu = s >> 1;
        const int sg = s / T_SEG, b = sg & 1;
        const bool first = (s % T_SEG) == 0;
        // a segment's accumulator is free once the converter warps have
        // added the segment two back into their registers
        if (first && sg >= 2 && !mbar_wait(accempty(b), (uint32_t)((sg >> 1) - 1) & 1u)) break;
        if (!mbar_wait(bfull(bs), bu & 1)) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(bst + bs * TS_STAGE), sb = sa + 3 * TS_SPLIT;
        const uint32_t acc = tmem + (uint32_t)(b * BN);
#pragma unroll
        for (int kk = 0; kk < TBK / 16; ++kk) {
#pragma unroll
          for (int t = 0; t < 6; ++t) {
            // split pairs (a, b) with a + b <= 2: hh, hm, mh, hl, lh, mm
            const int pa = (t == 2 || t == 5) ? 1 : (t == 4 ? 2 : 0);
            const int pb = (t == 1 || t == 5) ? 1 : (t == 3 ? 2 : 0);
            const uint64_t da = smem_desc_sw128(sa + pa * TS_SPLIT + kk * 2048, TS_BOX, 1024);
            const uint64_t db = smem_desc_sw128(sb + pb * TS_SPLIT + kk * 2048, TS_BOX, 1024);
            mma_bf16(acc, da, db, idesc, (!first || kk > 0 || t > 0) ? 1u : 0u);
          }
        }
        mma_commit(bempty(bs));
        if (s % T_SEG == T_SEG - 1 || s == nchunks - 1) mma_commit(accfull(b));
      }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, T_TMEM_COLS);
  }
}

}  // namespace

cudaError_t status_fetch_trigemm(int* out, cudaStream_t s) {
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

kronq_status trigemm_tc(const TriGemm& t, cudaStream_t s) {
  if (t.M <= 0 || t.N <= 0) return KRONQ_OK;
  if (t.a_upper == t.b_upper) return fail(KRONQ_ERR_INVALID_ARG, "trigemm_tc: exactly one triangular operand");
  if (t.M > (int64_t)1 << 30 || t.N > (int64_t)1 << 30 || t.K > (int64_t)1 << 30)
    return fail(KRONQ_ERR_INVALID_ARG, "trigemm_tc: size out of range");
  TriArgs g;
  g.A = t.A; g.B = t.B; g.C = t.C;
  g.lda = t.lda; g.ldb = t.ldb; g.ldc = t.ldc;
  g.strideA = t.strideA; g.strideB = t.strideB; g.strideC = t.strideC;
  g.M = (int)t.M; g.N = (int)t.N; g.K = (int)t.K;
  g.alpha = t.alpha;
  g.a_upper = t.a_upper ? 1 : 0;
  g.b_upper = t.b_upper ? 1 : 0;
  g.tiles_m = (int)ceil_div(t.M, BM);
  g.tiles_n = (int)ceil_div(t.N, BN);
  auto vec_ok = [&](const float* p, int64_t ld, int64_t stride) {
    return aligned(p, 16) && (ld % 4) == 0 && (t.batch <= 1 || (stride % 4) == 0);
  };
  g.vecA = vec_ok(t.A, t.lda, t.strideA) ? 1 : 0;
  g.vecB = vec_ok(t.B, t.ldb, t.strideB) ? 1 : 0;
  g.vecC = vec_ok(t.C, t.ldc, t.strideC) ? 1 : 0;
  g.info = t.info;
  dim3 grid((unsigned)(g.tiles_m * g.tiles_n), (unsigned)t.batch);
  // TMA path: 16-byte row strides and origins, x coordinates on 4 floats.
  TriTma tt;
  CUtensorMap mA, mB;
  auto origin = [](const float* hold, int64_t ld, const float* p, int64_t stride, int& x0, int& y0,
                   int& dx, int& dy) {
    const int64_t off = p - hold;
    if (off < 0 || ld <= 0) return false;
    x0 = (int)(off % ld);
    y0 = (int)(off / ld);
    dx = (int)(stride % ld);
    dy = (int)(stride / ld);
    return (x0 % 4) == 0 && (dx % 4) == 0 && stride >= 0;
  };
  bool use_tma = t.holdA && t.holdB && (t.lda % 4) == 0 && (t.ldb % 4) == 0 &&
                 aligned(t.holdA, 16) && aligned(t.holdB, 16) &&
                 origin(t.holdA, t.lda, t.A, t.batch > 1 ? t.strideA : 0, tt.ax0, tt.ay0, tt.adx, tt.ady) &&
                 origin(t.holdB, t.ldb, t.B, t.batch > 1 ? t.strideB : 0, tt.bx0, tt.by0, tt.bdx, tt.bdy);
  if (use_tma) {
    use_tma = tma_map_2d(&mA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, t.holdA, t.holdA_cols, t.holdA_rows,
                         t.lda, 32, BM) &&
              tma_map_2d(&mB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, t.holdB, t.holdB_cols, t.holdB_rows,
                         t.ldb, 32, TBK);
  }
  if (use_tma) {
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(&trigemm_tma_kernel), T_SMEM);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(trigemm tma)");
    trigemm_tma_kernel<<<grid, T_THREADS, T_SMEM, s>>>(mA, mB, g, tt);
    KQ_LAUNCH_CHECK("trigemm_tma_kernel");
    return KRONQ_OK;
  }
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(&trigemm_tc_kernel), SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(trigemm)");
  trigemm_tc_kernel<<<grid, THREADS, SMEM_BYTES, s>>>(g);
  KQ_LAUNCH_CHECK("trigemm_tc_kernel");
  return KRONQ_OK;
}

}  // namespace kq

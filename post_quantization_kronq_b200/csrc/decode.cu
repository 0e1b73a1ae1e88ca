// Deploy-path matvec from packed codes: y = D_o^-1 U^T Q V D_i^-1 x.
//
// KronQ README intro: quantized weights are stored packed int4/int2 and a
// fused dequant + BiIP matvec unpacks them on the fly for single-token
// decode.  Q[i, j] = scale[i, g(j)] (q[i, j] - zero[i, g(j)]) with q from the
// uint32 words of kronq_pack (least significant bits first, along n).
//
// Three steps on the stream: x' = V D_i^-1 x (the BiIP row transform on a
// one-row matrix), y' = Q x' (below), y = D_o^-1 U^T y' (the inverse row
// transform).  The matvec reads each packed word once: a warp per row, a lane
// per word, x' staged in shared memory once per CTA; per word the group's
// scale and zero enter as scale (sum q x - zero sum x).  HBM-bound on the
// words: m n b / 8 bytes.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

constexpr int MV_THREADS = 256;

template <int BITS>
__global__ void __launch_bounds__(MV_THREADS)
    dequant_matvec_kernel(const uint32_t* P, const float* sc, const float* zp, int64_t m, int64_t n,
                          int64_t ngroups, int group, const float* xr, float* yr) {
  constexpr int PER = 32 / BITS;
  constexpr uint32_t MASK = (1u << BITS) - 1u;
  extern __shared__ float xs[];
  const int64_t wpr = (n * BITS + 31) / 32;
  for (int64_t j = threadIdx.x; j < wpr * PER; j += blockDim.x) xs[j] = (j < n) ? xr[j] : 0.f;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int WPC = MV_THREADS / 32;
  for (int64_t r = (int64_t)blockIdx.x * WPC + warp; r < m; r += (int64_t)gridDim.x * WPC) {
    const uint32_t* pw = P + r * wpr;
    const float* scr = sc + r * ngroups;
    const float* zpr = zp + r * ngroups;
    float acc = 0.f;
    for (int64_t w = lane; w < wpr; w += 32) {
      const uint32_t word = pw[w];
      const int64_t j0 = w * PER;
      const float* xv = xs + j0;
      const int64_t g0 = (group < 0) ? 0 : j0 / group;
      const int64_t g1 = (group < 0) ? 0 : (j0 + PER - 1) / group;
      if (g0 == g1) {
        float dot = 0.f, sx = 0.f;
#pragma unroll
        for (int c = 0; c < PER; ++c) {
          const float xc = xv[c];
          dot = fmaf((float)((word >> (BITS * c)) & MASK), xc, dot);
          sx += xc;
        }
        acc = fmaf(scr[g0], dot - zpr[g0] * sx, acc);
      } else {
        // the word straddles a group boundary (groups smaller than a word,
        // or the ragged end of a row)
        for (int c = 0; c < PER; ++c) {
          const int64_t j = j0 + c;
          if (j >= n) break;
          const int64_t g = j / group;
          acc = fmaf(scr[g] * ((float)((word >> (BITS * c)) & MASK) - zpr[g]), xv[c], acc);
        }
      }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) yr[r] = acc;
  }
}

int64_t odd_of(int64_t n) {
  while (n > 0 && (n % 2) == 0) n /= 2;
  return n;
}

}  // namespace
}  // namespace kq

using namespace kq;

extern "C" {

size_t kronq_decode_matvec_workspace_bytes(int64_t m, int64_t n) {
  if (m <= 0 || n <= 0) return 0;
  return (size_t)(((n * 4 + 255) / 256) * 256 + ((m * 4 + 255) / 256) * 256);
}

kronq_status kronq_decode_matvec(const uint32_t* packed, const float* scales, const float* zeros,
                                 int64_t m, int64_t n, int bits, int group, uint64_t seed,
                                 kronq_biip_mode mode, const float* d_in, const float* d_out,
                                 const void* x, kronq_dtype xdt, float* y, void* workspace,
                                 size_t ws_bytes, kronq_stream_t s) {
  if (!packed || !scales || !zeros || !d_in || !d_out || !x || !y)
    return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: NULL pointer");
  if (m <= 0 || n <= 0 || n > (1 << 24) || m > (1 << 24))
    return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: sizes out of range");
  if (bits != 2 && bits != 4) return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: bits must be 2 or 4");
  if (!(group == -1 || group > 0)) return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: group must be -1 or > 0");
  if (xdt != KRONQ_BF16 && xdt != KRONQ_F32) return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: bad dtype");
  if (mode < KRONQ_BIIP_FULL || mode > KRONQ_BIIP_SV_ONLY)
    return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: bad mode");
  const bool use_in = mode != KRONQ_BIIP_SU_ONLY;
  const bool use_out = mode != KRONQ_BIIP_SV_ONLY;
  if ((use_in && odd_of(n) > 255) || (use_out && odd_of(m) > 255))
    return fail(KRONQ_ERR_UNSUPPORTED, "decode_matvec: odd factor of a rotated dimension exceeds 255");
  if (!workspace || ws_bytes < kronq_decode_matvec_workspace_bytes(m, n) || !aligned(workspace, 256))
    return fail(KRONQ_ERR_INVALID_ARG, "decode_matvec: workspace too small or not 256-byte aligned");
  const int per = 32 / bits;
  const int64_t wpr = (n * bits + 31) / 32;
  const size_t xs_bytes = (size_t)(wpr * per) * sizeof(float);
  if (xs_bytes > 200 * 1024) return fail(KRONQ_ERR_UNSUPPORTED, "decode_matvec: row too long");
  cudaStream_t st = as_stream(s);
  float* xr = static_cast<float*>(workspace);
  float* yr = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ((n * 4 + 255) / 256) * 256);
  // x' = V D_i^-1 x: the input-side row transform of a one-row matrix
  RowPass p1;
  p1.in = x; p1.in_bf16 = xdt == KRONQ_BF16; p1.ld_in = n;
  p1.out = xr; p1.ld_out = 1; p1.rows = 1; p1.L = n;
  p1.scale = d_in; p1.scale_mode = 2; p1.rotate = use_in; p1.inverse = false;
  p1.sign_state = 2ull * seed;
  kronq_status r = rowpass(p1, st);
  if (r != KRONQ_OK) return r;
  // y' = Q x'
  const int64_t ngroups = (group == -1) ? 1 : (n + group - 1) / group;
  const int64_t rows_per_cta = MV_THREADS / 32;
  const int64_t want = ceil_div(m, rows_per_cta);
  const int64_t cap = 4 * (int64_t)sm_count();
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  const void* fn = bits == 2 ? reinterpret_cast<const void*>(&dequant_matvec_kernel<2>)
                             : reinterpret_cast<const void*>(&dequant_matvec_kernel<4>);
  cudaError_t e = allow_smem(fn, (int)xs_bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode matvec)");
  if (bits == 2)
    dequant_matvec_kernel<2><<<grid, MV_THREADS, xs_bytes, st>>>(packed, scales, zeros, m, n, ngroups, group, xr, yr);
  else
    dequant_matvec_kernel<4><<<grid, MV_THREADS, xs_bytes, st>>>(packed, scales, zeros, m, n, ngroups, group, xr, yr);
  KQ_LAUNCH_CHECK("dequant_matvec_kernel");
  // y = D_o^-1 U^T y': the inverse output-side row transform
  RowPass p2;
  p2.in = yr; p2.in_bf16 = false; p2.ld_in = m;
  p2.out = y; p2.ld_out = 1; p2.rows = 1; p2.L = m;
  p2.scale = d_out; p2.scale_mode = 2; p2.rotate = use_out; p2.inverse = true;
  p2.sign_state = 2ull * seed + 1ull;
  return rowpass(p2, st);
}

}  // extern "C"

// Packed int4 / int2 code storage (KronQ README, "Model zoo": W4/W2 stored
// as real packed int4/int2; W3 is not bit-packable).  Layout: per row, along
// n, codes fill uint32 words from the least significant bit up; a ragged
// last word is zero-padded.  Rows of whole 4-word quads: one thread per quad
// with 16-byte loads and stores; otherwise one thread per output word.
#include "common.cuh"
#include "internal.h"

namespace kq {
namespace {

__global__ void pack_kernel(const uint8_t* codes, int64_t m, int64_t n, int bits, int64_t wpr,
                            uint32_t* out) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= m * wpr) return;
  const int64_t r = t / wpr, w = t - r * wpr;
  const int per = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const int64_t c0 = w * per;
  const uint8_t* src = codes + r * n + c0;
  uint32_t word = 0;
  if (c0 + per <= n && ((reinterpret_cast<uintptr_t>(src) & 7) == 0)) {
    if (per == 8) {
      const uint2 x = *reinterpret_cast<const uint2*>(src);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        word |= (((x.x >> (8 * k)) & mask) << (bits * k));
        word |= (((x.y >> (8 * k)) & mask) << (bits * (k + 4)));
      }
    } else {
      const uint2 x0 = *reinterpret_cast<const uint2*>(src);
      const uint2 x1 = *reinterpret_cast<const uint2*>(src + 8);
      const uint32_t xs[4] = {x0.x, x0.y, x1.x, x1.y};
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int k = 0; k < 4; ++k) word |= (((xs[q] >> (8 * k)) & mask) << (bits * (4 * q + k)));
    }
  } else {
    for (int k = 0; k < per; ++k) {
      const int64_t c = c0 + k;
      if (c < n) word |= ((uint32_t)src[k] & mask) << (bits * k);
    }
  }
  out[t] = word;
}

// Four codes of a 32-bit lane (one per byte, each below 2^b) side by side in
// the low 4 b bits: pairs of fields are merged in two shift-or steps.
__device__ __forceinline__ uint32_t squeeze2(uint32_t x) {
  uint32_t v = x & 0x03030303u;
  v = (v | (v >> 6)) & 0x000F000Fu;
  return (v | (v >> 12)) & 0xFFu;
}
__device__ __forceinline__ uint32_t squeeze4(uint32_t x) {
  uint32_t v = x & 0x0F0F0F0Fu;
  v = (v | (v >> 4)) & 0x00FF00FFu;
  return (v | (v >> 8)) & 0xFFFFu;
}

// Rows of a whole number of 4-word quads (n a multiple of 4 x 32 / b), 16-byte
// aligned: one thread per quad, 16-byte loads of the codes (4 at 2 bits, 2 at
// 4 bits) and one 16-byte store, so that every thread keeps 32 - 64 bytes of
// loads in flight.  Quads never straddle rows, so the arrays are read flat.
__global__ void __launch_bounds__(256) pack_quad_kernel(const uint4* codes, int64_t nquad, int bits,
                                                        uint4* out) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= nquad) return;
  uint32_t w[4];
  if (bits == 2) {
    const uint4* src = codes + 4 * t;
    uint4 x[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) x[q] = src[q];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = squeeze2(x[q].x) | (squeeze2(x[q].y) << 8) | (squeeze2(x[q].z) << 16) | (squeeze2(x[q].w) << 24);
  } else {
    const uint4* src = codes + 2 * t;
    const uint4 x0 = src[0], x1 = src[1];
    w[0] = squeeze4(x0.x) | (squeeze4(x0.y) << 16);
    w[1] = squeeze4(x0.z) | (squeeze4(x0.w) << 16);
    w[2] = squeeze4(x1.x) | (squeeze4(x1.y) << 16);
    w[3] = squeeze4(x1.z) | (squeeze4(x1.w) << 16);
  }
  out[t] = make_uint4(w[0], w[1], w[2], w[3]);
}

__global__ void unpack_kernel(const uint32_t* in, int64_t m, int64_t n, int bits, int64_t wpr,
                              uint8_t* codes) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= m * wpr) return;
  const int64_t r = t / wpr, w = t - r * wpr;
  const int per = 32 / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const uint32_t word = in[t];
  const int64_t c0 = w * per;
  uint8_t* dst = codes + r * n + c0;
  for (int k = 0; k < per; ++k)
    if (c0 + k < n) dst[k] = (uint8_t)((word >> (bits * k)) & mask);
}

}  // namespace

kronq_status pack_codes(const uint8_t* codes, int64_t m, int64_t n, int bits, uint32_t* out,
                        cudaStream_t s) {
  const int64_t wpr = ceil_div(n * bits, 32);
  const int64_t tot = m * wpr;
  if (tot == 0) return KRONQ_OK;
  if (n % (4 * (32 / bits)) == 0 && aligned(codes, 16) && aligned(out, 16)) {
    const int64_t nquad = tot / 4;
    pack_quad_kernel<<<(unsigned)ceil_div(nquad, 256), 256, 0, s>>>(reinterpret_cast<const uint4*>(codes), nquad,
                                                                    bits, reinterpret_cast<uint4*>(out));
    KQ_LAUNCH_CHECK("pack_quad_kernel");
    return KRONQ_OK;
  }
  pack_kernel<<<(unsigned)ceil_div(tot, 256), 256, 0, s>>>(codes, m, n, bits, wpr, out);
  KQ_LAUNCH_CHECK("pack_kernel");
  return KRONQ_OK;
}

kronq_status unpack_codes(const uint32_t* in, int64_t m, int64_t n, int bits, uint8_t* codes,
                          cudaStream_t s) {
  const int64_t wpr = ceil_div(n * bits, 32);
  const int64_t tot = m * wpr;
  if (tot == 0) return KRONQ_OK;
  unpack_kernel<<<(unsigned)ceil_div(tot, 256), 256, 0, s>>>(in, m, n, bits, wpr, codes);
  KQ_LAUNCH_CHECK("unpack_kernel");
  return KRONQ_OK;
}

}  // namespace kq

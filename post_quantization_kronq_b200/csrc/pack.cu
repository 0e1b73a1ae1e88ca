// Packed int4 / int2 code storage (KronQ README, "Model zoo": W4/W2 stored
// as real packed int4/int2; W3 is not bit-packable).  Layout: per row, along
// n, codes fill uint32 words from the least significant bit up; a ragged
// last word is zero-padded.  One thread per output word (coalesced words,
// 8- or 16-byte contiguous code runs per thread).
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

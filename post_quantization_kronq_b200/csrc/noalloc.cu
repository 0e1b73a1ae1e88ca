// kronq_quantize_layer_static: the quantize call for callers that cannot
// allocate device memory.
//
// Some callers only hold device pointers handed to them by another runtime:
// a plugin inside a host framework whose memory pool owns all device memory
// and exposes no allocator to plugins, or a foreign-language caller whose
// runtime has no CUDA allocation binding.  Others run on paths where
// cudaMalloc is not allowed because it synchronises the device.  They still
// own their inputs and outputs, but cannot provide the scratch workspace that
// kronq_quantize_layer asks for.  This entry point takes its scratch from a
// file-scope static device array instead, then runs the same code path as
// kronq_quantize_layer.
//
// The array is part of the library's device image: every GPU that loads the
// library holds its kStaticScratchBytes until the process exits.  All calls
// on a device share it and it keeps the last call's contents; nothing in it
// has to start at zero (each call writes every scratch byte before reading
// it), but calls whose executions overlap on the GPU -- on two streams, or
// from two threads -- race on it.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_quant_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_quant_scratch on the current device.  The host-side
// name is only a stand-in for the symbol; the address comes from
// cudaGetSymbolAddress, called once per device with that device current.
kronq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return kq::cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return kq::fail(KRONQ_ERR_UNSUPPORTED, "device index out of range");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_quant_scratch);
    if (e != cudaSuccess || !p) return kq::cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KRONQ_OK;
}

}  // namespace

extern "C" kronq_status kronq_quantize_layer_static(float* Wt, float* HX, int64_t m, int64_t n,
                                                    const kronq_quant_params* p, uint8_t* codes,
                                                    float* scales, float* zeros, float* E, int* info,
                                                    kronq_stream_t s) {
  if (!p) return kq::fail(KRONQ_ERR_INVALID_ARG, "quantize_layer_static: params is NULL");
  if (m <= 0 || n <= 0) return kq::fail(KRONQ_ERR_INVALID_ARG, "quantize_layer_static: non-positive size");
  const size_t need = kronq_quantize_workspace_bytes(m, n, p);
  if (need > kStaticScratchBytes)
    return kq::fail(KRONQ_ERR_INVALID_ARG,
                    "quantize_layer_static: this layer needs " + std::to_string(need) +
                        " bytes of scratch but the static scratch holds " +
                        std::to_string(kStaticScratchBytes) +
                        " bytes (64 MiB); use kronq_quantize_layer with a caller workspace");
  void* scratch = nullptr;
  kronq_status r = scratch_address(&scratch);
  if (r != KRONQ_OK) return r;
  return kronq_quantize_layer(Wt, HX, m, n, p, codes, scales, zeros, E, info, scratch,
                              kStaticScratchBytes, s);
}

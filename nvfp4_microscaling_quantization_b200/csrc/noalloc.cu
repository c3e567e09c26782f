// noalloc.cu -- nvfp4_quantize_noalloc: the quantizer for callers that cannot
// hand the library any device memory of their own beyond the tensors.
//
// nvfp4_quantize needs a small workspace when it computes the tensor amax
// itself.  Some callers have no way to provide one: a plugin slot in an
// inference or training engine that passes only input and output buffers, or
// a process whose framework has reserved all device memory in its own caching
// pool, where a fresh cudaMalloc would fail or block the host until the
// device is idle.  For them this entry point keeps that scratch in a
// fixed-size array of device memory that is part of the library image itself,
// so nothing is allocated at call time.
#include <cstdint>
#include <map>
#include <mutex>

#include <cuda_runtime.h>

#include "launch_config.h"
#include "nvfp4.h"

namespace {

// The scratch every nvfp4_quantize_noalloc call on a device uses.  Each GPU
// that loads the library holds these bytes until the process exits.
constexpr size_t kScratchBytes = 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// In host code g_noalloc_scratch names a host-side stand-in, not device
// memory.  The device address is looked up with the device current, once per
// CUDA context (the first call in a context does it) and kept for later calls
// in that context.  The key is the context's process-unique id, so a context
// created again on the same device (after cudaDeviceReset) looks the address
// up again instead of reusing a stale one; a failed lookup is not kept.
int scratch_for_current_device(void** out) {
  static std::mutex mu;
  static std::map<uint64_t, void*> by_context;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
  uint64_t ctx = nvfp4::current_context_id();
  if (ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    auto it = by_context.find(ctx);
    if (it != by_context.end()) {
      *out = it->second;
      return NVFP4_OK;
    }
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
  // the lookup made the device's context current if it was not yet
  if (ctx == 0) ctx = nvfp4::current_context_id();
  if (ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    by_context[ctx] = p;
  }
  *out = p;
  return NVFP4_OK;
}

}  // namespace

extern "C" {

int nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout,
                           int mode, int rht_group, uint64_t seed, const float* amax_in,
                           uint8_t* codes, uint8_t* scales, float* global_scale, void* stream) {
  if (amax_in) {
    // the tensor amax is supplied: no scratch is touched at all
    return nvfp4_quantize(x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, codes, scales,
                          global_scale, nullptr, 0, stream);
  }
  const size_t need = nvfp4_workspace_bytes(rows, cols, layout, mode, rht_group);
  if (need == 0)  // invalid layout, mode, group or size: let the checks name it, nothing is launched
    return nvfp4_quantize(x, rows, cols, ld, layout, mode, rht_group, seed, nullptr, codes, scales,
                          global_scale, nullptr, 0, stream);
  if (need > kScratchBytes) return NVFP4_ERR_WORKSPACE;  // more than the built-in scratch holds
  void* scratch = nullptr;
  const int st = scratch_for_current_device(&scratch);
  if (st) return st;
  // nvfp4_quantize zeroes the amax word in the scratch on `stream` before the
  // pre-pass, so whatever the previous call left there does not matter.
  return nvfp4_quantize(x, rows, cols, ld, layout, mode, rht_group, seed, nullptr, codes, scales,
                        global_scale, scratch, kScratchBytes, stream);
}

}  // extern "C"

// launch_config.h -- grid sizing of the persistent kernels: how many CTAs of a
// kernel are resident on one SM at once, and a cache of that set-up so that a
// launch after the first does no attribute calls or device queries.
#pragma once

#include <cstdint>
#include <map>
#include <mutex>
#include <tuple>

#include <cuda.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// Sets the largest shared-memory carveout for `kernel` and returns in *per_sm
// the CTAs that fit on one SM by shared memory, registers and threads, capped
// at `cap`.  Counted from the kernel's attributes because the occupancy
// calculator does not apply the carveout preference (it reports fewer CTAs
// than the hardware then runs).
template <typename Kernel>
cudaError_t resident_ctas(Kernel kernel, int threads, size_t dyn_smem, int cap, int* per_sm) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                       cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  int dev = 0, smem_sm = 0, reserved = 0, regs_sm = 0, threads_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev);
  cudaDeviceGetAttribute(&threads_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev);
  const size_t smem_cta = dyn_smem + fa.sharedSizeBytes + static_cast<size_t>(reserved);
  // registers are allocated per warp in units of 256 (8 per thread)
  const int warps = (threads + 31) / 32;
  const int regs_cta = ((fa.numRegs + 7) / 8) * 8 * 32 * warps;
  int n = cap;
  if (smem_cta > 0 && static_cast<size_t>(n) * smem_cta > static_cast<size_t>(smem_sm))
    n = static_cast<int>(static_cast<size_t>(smem_sm) / smem_cta);
  if (regs_cta > 0 && n * regs_cta > regs_sm) n = regs_sm / regs_cta;
  if (n * threads > threads_sm) n = threads_sm / threads;
  *per_sm = n < 1 ? 1 : n;
  return cudaSuccess;
}

// The unique id of the CUDA context current on this thread (cuCtxGetId: ids
// are never reused within a process, so a context created again after
// cudaDeviceReset gets a new one).  0 if it cannot be read.
inline uint64_t current_context_id() {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static const std::pair<GetCurrentFn, GetIdFn> fns = [] {
    void* cur = nullptr;
    void* id = nullptr;
    cudaDriverEntryPointQueryResult q1 = cudaDriverEntryPointSymbolNotFound, q2 = q1;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &cur, 12000, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess)
      cur = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &id, 12000, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      id = nullptr;
    return std::make_pair(reinterpret_cast<GetCurrentFn>(cur), reinterpret_cast<GetIdFn>(id));
  }();
  if (!fns.first || !fns.second) return 0;
  CUcontext ctx = nullptr;
  if (fns.first(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  return fns.second(ctx, &id) == CUDA_SUCCESS ? static_cast<uint64_t>(id) : 0;
}

// Launch geometry of one kernel in the current context.
struct LaunchGeom {
  int sms;     // streaming multiprocessors of the device
  int per_sm;  // CTAs of the kernel resident on one SM at once
};

// The first launch of `kernel` (with this block size, dynamic shared memory
// and cap) in a context sets its dynamic shared-memory limit and carveout,
// counts its resident CTAs and reads the SM count; later launches in the same
// context read the cached result.  The runtime calls made here (attributes,
// device queries) are host-side and allowed during stream capture.
template <typename Kernel>
cudaError_t launch_geometry(Kernel kernel, int threads, size_t dyn_smem, int cap, LaunchGeom* out) {
  using Key = std::tuple<const void*, uint64_t, int, int, size_t, int>;
  static std::mutex mu;
  static std::map<Key, LaunchGeom> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // 0 until a runtime call has made the device's context current on this
  // thread: such a launch sets up without caching
  const uint64_t ctx = current_context_id();
  const Key key{reinterpret_cast<const void*>(kernel), ctx, dev, threads, dyn_smem, cap};
  if (ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *out = it->second;
      return cudaSuccess;
    }
  }
  if (dyn_smem > 0) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(dyn_smem));
    if (e != cudaSuccess) return e;
  }
  LaunchGeom g{148, 1};
  if ((e = resident_ctas(kernel, threads, dyn_smem, cap, &g.per_sm)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&g.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if (ctx != 0) {
    std::lock_guard<std::mutex> lock(mu);
    cache[key] = g;
  }
  *out = g;
  return cudaSuccess;
}

// Launch `kernel` with programmatic stream serialization: it may begin (its
// CTAs scheduled, its prologue run) while the previous kernel on the stream
// finishes; the kernel itself calls grid_dependency_wait() before touching
// global memory.  For the persistent kernels, whose one CTA per SM cannot
// share an SM with the previous kernel's, the overlap is the next kernel's
// prologue (barrier set-up, tensor-memory allocation, the rotation matrix)
// with the previous kernel's last tiles.
template <typename... ExpTypes, typename... ActTypes>
cudaError_t launch_overlapped(void (*kernel)(ExpTypes...), unsigned grid, unsigned threads, size_t smem,
                              cudaStream_t stream, ActTypes&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<ActTypes&&>(args)...);
}

}  // namespace nvfp4

// launch_config.h -- grid sizing of the persistent kernels: how many CTAs of a
// kernel are resident on one SM at once.
#pragma once

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

}  // namespace nvfp4

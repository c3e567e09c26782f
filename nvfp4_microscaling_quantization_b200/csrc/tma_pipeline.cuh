// tma_pipeline.cuh -- the shared-memory pipeline of the sm_100a quantizer:
// TMA tile loads (cp.async.bulk.tensor, no multicast) completing on mbarriers,
// consumer release through a second mbarrier per stage, and bounded waits.
//
// Every wait is bounded: after a few plain polls it sleeps on the barrier in
// slices of at most kSuspendNs nanoseconds (the thread wakes as soon as the
// phase completes) until kWaitLimitNs of wall time (%globaltimer) have passed.
// A wait
// that runs out (which only a broken device or driver could cause) raises the
// CTA's abort flag; the kernel then stops issuing loads, waits (again bounded)
// for the loads it has in flight, reports the failure through a NaN in its
// scalar output and returns, so the context stays usable.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace nvfp4 {

constexpr uint32_t kSuspendNs = 1u << 16;            // ~65 us per sleep
constexpr uint64_t kWaitLimitNs = 2000000000ull;     // 2 s in all

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
      : "memory");
  return done != 0;
}

// Wait for the phase with the given parity to complete; false if it has not
// completed within kWaitLimitNs.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity) {
  const uint64_t start = global_timer_ns();
  do {
    if (mbar_try_wait_sleep(bar, parity)) return true;
  } while (global_timer_ns() - start < kWaitLimitNs);
  return mbar_try_wait(bar, parity);
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
#pragma unroll 1
  for (int i = 0; i < 32; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity);
}

// 2-D tiled TMA load of one box into shared memory; x is the innermost
// coordinate (elements), always a multiple of 64 here (128 bytes).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Programmatic dependent launch.  grid_dependency_wait(): wait until the
// grids this one depends on (the previous kernel on the stream) have
// completed and their memory operations are visible -- called by every thread
// before its first global-memory access, so a kernel launched early never
// reads an input its predecessor is still writing or overwrites an output it
// is still reading; it returns at once for a launch without that dependency.
// allow_dependent_launch(): this CTA lets the next kernel on the stream begin
// launching (its CTAs then take SMs as this grid's CTAs exit and run their
// prologue, before their own grid_dependency_wait).
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependent_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Byte offset of a 16-byte chunk inside a tile written with the 128-byte
// swizzle: within each 1024-byte atom the chunk index (bits 4..6) is XORed
// with the 128-byte row index (bits 7..9).  Tiles start 1024-byte aligned.
__device__ __forceinline__ uint32_t swizzle128(uint32_t offset) {
  return offset ^ ((offset >> 3) & 0x70u);
}

}  // namespace nvfp4

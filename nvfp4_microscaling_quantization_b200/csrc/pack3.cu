// pack3.cu -- packed storage of the 3-bit formats (NVFP3, NVINT3, IF3, MXFP3).
//
// The quantizer holds a 3-bit code in a nibble (sign bit 3, magnitude code in
// bits 0..1, bit 2 always clear).  The packed layout keeps 3 bits per element:
// the 16 codes of a block in 6 bytes, element i in bits 3i .. 3i+2 of the
// block's 48-bit little-endian field (bit 3i+2 = sign, bits 3i .. 3i+1 =
// magnitude code).  NVFP3, NVINT3 and IF3 keep their E4M3 scale byte per
// 16 elements (3 + 8/16 = 3.5 bits per value); MXFP3 keeps one UE8M0 byte per
// 32-element group instead of the quantizer's copy in each 16-element half
// (3 + 8/32 = 3.25 bits per value) -- the bits per value of the IF4 paper
// page's 3-bit formats table.  One thread per 16-element block.
#include "kernels.h"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
pack3_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales, int64_t blocks, int mx,
             uint8_t* __restrict__ pcodes, uint8_t* __restrict__ pscales) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t b = int64_t(blockIdx.x) * kThreads + threadIdx.x; b < blocks; b += stride) {
    const uint2 c = *reinterpret_cast<const uint2*>(codes + b * 8);
    uint64_t bits = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t nib = ((i < 8 ? c.x : c.y) >> (4 * (i & 7))) & 15u;
      const uint64_t v3 = (nib & 3u) | ((nib >> 1) & 4u);
      bits |= v3 << (3 * i);
    }
    uint16_t* dst = reinterpret_cast<uint16_t*>(pcodes + b * 6);
    dst[0] = static_cast<uint16_t>(bits);
    dst[1] = static_cast<uint16_t>(bits >> 16);
    dst[2] = static_cast<uint16_t>(bits >> 32);
    if (!mx) pscales[b] = scales[b];
    else if ((b & 1) == 0) pscales[b >> 1] = scales[b];
  }
}

__global__ void __launch_bounds__(kThreads)
unpack3_kernel(const uint8_t* __restrict__ pcodes, const uint8_t* __restrict__ pscales, int64_t blocks, int mx,
               uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t b = int64_t(blockIdx.x) * kThreads + threadIdx.x; b < blocks; b += stride) {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(pcodes + b * 6);
    const uint64_t bits = uint64_t(src[0]) | (uint64_t(src[1]) << 16) | (uint64_t(src[2]) << 32);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t v3 = static_cast<uint32_t>(bits >> (3 * i)) & 7u;
      const uint32_t nib = (v3 & 3u) | ((v3 & 4u) << 1);
      if (i < 8) lo |= nib << (4 * i);
      else hi |= nib << (4 * (i - 8));
    }
    *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(lo, hi);
    scales[b] = mx ? pscales[b >> 1] : pscales[b];
  }
}

int grid_of(int64_t blocks) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (blocks + kThreads - 1) / kThreads;
  return static_cast<int>(need < int64_t(sms) * 8 ? need : int64_t(sms) * 8);
}

}  // namespace

cudaError_t launch_pack3(const uint8_t* codes, const uint8_t* scales, int64_t blocks, int mx, uint8_t* pcodes,
                         uint8_t* pscales, cudaStream_t stream) {
  const int grid = grid_of(blocks);
  if (grid == 0) return cudaSuccess;
  pack3_kernel<<<grid, kThreads, 0, stream>>>(codes, scales, blocks, mx, pcodes, pscales);
  return cudaGetLastError();
}

cudaError_t launch_unpack3(const uint8_t* pcodes, const uint8_t* pscales, int64_t blocks, int mx, uint8_t* codes,
                           uint8_t* scales, cudaStream_t stream) {
  const int grid = grid_of(blocks);
  if (grid == 0) return cudaSuccess;
  unpack3_kernel<<<grid, kThreads, 0, stream>>>(pcodes, pscales, blocks, mx, codes, scales);
  return cudaGetLastError();
}

}  // namespace nvfp4

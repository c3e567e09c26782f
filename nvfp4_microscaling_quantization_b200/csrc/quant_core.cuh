// quant_core.cuh -- the per-thread quantization core shared by the tiled
// kernels: four 16-element blocks of one view row held as two float2[16]
// pairs (block 0 | block 1, block 2 | block 3), quantized and stored.
#pragma once

#include <cstdint>

#include "nvfp4_device.cuh"

namespace nvfp4 {

__device__ __forceinline__ float absmax64(const float2 (&z)[2][16]) {
  float aa, ab, ac, ad;
  absmax_pair(z[0], aa, ab);
  absmax_pair(z[1], ac, ad);
  return fmaxf(max3(aa, ab, ac), ad);
}

// Store the codes and scales of the four blocks of view row `vrow` starting at
// view column `vcol0` (blocks at or beyond vcols are skipped).
__device__ __forceinline__ void store64(const BlockOut (&o)[4], int64_t vrow, int64_t vcol0, int64_t vcols,
                                        uint8_t* codes, uint8_t* scales, bool codes_aligned16, bool scales_aligned4) {
  const int64_t left = (vcols - vcol0) / 16;
  const int nvalid = left < 4 ? static_cast<int>(left) : 4;
  uint8_t* cdst = codes + vrow * (vcols / 2) + vcol0 / 2;
  uint8_t* sdst = scales + vrow * (vcols / 16) + vcol0 / 16;
  if (nvalid == 4 && codes_aligned16) {
    reinterpret_cast<uint4*>(cdst)[0] = make_uint4(o[0].lo, o[0].hi, o[1].lo, o[1].hi);
    reinterpret_cast<uint4*>(cdst)[1] = make_uint4(o[2].lo, o[2].hi, o[3].lo, o[3].hi);
  } else {
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (b < nvalid) reinterpret_cast<uint2*>(cdst)[b] = make_uint2(o[b].lo, o[b].hi);
  }
  if (nvalid == 4 && scales_aligned4) {
    *reinterpret_cast<uint32_t*>(sdst) = (o[0].scale & 0xFFu) | ((o[1].scale & 0xFFu) << 8) |
                                         ((o[2].scale & 0xFFu) << 16) | ((o[3].scale & 0xFFu) << 24);
  } else {
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (b < nvalid) sdst[b] = static_cast<uint8_t>(o[b].scale);
  }
}

// Quantize the four blocks of view row `vrow` starting at view column `vcol0`
// and store their codes and scales (blocks at or beyond vcols are skipped).
template <int MODE, bool TBL = true>
__device__ __forceinline__ void quantize_store64(const float2 (&z)[2][16], const ScaleCtx& sc, PhiloxKey key,
                                                 int64_t vrow, int64_t vcol0, int64_t vcols, uint8_t* codes,
                                                 uint8_t* scales, bool codes_aligned16, bool scales_aligned4) {
  const uint64_t e0 = static_cast<uint64_t>(vrow) * static_cast<uint64_t>(vcols) + static_cast<uint64_t>(vcol0);
  uint32_t kd[4] = {0u, 0u, 0u, 0u};
  if constexpr (MODE == kMSEDEN) block_draws<4>(key, e0 >> 4, kd);
  BlockOut o[4];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const PairRng rng{key, e0 + 32 * p, e0 + 32 * p + 16, kd[2 * p], kd[2 * p + 1]};
    quantize_pair<MODE, TBL>(z[p], sc, rng, o[2 * p], o[2 * p + 1]);
  }
  store64(o, vrow, vcol0, vcols, codes, scales, codes_aligned16, scales_aligned4);
}

}  // namespace nvfp4

// quantize_kernels.cu -- the quantization kernels (row-wise and transposed)
// and the tensor-amax pre-pass, for sm_100a.
//
// Row-wise (blocks of 16 along a row of X): one thread owns one 16-element
// block, loaded with two 16-byte vector loads; a warp covers 512 consecutive
// elements.  With a rotation of g = 32..128 elements, the g/16 lanes holding
// one group exchange values with warp shuffles for the cross-lane butterfly
// stages.
//
// Transposed (blocks of 16 down a column of X, output X^T): a CTA stages a
// 128-row x 64-column tile of X in shared memory with coalesced 16-byte loads
// (row chunks XOR-swizzled so the column reads below are conflict-free), then
// each thread reads 2 adjacent columns x 16 rows (one 16-block of two output
// rows); the 8 threads sharing a column pair sit in consecutive lanes, so the
// rotation's cross-lane stages are shuffles again.  Output rows (columns of X)
// are written as 64-byte code runs and 8-byte scale runs.
//
// The amax pre-pass is the same kernel with AMAX_ONLY set: it rotates, takes
// max |z| and folds it into one float with an atomic max on the bit pattern
// (valid for non-negative floats).
#include "kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void load_block16(const uint16_t* p, float* z) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
  bf16x2_to_f32(a.x, z[0], z[1]);
  bf16x2_to_f32(a.y, z[2], z[3]);
  bf16x2_to_f32(a.z, z[4], z[5]);
  bf16x2_to_f32(a.w, z[6], z[7]);
  bf16x2_to_f32(b.x, z[8], z[9]);
  bf16x2_to_f32(b.y, z[10], z[11]);
  bf16x2_to_f32(b.z, z[12], z[13]);
  bf16x2_to_f32(b.w, z[14], z[15]);
}

// Reduce a non-negative per-thread max over the CTA and fold it into *accum.
__device__ __forceinline__ void cta_amax_fold(float local, unsigned int* accum) {
  __shared__ unsigned int warp_max[kThreads / 32];
  unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(local));
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) warp_max[warp] = bits;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned int m = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) m = max(m, warp_max[w]);
    atomicMax(accum, m);
  }
}

template <int MODE, int G, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads)
rowwise_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
               const float* __restrict__ amax, unsigned int* __restrict__ amax_accum,
               uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ gscale) {
  constexpr uint32_t kLanesPerGroup = G > 16 ? G / 16 : 1;
  const int64_t nb = cols / 16;
  const int64_t total = rows * nb;
  const int64_t total_warps = (total + 31) & ~int64_t(31);  // whole warps iterate together
  const PhiloxKey key = philox_key(seed);
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t lig = lane & (kLanesPerGroup - 1u);
  uint32_t sign_bits = 0;
  if constexpr (G > 0) sign_bits = rht_sign_bits(key, lig);
  float s_g = 1.0f;
  if constexpr (!AMAX_ONLY) {
    s_g = global_scale_of<MODE>(*amax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *gscale = s_g;
  }
  const bool dense = ld == cols;
  float local_max = 0.0f;
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t b = int64_t(blockIdx.x) * kThreads + threadIdx.x; b < total_warps; b += stride) {
    const bool valid = b < total;
    float z[16];
    if (valid) {
      int64_t offset;
      if (dense) {
        offset = b * 16;
      } else {
        const int64_t row = b / nb;
        offset = row * ld + (b - row * nb) * 16;
      }
      load_block16(x + offset, z);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) z[i] = 0.0f;
    }
    if constexpr (G > 0) rht_forward<G>(z, sign_bits, lig);
    if constexpr (AMAX_ONLY) {
      local_max = fmaxf(local_max, block_absmax(z));
    } else {
      if (valid) {
        const BlockRng rng{key, static_cast<uint64_t>(b) * 16u, static_cast<uint64_t>(b)};
        const BlockOut o = quantize_block<MODE>(z, s_g, rng);
        *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(o.lo, o.hi);
        scales[b] = static_cast<uint8_t>(o.scale);
      }
    }
  }
  if constexpr (AMAX_ONLY) cta_amax_fold(local_max, amax_accum);
}

constexpr int kTileRows = 128;  // rows of X per tile (the block dimension of X^T)
constexpr int kTileCols = 64;   // columns of X per tile (output rows)
constexpr int kChunks = kTileCols / 8;  // 16-byte chunks per tile row

template <int MODE, int G, bool AMAX_ONLY>
__global__ void __launch_bounds__(kThreads)
transposed_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld, uint64_t seed,
                  const float* __restrict__ amax, unsigned int* __restrict__ amax_accum,
                  uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ gscale) {
  constexpr uint32_t kLanesPerGroup = G > 16 ? G / 16 : 1;
  __shared__ uint4 tile[kTileRows * kChunks];
  const uint32_t* tile_words = reinterpret_cast<const uint32_t*>(tile);

  const int64_t tiles_r = (rows + kTileRows - 1) / kTileRows;
  const int64_t tiles_c = (cols + kTileCols - 1) / kTileCols;
  const int64_t n_tiles = tiles_r * tiles_c;
  const PhiloxKey key = philox_key(seed);
  const uint32_t tid = threadIdx.x;
  const uint32_t lane = tid & 31u, warp = tid >> 5;
  const uint32_t k = lane & 7u;          // 16-row block inside the tile
  const uint32_t p = warp * 4u + (lane >> 3);  // column pair inside the tile (0..31)
  const uint32_t lig = k & (kLanesPerGroup - 1u);
  uint32_t sign_bits = 0;
  if constexpr (G > 0) sign_bits = rht_sign_bits(key, lig);
  float s_g = 1.0f;
  if constexpr (!AMAX_ONLY) {
    s_g = global_scale_of<MODE>(*amax);
    if (blockIdx.x == 0 && tid == 0) *gscale = s_g;
  }
  const int64_t out_code_pitch = rows / 2;   // bytes per output row (a column of X)
  const int64_t out_scale_pitch = rows / 16;
  float local_max = 0.0f;

  for (int64_t t = blockIdx.x; t < n_tiles; t += gridDim.x) {
    const int64_t tr = t / tiles_c, tc = t - tr * tiles_c;
    const int64_t r0 = tr * kTileRows, c0 = tc * kTileCols;
    // stage the tile: thread -> chunk j of rows (tid/8) + 32 it
    uint4 v[kTileRows * kChunks / kThreads];
#pragma unroll
    for (int it = 0; it < kTileRows * kChunks / kThreads; ++it) {
      const int64_t r = (tid >> 3) + 32 * it, gr = r0 + r, gc = c0 + 8 * (tid & 7u);
      v[it] = (gr < rows && gc < cols) ? __ldg(reinterpret_cast<const uint4*>(x + gr * ld + gc))
                                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < kTileRows * kChunks / kThreads; ++it) {
      const uint32_t r = (tid >> 3) + 32 * it, j = tid & 7u;
      tile[r * kChunks + (j ^ ((r >> 4) & 7u))] = v[it];
    }
    __syncthreads();

    float z0[16], z1[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t r = 16u * k + i;
      const uint32_t w = tile_words[r * (kChunks * 4) + (((p >> 2) ^ k) << 2) + (p & 3u)];
      bf16x2_to_f32(w, z0[i], z1[i]);
    }
    __syncthreads();  // the tile buffer is free for the next iteration

    const int64_t gcol = c0 + 2 * p;        // first of this thread's two columns of X
    const int64_t grow = r0 + 16 * k;       // first row of this thread's block
    const bool valid = gcol < cols && grow < rows;  // cols % 8 == 0: both columns valid together
    if constexpr (G > 0) {
      rht_forward<G>(z0, sign_bits, lig);
      rht_forward<G>(z1, sign_bits, lig);
    }
    if constexpr (AMAX_ONLY) {
      if (valid) local_max = fmaxf(local_max, fmaxf(block_absmax(z0), block_absmax(z1)));
    } else {
      if (valid) {
#pragma unroll
        for (int col = 0; col < 2; ++col) {
          const int64_t orow = gcol + col;  // output row = column of X
          const uint64_t blk = static_cast<uint64_t>(orow * out_scale_pitch + grow / 16);
          const BlockRng rng{key, static_cast<uint64_t>(orow * rows + grow), blk};
          const BlockOut o = quantize_block<MODE>(col == 0 ? z0 : z1, s_g, rng);
          *reinterpret_cast<uint2*>(codes + orow * out_code_pitch + grow / 2) = make_uint2(o.lo, o.hi);
          scales[blk] = static_cast<uint8_t>(o.scale);
        }
      }
    }
  }
  if constexpr (AMAX_ONLY) cta_amax_fold(local_max, amax_accum);
}

template <int MODE, int G, bool AMAX_ONLY>
cudaError_t launch_one(const QuantArgs& a) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const uint16_t* x = static_cast<const uint16_t*>(a.x);
  unsigned int* accum = reinterpret_cast<unsigned int*>(a.amax_accum);
  if (a.layout == 0) {
    const int64_t total = a.rows * (a.cols / 16);
    const int64_t need = (total + kThreads - 1) / kThreads;
    int64_t grid = need < int64_t(sms) * 8 ? need : int64_t(sms) * 8;
    if (grid == 0) {
      if (AMAX_ONLY) return cudaSuccess;
      grid = 1;  // an empty tensor still gets its tensor scale written
    }
    rowwise_kernel<MODE, G, AMAX_ONLY><<<static_cast<unsigned>(grid), kThreads, 0, a.stream>>>(
        x, a.rows, a.cols, a.ld, a.seed, a.amax, accum, a.codes, a.scales, a.gscale);
  } else {
    const int64_t tiles = ((a.rows + kTileRows - 1) / kTileRows) * ((a.cols + kTileCols - 1) / kTileCols);
    int64_t grid = tiles < int64_t(sms) * 8 ? tiles : int64_t(sms) * 8;
    if (grid == 0) {
      if (AMAX_ONLY) return cudaSuccess;
      grid = 1;
    }
    transposed_kernel<MODE, G, AMAX_ONLY><<<static_cast<unsigned>(grid), kThreads, 0, a.stream>>>(
        x, a.rows, a.cols, a.ld, a.seed, a.amax, accum, a.codes, a.scales, a.gscale);
  }
  return cudaGetLastError();
}

template <int MODE, bool AMAX_ONLY>
cudaError_t dispatch_group(const QuantArgs& a) {
  switch (a.rht_group) {
    case 0: return launch_one<MODE, 0, AMAX_ONLY>(a);
    case 16: return launch_one<MODE, 16, AMAX_ONLY>(a);
    case 32: return launch_one<MODE, 32, AMAX_ONLY>(a);
    case 64: return launch_one<MODE, 64, AMAX_ONLY>(a);
    case 128: return launch_one<MODE, 128, AMAX_ONLY>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_amax(const QuantArgs& a) {
  if (mma_path_applies(a)) return launch_amax_mma(a);
  if (tma_path_applies(a)) return launch_amax_tma(a);
  return dispatch_group<kRTN, true>(a);
}

// The tensor scale of an empty MXFP4 / MXFP3 call (they have none: 1).
__global__ void set_one_kernel(float* p) { *p = 1.0f; }

cudaError_t launch_quantize(const QuantArgs& a) {
  if (mma_path_applies(a)) return launch_quantize_mma(a);
  if (tma_path_applies(a)) return launch_quantize_tma(a);
  if (a.mode == kMXFP4 || a.mode == kMXFP3) {
    // MXFP4 groups are the block pairs of the tiled kernels; the one-block
    // kernels do not form them (the C ABI rejects such shapes up front)
    if (a.rows != 0 && a.cols != 0) return cudaErrorNotSupported;
    set_one_kernel<<<1, 1, 0, a.stream>>>(a.gscale);
    return cudaGetLastError();
  }
  switch (a.mode) {
    case kRTN: return dispatch_group<kRTN, false>(a);
    case kSR: return dispatch_group<kSR, false>(a);
    case kMSEDEN: return dispatch_group<kMSEDEN, false>(a);
    case kIF4: return dispatch_group<kIF4, false>(a);
    case k4over6: return dispatch_group<k4over6, false>(a);
    case kScaleSearch: return dispatch_group<kScaleSearch, false>(a);
    case kNVINT4: return dispatch_group<kNVINT4, false>(a);
    case kNVFP3: return dispatch_group<kNVFP3, false>(a);
    case kNVINT3: return dispatch_group<kNVINT3, false>(a);
    case kIF3: return dispatch_group<kIF3, false>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4

// rotate_mma.cu -- quantization with the random Hadamard rotation on the
// sm_100a tensor cores.
//
// The rotation of a g-group is a dense product: for a 128 x 128 tile of X,
// D = A . B with A the tile (bf16) and B[k][n] = sigma_k H_g[n][k] (bf16 +-1,
// block-diagonal when g < 128), accumulated in fp32 in tensor memory; then
// z = RN(c_g * D).  Row-wise tiles are K-major A operands (K = the tile's
// columns), transposed tiles are the same TMA boxes read MN-major (K = the
// tile's rows), so both layouts share one kernel and one load pattern.
//
// Warp roles in a CTA of 10 warps (two CTAs per SM):
//   warps 0-7  epilogue: thread (lane quarter q = warp % 4, half j = warp / 4)
//              owns view row 32q + lane of the tile and its 64 columns
//              64j .. 64j+63 (four 16-element blocks); it loads them from
//              tensor memory, scales by c_g and quantizes (or takes max|z|, or
//              stores z).
//   warp 8     TMA producer: two 64-column boxes of 128 rows per tile into a
//              2-stage shared-memory ring.
//   warp 9     allocates tensor memory (2 accumulators x 128 columns), and one
//              lane issues the 8 MMAs (K = 16 each) of a tile, committing
//              "stage free" and "accumulator full" mbarriers.
// Every wait is bounded (tma_pipeline.cuh); on a failed wait the CTA drains
// what it issued, frees tensor memory and reports NaN in its scalar output.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kernels.h"
#include "nvfp4_device.cuh"
#include "quant_core.cuh"
#include "tcgen05.cuh"
#include "tma_pipeline.cuh"

namespace nvfp4 {

namespace {

constexpr int kEpiWarps = 8;
constexpr int kThreads = (kEpiWarps + 2) * 32;
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kStagesA = 2;                 // A tiles in flight
constexpr int kAccum = 2;                   // accumulators in tensor memory
constexpr int kTile = 128;                  // tile rows and columns of X
constexpr uint32_t kTileBytes = kTile * kTile * 2;
constexpr uint32_t kBoxBytes = kTile * 128;  // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = kAccum * kTile;
constexpr size_t kDynSmem = (kStagesA + 1) * kTileBytes + 1024;

enum Kind { kQuantize = 0, kAmax = 1, kStoreZ = 2 };

struct MmaShared {
  uint64_t full[kStagesA];   // A tile landed (TMA transaction bytes)
  uint64_t sfree[kStagesA];  // MMAs reading the A tile are done (tcgen05.commit)
  uint64_t tfull[kAccum];    // accumulator ready (tcgen05.commit)
  uint64_t tfree[kAccum];    // accumulator read by the epilogue warps
  uint32_t tmem_base;
  uint32_t issued_a;         // bit s: a load went into stage s; bit 8+s: its phase parity
  uint32_t issued_mma;       // bit a: MMAs went into accumulator a; bit 8+a: parity
  int abort_flag;
  unsigned int warp_max[kEpiWarps];
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

// B operand, K-major with the 128-byte swizzle: two 64-wide K halves of 128
// rows (n) x 128 bytes; element (n, k) = sigma_(k mod G) * H_G[n mod G][k mod G]
// inside the diagonal G x G blocks, 0 elsewhere.  bf16 +1 = 0x3F80, -1 = 0xBF80.
template <int G>
__device__ __forceinline__ void build_hadamard_b(uint8_t* bmat, PhiloxKey key, uint32_t tid) {
  const uint4 w = philox_call(key, 0, kTagSigns);
  for (uint32_t c = tid; c < 2048; c += kThreads) {
    const uint32_t half = c >> 10, n = (c >> 3) & 127u, kc = c & 7u;
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t two = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t k = half * 64 + kc * 8 + 2 * i + h;
        uint32_t v = 0;
        if (n / G == k / G) {
          const uint32_t kg = k % G, ng = n % G;
          const uint32_t neg = ((word_of(w, kg >> 5) >> (kg & 31)) ^ __popc(ng & kg)) & 1u;
          v = neg ? 0xBF80u : 0x3F80u;
        }
        two |= v << (16 * h);
      }
      packed[i] = two;
    }
    *reinterpret_cast<uint4*>(bmat + half * kBoxBytes + n * 128 + ((kc ^ (n & 7u)) << 4)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

template <int MODE, int G, int KIND, bool ROWWISE>
__global__ void __launch_bounds__(kThreads, 2)
rotate_mma_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols, uint64_t seed,
                  const float* __restrict__ amax, unsigned int* __restrict__ amax_accum, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ scales, float* __restrict__ gscale, float* __restrict__ zout) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) MmaShared sh;
  uint8_t* a_tiles = align_1024(dyn_smem);
  uint8_t* bmat = a_tiles + kStagesA * kTileBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const int64_t n_ct = (cols + kTile - 1) / kTile;
  const int64_t n_tiles = ((rows + kTile - 1) / kTile) * n_ct;

  if (tid == kProducerWarp * 32) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sfree[s], 1);
    }
    for (int a = 0; a < kAccum; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], kEpiWarps);
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  build_hadamard_b<G>(bmat, key, tid);
  fence_proxy_async_smem();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = sh.tmem_base;
  const int64_t step = gridDim.x;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      prefetch_tensormap(&tmap);
      int k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++k) {
        const int s = k % kStagesA;
        const uint32_t u = k / kStagesA;
        if (k >= kStagesA && !mbar_wait(&sh.sfree[s], (u - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) break;
        const int64_t rt = t / n_ct, ct = t - rt * n_ct;
        const int32_t x = static_cast<int32_t>(ct * kTile), y = static_cast<int32_t>(rt * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kTileBytes);
        uint8_t* dst = a_tiles + s * kTileBytes;
        tma_load_2d(dst, &tmap, x, y, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &tmap, x + 64, y, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kTile, kTile, ROWWISE ? 0u : 1u);
      const uint32_t b_addr = smem_u32(bmat);
      int k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++k) {
        const int s = k % kStagesA, a = k % kAccum;
        const uint32_t us = k / kStagesA, ua = k / kAccum;
        if (!mbar_wait(&sh.full[s], us & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (k >= kAccum && !mbar_wait(&sh.tfree[a], (ua - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(a_tiles + s * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // K-major A: 32 bytes of K per step inside a 64-wide half; MN-major A:
          // two 8-row K groups (2 x 1024 bytes) per step, the two M halves 16 KB apart.
          const uint64_t adesc = ROWWISE ? smem_desc_sw128(a_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024)
                                         : smem_desc_sw128(a_addr + kk * 2048, kBoxBytes, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
          umma_bf16(tmem_base + a * kTile, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sh.sfree[s]);
        umma_commit(&sh.tfull[a]);
        sh.issued_mma = (sh.issued_mma & ~(0x101u << a)) | (1u << a) | ((ua & 1u) << (8 + a));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u, j = warp >> 2;
    ScaleCtx sc{1.0f, 0.0f, 0.0f};
    if constexpr (KIND == kQuantize) {
      sc.s_g = global_scale_of<MODE>(*amax);
      sc.q6 = __fmul_rn(6.0f, sc.s_g);
      sc.q4 = __fmul_rn(4.0f, sc.s_g);
      if (blockIdx.x == 0 && tid == 0) *gscale = sc.s_g;
    }
    const int64_t vcols = ROWWISE ? cols : rows;
    const bool codes_aligned16 = ((vcols / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(codes) % 16) == 0;
    const bool scales_aligned4 = ((vcols / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(scales) % 4) == 0;
    const float2 c2 = f2(RhtConst<G>::c, RhtConst<G>::c);
    float local_max = 0.0f;
    int k = 0;
    for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++k) {
      const int a = k % kAccum;
      if (!mbar_wait(&sh.tfull[a], (k / kAccum) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      const uint32_t taddr = tmem_base + ((32u * q) << 16) + a * kTile + j * 64;
      const int64_t rt = t / n_ct, ct = t - rt * n_ct;
      // view row of this thread and view column of its first element
      const int64_t vrow = (ROWWISE ? rt : ct) * kTile + 32 * q + lane;
      const int64_t vcol0 = (ROWWISE ? ct : rt) * kTile + 64 * j;
      const int64_t vrows = ROWWISE ? rows : cols;

      if constexpr (KIND == kQuantize) {
        // one pair of blocks at a time: load 32 columns, quantize, then the next 32
        const bool valid = vrow < vrows && vcol0 < vcols;
        const uint64_t e0 = static_cast<uint64_t>(vrow) * static_cast<uint64_t>(vcols) + static_cast<uint64_t>(vcol0);
        float u[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        if constexpr (MODE == kMSEDEN) block_uniforms4(key, e0 >> 4, u);
        BlockOut o[4];
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          float v[32];
          tmem_ld32_wait(taddr + 32 * p, v);
          if (p == 1) {
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.tfree[a]);
          }
          float2 zp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) zp[i] = __fmul2_rn(f2(v[i], v[16 + i]), c2);
          const PairRng rng{key, e0 + 32 * p, e0 + 32 * p + 16, u[2 * p], u[2 * p + 1]};
          quantize_pair<MODE>(zp, sc.s_g, sc.q6, sc.q4, rng, o[2 * p], o[2 * p + 1]);
        }
        if (valid) store64(o, vrow, vcol0, vcols, codes, scales, codes_aligned16, scales_aligned4);
        continue;
      }

      float v[64];
      tmem_ld64_wait(taddr, v);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tfree[a]);

      float2 z[2][16];
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int i = 0; i < 16; ++i) z[p][i] = __fmul2_rn(f2(v[32 * p + i], v[32 * p + 16 + i]), c2);

      if constexpr (KIND == kAmax) {
        local_max = fmaxf(local_max, absmax64(z));
      } else if constexpr (KIND == kStoreZ) {
        if (vrow < vrows && vcol0 < vcols) {
          float4* dst = reinterpret_cast<float4*>(zout + vrow * vcols + vcol0);
          const int64_t left = (vcols - vcol0) / 16;
          const int nvalid = left < 4 ? static_cast<int>(left) : 4;
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            if (b >= nvalid) continue;
            const int p = b >> 1;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * e;
              dst[4 * b + e] = (b & 1) ? make_float4(z[p][i].y, z[p][i + 1].y, z[p][i + 2].y, z[p][i + 3].y)
                                       : make_float4(z[p][i].x, z[p][i + 1].x, z[p][i + 2].x, z[p][i + 3].x);
            }
          }
        }
      }
    }
    if constexpr (KIND == kAmax) {
      const unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(local_max));
      if (lane == 0) sh.warp_max[warp] = bits;
    }
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    // let every load and MMA still in flight finish before the CTA lets go
    if (tid == kProducerWarp * 32)
      for (int s = 0; s < kStagesA; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == kMmaWarp * 32)
      for (int a = 0; a < kAccum; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
  }
  if (tid == 0) {
    if constexpr (KIND == kAmax) {
      unsigned int m = 0;
#pragma unroll
      for (int w = 0; w < kEpiWarps; ++w) m = max(m, sh.warp_max[w]);
      atomicMax(amax_accum, failed ? 0x7FC00000u : m);
    } else if constexpr (KIND == kQuantize) {
      if (failed) *gscale = __uint_as_float(0x7FC00000u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// --------------------------------------------------------------------- host
using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

bool make_map(CUtensorMap* map, const void* x, int64_t rows, int64_t cols, int64_t ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, kTile};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int G, int KIND, bool ROWWISE>
cudaError_t launch_one(const QuantArgs& a, float* zout) {
  CUtensorMap map;
  if (!make_map(&map, a.x, a.rows, a.cols, a.ld)) return cudaErrorInvalidValue;
  auto kernel = rotate_mma_kernel<MODE, G, KIND, ROWWISE>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDynSmem));
  if (e != cudaSuccess) return e;
  // two CTAs per SM need the largest shared-memory carveout
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, kDynSmem);
  if (e != cudaSuccess) return e;
  per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);  // tensor memory holds two CTAs' accumulators
  const int64_t n_tiles = ((a.rows + kTile - 1) / kTile) * ((a.cols + kTile - 1) / kTile);
  int64_t grid = n_tiles < int64_t(sms) * per_sm ? n_tiles : int64_t(sms) * per_sm;
  if (grid == 0) {
    if (KIND == kAmax) return cudaSuccess;
    grid = 1;
  }
  kernel<<<static_cast<unsigned>(grid), kThreads, kDynSmem, a.stream>>>(
      map, a.rows, a.cols, a.seed, a.amax, reinterpret_cast<unsigned int*>(a.amax_accum), a.codes, a.scales,
      a.gscale, zout);
  return cudaGetLastError();
}

template <int MODE, int KIND>
cudaError_t dispatch(const QuantArgs& a, float* zout) {
  const bool row = a.layout == 0;
  switch (a.rht_group) {
    case 16: return row ? launch_one<MODE, 16, KIND, true>(a, zout) : launch_one<MODE, 16, KIND, false>(a, zout);
    case 32: return row ? launch_one<MODE, 32, KIND, true>(a, zout) : launch_one<MODE, 32, KIND, false>(a, zout);
    case 64: return row ? launch_one<MODE, 64, KIND, true>(a, zout) : launch_one<MODE, 64, KIND, false>(a, zout);
    case 128: return row ? launch_one<MODE, 128, KIND, true>(a, zout) : launch_one<MODE, 128, KIND, false>(a, zout);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool mma_path_applies(const QuantArgs& a) {
  if (a.rht_group == 0) return false;
  if (a.rows < kTile || a.cols < kTile) return false;
  if (a.rows >= (int64_t(1) << 31) || a.cols >= (int64_t(1) << 31)) return false;
  // the tensor map needs a 16-byte aligned base and row pitch
  if (reinterpret_cast<uintptr_t>(a.x) % 16 != 0 || a.ld % 8 != 0) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_amax_mma(const QuantArgs& a) { return dispatch<kRTN, kAmax>(a, nullptr); }

cudaError_t launch_rotate_mma(const QuantArgs& a, float* zout) { return dispatch<kRTN, kStoreZ>(a, zout); }

cudaError_t launch_quantize_mma(const QuantArgs& a) {
  switch (a.mode) {
    case kRTN: return dispatch<kRTN, kQuantize>(a, nullptr);
    case kSR: return dispatch<kSR, kQuantize>(a, nullptr);
    case kMSEDEN: return dispatch<kMSEDEN, kQuantize>(a, nullptr);
    case kIF4: return dispatch<kIF4, kQuantize>(a, nullptr);
    case k4over6: return dispatch<k4over6, kQuantize>(a, nullptr);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4

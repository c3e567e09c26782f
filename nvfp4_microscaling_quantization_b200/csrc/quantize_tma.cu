// quantize_tma.cu -- the tiled quantization kernels for sm_100a.
//
// A persistent CTA of 128 threads streams tiles of X through a ring of
// shared-memory stages filled by TMA (cp.async.bulk.tensor 2-D, 128-byte
// swizzle, no multicast).  Each warp releases a stage once it has read its
// part (one arrival on the stage's "empty" mbarrier) and takes a ticket; the
// warp that takes the last ticket refills the stage with the CTA's tile that
// many stages ahead and arms the stage's "full" mbarrier with the tile's byte
// count, so no thread ever waits to refill.  Every thread owns 64 elements = four 16-element blocks
// of one view row, held as two float2[16] pairs (block 0 | block 1, block 2 |
// block 3), so each per-element step of two blocks is one packed f32x2
// instruction.
//
// Row-wise tile: 16 rows x 512 columns of X (8 TMA boxes of 16 x 64); thread
// (row j, piece p) owns columns 64p .. 64p+63 of row j; reads are 16-byte
// chunks, conflict-free thanks to the swizzle.
// Transposed tile: 128 rows x 64 columns of X (one box); thread (column c,
// half h) owns rows 64h .. 64h+63 of column c, i.e. four blocks of output row
// c; reads are 2-byte elements.
// In both, the two 64-element halves of a 128-element rotation group sit in
// lanes l and l ^ 16, which exchange values once for the h = 64 butterfly
// stage; all other stages stay inside the thread.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kernels.h"
#include "launch_config.h"
#include "nvfp4_device.cuh"
#include "quant_core.cuh"
#include "tma_pipeline.cuh"

namespace nvfp4 {

namespace {

#ifndef NVFP4_TMA_STAGES
#define NVFP4_TMA_STAGES 3
#endif
#ifndef NVFP4_TMA_MIN_BLOCKS
#define NVFP4_TMA_MIN_BLOCKS 4
#endif

constexpr int kNT = 128;                   // threads per CTA
constexpr int kStages = NVFP4_TMA_STAGES;  // ring depth
constexpr int kMinBlocks = NVFP4_TMA_MIN_BLOCKS;
constexpr uint32_t kStageBytes = 16384;

// row-wise: 8 boxes of 16 rows x 64 columns
constexpr int kRowBoxRows = 16, kRowBoxes = 8, kRowTileCols = kRowBoxes * 64;
constexpr uint32_t kRowBoxBytes = kRowBoxRows * 128;
// transposed: 1 box of 128 rows x 64 columns
constexpr int kColTileRows = 128, kColTileCols = 64;

static_assert(kRowBoxes * kRowBoxBytes == kStageBytes, "row-wise stage size");
static_assert(kColTileRows * 128 == kStageBytes, "transposed stage size");

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

// ---------------------------------------------------------------- the ring
constexpr int kWarps = kNT / 32;

struct Ring {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  unsigned int tickets[kStages];
  unsigned int issued_mask;   // stages that ever received a load
  unsigned int last_parity;   // bit s: phase parity of the last load issued into stage s
  int abort_flag;
};

// (tile row, tile column) of the tiles a CTA visits: blockIdx.x, then every
// gridDim.x-th tile, advanced without a division per step.
struct TileCursor {
  int64_t t, rt, ct;
  __device__ __forceinline__ void start(int64_t t0, int64_t n_ct) {
    t = t0;
    rt = t0 / n_ct;
    ct = t0 - rt * n_ct;
  }
  __device__ __forceinline__ void advance(int64_t step, int64_t drt, int64_t dct, int64_t n_ct) {
    t += step;
    rt += drt;
    ct += dct;
    if (ct >= n_ct) {
      ct -= n_ct;
      ++rt;
    }
  }
};

template <bool ROWWISE>
__device__ __forceinline__ void issue_tile(const CUtensorMap* map, uint8_t* stage, uint64_t* full, int64_t rt,
                                           int64_t ct) {
  mbar_arrive_expect_tx(full, kStageBytes);
  if constexpr (ROWWISE) {
    const int32_t x = static_cast<int32_t>(ct * kRowTileCols), y = static_cast<int32_t>(rt * kRowBoxRows);
#pragma unroll
    for (int b = 0; b < kRowBoxes; ++b) tma_load_2d(stage + b * kRowBoxBytes, map, x + 64 * b, y, full);
  } else {
    tma_load_2d(stage, map, static_cast<int32_t>(ct * kColTileCols), static_cast<int32_t>(rt * kColTileRows), full);
  }
}

// ------------------------------------------------------ the 64-element core
// z[p][i]: element i of block 2p (.x) and of block 2p+1 (.y).  Butterfly
// stages in the oracle's order: h = 1, 2, 4, 8 inside a block, h = 16 between
// the blocks of a pair, h = 32 between the pairs, h = 64 with lane ^ 16.
template <int G>
__device__ __forceinline__ void rotate64(float2 (&z)[2][16], bool upper_half) {
#pragma unroll
  for (int h = 1; h < 16 && h < G; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i & h) continue;
        const float2 a = z[p][i], b = z[p][i + h];
        z[p][i] = add2_rn(a, b);
        z[p][i + h] = sub2_rn(a, b);
      }
  }
  if constexpr (G >= 32) {
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = z[p][i].x, b = z[p][i].y;
        z[p][i] = f2(__fadd_rn(a, b), __fsub_rn(a, b));
      }
  }
  if constexpr (G >= 64) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 a = z[0][i], b = z[1][i];
      z[0][i] = add2_rn(a, b);
      z[1][i] = sub2_rn(a, b);
    }
  }
  if constexpr (G == 128) {
    // lower half: mine + other; upper half: other - mine (one RN operation each)
    const float2 sgn = upper_half ? f2(-1.0f, -1.0f) : f2(1.0f, 1.0f);
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 other =
            f2(__shfl_xor_sync(0xFFFFFFFFu, z[p][i].x, 16), __shfl_xor_sync(0xFFFFFFFFu, z[p][i].y, 16));
        z[p][i] = fma2_rn(sgn, z[p][i], other);
      }
  }
  const float2 c2 = f2(RhtConst<G>::c, RhtConst<G>::c);
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int i = 0; i < 16; ++i) z[p][i] = mul2_rn(z[p][i], c2);
}

// -------------------------------------------------------------- the kernel
template <int MODE, int G, bool AMAX_ONLY, bool ROWWISE>
__global__ void __launch_bounds__(kNT, kMinBlocks)
quantize_tma_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols, uint64_t seed,
                    const float* __restrict__ amax, unsigned int* __restrict__ amax_accum,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ gscale) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) Ring ring;
  __shared__ __align__(16) uint32_t sign_tab[128];
  __shared__ unsigned int warp_max[kNT / 32];
  __shared__ __align__(16) float4 scale_tbl[128];  // block-scale constants per E4M3 code
  uint8_t* stages = align_1024(dyn_smem);

  const uint32_t tid = threadIdx.x;
  const PhiloxKey key = philox_key(seed);
  const int64_t n_ct = ROWWISE ? (cols + kRowTileCols - 1) / kRowTileCols : (cols + kColTileCols - 1) / kColTileCols;
  const int64_t n_tiles = ROWWISE ? ((rows + kRowBoxRows - 1) / kRowBoxRows) * n_ct
                                  : ((rows + kColTileRows - 1) / kColTileRows) * n_ct;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ring.full[s], 1);
      mbar_init(&ring.empty[s], kWarps);
      ring.tickets[s] = 0;
    }
    ring.issued_mask = 0;
    ring.last_parity = 0;
    ring.abort_flag = 0;
    fence_barrier_init();
  }
  if constexpr (G > 0) {
    // row-wise: mask of element pair (2q, 2q+1) of a 128-element window (bits 15 and 31);
    // transposed: mask of row q (bit 31 of the fp32 pattern).  Sign of position e: sigma_(e mod G).
    const uint4 w = philox_call(key, 0, kTagSigns);
    auto sgn = [&](uint32_t e) { e %= G; return (word_of(w, e >> 5) >> (e & 31)) & 1u; };
    if constexpr (ROWWISE) {
      if (tid < 64) sign_tab[tid] = (sgn(2 * tid) << 15) | (sgn(2 * tid + 1) << 31);
    } else {
      sign_tab[tid] = sgn(tid) << 31;
    }
  }
  __syncthreads();
  const int64_t step = gridDim.x, drt = step / n_ct, dct = step - drt * n_ct;
  // load the CTA's k-th tile (sequence index) into stage k mod kStages
  auto load = [&](int64_t kseq) {
    const int64_t tn = blockIdx.x + kseq * step;
    if (tn >= n_tiles) return;
    const int st = static_cast<int>(kseq % kStages);
    const int64_t rt = tn / n_ct;
    issue_tile<ROWWISE>(&tmap, stages + st * kStageBytes, &ring.full[st], rt, tn - rt * n_ct);
    atomicOr(&ring.issued_mask, 1u << st);
    if ((kseq / kStages) & 1) atomicOr(&ring.last_parity, 1u << st);
    else atomicAnd(&ring.last_parity, ~(1u << st));
  };
  if (tid == 0) {
    prefetch_tensormap(&tmap);
    for (int k = 0; k < kStages; ++k) load(k);
  }

  ScaleCtx sc{1.0f, 6.0f, 4.0f, 1.0f / 6.0f, 0.25f, -0.0f, false, nullptr};
  if constexpr (!AMAX_ONLY) {
    // the first loads are in flight: build the scale table meanwhile
    build_scale_table(scale_tbl, global_scale_of<MODE>(*amax), tid, kNT);
    __syncthreads();
    sc = make_scale_ctx<MODE>(*amax);
    sc.tbl = scale_tbl;
    if (blockIdx.x == 0 && tid == 0) *gscale = sc.s_g;
  }
  // thread roles
  const uint32_t j = tid & 15u, piece = tid >> 4;                    // row-wise: row, 64-column piece
  const uint32_t col = (tid >> 5) * 16u + (tid & 15u), half = (tid >> 4) & 1u;  // transposed: column, row half
  const bool upper_half = ROWWISE ? (piece & 1u) != 0 : half != 0;
  const int64_t vcols = ROWWISE ? cols : rows;
  const bool codes_aligned16 = ((vcols / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(codes) % 16) == 0;
  const bool scales_aligned4 = ((vcols / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(scales) % 4) == 0;
  float local_max = 0.0f;
  const uint32_t lane = tid & 31u;
  // A warp is done with stage s: release it, and refill it if it was the last.
  auto release = [&](int s, int k) {
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&ring.empty[s]);
      if (atomicAdd(&ring.tickets[s], 1u) == kWarps - 1) {
        atomicExch(&ring.tickets[s], 0u);
        if (blockIdx.x + int64_t(k + kStages) * step < n_tiles) {
          if (mbar_wait(&ring.empty[s], (k / kStages) & 1u)) load(k + kStages);
          else atomicExch(&ring.abort_flag, 1);
        }
      }
    }
  };

  TileCursor cur;
  cur.start(blockIdx.x, n_ct);
  int k = 0;
  for (; cur.t < n_tiles; cur.advance(step, drt, dct, n_ct), ++k) {
    const int s = k % kStages;
    if (!mbar_wait(&ring.full[s], (k / kStages) & 1u)) {
      atomicExch(&ring.abort_flag, 1);
      break;
    }
    const uint8_t* tile = stages + s * kStageBytes;
    float2 z[2][16];
    if constexpr (ROWWISE) {
      const uint8_t* rowp = tile + piece * kRowBoxBytes;
      uint4 ch[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) ch[c] = *reinterpret_cast<const uint4*>(rowp + swizzle128(j * 128u + c * 16u));
      release(s, k);
      const uint32_t* masks = sign_tab + 32 * (piece & 1u);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 mk = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (G > 0) mk = *reinterpret_cast<const uint4*>(masks + 4 * c);
        const uint32_t wv[4] = {ch[c].x ^ mk.x, ch[c].y ^ mk.y, ch[c].z ^ mk.z, ch[c].w ^ mk.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float lo = __uint_as_float(wv[m] << 16), hi = __uint_as_float(wv[m] & 0xFFFF0000u);
          const int blk = c >> 1, i = 8 * (c & 1) + 2 * m;
          if (blk & 1) {
            z[blk >> 1][i].y = lo;
            z[blk >> 1][i + 1].y = hi;
          } else {
            z[blk >> 1][i].x = lo;
            z[blk >> 1][i + 1].x = hi;
          }
        }
      }
    } else {
      // element (row r, column col): chunk col/8 of row r, XOR-swizzled by r mod 8 (= i mod 8)
      const uint8_t* colp = tile + half * (64u * 128u) + ((col & 7u) << 1);
      uint32_t v[64];
#pragma unroll
      for (int e = 0; e < 64; ++e)
        v[e] = *reinterpret_cast<const uint16_t*>(colp + e * 128u + ((((col >> 3) ^ (e & 7)) & 7u) << 4));
      release(s, k);
      const uint32_t* masks = sign_tab + 64 * half;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        uint4 mk = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (G > 0) mk = *reinterpret_cast<const uint4*>(masks + 4 * q);
        const uint32_t mv[4] = {mk.x, mk.y, mk.z, mk.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int e = 4 * q + m, blk = e >> 4, i = e & 15;
          const float x = __uint_as_float((v[e] << 16) ^ mv[m]);
          if (blk & 1) z[blk >> 1][i].y = x;
          else z[blk >> 1][i].x = x;
        }
      }
    }

    if constexpr (G > 0) rotate64<G>(z, upper_half);

    const int64_t rt = cur.rt, ct = cur.ct;
    if constexpr (AMAX_ONLY) {
      local_max = fmaxf(local_max, absmax64(z));
    } else if constexpr (ROWWISE) {
      const int64_t row = rt * kRowBoxRows + j, col0 = ct * kRowTileCols + 64 * piece;
      if (row < rows && col0 < cols)
        quantize_store64<MODE>(z, sc, key, row, col0, cols, codes, scales, codes_aligned16, scales_aligned4);
    } else {
      const int64_t vrow = ct * kColTileCols + col, vcol0 = rt * kColTileRows + 64 * half;
      if (vrow < cols && vcol0 < rows)
        quantize_store64<MODE>(z, sc, key, vrow, vcol0, rows, codes, scales, codes_aligned16, scales_aligned4);
    }
  }

  if constexpr (AMAX_ONLY) {
    const unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(local_max));
    if ((tid & 31u) == 0) warp_max[tid >> 5] = bits;
  }
  __syncthreads();
  // After a failed wait: let every load still in flight land before the CTA exits.
  if (tid == 0 && *reinterpret_cast<volatile int*>(&ring.abort_flag)) {
    for (int st = 0; st < kStages; ++st)
      if ((ring.issued_mask >> st) & 1u) mbar_wait(&ring.full[st], (ring.last_parity >> st) & 1u);
  }
  if (tid == 0) {
    const bool failed = *reinterpret_cast<volatile int*>(&ring.abort_flag) != 0;
    if constexpr (AMAX_ONLY) {
      unsigned int m = 0;
#pragma unroll
      for (int w = 0; w < kNT / 32; ++w) m = max(m, warp_max[w]);
      atomicMax(amax_accum, failed ? 0x7FC00000u : m);
    } else {
      if (failed) *gscale = __uint_as_float(0x7FC00000u);
    }
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

bool make_map(CUtensorMap* map, const void* x, int64_t rows, int64_t cols, int64_t ld, uint32_t box_x,
              uint32_t box_y) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {box_x, box_y};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, int G, bool AMAX_ONLY, bool ROWWISE>
cudaError_t launch_tma_one(const QuantArgs& a) {
  CUtensorMap map;
  if (!make_map(&map, a.x, a.rows, a.cols, a.ld, 64, ROWWISE ? kRowBoxRows : kColTileRows))
    return cudaErrorInvalidValue;
  auto kernel = quantize_tma_kernel<MODE, G, AMAX_ONLY, ROWWISE>;
  const size_t smem = kStages * kStageBytes + 1024;
  LaunchGeom geom;
  const cudaError_t e = launch_geometry(kernel, kNT, smem, 32, &geom);
  if (e != cudaSuccess) return e;
  const int sms = geom.sms, per_sm = geom.per_sm;
  const int64_t n_ct = ROWWISE ? (a.cols + kRowTileCols - 1) / kRowTileCols : (a.cols + kColTileCols - 1) / kColTileCols;
  const int64_t n_tiles = ROWWISE ? ((a.rows + kRowBoxRows - 1) / kRowBoxRows) * n_ct
                                  : ((a.rows + kColTileRows - 1) / kColTileRows) * n_ct;
  int64_t grid = n_tiles < int64_t(sms) * per_sm ? n_tiles : int64_t(sms) * per_sm;
  if (grid == 0) {
    if (AMAX_ONLY) return cudaSuccess;
    grid = 1;
  }
  kernel<<<static_cast<unsigned>(grid), kNT, smem, a.stream>>>(map, a.rows, a.cols, a.seed, a.amax,
                                                              reinterpret_cast<unsigned int*>(a.amax_accum),
                                                              a.codes, a.scales, a.gscale);
  return cudaGetLastError();
}

template <int MODE, int G, bool AMAX_ONLY>
cudaError_t launch_layout(const QuantArgs& a) {
  return a.layout == 0 ? launch_tma_one<MODE, G, AMAX_ONLY, true>(a) : launch_tma_one<MODE, G, AMAX_ONLY, false>(a);
}

template <int MODE, bool AMAX_ONLY>
cudaError_t dispatch_tma(const QuantArgs& a) {
  switch (a.rht_group) {
    case 0: return launch_layout<MODE, 0, AMAX_ONLY>(a);
    case 16: return launch_layout<MODE, 16, AMAX_ONLY>(a);
    case 32: return launch_layout<MODE, 32, AMAX_ONLY>(a);
    case 64: return launch_layout<MODE, 64, AMAX_ONLY>(a);
    case 128: return launch_layout<MODE, 128, AMAX_ONLY>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool tma_path_applies(const QuantArgs& a) {
  if (a.rows >= (int64_t(1) << 31) || a.cols >= (int64_t(1) << 31)) return false;
  if (encode_fn() == nullptr) return false;
  if (a.layout == 0) return a.cols >= 64 && a.rows >= kRowBoxRows;
  return a.cols >= kColTileCols && a.rows >= kColTileRows;
}

cudaError_t launch_amax_tma(const QuantArgs& a) { return dispatch_tma<kRTN, true>(a); }

cudaError_t launch_quantize_tma(const QuantArgs& a) {
  switch (a.mode) {
    case kRTN: return dispatch_tma<kRTN, false>(a);
    case kSR: return dispatch_tma<kSR, false>(a);
    case kMSEDEN: return dispatch_tma<kMSEDEN, false>(a);
    case kIF4: return dispatch_tma<kIF4, false>(a);
    case k4over6: return dispatch_tma<k4over6, false>(a);
    case kScaleSearch: return dispatch_tma<kScaleSearch, false>(a);
    case kMXFP4: return dispatch_tma<kMXFP4, false>(a);
    case kNVINT4: return dispatch_tma<kNVINT4, false>(a);
    case kNVFP3: return dispatch_tma<kNVFP3, false>(a);
    case kNVINT3: return dispatch_tma<kNVINT3, false>(a);
    case kIF3: return dispatch_tma<kIF3, false>(a);
    case kMXFP3: return dispatch_tma<kMXFP3, false>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4

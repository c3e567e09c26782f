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
// One CTA per SM (it allocates all 512 tensor-memory columns).  Warp roles:
//   epilogue   groups of four warps (Shape: four groups, three for SR), each
//              owning one 128-column fp32 accumulator and taking every
//              groups-th tile of the CTA; warp w reads lane quarter w % 4 (as
//              tensor memory requires), so its thread owns one tile row, all
//              128 columns (eight 16-element blocks), loaded 32 columns at a
//              time, scaled by c_g and quantized two blocks at a time (or
//              reduced to max|z|, or stored).  The accumulator columns are
//              permuted so a load yields (block a, block b) register pairs.
//   producer   one lane issues the TMA loads: two 64-column boxes of 128 rows
//              per tile into a kStagesA-stage shared-memory ring.
//   MMA        allocates the tensor memory, and one lane issues the 8 MMAs
//              (K = 16 each) of a tile into the accumulator of the group that
//              takes it, committing "stage free" and "accumulator full"
//              mbarriers.
// Every wait is bounded (tma_pipeline.cuh); on a failed wait the CTA drains
// what it issued, frees tensor memory and reports NaN in its scalar output.
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>

#include "kernels.h"
#include "launch_config.h"
#include "nvfp4_device.cuh"
#include "quant_core.cuh"
#include "tcgen05.cuh"
#include "tma_pipeline.cuh"

namespace nvfp4 {

namespace {

#ifndef NVFP4_MMA_STAGES
#define NVFP4_MMA_STAGES 3
#endif

enum Kind { kQuantize = 0, kAmax = 1, kStoreZ = 2 };

// Launch shape of one instantiation: epilogue groups of four warps, each
// owning one 128-column accumulator and taking every groups-th tile of the
// CTA; one TMA producer warp and one MMA warp.  SR runs three groups (14
// warps, 128 registers a thread: its Philox-heavy epilogue spills at 96),
// everything else four (18 warps, 96 registers).
template <int MODE, int KIND>
struct Shape {
  // SR (Philox) and scale search (19 candidates) get 128 registers a thread
  static constexpr int groups = (KIND == kQuantize && (MODE == kSR || MODE == kScaleSearch)) ? 3 : 4;
  static constexpr int epi_warps = 4 * groups;
  static constexpr int producer_warp = epi_warps, mma_warp = epi_warps + 1;
  static constexpr int threads = (epi_warps + 2) * 32;
};
constexpr int kMaxGroups = 4;
constexpr int kStagesA = NVFP4_MMA_STAGES;   // A tiles in flight
constexpr int kTile = 128;                   // tile rows and columns of X
constexpr uint32_t kTileBytes = kTile * kTile * 2;
constexpr uint32_t kBoxBytes = kTile * 128;  // 128 rows x 64 bf16
constexpr uint32_t kTmemCols = 512;          // up to four 128-column accumulators (a power of two)
constexpr size_t kDynSmem = (kStagesA + 1) * kTileBytes + 1024;

#ifndef NVFP4_MMA_BAND_ROWS
#define NVFP4_MMA_BAND_ROWS 1
#endif
#ifndef NVFP4_MMA_BAND_ROWS_T
#define NVFP4_MMA_BAND_ROWS_T 16
#endif

// Tile order: tiles are taken in bands of `band` tile rows, column by column
// inside a band (tile t -> (rt, ct)), so the tiles in flight at once read
// long runs of each input row and, for the transposed layout, write long
// runs of each output row.  32-bit arithmetic: the routing admits fewer than
// 2^31 tiles.
struct TileGrid {
  uint32_t n_rt, n_ct, band;
  __device__ __forceinline__ void coords(uint32_t t, uint32_t& rt, uint32_t& ct) const {
    const uint32_t per_band = band * n_ct;
    const uint32_t bg = t / per_band, r = t - bg * per_band;
    const uint32_t left = n_rt - bg * band;
    const uint32_t h = left < band ? left : band;  // tile rows in this band
    ct = r / h;
    rt = bg * band + (r - ct * h);
  }
};

struct MmaShared {
  uint64_t full[kStagesA];   // A tile landed (TMA transaction bytes)
  uint64_t sfree[kStagesA];  // MMAs reading the A tile are done (tcgen05.commit)
  uint64_t tfull[kMaxGroups];  // the group's accumulator ready (tcgen05.commit)
  uint64_t tfree[kMaxGroups];  // the group's accumulator read by its warps
  uint32_t tmem_base;
  uint32_t issued_a;         // bit s: a load went into stage s; bit 8+s: its phase parity
  uint32_t issued_mma;       // bit a: MMAs went into accumulator a; bit 8+a: parity
  int abort_flag;
  unsigned int warp_max[4 * kMaxGroups];
  float4 scale_tbl[128];     // the launch's block-scale constants per E4M3 code
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return p + ((1024u - (smem_u32(p) & 1023u)) & 1023u);
}

// Accumulator column of output column n: inside each 32-column group the two
// 16-element blocks are interleaved (block a element i at 2i, block b element
// i at 2i + 1), so a 32-column load from tensor memory yields the (a_i, b_i)
// register pairs that the packed f32x2 arithmetic works on.
__device__ __forceinline__ uint32_t output_col_of(uint32_t acc_col) {
  return (acc_col & ~31u) | ((acc_col & 1u) << 4) | ((acc_col & 31u) >> 1);
}

// B operand, K-major with the 128-byte swizzle: two 64-wide K halves of 128
// rows x 128 bytes; row r holds output column n = output_col_of(r), element
// (n, k) = sigma_(k mod G) * H_G[n mod G][k mod G] inside the diagonal G x G
// blocks, 0 elsewhere.  bf16 +1 = 0x3F80, -1 = 0xBF80.
template <int G>
__device__ __forceinline__ void build_hadamard_b(uint8_t* bmat, PhiloxKey key, uint32_t tid, uint32_t nthreads) {
  const uint4 w = philox_call(key, 0, kTagSigns);
  for (uint32_t c = tid; c < 2048; c += nthreads) {
    const uint32_t half = c >> 10, r = (c >> 3) & 127u, kc = c & 7u;
    const uint32_t n = output_col_of(r);
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
    *reinterpret_cast<uint4*>(bmat + half * kBoxBytes + r * 128 + ((kc ^ (r & 7u)) << 4)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

// Quantize one thread's row of a 128 x 128 tile of a view from tensor memory:
// the accumulator columns at taddr (this thread's lane; columns permuted by
// output_col_of) hold the unscaled rotation sums of view row vrow, view
// columns vcol_base .. vcol_base + 127.  Each 32-column load is scaled by
// c_G and quantized two blocks at a time; lane 0 of the warp arrives on
// free_bar once the warp's last columns are loaded.  Blocks outside the view
// are not stored.
template <int MODE, int G>
__device__ __forceinline__ void quantize_tmem_row(uint32_t taddr, uint64_t* free_bar, const ScaleCtx& sc,
                                                  PhiloxKey key, int64_t vrow, int64_t vcol_base, int64_t vrows,
                                                  int64_t vcols, bool row_blocks8, bool codes_aligned16,
                                                  bool scales_aligned4, uint8_t* codes, uint8_t* scales) {
  const uint32_t lane = threadIdx.x & 31u;
  const float2 c2 = f2(RhtConst<G>::c, RhtConst<G>::c);
  // MS-EDEN scale draws: when a thread owns a whole 128-column row of the
  // tile and view rows hold whole groups of eight blocks, its eight blocks
  // take the eight draws of one Philox call
  uint4 wu = make_uint4(0u, 0u, 0u, 0u);
  if constexpr (MODE == kMSEDEN) {
    if (row_blocks8)
      wu = philox_call(key, (static_cast<uint64_t>(vrow) * static_cast<uint64_t>(vcols / 16) +
                             static_cast<uint64_t>(vcol_base / 16)) >> 3,
                       kTagBlock);
  }
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int64_t vcol0 = vcol_base + 64 * h;  // view column of the first element
    const bool last = h == 1;
    // one pair of blocks at a time: load 32 columns, quantize, then the next 32
    const bool valid = vrow < vrows && vcol0 < vcols;
    const uint64_t e0 = static_cast<uint64_t>(vrow) * static_cast<uint64_t>(vcols) + static_cast<uint64_t>(vcol0);
    uint32_t kd[4] = {0u, 0u, 0u, 0u};
    if constexpr (MODE == kMSEDEN) {
      if (row_blocks8) {
#pragma unroll
        for (int b = 0; b < 4; ++b) kd[b] = half_word(wu, 4 * h + b);
      } else {
        block_draws<4>(key, e0 >> 4, kd);
      }
    }
    BlockOut o[4];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      float v[32];
      tmem_ld32_wait(taddr + 64 * h + 32 * p, v);
      if (last && p == 1) {
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(free_bar);
      }
      float2 zp[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) zp[i] = mul2_rn(f2(v[2 * i], v[2 * i + 1]), c2);
      const PairRng rng{key, e0 + 32 * p, e0 + 32 * p + 16, kd[2 * p], kd[2 * p + 1]};
      quantize_pair<MODE>(zp, sc, rng, o[2 * p], o[2 * p + 1]);
    }
    if (valid) store64(o, vrow, vcol0, vcols, codes, scales, codes_aligned16, scales_aligned4);
  }
}

template <int MODE, int G, int KIND, bool ROWWISE>
__global__ void __launch_bounds__(Shape<MODE, KIND>::threads, 1)
rotate_mma_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols, uint64_t seed,
                  const float* __restrict__ amax, unsigned int* __restrict__ amax_accum, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ scales, float* __restrict__ gscale, float* __restrict__ zout) {
  using S = Shape<MODE, KIND>;
  constexpr int kGroups = S::groups, kAccum = S::groups;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) MmaShared sh;
  uint8_t* a_tiles = align_1024(dyn_smem);
  uint8_t* bmat = a_tiles + kStagesA * kTileBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const TileGrid tg{static_cast<uint32_t>((rows + kTile - 1) / kTile), static_cast<uint32_t>((cols + kTile - 1) / kTile),
                    static_cast<uint32_t>(ROWWISE ? NVFP4_MMA_BAND_ROWS : NVFP4_MMA_BAND_ROWS_T)};
  const int64_t n_tiles = static_cast<int64_t>(tg.n_rt) * tg.n_ct;

  if (tid == S::producer_warp * 32) {
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sfree[s], 1);
    }
    for (int a = 0; a < kAccum; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], 4);  // the four warps of one epilogue group
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == S::mma_warp) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;
  const int64_t step = gridDim.x;
  if (warp != S::producer_warp) {
    // B is built by every warp but the producer, which starts loading tiles
    // meanwhile; the builders meet at barrier 2 before the first MMA
    const uint32_t bt = warp < S::producer_warp ? tid : tid - 32, nb = S::threads - 32;
    build_hadamard_b<G>(bmat, key, bt, nb);
    fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"r"(nb) : "memory");
  }

  if (warp == S::producer_warp) {
    if (lane == 0) {
      grid_dependency_wait();
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
        uint32_t rt, ct;
        tg.coords(static_cast<uint32_t>(t), rt, ct);
        const int32_t x = static_cast<int32_t>(ct * kTile), y = static_cast<int32_t>(rt * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kTileBytes);
        uint8_t* dst = a_tiles + s * kTileBytes;
        tma_load_2d(dst, &tmap, x, y, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &tmap, x + 64, y, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == S::mma_warp) {
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
    // group `grp` takes the CTA's tiles k = grp, grp + groups, ... into its
    // accumulator grp; a warp reads lane quarter q (= warp % 4, as tensor
    // memory requires): its thread owns one tile row, all 128 columns
    const uint32_t q = warp & 3u, grp = warp >> 2;
    grid_dependency_wait();
    ScaleCtx sc{1.0f, 6.0f, 4.0f, 1.0f / 6.0f, 0.25f, -0.0f, false, nullptr};
    if constexpr (KIND == kQuantize) {
      sc = make_scale_ctx<MODE>(*amax);
      // the scale table, built by the epilogue warps while the first tiles load
      build_scale_table(sh.scale_tbl, sc.s_g, tid, S::epi_warps * 32);
      asm volatile("bar.sync 1, %0;" ::"r"(S::epi_warps * 32) : "memory");
      sc.tbl = sh.scale_tbl;
      if (blockIdx.x == 0 && tid == 0) *gscale = sc.s_g;
    }
    const int64_t vcols = ROWWISE ? cols : rows;
    const int64_t vrows = ROWWISE ? rows : cols;
    const bool codes_aligned16 = ((vcols / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(codes) % 16) == 0;
    const bool scales_aligned4 = ((vcols / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(scales) % 4) == 0;
    const bool row_blocks8 = ((vcols / 16) % 8) == 0;
    const float2 c2 = f2(RhtConst<G>::c, RhtConst<G>::c);
    float local_max = 0.0f;
    int k = static_cast<int>(grp);
    for (int64_t t = blockIdx.x + grp * step; t < n_tiles; t += kGroups * step, k += kGroups) {
      const int a = k % kAccum;
      if (!mbar_wait(&sh.tfull[a], (k / kAccum) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      uint32_t rt, ct;
      tg.coords(static_cast<uint32_t>(t), rt, ct);
      // view row of this thread
      const int64_t vrow = (ROWWISE ? rt : ct) * kTile + 32 * q + lane;
      if constexpr (KIND == kQuantize) {
        quantize_tmem_row<MODE, G>(tmem_base + ((32u * q) << 16) + a * kTile, &sh.tfree[a], sc, key, vrow,
                                   static_cast<int64_t>(ROWWISE ? ct : rt) * kTile, vrows, vcols, row_blocks8,
                                   codes_aligned16, scales_aligned4, codes, scales);
      } else {
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const uint32_t taddr = tmem_base + ((32u * q) << 16) + a * kTile + h * 64;
          const int64_t vcol0 = (ROWWISE ? ct : rt) * kTile + 64 * h;  // view column of the first element
          const bool last = h == 1;
          // max |z| or z itself, one pair of blocks (32 columns) at a time
#pragma unroll
          for (int p = 0; p < 2; ++p) {
            float v[32];
            tmem_ld32_wait(taddr + 32 * p, v);
            if (last && p == 1) {
              tc_fence_before_sync();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sh.tfree[a]);
            }
            if constexpr (KIND == kAmax) {
              local_max = fmaxf(local_max, absmax_tree<32>(v));  // of |acc|: scaled by c_g at the end
            } else {
              float2 zp[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) zp[i] = mul2_rn(f2(v[2 * i], v[2 * i + 1]), c2);
              const int64_t c0 = vcol0 + 32 * p;  // view column of block 2p
              if (vrow < vrows && c0 < vcols) {
                float4* dst = reinterpret_cast<float4*>(zout + vrow * vcols + c0);
                const bool second = c0 + 16 < vcols;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int i = 4 * e;
                  dst[e] = make_float4(zp[i].x, zp[i + 1].x, zp[i + 2].x, zp[i + 3].x);
                  if (second) dst[4 + e] = make_float4(zp[i].y, zp[i + 1].y, zp[i + 2].y, zp[i + 3].y);
                }
              }
            }
          }
        }
      }
    }
    if constexpr (KIND == kAmax) {
      // RN(c t) is monotone in t >= 0: max RN(c |acc|) = RN(c max |acc|)
      local_max = __fmul_rn(RhtConst<G>::c, local_max);
      const unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(local_max));
      if (lane == 0) sh.warp_max[warp] = bits;
    }
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    // let every load and MMA still in flight finish before the CTA lets go
    if (tid == S::producer_warp * 32)
      for (int s = 0; s < kStagesA; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == S::mma_warp * 32)
      for (int a = 0; a < kAccum; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
  }
  if (tid == 0) {
    if constexpr (KIND == kAmax) {
      unsigned int m = 0;
#pragma unroll
      for (int w = 0; w < S::epi_warps; ++w) m = max(m, sh.warp_max[w]);
      atomicMax(amax_accum, failed ? 0x7FC00000u : m);
    } else if constexpr (KIND == kQuantize) {
      if (failed) *gscale = __uint_as_float(0x7FC00000u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == S::mma_warp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------- both layouts at once
// The tensor amax of the row-wise view (rotated along rows with group g_r)
// and of the transposed view (rotated along columns with group g_c) from one
// read of X.  Every tile goes through the MMAs its views need -- the K-major
// one against B_r (when g_r > 0) and the MN-major one against B_c (g_c = 0:
// the identity, z = x exactly) -- each into the next of four 128-column
// accumulator slots (all 512 tensor-memory columns), each slot with its own
// "full" and "free" barriers, so a view's epilogue starts as soon as its own
// MMAs land and the MMA warp refills a slot as soon as it is read.  Slot s is
// read by epilogue warps 4s .. 4s+3 (warp 4s + q reads lane quarter q).
// With g_r = 0 (the forward RTN operands X and W) the row view needs no MMA:
// the slot's warps also take max|x| straight from the staged tile before its
// stage is released, and four tiles are in flight in tensor memory.
// Because RN(c t) is monotone in t >= 0, the epilogue keeps max |acc| and
// scales once at the end: max RN(c |acc|) = RN(c max |acc|), so the results
// are those of the single-layout pre-passes bit for bit.

#ifndef NVFP4_DUAL_STAGES
#define NVFP4_DUAL_STAGES 4
#endif
constexpr int kDualStages = NVFP4_DUAL_STAGES;  // A tiles in flight (each held until its MMAs are done)
constexpr int kDualSlots = 4;                   // 128-column accumulator slots
constexpr int kDualEpiWarps = 4 * kDualSlots;
constexpr int kDualThreads = (kDualEpiWarps + 2) * 32;
constexpr int kDualProducerWarp = kDualEpiWarps, kDualMmaWarp = kDualEpiWarps + 1;
constexpr size_t kDualDynSmem = (kDualStages + 2) * kTileBytes + 1024;

struct DualShared {
  uint64_t full[kDualStages];
  uint64_t sfree[kDualStages];
  uint64_t tfull[kDualSlots];   // the slot's accumulator is ready
  uint64_t tfree[kDualSlots];   // the slot's accumulator has been read by its four warps
  uint32_t tmem_base;
  uint32_t issued_a;
  uint32_t issued_mma;
  int abort_flag;
  unsigned int warp_max[2][kMaxDualMembers][kDualEpiWarps];
};

__device__ __forceinline__ float rht_scale_of(int g) {
  return g == 16 ? RhtConst<16>::c : g == 32 ? RhtConst<32>::c : g == 64 ? RhtConst<64>::c
                                                                         : g == 128 ? RhtConst<128>::c : 1.0f;
}

// B for a rotation group g chosen at run time, laid out like build_hadamard_b;
// g = 0 gives the identity (row r holds output column output_col_of(r)).
__device__ __forceinline__ void build_rotation_b(uint8_t* bmat, PhiloxKey key, uint32_t tid, uint32_t nthreads,
                                                 int g) {
  const uint4 w = philox_call(key, 0, kTagSigns);
  const uint32_t gg = g > 0 ? static_cast<uint32_t>(g) : 1u;
  for (uint32_t c = tid; c < 2048; c += nthreads) {
    const uint32_t half = c >> 10, r = (c >> 3) & 127u, kc = c & 7u;
    const uint32_t n = output_col_of(r);
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t two = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t k = half * 64 + kc * 8 + 2 * i + h;
        uint32_t v = 0;
        if (g == 0) {
          v = n == k ? 0x3F80u : 0u;
        } else if (n / gg == k / gg) {
          const uint32_t kg = k % gg, ng = n % gg;
          const uint32_t neg = ((word_of(w, kg >> 5) >> (kg & 31)) ^ __popc(ng & kg)) & 1u;
          v = neg ? 0xBF80u : 0x3F80u;
        }
        two |= v << (16 * h);
      }
      packed[i] = two;
    }
    *reinterpret_cast<uint4*>(bmat + half * kBoxBytes + r * 128 + ((kc ^ (r & 7u)) << 4)) =
        make_uint4(packed[0], packed[1], packed[2], packed[3]);
  }
}

// max |v| over 64 accumulator values (and m), as a tree: short dependency
// chains, so a warp's reduction does not wait on its own previous result.
__device__ __forceinline__ float absmax64(const float (&v)[64], float m) { return fmaxf(m, absmax_tree<64>(v)); }

// A group of tensors measured or quantized by one launch: the same rotation
// groups, modes and seed for every member; the members' tiles are numbered
// one member after the other (member i owns tiles tile0 .. tile0 + its count
// - 1), so one persistent grid walks them all and pays one ramp and one tail.
struct DualMember {
  int64_t rows, cols;   // the tensor (row view rows x cols, column view cols x rows)
  int64_t tile0;        // its first tile in the group's numbering
  uint32_t n_rt, n_ct;  // its grid of 128 x 128 tiles
  const float* amax_r;  // quantize: the tensor amax of each view
  const float* amax_c;
  uint8_t* codes_r;
  uint8_t* scales_r;
  float* gscale_r;
  uint8_t* codes_c;
  uint8_t* scales_c;
  float* gscale_c;
  unsigned int* max_r;  // pre-pass: the amax of each view (binary32 patterns, atomicMax)
  unsigned int* max_c;
};
struct DualGroup {
  CUtensorMap map[kMaxDualMembers];
  DualMember m[kMaxDualMembers];
  int64_t n_tiles;      // all members' tiles
  int n;                // members
};

// The member that owns tile t of the group (members without tiles own none).
__device__ __forceinline__ int group_member(const DualGroup& g, int64_t t) {
  int i = 0;
#pragma unroll
  for (int j = 1; j < kMaxDualMembers; ++j)
    if (j < g.n && t >= g.m[j].tile0) i = j;
  return i;
}
// Tile t of the group as (member, tile row, tile column) of the member.
__device__ __forceinline__ int group_tile(const DualGroup& g, int64_t t, uint32_t band, uint32_t& rt, uint32_t& ct) {
  const int i = group_member(g, t);
  const TileGrid tg{g.m[i].n_rt, g.m[i].n_ct, band};
  tg.coords(static_cast<uint32_t>(t - g.m[i].tile0), rt, ct);
  return i;
}

__global__ void __launch_bounds__(kDualThreads, 1)
dual_amax_kernel(const __grid_constant__ DualGroup grp, uint64_t seed, int g_r, int g_c) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) DualShared sh;
  uint8_t* a_tiles = align_1024(dyn_smem);
  uint8_t* b_r = a_tiles + kDualStages * kTileBytes;
  uint8_t* b_c = b_r + kTileBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const uint32_t band = static_cast<uint32_t>(NVFP4_MMA_BAND_ROWS);
  const int64_t n_tiles = grp.n_tiles;
  const int64_t step = gridDim.x;
  // this CTA's tiles: blockIdx.x, blockIdx.x + step, ...
  const int64_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + step - 1) / step : 0;
  // accumulators per tile: the row view's (if rotated) then the column view's
  const int views = g_r != 0 ? 2 : 1;
  const bool row_from_smem = g_r == 0;

  if (tid == kDualProducerWarp * 32) {
    for (int s = 0; s < kDualStages; ++s) {
      mbar_init(&sh.full[s], 1);
      // released by the MMA commit, and with the row view taken from shared
      // memory also by the four warps of the slot that reads the tile
      mbar_init(&sh.sfree[s], row_from_smem ? 5 : 1);
    }
    for (int a = 0; a < kDualSlots; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], 4);
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kDualMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;
  if (warp != kDualProducerWarp) {
    // the B matrices, built while the producer starts loading (barrier 2)
    const uint32_t bt = warp < kDualProducerWarp ? tid : tid - 32, nb = kDualThreads - 32;
    if (g_r != 0) build_rotation_b(b_r, key, bt, nb, g_r);
    build_rotation_b(b_c, key, bt, nb, g_c);
    fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"r"(nb) : "memory");
  }

  if (warp == kDualProducerWarp) {
    if (lane == 0) {
      grid_dependency_wait();
      for (int i = 0; i < grp.n; ++i) prefetch_tensormap(&grp.map[i]);
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = static_cast<int>(k % kDualStages);
        const uint32_t u = static_cast<uint32_t>(k / kDualStages);
        if (k >= kDualStages && !mbar_wait(&sh.sfree[s], (u - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) break;
        uint32_t rt, ct;
        const int mi = group_tile(grp, blockIdx.x + k * step, band, rt, ct);
        const int32_t x = static_cast<int32_t>(ct * kTile), y = static_cast<int32_t>(rt * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kTileBytes);
        uint8_t* dst = a_tiles + s * kTileBytes;
        tma_load_2d(dst, &grp.map[mi], x, y, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &grp.map[mi], x + 64, y, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == kDualMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_r = idesc_bf16_f32(kTile, kTile, 0u);
      constexpr uint32_t idesc_c = idesc_bf16_f32(kTile, kTile, 1u);
      const uint32_t br_addr = smem_u32(b_r), bc_addr = smem_u32(b_c);
      int64_t j = 0;  // running accumulator index: slot j % 4, use j / 4
      for (int64_t k = 0; k < my_tiles && !*reinterpret_cast<volatile int*>(&sh.abort_flag); ++k) {
        const int s = static_cast<int>(k % kDualStages);
        if (!mbar_wait(&sh.full[s], static_cast<uint32_t>(k / kDualStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(a_tiles + s * kTileBytes);
        bool ok = true;
        for (int v = 0; v < views; ++v, ++j) {
          const int a = static_cast<int>(j % kDualSlots);
          const uint32_t use = static_cast<uint32_t>(j / kDualSlots);
          if (use > 0 && !mbar_wait(&sh.tfree[a], (use - 1) & 1u)) {
            atomicExch(&sh.abort_flag, 1);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d = tmem_base + a * kTile;
          if (v == 0 && views == 2) {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(br_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              umma_bf16(d, adesc, bdesc, idesc_r, kk > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_addr + kk * 2048, kBoxBytes, 1024);
              const uint64_t bdesc = smem_desc_sw128(bc_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              umma_bf16(d, adesc, bdesc, idesc_c, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&sh.tfull[a]);
          sh.issued_mma = (sh.issued_mma & ~(0x101u << a)) | (1u << a) | ((use & 1u) << (8 + a));
        }
        if (!ok) break;
        umma_commit(&sh.sfree[s]);
      }
    }
  } else {
    // epilogue: slot `slot`, lane quarter q
    const uint32_t q = warp & 3u, slot = warp >> 2;
    grid_dependency_wait();
    // per member: max |acc| (unscaled) of the row and column views; max |x| from smem
    float m_r[kMaxDualMembers], m_c[kMaxDualMembers];
#pragma unroll
    for (int i = 0; i < kMaxDualMembers; ++i) m_r[i] = m_c[i] = 0.0f;
    const int64_t n_acc = my_tiles * views;
    const uint32_t part = q * 32u + lane;
    for (int64_t j = slot; j < n_acc; j += kDualSlots) {
      const int64_t k = j / views;
      const int v = static_cast<int>(j % views);
      const int mi = group_member(grp, blockIdx.x + k * step);
      if (row_from_smem) {
        // max|x| of the staged tile for the row view: 128 threads, 256 bytes
        // each (the order of the swizzled bytes does not matter to a
        // maximum); bf16 -> f32 is exact
        const int s = static_cast<int>(k % kDualStages);
        if (!mbar_wait(&sh.full[s], static_cast<uint32_t>(k / kDualStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a_tiles + s * kTileBytes) + part;
        uint32_t bmax = 0;  // max of |x| as bf16 bit-pattern pairs (monotone for non-negative values)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 w4 = src[i * 128];
          bmax = __vmaxu2(bmax, __vmaxu2(__vmaxu2(w4.x & 0x7FFF7FFFu, w4.y & 0x7FFF7FFFu),
                                         __vmaxu2(w4.z & 0x7FFF7FFFu, w4.w & 0x7FFF7FFFu)));
        }
        const float mx = __uint_as_float(max(bmax & 0xFFFFu, bmax >> 16) << 16);
#pragma unroll
        for (int i = 0; i < kMaxDualMembers; ++i)
          if (i == mi) m_r[i] = fmaxf(m_r[i], mx);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.sfree[s]);
      }
      if (!mbar_wait(&sh.tfull[slot], static_cast<uint32_t>(j / kDualSlots) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      const uint32_t base = tmem_base + ((32u * q) << 16) + slot * kTile;
      float m = 0.0f;
      {
        float v0[64];
        tmem_ld64_wait(base, v0);
        m = absmax64(v0, m);
      }
      {
        float v1[64];
        tmem_ld64_wait(base + 64, v1);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.tfree[slot]);
        m = absmax64(v1, m);
      }
      const bool row = v == 0 && views == 2;
#pragma unroll
      for (int i = 0; i < kMaxDualMembers; ++i)
        if (i == mi) {
          if (row) m_r[i] = fmaxf(m_r[i], m);
          else m_c[i] = fmaxf(m_c[i], m);
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxDualMembers; ++i) {
      const unsigned int br = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m_r[i]));
      const unsigned int bc = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m_c[i]));
      if (lane == 0) {
        sh.warp_max[0][i][warp] = br;
        sh.warp_max[1][i][warp] = bc;
      }
    }
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    if (tid == kDualProducerWarp * 32)
      for (int s = 0; s < kDualStages; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == kDualMmaWarp * 32)
      for (int a = 0; a < kDualSlots; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
  }
  if (tid < static_cast<uint32_t>(grp.n)) {
    // thread i finishes member i
    const int i = static_cast<int>(tid);
    unsigned int mr = 0, mc = 0;
#pragma unroll
    for (int w = 0; w < kDualEpiWarps; ++w) {
      mr = max(mr, sh.warp_max[0][i][w]);
      mc = max(mc, sh.warp_max[1][i][w]);
    }
    // one rounding of the largest magnitude by the rotation constant (the
    // row view read from shared memory is x itself)
    const float cr = row_from_smem ? 1.0f : rht_scale_of(g_r), cc = rht_scale_of(g_c);
    const unsigned int sr = __float_as_uint(__fmul_rn(__uint_as_float(mr), cr));
    const unsigned int sc = __float_as_uint(__fmul_rn(__uint_as_float(mc), cc));
    atomicMax(grp.m[i].max_r, failed ? 0x7FC00000u : sr);
    atomicMax(grp.m[i].max_c, failed ? 0x7FC00000u : sc);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kDualMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}

// The same pre-pass when both views are rotated with different group sizes,
// in groups: two epilogue groups of eight warps, each owning two 128-column
// accumulators (row view and column view of one tile, one commit for both);
// warp (q, j) of a group reads lane quarter q of view j, 64 columns per load,
// scales by c_g and reduces with a tree.  Measured faster than the slot ring
// when every tile carries two MMAs; the results are identical.  With one
// group size for both views (dY of the backward pass) the pair kernel below
// does the same work in half the MMA instructions.
constexpr int kGrpStages = 5;     // A tiles in flight (each held until both MMAs are done)
constexpr int kGrpGroups = 2;
constexpr int kGrpEpiWarps = 8 * kGrpGroups;
constexpr int kGrpThreads = (kGrpEpiWarps + 2) * 32;
constexpr int kGrpProducerWarp = kGrpEpiWarps, kGrpMmaWarp = kGrpEpiWarps + 1;
constexpr size_t kGrpDynSmem = (kGrpStages + 2) * kTileBytes + 1024;

struct GroupDualShared {
  uint64_t full[kGrpStages];
  uint64_t sfree[kGrpStages];
  uint64_t tfull[kGrpGroups];   // both accumulators of the group ready
  uint64_t tfree[kGrpGroups];   // both loaded by the group
  uint32_t tmem_base;
  uint32_t issued_a;
  uint32_t issued_mma;
  int abort_flag;
  unsigned int warp_max[2][kGrpEpiWarps];
};
// 227 KB of shared memory per CTA on sm_100
static_assert(kGrpDynSmem + sizeof(GroupDualShared) <= 227u * 1024u, "group pre-pass shared memory");

__global__ void __launch_bounds__(kGrpThreads, 1)
dual_amax_group_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols, uint64_t seed, int g_r,
                 int g_c, unsigned int* __restrict__ amax_r, unsigned int* __restrict__ amax_c) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) GroupDualShared sh;
  uint8_t* a_tiles = align_1024(dyn_smem);
  uint8_t* b_r = a_tiles + kGrpStages * kTileBytes;
  uint8_t* b_c = b_r + kTileBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const TileGrid tg{static_cast<uint32_t>((rows + kTile - 1) / kTile), static_cast<uint32_t>((cols + kTile - 1) / kTile),
                    static_cast<uint32_t>(NVFP4_MMA_BAND_ROWS)};
  const int64_t n_tiles = static_cast<int64_t>(tg.n_rt) * tg.n_ct;

  if (tid == kGrpProducerWarp * 32) {
    // with g_r = 0 the row view needs no MMA: the group's four row-view
    // warps take max|x| from the staged tile and release the stage themselves
    for (int s = 0; s < kGrpStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sfree[s], g_r == 0 ? 5 : 1);
    }
    for (int a = 0; a < kGrpGroups; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], g_r == 0 ? 4 : 8);
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kGrpMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;
  const int64_t step = gridDim.x;
  if (warp != kGrpProducerWarp) {
    // the B matrices, built while the producer starts loading (barrier 2)
    const uint32_t bt = warp < kGrpProducerWarp ? tid : tid - 32, nb = kGrpThreads - 32;
    if (g_r != 0) build_rotation_b(b_r, key, bt, nb, g_r);
    build_rotation_b(b_c, key, bt, nb, g_c);
    fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"r"(nb) : "memory");
  }

  if (warp == kGrpProducerWarp) {
    if (lane == 0) {
      grid_dependency_wait();
      prefetch_tensormap(&tmap);
      int k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++k) {
        const int s = k % kGrpStages;
        const uint32_t u = k / kGrpStages;
        if (k >= kGrpStages && !mbar_wait(&sh.sfree[s], (u - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) break;
        uint32_t rt, ct;
        tg.coords(static_cast<uint32_t>(t), rt, ct);
        const int32_t x = static_cast<int32_t>(ct * kTile), y = static_cast<int32_t>(rt * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kTileBytes);
        uint8_t* dst = a_tiles + s * kTileBytes;
        tma_load_2d(dst, &tmap, x, y, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &tmap, x + 64, y, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == kGrpMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_r = idesc_bf16_f32(kTile, kTile, 0u);
      constexpr uint32_t idesc_c = idesc_bf16_f32(kTile, kTile, 1u);
      const uint32_t br_addr = smem_u32(b_r), bc_addr = smem_u32(b_c);
      int k = 0;
      for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++k) {
        const int s = k % kGrpStages, a = k % kGrpGroups;
        const uint32_t use = k / kGrpGroups;
        if (!mbar_wait(&sh.full[s], (k / kGrpStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (use > 0 && !mbar_wait(&sh.tfree[a], (use - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(a_tiles + s * kTileBytes);
        const uint32_t d_r = tmem_base + a * 256, d_c = d_r + 128;
        if (g_r != 0) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(a_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(br_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
            umma_bf16(d_r, adesc, bdesc, idesc_r, kk > 0 ? 1u : 0u);
          }
        }
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t adesc = smem_desc_sw128(a_addr + kk * 2048, kBoxBytes, 1024);
          const uint64_t bdesc = smem_desc_sw128(bc_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
          umma_bf16(d_c, adesc, bdesc, idesc_c, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sh.sfree[s]);
        umma_commit(&sh.tfull[a]);
        sh.issued_mma = (sh.issued_mma & ~(0x101u << a)) | (1u << a) | ((use & 1u) << (8 + a));
      }
    }
  } else {
    const uint32_t q = warp & 3u, j = (warp >> 2) & 1u, grp = warp >> 3;
    grid_dependency_wait();
    const float c = rht_scale_of(j == 0 ? g_r : g_c);
    float m = 0.0f;
    int k = static_cast<int>(grp);
    if (j == 0 && g_r == 0) {
      // max|x| of the staged tile: 128 threads, 256 bytes each (the order of
      // the swizzled bytes does not matter to a maximum); bf16 -> f32 is exact
      const uint32_t part = (warp & 3u) * 32u + lane;
      for (int64_t t = blockIdx.x + grp * step; t < n_tiles; t += kGrpGroups * step, k += kGrpGroups) {
        const int s = k % kGrpStages;
        if (!mbar_wait(&sh.full[s], (k / kGrpStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a_tiles + s * kTileBytes) + part;
        uint32_t bmax = 0;  // max of |x| as bf16 bit patterns (monotone for non-negative values)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 w4 = src[i * 128];
          const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) bmax = max(bmax, max(w[e] & 0x7FFFu, (w[e] >> 16) & 0x7FFFu));
        }
        m = fmaxf(m, __uint_as_float(bmax << 16));
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.sfree[s]);
      }
    } else {
    for (int64_t t = blockIdx.x + grp * step; t < n_tiles; t += kGrpGroups * step, k += kGrpGroups) {
      if (!mbar_wait(&sh.tfull[grp], (k / kGrpGroups) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      const uint32_t base = tmem_base + ((32u * q) << 16) + grp * 256 + j * 128;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float v[64];
        tmem_ld64_wait(base + 64 * h, v);
        if (h == 1) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.tfree[grp]);
        }
        m = absmax64(v, m);
      }
    }
    // max |acc| so far: RN(c t) is monotone in t >= 0, so max RN(c |acc|) = RN(c max |acc|)
    m = __fmul_rn(c, m);
    }
    const unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
    if (lane == 0) sh.warp_max[j][warp] = bits;
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    if (tid == kGrpProducerWarp * 32)
      for (int s = 0; s < kGrpStages; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == kGrpMmaWarp * 32)
      for (int a = 0; a < kGrpGroups; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
  }
  if (tid == 0) {
    unsigned int mr = 0, mc = 0;
#pragma unroll
    for (int w = 0; w < kGrpEpiWarps; ++w) {
      // warps with (w >> 2) odd read the column view
      if (((w >> 2) & 1) == 0) mr = max(mr, sh.warp_max[0][w]);
      else mc = max(mc, sh.warp_max[1][w]);
    }
    atomicMax(amax_r, failed ? 0x7FC00000u : mr);
    atomicMax(amax_c, failed ? 0x7FC00000u : mc);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kGrpMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}


// ------------------------------------ both views rotated with one group size
// Pairs of tiles: the rotation matrix is the A operand of every MMA and the
// two tiles of a pair together the N = 256 B operand (an amax does not care
// how D is laid out): D_row[n][r] = sum_k B[k][n] T[r][k] over the pair's 256
// tile rows r (K-major B), D_col[n][c] = sum_r B[r][n] T[r][c] over its 256
// tile columns c (MN-major B).  A stage holds a pair with its 64-column boxes
// interleaved -- tile 0 box 0, tile 1 box 0, tile 0 box 1, tile 1 box 1 -- so
// that both B operands have regular strides; a CTA's odd last tile is loaded
// twice.  Half the MMA instructions of the group kernel for the same work,
// and a quarter fewer operand bytes read from shared memory.
constexpr int kPairStages = 3;
constexpr uint32_t kPairBytes = 2 * kTileBytes;
constexpr int kPairEpiWarps = 16;  // eight per view: lane quarter q, column half h
constexpr int kPairThreads = (kPairEpiWarps + 2) * 32;
constexpr int kPairProducerWarp = kPairEpiWarps, kPairMmaWarp = kPairEpiWarps + 1;
constexpr size_t kPairDynSmem = kPairStages * kPairBytes + kTileBytes + 1024;

struct PairDualShared {
  uint64_t full[kPairStages];
  uint64_t sfree[kPairStages];
  uint64_t tfull[2];  // view v's accumulator holds the pair's result
  uint64_t tfree[2];  // ... and has been loaded by the view's eight warps
  uint32_t tmem_base;
  uint32_t issued_a;
  uint32_t issued_mma;
  int abort_flag;
  unsigned int warp_max[2][kPairEpiWarps];
};
static_assert(kPairDynSmem + sizeof(PairDualShared) <= 227u * 1024u, "pair pre-pass shared memory");

__global__ void __launch_bounds__(kPairThreads, 1)
dual_amax_pair_kernel(const __grid_constant__ CUtensorMap tmap, int64_t rows, int64_t cols, uint64_t seed, int g,
                      unsigned int* __restrict__ amax_r, unsigned int* __restrict__ amax_c) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) PairDualShared sh;
  uint8_t* pairs = align_1024(dyn_smem);
  uint8_t* bmat = pairs + kPairStages * kPairBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const TileGrid tg{static_cast<uint32_t>((rows + kTile - 1) / kTile), static_cast<uint32_t>((cols + kTile - 1) / kTile),
                    static_cast<uint32_t>(NVFP4_MMA_BAND_ROWS)};
  const int64_t n_tiles = static_cast<int64_t>(tg.n_rt) * tg.n_ct;
  const int64_t step = gridDim.x;
  const int64_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + step - 1) / step : 0;
  const int64_t my_pairs = (my_tiles + 1) / 2;

  if (tid == kPairProducerWarp * 32) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sfree[s], 1);
    }
    for (int v = 0; v < 2; ++v) {
      mbar_init(&sh.tfull[v], 1);
      mbar_init(&sh.tfree[v], 8);
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;
  if (warp != kPairProducerWarp) {
    const uint32_t bt = warp < kPairProducerWarp ? tid : tid - 32, nb = kPairThreads - 32;
    build_rotation_b(bmat, key, bt, nb, g);
    fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"r"(nb) : "memory");
  }

  if (warp == kPairProducerWarp) {
    if (lane == 0) {
      grid_dependency_wait();
      prefetch_tensormap(&tmap);
      for (int64_t p = 0; p < my_pairs; ++p) {
        const int s = static_cast<int>(p % kPairStages);
        const uint32_t u = static_cast<uint32_t>(p / kPairStages);
        if (p >= kPairStages && !mbar_wait(&sh.sfree[s], (u - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) break;
        const int64_t t0 = blockIdx.x + 2 * p * step;
        const int64_t t1 = 2 * p + 1 < my_tiles ? t0 + step : t0;
        uint32_t rt0, ct0, rt1, ct1;
        tg.coords(static_cast<uint32_t>(t0), rt0, ct0);
        tg.coords(static_cast<uint32_t>(t1), rt1, ct1);
        const int32_t x0 = static_cast<int32_t>(ct0 * kTile), y0 = static_cast<int32_t>(rt0 * kTile);
        const int32_t x1 = static_cast<int32_t>(ct1 * kTile), y1 = static_cast<int32_t>(rt1 * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kPairBytes);
        uint8_t* dst = pairs + s * kPairBytes;
        tma_load_2d(dst, &tmap, x0, y0, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &tmap, x1, y1, &sh.full[s]);
        tma_load_2d(dst + 2 * kBoxBytes, &tmap, x0 + 64, y0, &sh.full[s]);
        tma_load_2d(dst + 3 * kBoxBytes, &tmap, x1 + 64, y1, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == kPairMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_r = idesc_bf16_f32(kTile, 2 * kTile, 0u);
      constexpr uint32_t idesc_c = idesc_bf16_f32(kTile, 2 * kTile, 0u) | (1u << 16);  // B MN-major
      const uint32_t b_addr = smem_u32(bmat);
      for (int64_t p = 0; p < my_pairs; ++p) {
        const int s = static_cast<int>(p % kPairStages);
        if (!mbar_wait(&sh.full[s], static_cast<uint32_t>(p / kPairStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        const uint32_t pair_addr = smem_u32(pairs + s * kPairBytes);
        bool ok = true;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          if (p > 0 && !mbar_wait(&sh.tfree[v], static_cast<uint32_t>(p - 1) & 1u)) {
            atomicExch(&sh.abort_flag, 1);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d = tmem_base + v * 256;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(b_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = v == 0 ? smem_desc_sw128(pair_addr + (kk >> 2) * 2 * kBoxBytes + (kk & 3) * 32, 16, 1024)
                                          : smem_desc_sw128(pair_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16(d, adesc, bdesc, v == 0 ? idesc_r : idesc_c, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sh.tfull[v]);
          sh.issued_mma = (sh.issued_mma & ~(0x101u << v)) | (1u << v) | ((static_cast<uint32_t>(p) & 1u) << (8 + v));
        }
        if (!ok) break;
        umma_commit(&sh.sfree[s]);
      }
    }
  } else {
    const uint32_t v = warp >> 3, q = warp & 3u, h = (warp >> 2) & 1u;
    grid_dependency_wait();
    float m = 0.0f;
    for (int64_t p = 0; p < my_pairs; ++p) {
      if (!mbar_wait(&sh.tfull[v], static_cast<uint32_t>(p) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      const uint32_t base = tmem_base + ((32u * q) << 16) + v * 256 + h * 128;
#pragma unroll 1
      for (int hh = 0; hh < 2; ++hh) {
        float vals[64];
        tmem_ld64_wait(base + 64 * hh, vals);
        if (hh == 1) {
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.tfree[v]);
        }
        m = absmax64(vals, m);
      }
    }
    m = __fmul_rn(rht_scale_of(g), m);
    const unsigned int bits = __reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m));
    if (lane == 0) sh.warp_max[v][warp & 7u] = bits;
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    if (tid == kPairProducerWarp * 32)
      for (int s = 0; s < kPairStages; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == kPairMmaWarp * 32)
      for (int v = 0; v < 2; ++v)
        if ((sh.issued_mma >> v) & 1u) mbar_wait(&sh.tfull[v], (sh.issued_mma >> (8 + v)) & 1u);
  }
  if (tid == 0) {
    unsigned int mr = 0, mc = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      mr = max(mr, sh.warp_max[0][w]);
      mc = max(mc, sh.warp_max[1][w]);
    }
    atomicMax(amax_r, failed ? 0x7FC00000u : mr);
    atomicMax(amax_c, failed ? 0x7FC00000u : mc);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kPairMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
  }
}


// ------------------------------------------------ both layouts' quantization
// One read of X for both views' codes and scales (given both tensor amaxes):
// the pre-pass structure above -- four accumulator slots, per-slot barriers,
// the row view's MMA against B_r when it is rotated (G_R > 0) and the column
// view's MN-major MMA against B_c -- with quantizing epilogues.  A slot's four
// warps quantize the view held in it (quantize_tmem_row, the code path of the
// single-layout kernel); with G_R = 0 they also quantize the row view straight
// from the staged tile (quantize_smem_row) before releasing its stage.  The
// outputs equal those of two single-layout calls bit for bit: the same MMAs
// give the same rotated values and the same per-pair arithmetic follows.
// `reverse` walks the tiles from the last one back, so that a launch right
// after the pre-pass starts on the tiles the pre-pass read last (still in L2).

// Quantize row r of the staged 128 x 128 tile (two 64-column boxes, 128-byte
// swizzle): view row vrow, view columns vcol_base .. +127, no rotation.
template <int MODE>
__device__ __forceinline__ void quantize_smem_row(const uint8_t* tile, uint32_t r, const ScaleCtx& sc, PhiloxKey key,
                                                  int64_t vrow, int64_t vcol_base, int64_t vrows, int64_t vcols,
                                                  bool codes_aligned16, bool scales_aligned4, uint8_t* codes,
                                                  uint8_t* scales) {
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const int64_t vcol0 = vcol_base + 64 * h;
    const bool valid = vrow < vrows && vcol0 < vcols;
    const uint64_t e0 = static_cast<uint64_t>(vrow) * static_cast<uint64_t>(vcols) + static_cast<uint64_t>(vcol0);
    const uint8_t* rowp = tile + h * kBoxBytes + r * 128u;
    BlockOut o[4];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      // block a = columns 32p .. 32p+15 (16-byte chunks 4p, 4p+1), block b =
      // columns 32p+16 .. 32p+31 (chunks 4p+2, 4p+3)
      uint32_t wa[8], wb[8];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint4 ua = *reinterpret_cast<const uint4*>(rowp + (((4u * p + c) ^ (r & 7u)) << 4));
        const uint4 ub = *reinterpret_cast<const uint4*>(rowp + (((4u * p + 2u + c) ^ (r & 7u)) << 4));
        wa[4 * c] = ua.x; wa[4 * c + 1] = ua.y; wa[4 * c + 2] = ua.z; wa[4 * c + 3] = ua.w;
        wb[4 * c] = ub.x; wb[4 * c + 1] = ub.y; wb[4 * c + 2] = ub.z; wb[4 * c + 3] = ub.w;
      }
      float2 z[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float a0, a1, b0, b1;
        bf16x2_to_f32(wa[i], a0, a1);
        bf16x2_to_f32(wb[i], b0, b1);
        z[2 * i] = f2(a0, b0);
        z[2 * i + 1] = f2(a1, b1);
      }
      const PairRng rng{key, e0 + 32 * p, e0 + 32 * p + 16, 0u, 0u};
      quantize_pair<MODE>(z, sc, rng, o[2 * p], o[2 * p + 1]);
    }
    if (valid) store64(o, vrow, vcol0, vcols, codes, scales, codes_aligned16, scales_aligned4);
  }
}

// Tile k of this CTA (tiles blockIdx.x, blockIdx.x + gridDim.x, ...), or
// counted from the last tile back when `reverse` is set.
__device__ __forceinline__ uint32_t dual_tile_index(int64_t k, int64_t n_tiles, int reverse) {
  const int64_t t = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
  return static_cast<uint32_t>(reverse ? n_tiles - 1 - t : t);
}

struct DualQuantShared {
  uint64_t full[kDualStages];
  uint64_t sfree[kDualStages];
  uint64_t tfull[kDualSlots];
  uint64_t tfree[kDualSlots];
  uint32_t tmem_base;
  uint32_t issued_a;
  uint32_t issued_mma;
  int abort_flag;
  float4 scale_tbl[kMaxDualMembers][2][128];  // block-scale constants per E4M3 code: member, view
  ScaleCtx sc[kMaxDualMembers][2];             // each member's scale constants: row and column view
};
// 227 KB of shared memory per CTA on sm_100
static_assert(kDualDynSmem + sizeof(DualQuantShared) <= 227u * 1024u, "both-layout quantize shared memory");

#ifndef NVFP4_DUALQ_BAND_ROWS
#define NVFP4_DUALQ_BAND_ROWS 1
#endif

template <int MODE_R, int G_R, int MODE_C, int G_C, bool MULTI>
__global__ void __launch_bounds__(kDualThreads, 1)
dual_quantize_kernel(const __grid_constant__ DualGroup grp, uint64_t seed, int reverse) {
  static_assert(G_C > 0, "the column view is rotated on the tensor cores");
  constexpr int kViews = G_R != 0 ? 2 : 1;
  constexpr bool kRowFromSmem = G_R == 0;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(16) DualQuantShared sh;
  uint8_t* a_tiles = align_1024(dyn_smem);
  uint8_t* b_r = a_tiles + kDualStages * kTileBytes;
  uint8_t* b_c = b_r + kTileBytes;

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const PhiloxKey key = philox_key(seed);
  const uint32_t band = static_cast<uint32_t>(NVFP4_DUALQ_BAND_ROWS);
  const int64_t n_tiles = grp.n_tiles;
  const int64_t step = gridDim.x;
  const int64_t my_tiles = n_tiles > blockIdx.x ? (n_tiles - blockIdx.x + step - 1) / step : 0;

  if (tid == kDualProducerWarp * 32) {
    for (int s = 0; s < kDualStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sfree[s], kRowFromSmem ? 5 : 1);
    }
    for (int a = 0; a < kDualSlots; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], 4);
    }
    sh.issued_a = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kDualMmaWarp) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;
  if (warp != kDualProducerWarp) {
    const uint32_t bt = warp < kDualProducerWarp ? tid : tid - 32, nb = kDualThreads - 32;
    if constexpr (G_R != 0) build_hadamard_b<G_R>(b_r, key, bt, nb);
    build_hadamard_b<G_C>(b_c, key, bt, nb);
    fence_proxy_async_smem();
    asm volatile("bar.sync 2, %0;" ::"r"(nb) : "memory");
  }

  if (warp == kDualProducerWarp) {
    if (lane == 0) {
      grid_dependency_wait();
      for (int i = 0; i < grp.n; ++i) prefetch_tensormap(&grp.map[i]);
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = static_cast<int>(k % kDualStages);
        const uint32_t u = static_cast<uint32_t>(k / kDualStages);
        if (k >= kDualStages && !mbar_wait(&sh.sfree[s], (u - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&sh.abort_flag)) break;
        uint32_t rt, ct;
        const int mi = group_tile(grp, dual_tile_index(k, n_tiles, reverse), band, rt, ct);
        const int32_t x = static_cast<int32_t>(ct * kTile), y = static_cast<int32_t>(rt * kTile);
        mbar_arrive_expect_tx(&sh.full[s], kTileBytes);
        uint8_t* dst = a_tiles + s * kTileBytes;
        tma_load_2d(dst, &grp.map[mi], x, y, &sh.full[s]);
        tma_load_2d(dst + kBoxBytes, &grp.map[mi], x + 64, y, &sh.full[s]);
        sh.issued_a = (sh.issued_a & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
      }
    }
  } else if (warp == kDualMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc_r = idesc_bf16_f32(kTile, kTile, 0u);
      constexpr uint32_t idesc_c = idesc_bf16_f32(kTile, kTile, 1u);
      const uint32_t br_addr = smem_u32(b_r), bc_addr = smem_u32(b_c);
      int64_t j = 0;
      for (int64_t k = 0; k < my_tiles && !*reinterpret_cast<volatile int*>(&sh.abort_flag); ++k) {
        const int s = static_cast<int>(k % kDualStages);
        if (!mbar_wait(&sh.full[s], static_cast<uint32_t>(k / kDualStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        tc_fence_after_sync();
        const uint32_t a_addr = smem_u32(a_tiles + s * kTileBytes);
        bool ok = true;
#pragma unroll
        for (int v = 0; v < kViews; ++v) {
          const int a = static_cast<int>(j % kDualSlots);
          const uint32_t use = static_cast<uint32_t>(j / kDualSlots);
          ++j;
          if (use > 0 && !mbar_wait(&sh.tfree[a], (use - 1) & 1u)) {
            atomicExch(&sh.abort_flag, 1);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t d = tmem_base + a * kTile;
          if (kViews == 2 && v == 0) {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(br_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              umma_bf16(d, adesc, bdesc, idesc_r, kk > 0 ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_addr + kk * 2048, kBoxBytes, 1024);
              const uint64_t bdesc = smem_desc_sw128(bc_addr + (kk >> 2) * kBoxBytes + (kk & 3) * 32, 16, 1024);
              umma_bf16(d, adesc, bdesc, idesc_c, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&sh.tfull[a]);
          sh.issued_mma = (sh.issued_mma & ~(0x101u << a)) | (1u << a) | ((use & 1u) << (8 + a));
        }
        if (!ok) break;
        umma_commit(&sh.sfree[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const uint32_t q = warp & 3u, slot = warp >> 2;
    grid_dependency_wait();
    // every member's scale constants and tables, once per CTA
    for (int i = 0; i < grp.n; ++i) {
      const float s_r = global_scale_of<MODE_R>(*grp.m[i].amax_r), s_c = global_scale_of<MODE_C>(*grp.m[i].amax_c);
      build_scale_table(sh.scale_tbl[i][0], s_r, tid, kDualEpiWarps * 32);
      build_scale_table(sh.scale_tbl[i][1], s_c, tid, kDualEpiWarps * 32);
      if (tid == 0) {
        sh.sc[i][0] = make_scale_ctx<MODE_R>(*grp.m[i].amax_r);
        sh.sc[i][1] = make_scale_ctx<MODE_C>(*grp.m[i].amax_c);
        sh.sc[i][0].tbl = sh.scale_tbl[i][0];
        sh.sc[i][1].tbl = sh.scale_tbl[i][1];
        if (blockIdx.x == 0) {
          *grp.m[i].gscale_r = sh.sc[i][0].s_g;
          *grp.m[i].gscale_c = sh.sc[i][1].s_g;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(kDualEpiWarps * 32) : "memory");
    const int64_t n_acc = my_tiles * kViews;
    const uint32_t r_in_tile = 32u * q + lane;
    // a group of one (MULTI false): the member's constants once, before the
    // loop; a larger group: looked up for each tile's member
    const DualMember& m0 = grp.m[0];
    const ScaleCtx sc_r0 = MULTI ? ScaleCtx{} : sh.sc[0][0], sc_c0 = MULTI ? ScaleCtx{} : sh.sc[0][1];
    const bool r_codes16_0 = ((m0.cols / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(m0.codes_r) % 16) == 0;
    const bool r_scales4_0 = ((m0.cols / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(m0.scales_r) % 4) == 0;
    const bool c_codes16_0 = ((m0.rows / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(m0.codes_c) % 16) == 0;
    const bool c_scales4_0 = ((m0.rows / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(m0.scales_c) % 4) == 0;
    for (int64_t j = slot; j < n_acc; j += kDualSlots) {
      const int64_t k = j / kViews;
      const int v = static_cast<int>(j % kViews);
      uint32_t rt, ct;
      int mi = 0;
      if constexpr (MULTI) {
        mi = group_tile(grp, dual_tile_index(k, n_tiles, reverse), band, rt, ct);
      } else {
        const TileGrid tg{m0.n_rt, m0.n_ct, band};
        tg.coords(dual_tile_index(k, n_tiles, reverse), rt, ct);
      }
      const DualMember& mb = MULTI ? grp.m[mi] : m0;
      const int64_t rows = mb.rows, cols = mb.cols;
      const ScaleCtx sc_r = MULTI ? sh.sc[mi][0] : sc_r0, sc_c = MULTI ? sh.sc[mi][1] : sc_c0;
      uint8_t* const codes_r = mb.codes_r;
      uint8_t* const scales_r = mb.scales_r;
      uint8_t* const codes_c = mb.codes_c;
      uint8_t* const scales_c = mb.scales_c;
      // row view: rows x cols; column view: cols x rows
      const bool r_codes16 =
          MULTI ? ((cols / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(codes_r) % 16) == 0 : r_codes16_0;
      const bool r_scales4 =
          MULTI ? ((cols / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(scales_r) % 4) == 0 : r_scales4_0;
      const bool c_codes16 =
          MULTI ? ((rows / 2) % 16) == 0 && (reinterpret_cast<uintptr_t>(codes_c) % 16) == 0 : c_codes16_0;
      const bool c_scales4 =
          MULTI ? ((rows / 16) % 4) == 0 && (reinterpret_cast<uintptr_t>(scales_c) % 4) == 0 : c_scales4_0;
      const bool r_blocks8 = ((cols / 16) % 8) == 0, c_blocks8 = ((rows / 16) % 8) == 0;
      if constexpr (kRowFromSmem) {
        const int s = static_cast<int>(k % kDualStages);
        if (!mbar_wait(&sh.full[s], static_cast<uint32_t>(k / kDualStages) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        quantize_smem_row<MODE_R>(a_tiles + s * kTileBytes, r_in_tile, sc_r, key,
                                  static_cast<int64_t>(rt) * kTile + r_in_tile, static_cast<int64_t>(ct) * kTile, rows,
                                  cols, r_codes16, r_scales4, codes_r, scales_r);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.sfree[s]);
      }
      if (!mbar_wait(&sh.tfull[slot], static_cast<uint32_t>(j / kDualSlots) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      tc_fence_after_sync();
      const uint32_t base = tmem_base + ((32u * q) << 16) + slot * kTile;
      if constexpr (kViews == 2 && MODE_R == MODE_C && G_R == G_C) {
        // both views run the same code: one call site with the view's
        // parameters selected, so the epilogue is one copy of the code in
        // the instruction cache whichever view a warp holds
        const bool row = v == 0;
        quantize_tmem_row<MODE_C, G_C>(
            base, &sh.tfree[slot], row ? sc_r : sc_c, key,
            static_cast<int64_t>(row ? rt : ct) * kTile + r_in_tile, static_cast<int64_t>(row ? ct : rt) * kTile,
            row ? rows : cols, row ? cols : rows, row ? r_blocks8 : c_blocks8, row ? r_codes16 : c_codes16,
            row ? r_scales4 : c_scales4, row ? codes_r : codes_c, row ? scales_r : scales_c);
      } else if (kViews == 2 && v == 0) {
        if constexpr (G_R != 0)
          quantize_tmem_row<MODE_R, (G_R != 0 ? G_R : 16)>(
              base, &sh.tfree[slot], sc_r, key, static_cast<int64_t>(rt) * kTile + r_in_tile,
              static_cast<int64_t>(ct) * kTile, rows, cols, r_blocks8, r_codes16, r_scales4, codes_r, scales_r);
      } else {
        quantize_tmem_row<MODE_C, G_C>(base, &sh.tfree[slot], sc_c, key, static_cast<int64_t>(ct) * kTile + r_in_tile,
                                       static_cast<int64_t>(rt) * kTile, cols, rows, c_blocks8, c_codes16, c_scales4,
                                       codes_c, scales_c);
      }
    }
  }

  __syncthreads();
  const bool failed = *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
  if (failed) {
    if (tid == kDualProducerWarp * 32)
      for (int s = 0; s < kDualStages; ++s)
        if ((sh.issued_a >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_a >> (8 + s)) & 1u);
    if (tid == kDualMmaWarp * 32)
      for (int a = 0; a < kDualSlots; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
    if (tid < static_cast<uint32_t>(grp.n)) {
      *grp.m[tid].gscale_r = __uint_as_float(0x7FC00000u);
      *grp.m[tid].gscale_c = __uint_as_float(0x7FC00000u);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kDualMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, 512);
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
  // one CTA per SM: it allocates all of tensor memory
  constexpr int threads = Shape<MODE, KIND>::threads;
  LaunchGeom geom;
  cudaError_t e = launch_geometry(kernel, threads, kDynSmem, 1, &geom);
  if (e != cudaSuccess) return e;
  const int sms = geom.sms, per_sm = geom.per_sm;
  const int64_t n_tiles = ((a.rows + kTile - 1) / kTile) * ((a.cols + kTile - 1) / kTile);
  int64_t grid = n_tiles < int64_t(sms) * per_sm ? n_tiles : int64_t(sms) * per_sm;
  if (grid == 0) {
    if (KIND == kAmax) return cudaSuccess;
    grid = 1;
  }
  return launch_overlapped(kernel, static_cast<unsigned>(grid), threads, kDynSmem, a.stream, map, a.rows, a.cols,
                           a.seed, a.amax, reinterpret_cast<unsigned int*>(a.amax_accum), a.codes, a.scales, a.gscale,
                           zout);
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
  if (((a.rows + kTile - 1) / kTile) * ((a.cols + kTile - 1) / kTile) >= (int64_t(1) << 31)) return false;
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
    case kScaleSearch: return dispatch<kScaleSearch, kQuantize>(a, nullptr);
    case kMXFP4: return dispatch<kMXFP4, kQuantize>(a, nullptr);
    case kNVINT4: return dispatch<kNVINT4, kQuantize>(a, nullptr);
    case kNVFP3: return dispatch<kNVFP3, kQuantize>(a, nullptr);
    case kNVINT3: return dispatch<kNVINT3, kQuantize>(a, nullptr);
    case kIF3: return dispatch<kIF3, kQuantize>(a, nullptr);
    case kMXFP3: return dispatch<kMXFP3, kQuantize>(a, nullptr);
    default: return cudaErrorInvalidValue;
  }
}

bool dual_mma_path_applies(const void* x, int64_t rows, int64_t cols, int64_t ld) {
  QuantArgs a{x, rows, cols, ld, 0, kRTN, 128, 0, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};
  return mma_path_applies(a);
}

namespace {

// A group's kernel parameter from up to kMaxDualMembers non-empty tensors;
// false if a tensor map cannot be encoded.
bool make_group(DualGroup& g, int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                const int64_t* ld) {
  std::memset(&g, 0, sizeof(g));
  g.n = n;
  int64_t t0 = 0;
  for (int i = 0; i < n; ++i) {
    if (!make_map(&g.map[i], x[i], rows[i], cols[i], ld[i])) return false;
    DualMember& m = g.m[i];
    m.rows = rows[i];
    m.cols = cols[i];
    m.tile0 = t0;
    m.n_rt = static_cast<uint32_t>((rows[i] + kTile - 1) / kTile);
    m.n_ct = static_cast<uint32_t>((cols[i] + kTile - 1) / kTile);
    t0 += static_cast<int64_t>(m.n_rt) * m.n_ct;
  }
  g.n_tiles = t0;
  return true;
}

}  // namespace

cudaError_t launch_amax_dual_ring(int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                                  const int64_t* ld, int g_r, int g_c, uint64_t seed, float* const* amax_r,
                                  float* const* amax_c, cudaStream_t stream) {
  if (n < 1 || n > kMaxDualMembers) return cudaErrorInvalidValue;
  DualGroup g;
  if (!make_group(g, n, x, rows, cols, ld)) return cudaErrorInvalidValue;
  for (int i = 0; i < n; ++i) {
    g.m[i].max_r = reinterpret_cast<unsigned int*>(amax_r[i]);
    g.m[i].max_c = reinterpret_cast<unsigned int*>(amax_c[i]);
  }
  LaunchGeom geom;
  cudaError_t e = launch_geometry(dual_amax_kernel, kDualThreads, kDualDynSmem, 1, &geom);
  if (e != cudaSuccess) return e;
  const int64_t grid = g.n_tiles < int64_t(geom.sms) ? g.n_tiles : int64_t(geom.sms);
  if (grid == 0) return cudaSuccess;
  return launch_overlapped(dual_amax_kernel, static_cast<unsigned>(grid), kDualThreads, kDualDynSmem, stream, g, seed,
                           g_r, g_c);
}

cudaError_t launch_amax_dual_mma(const void* x, int64_t rows, int64_t cols, int64_t ld, int g_r, int g_c,
                                 uint64_t seed, float* amax_r, float* amax_c, cudaStream_t stream) {
  // the row view straight from the tile: the slot ring, a group of one
  if (g_r == 0) return launch_amax_dual_ring(1, &x, &rows, &cols, &ld, g_r, g_c, seed, &amax_r, &amax_c, stream);
  CUtensorMap map;
  if (!make_map(&map, x, rows, cols, ld)) return cudaErrorInvalidValue;
  LaunchGeom geom;
  if (g_r == g_c) {
    // both views rotated with one group size: pairs of tiles per MMA
    cudaError_t e = launch_geometry(dual_amax_pair_kernel, kPairThreads, kPairDynSmem, 1, &geom);
    if (e != cudaSuccess) return e;
    const int64_t n_tiles = ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile);
    const int64_t grid = n_tiles < int64_t(geom.sms) ? n_tiles : int64_t(geom.sms);
    if (grid == 0) return cudaSuccess;
    return launch_overlapped(dual_amax_pair_kernel, static_cast<unsigned>(grid), kPairThreads, kPairDynSmem, stream,
                             map, rows, cols, seed, g_r, reinterpret_cast<unsigned int*>(amax_r),
                             reinterpret_cast<unsigned int*>(amax_c));
  }
  // both views rotated, different group sizes: the group kernel
  cudaError_t e = launch_geometry(dual_amax_group_kernel, kGrpThreads, kGrpDynSmem, 1, &geom);
  if (e != cudaSuccess) return e;
  const int64_t n_tiles = ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile);
  const int64_t grid = n_tiles < int64_t(geom.sms) ? n_tiles : int64_t(geom.sms);
  if (grid == 0) return cudaSuccess;
  return launch_overlapped(dual_amax_group_kernel, static_cast<unsigned>(grid), kGrpThreads, kGrpDynSmem, stream, map,
                           rows, cols, seed, g_r, g_c, reinterpret_cast<unsigned int*>(amax_r),
                           reinterpret_cast<unsigned int*>(amax_c));
}

namespace {

// One launch for members a[0 .. n-1] (the same modes, groups, seed, stream
// and tile order; each fused).
template <int MODE_R, int G_R, int MODE_C, int G_C>
cudaError_t launch_dual_quantize_t(const DualQuantArgs* a, int n) {
  const void* x[kMaxDualMembers];
  int64_t rows[kMaxDualMembers], cols[kMaxDualMembers], ld[kMaxDualMembers];
  for (int i = 0; i < n; ++i) {
    x[i] = a[i].x;
    rows[i] = a[i].rows;
    cols[i] = a[i].cols;
    ld[i] = a[i].ld;
  }
  DualGroup g;
  if (!make_group(g, n, x, rows, cols, ld)) return cudaErrorInvalidValue;
  for (int i = 0; i < n; ++i) {
    DualMember& m = g.m[i];
    m.amax_r = a[i].amax_row;
    m.amax_c = a[i].amax_col;
    m.codes_r = a[i].codes_row;
    m.scales_r = a[i].scales_row;
    m.gscale_r = a[i].gscale_row;
    m.codes_c = a[i].codes_col;
    m.scales_c = a[i].scales_col;
    m.gscale_c = a[i].gscale_col;
  }
  auto kernel = n > 1 ? dual_quantize_kernel<MODE_R, G_R, MODE_C, G_C, true>
                      : dual_quantize_kernel<MODE_R, G_R, MODE_C, G_C, false>;
  LaunchGeom geom;
  cudaError_t e = launch_geometry(kernel, kDualThreads, kDualDynSmem, 1, &geom);
  if (e != cudaSuccess) return e;
  const int64_t grid = g.n_tiles < int64_t(geom.sms) ? g.n_tiles : int64_t(geom.sms);
  if (grid == 0) return cudaSuccess;
  return launch_overlapped(kernel, static_cast<unsigned>(grid), kDualThreads, kDualDynSmem, a[0].stream, g, a[0].seed,
                           a[0].reverse);
}

template <int G>
cudaError_t dispatch_dual_quantize(const DualQuantArgs* a, int n) {
  if (a[0].mode_row == kRTN && a[0].rht_group_row == 0) return launch_dual_quantize_t<kRTN, 0, kMSEDEN, G>(a, n);
  return launch_dual_quantize_t<kMSEDEN, G, kMSEDEN, G>(a, n);
}

}  // namespace

bool dual_quantize_fused(const DualQuantArgs& a) {
  if (!dual_mma_path_applies(a.x, a.rows, a.cols, a.ld)) return false;
  const int g = a.rht_group_col;
  if (a.mode_col != kMSEDEN || (g != 16 && g != 32 && g != 64 && g != 128)) return false;
  if (a.mode_row == kRTN && a.rht_group_row == 0) return true;
  return a.mode_row == kMSEDEN && a.rht_group_row == g;
}

cudaError_t launch_quantize_dual_group(const DualQuantArgs* a, int n) {
  if (n < 1 || n > kMaxDualMembers) return cudaErrorInvalidValue;
  switch (a[0].rht_group_col) {
    case 16: return dispatch_dual_quantize<16>(a, n);
    case 32: return dispatch_dual_quantize<32>(a, n);
    case 64: return dispatch_dual_quantize<64>(a, n);
    case 128: return dispatch_dual_quantize<128>(a, n);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_quantize_dual_mma(const DualQuantArgs& a) { return launch_quantize_dual_group(&a, 1); }

}  // namespace nvfp4

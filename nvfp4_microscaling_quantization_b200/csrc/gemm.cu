// gemm.cu -- the NVFP4 GEMM that consumes the quantizer's output on the
// sm_100a block-scaled tensor cores.
//
//   D[m][n] = gA * gB * sum_k (qA[m][k] * SA[m][k/16]) * (qB[n][k] * SB[n][k/16])
//
// qA, qB are E2M1 codes packed two per byte (element 2j in the low nibble),
// SA, SB their E4M3 block scales stored row-major ([rows][K/16] bytes), and
// gA, gB the FP32 tensor scales: exactly what nvfp4_quantize writes for an
// M x K (row-wise, or the transposed view of a K x M tensor) and an N x K
// operand.  Every GEMM of a fully-NVFP4 linear layer's training step takes
// this form (Quartet II article, sections "Quantisierung im
// Vorwaertsdurchlauf" and "... Rueckwaertsdurchlauf": Y = X W^T, dX = dY W,
// dW = dY^T X, each operand quantized along the reduction dimension; the
// Quartet II record's abstract: NVFP4 GEMMs in Blackwell hardware).
//
// Design (one persistent CTA per SM, 10 warps):
//   warp 0      TMA producer: 128 x 256 E2M1 tiles of A and B (128 bytes a
//               row, 128-byte swizzle) and their 128 x 16 scale bytes into
//               a 6-stage shared-memory ring;
//   warp 1      allocates all 512 tensor-memory columns; one thread issues
//               tcgen05.mma kind::mxf4nvf4 (M = N = 128, K = 64, UE4M3 scale
//               vector of 4 per row) -- four per K tile -- into one of two
//               128-column fp32 accumulators;
//   warps 2..5  scale-factor writers: move the stage's scale bytes from
//               shared memory into the stage's tensor-memory scale columns in
//               the layout the MMA reads (row 32h + l of a K step in byte f of
//               column 4 * step + h, lane l of every lane quarter);
//   warps 6..9  epilogue: drain an accumulator (tcgen05.ld), multiply by
//               gA * gB, store fp32 or bf16 rows of D, release the
//               accumulator, so the next tile's MMAs overlap the stores.
// Scale factors go to tensor memory through registers, so the GEMM reads the
// quantizer's row-major scale layout as it is: no reordered copy of the
// scales is needed in HBM.
//
// Every wait is bounded (tma_pipeline.cuh); a CTA whose wait runs out stops,
// lets its loads and MMAs in flight finish, and writes NaN to D[0][0].

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "kernels.h"
#include "launch_config.h"
#include "tcgen05.cuh"
#include "tma_pipeline.cuh"

namespace nvfp4 {
namespace {

constexpr int kGBM = 128;                        // output tile rows
constexpr int kGBK = 256;                        // K elements per stage = 128 bytes of E2M1 a row
constexpr uint32_t kGOpBytes = kGBM * kGBK / 2;  // 16 KB of A codes per stage
constexpr uint32_t kGSfBytes = kGBM * (kGBK / 16);  // 2 KB of A scale bytes per stage
constexpr uint32_t kGTmemCols = 512;
constexpr int kGProducerWarp = 0, kGMmaWarp = 1, kGEpiWarp0 = 6;  // scale writers: warps 2..5
static_assert(kGEpiWarp0 % 2 == 0, "each run of four epilogue warps covers the four lane quarters");

// The shape of one instance: output tiles of 128 x BN.
//   BN = 128: two 128-column accumulators (the next tile's MMAs overlap the
//             epilogue), six stages of 36 KB, four epilogue warps;
//   BN = 256: one 256-column accumulator (A is read once for twice the
//             columns: 25% fewer operand bytes per FLOP from L2), four
//             stages of 54 KB, eight epilogue warps (two per lane quarter,
//             128 columns each) to drain it quickly.
// Scale columns per stage: A 4 K steps x 4 columns, B 4 K steps x BN/32.
template <int BN>
struct GemmShape {
  static constexpr int accum = BN == 128 ? 2 : 1;
  static constexpr int stages = BN == 128 ? 6 : 4;
  static constexpr uint32_t b_bytes = BN * kGBK / 2;
  static constexpr uint32_t sfb_bytes = BN * (kGBK / 16);
  static constexpr uint32_t stage_bytes = kGOpBytes + b_bytes + kGSfBytes + sfb_bytes;  // a multiple of 1024
  static constexpr uint32_t sfb_cols_per_step = BN / 32;
  static constexpr uint32_t sf_cols = 16 + 4 * sfb_cols_per_step;
  static constexpr uint32_t sf_base = accum * BN;  // scale columns follow the accumulators
  static constexpr int epi_warps = 4 * (BN / 128);
  static constexpr int threads = (kGEpiWarp0 + epi_warps) * 32;
  static constexpr size_t dyn_smem = stages * stage_bytes + 1024;
  static_assert(sf_base + stages * sf_cols <= kGTmemCols, "tensor memory");
  static_assert(stage_bytes % 1024 == 0, "stage alignment");
};
constexpr int kGMaxStages = 6, kGMaxAccum = 2;

struct GemmShared {
  uint64_t full[kGMaxStages];     // A and B codes and scale bytes of the stage landed
  uint64_t sf_full[kGMaxStages];  // the stage's scale factors are in tensor memory (4 writer warps)
  uint64_t empty[kGMaxStages];    // the MMAs that read the stage completed
  uint64_t tfull[kGMaxAccum];     // accumulator holds a finished tile
  uint64_t tfree[kGMaxAccum];     // epilogue drained the accumulator (all epilogue warps)
  uint32_t tmem_base;
  uint32_t issued_ab;          // per stage: a load in flight (bit s) and its phase (bit 8 + s)
  uint32_t issued_mma;         // per accumulator: a commit pending (bit a) and its phase (bit 8 + a)
  int abort_flag;
};

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// One 32-byte global store (sm_100 st.global.v8.b32); dst 32-byte aligned.
__device__ __forceinline__ void st_global_32B(void* dst, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ bool aborted(GemmShared& sh) {
  return *reinterpret_cast<volatile int*>(&sh.abort_flag) != 0;
}

template <int OUT_BF16, int BN>
__global__ void __launch_bounds__(GemmShape<BN>::threads, 1)
nvfp4_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                  const __grid_constant__ CUtensorMap tmap_sa, const __grid_constant__ CUtensorMap tmap_sb,
                  const float* __restrict__ a_gscale, const float* __restrict__ b_gscale, int64_t m, int64_t n,
                  int64_t k, void* __restrict__ d, int64_t ldd) {
  using GS = GemmShape<BN>;
  constexpr int kGStages = GS::stages, kGAccum = GS::accum;
  constexpr uint32_t kGStageBytes = GS::stage_bytes, kGSfCols = GS::sf_cols, kGSfBase = GS::sf_base;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ __align__(8) GemmShared sh;
  uint8_t* tiles = align_1024(dyn_smem);

  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const int64_t n_tn = n / BN;
  const int64_t n_tiles = (m / kGBM) * n_tn;
  const int kt_count = static_cast<int>(k / kGBK);
  const int64_t step = gridDim.x;

  if (tid == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&sh.full[s], 1);
      mbar_init(&sh.sf_full[s], 4);
      mbar_init(&sh.empty[s], 1);
    }
    for (int a = 0; a < kGAccum; ++a) {
      mbar_init(&sh.tfull[a], 1);
      mbar_init(&sh.tfree[a], GS::epi_warps);
    }
    sh.issued_ab = 0;
    sh.issued_mma = 0;
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kGMmaWarp) {
    tmem_alloc(&sh.tmem_base, kGTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  allow_dependent_launch();
  const uint32_t tmem_base = sh.tmem_base;

  if (warp == kGProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      grid_dependency_wait();
      prefetch_tensormap(&tmap_a);
      prefetch_tensormap(&tmap_b);
      prefetch_tensormap(&tmap_sa);
      prefetch_tensormap(&tmap_sb);
      uint32_t it = 0;
      for (int64_t t = blockIdx.x; t < n_tiles && !aborted(sh); t += step) {
        const int32_t ya = static_cast<int32_t>((t / n_tn) * kGBM), yb = static_cast<int32_t>((t % n_tn) * BN);
        for (int kt = 0; kt < kt_count; ++kt, ++it) {
          const uint32_t s = it % kGStages, u = it / kGStages;
          if (it >= kGStages && !mbar_wait(&sh.empty[s], (u - 1) & 1u)) {
            atomicExch(&sh.abort_flag, 1);
            break;
          }
          if (aborted(sh)) break;
          uint8_t* dst = tiles + s * kGStageBytes;
          // codes (x in bytes, 128 per K tile), then the scale bytes (x = 16
          // per K tile): both multiples of 16.  Issuing the 16-byte scale rows
          // ahead of the codes measured slower.
          mbar_arrive_expect_tx(&sh.full[s], kGStageBytes);
          tma_load_2d(dst, &tmap_a, kt * (kGBK / 2), ya, &sh.full[s]);
          tma_load_2d(dst + kGOpBytes, &tmap_b, kt * (kGBK / 2), yb, &sh.full[s]);
          tma_load_2d(dst + kGOpBytes + GS::b_bytes, &tmap_sa, kt * (kGBK / 16), ya, &sh.full[s]);
          tma_load_2d(dst + kGOpBytes + GS::b_bytes + kGSfBytes, &tmap_sb, kt * (kGBK / 16), yb, &sh.full[s]);
          sh.issued_ab = (sh.issued_ab & ~(0x101u << s)) | (1u << s) | ((u & 1u) << (8 + s));
        }
      }
    }
  } else if (warp == kGMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_nvfp4_f32(kGBM, BN);
      uint32_t it = 0, tile = 0;
      for (int64_t t = blockIdx.x; t < n_tiles && !aborted(sh); t += step, ++tile) {
        const uint32_t a = tile % kGAccum, ua = tile / kGAccum;
        if (tile >= kGAccum && !mbar_wait(&sh.tfree[a], (ua - 1) & 1u)) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
        tc_fence_after_sync();
        bool ok = true;
        for (int kt = 0; kt < kt_count; ++kt, ++it) {
          const uint32_t s = it % kGStages, u = it / kGStages;
          if (!mbar_wait(&sh.full[s], u & 1u) || !mbar_wait(&sh.sf_full[s], u & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_u32(tiles + s * kGStageBytes), b_addr = a_addr + kGOpBytes;
          const uint32_t sf = tmem_base + kGSfBase + s * kGSfCols;
#pragma unroll
          for (int j = 0; j < kGBK / 64; ++j) {
            // K step j: 32 bytes further along each 128-byte swizzled row
            const uint64_t adesc = smem_desc_sw128(a_addr + j * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + j * 32, 16, 1024);
            umma_nvfp4(tmem_base + a * BN, adesc, bdesc, idesc, sf + 4 * j, sf + 16 + GS::sfb_cols_per_step * j,
                       (kt | j) != 0 ? 1u : 0u);
          }
          umma_commit(&sh.empty[s]);
        }
        // committed even after a failed wait, so the accumulator's phase is
        // tracked for the drain below
        umma_commit(&sh.tfull[a]);
        sh.issued_mma = (sh.issued_mma & ~(0x101u << a)) | (1u << a) | ((ua & 1u) << (8 + a));
        if (!ok) {
          atomicExch(&sh.abort_flag, 1);
          break;
        }
      }
    }
  } else if (warp < kGEpiWarp0) {
    // ------------------------------------------------- scale-factor writers
    // warp q = warp % 4 fills lane quarter q; its thread l carries rows l,
    // 32 + l, 64 + l, 96 + l of the tile, 16 scale bytes (one K tile) each.
    // The stage landing (full) also means the MMAs of the stage's previous
    // use have completed (the producer waited for them before loading), so
    // its scale columns are free.
    const uint32_t q = warp & 3u;
    uint32_t it = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < n_tiles && ok && !aborted(sh); t += step) {
      for (int kt = 0; kt < kt_count; ++kt, ++it) {
        const uint32_t s = it % kGStages, u = it / kGStages;
        if (!mbar_wait(&sh.full[s], u & 1u)) {
          ok = false;
          break;
        }
        const uint4* sa = reinterpret_cast<const uint4*>(tiles + s * kGStageBytes + kGOpBytes + GS::b_bytes);
        const uint4* sb = sa + kGBM;
        // A: column 4j + h holds the four factors of K step j of row 32h + l;
        // B: column (BN/32) j + h likewise for its BN rows
        constexpr int kHb = BN / 32;
        uint32_t ca[16], cb[4 * kHb];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint4 va = sa[32 * h + lane];
          ca[h] = va.x, ca[4 + h] = va.y, ca[8 + h] = va.z, ca[12 + h] = va.w;
        }
#pragma unroll
        for (int h = 0; h < kHb; ++h) {
          const uint4 vb = sb[32 * h + lane];
          cb[h] = vb.x, cb[kHb + h] = vb.y, cb[2 * kHb + h] = vb.z, cb[3 * kHb + h] = vb.w;
        }
        tc_fence_after_sync();
        const uint32_t sf = tmem_base + ((32u * q) << 16) + kGSfBase + s * kGSfCols;
        tmem_st16(sf, ca);
        tmem_st_wait();
#pragma unroll
        for (int c = 0; c < 4 * kHb; c += 16) {
          uint32_t part[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) part[i] = cb[c + i];
          tmem_st16(sf + 16 + c, part);
          tmem_st_wait();
        }
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.sf_full[s]);
      }
    }
    if (!ok) atomicExch(&sh.abort_flag, 1);
  } else {
    // ------------------------------------------------------------ epilogue
    // epilogue warp e = warp - kGEpiWarp0 reads the lane quarter tensor memory
    // allows it (warp % 4) and columns 128 (e / 4) .. +127: the epilogue warps
    // start at a multiple of four minus two, so each group of four consecutive
    // warps covers every lane quarter once
    const uint32_t e = warp - kGEpiWarp0, q = warp & 3u, c_begin = 128u * (e >> 2);
    grid_dependency_wait();
    const float gab = __fmul_rn(*a_gscale, *b_gscale);
    // 32-byte stores need D and its row pitch 32-byte aligned (one test for the launch)
    const bool wide_stores =
        ((reinterpret_cast<uintptr_t>(d) | static_cast<uintptr_t>(ldd * (OUT_BF16 ? 2 : 4))) & 31u) == 0;
    uint32_t tile = 0;
    for (int64_t t = blockIdx.x; t < n_tiles; t += step, ++tile) {
      const uint32_t a = tile % kGAccum;
      if (!mbar_wait(&sh.tfull[a], (tile / kGAccum) & 1u)) {
        atomicExch(&sh.abort_flag, 1);
        break;
      }
      if (aborted(sh)) break;
      tc_fence_after_sync();
      const int64_t row = (t / n_tn) * kGBM + 32 * q + lane, col0 = (t % n_tn) * BN;
      // all 128 columns of this warp's part in flight at once, one wait, then
      // the accumulator is released before the conversion and the stores, so
      // the next tile's MMAs overlap them
      uint32_t r[4][32];
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_ld32_nowait(tmem_base + ((32u * q) << 16) + a * BN + c_begin + 32 * c4, r[c4]);
      tmem_ld_wait();
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) tmem_regs_after_wait(r[c4]);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.tfree[a]);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {
        const uint32_t c = c_begin + 32u * c4;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[c4][i]);
        // each thread writes its own row: 32-byte stores fill whole L2 sectors
        // (half the store instructions and sector writes of 16-byte ones)
        if constexpr (OUT_BF16) {
          uint32_t w[16];
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(v[2 * k2], gab), __fmul_rn(v[2 * k2 + 1], gab));
            w[k2] = *reinterpret_cast<const uint32_t*>(&p);
          }
          uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<__nv_bfloat16*>(d) + row * ldd + col0 + c);
          if (wide_stores) {
            st_global_32B(dst, w);
            st_global_32B(dst + 32, w + 8);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              reinterpret_cast<uint4*>(dst)[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        } else {
          uint8_t* dst = reinterpret_cast<uint8_t*>(static_cast<float*>(d) + row * ldd + col0 + c);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) w[j] = __float_as_uint(__fmul_rn(v[8 * i + j], gab));
            if (wide_stores) {
              st_global_32B(dst + 32 * i, w);
            } else {
              reinterpret_cast<uint4*>(dst)[2 * i] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[2 * i + 1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
      }
    }
  }

  __syncthreads();
  const bool failed = aborted(sh);
  if (failed) {
    // let every load and MMA still in flight finish before the CTA lets go
    if (tid == kGProducerWarp * 32)
      for (int s = 0; s < kGStages; ++s)
        if ((sh.issued_ab >> s) & 1u) mbar_wait(&sh.full[s], (sh.issued_ab >> (8 + s)) & 1u);
    if (tid == kGMmaWarp * 32)
      for (int a = 0; a < kGAccum; ++a)
        if ((sh.issued_mma >> a) & 1u) mbar_wait(&sh.tfull[a], (sh.issued_mma >> (8 + a)) & 1u);
    if (tid == 0) {
      if (OUT_BF16)
        *static_cast<uint16_t*>(d) = 0x7FC0u;
      else
        *static_cast<uint32_t*>(d) = 0x7FC00000u;
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kGMmaWarp) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, kGTmemCols);
  }
}

using EncodeTiledFn = PFN_cuTensorMapEncodeTiled_v12000;

EncodeTiledFn gemm_encode_fn() {
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

// rows x (k / 2) bytes of packed E2M1, boxes of 128 bytes x box_rows rows.
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t k, uint32_t box_rows) {
  EncodeTiledFn fn = gemm_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 2)};
  cuuint32_t box[2] = {kGBK / 2, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rows x (k / 16) scale bytes, boxes of 16 bytes x box_rows rows (no swizzle).
bool make_scales_map(CUtensorMap* map, const uint8_t* scales, int64_t rows, int64_t k, uint32_t box_rows) {
  EncodeTiledFn fn = gemm_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(k / 16), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(k / 16)};
  cuuint32_t box[2] = {kGBK / 16, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(scales), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int OUT_BF16, int BN>
cudaError_t launch_gemm_t(const GemmArgs& g) {
  using GS = GemmShape<BN>;
  CUtensorMap ma, mb, msa, msb;
  if (!make_codes_map(&ma, g.a_codes, g.m, g.k, kGBM) || !make_codes_map(&mb, g.b_codes, g.n, g.k, BN) ||
      !make_scales_map(&msa, g.a_scales, g.m, g.k, kGBM) || !make_scales_map(&msb, g.b_scales, g.n, g.k, BN))
    return cudaErrorInvalidValue;
  auto kernel = nvfp4_gemm_kernel<OUT_BF16, BN>;
  LaunchGeom geom;
  const cudaError_t e = launch_geometry(kernel, GS::threads, GS::dyn_smem, 1, &geom);
  if (e != cudaSuccess) return e;
  const int sms = geom.sms;
  const int64_t n_tiles = (g.m / kGBM) * (g.n / BN);
  const int64_t grid = n_tiles < sms ? n_tiles : sms;
  if (grid == 0) return cudaSuccess;
  return launch_overlapped(kernel, static_cast<unsigned>(grid), GS::threads, GS::dyn_smem, g.stream, ma, mb, msa,
                           msb, g.a_gscale, g.b_gscale, g.m, g.n, g.k, g.d, g.ldd);
}

}  // namespace

bool gemm_available() { return gemm_encode_fn() != nullptr; }

// 128 x 256 tiles where n allows (the default), else 128 x 128; g.tile_n
// forces one (128 or 256) for tests.
cudaError_t launch_gemm(const GemmArgs& g) {
  const bool wide = g.tile_n == 256 || (g.tile_n == 0 && g.n % 256 == 0);
  if (wide) return g.out_bf16 ? launch_gemm_t<1, 256>(g) : launch_gemm_t<0, 256>(g);
  return g.out_bf16 ? launch_gemm_t<1, 128>(g) : launch_gemm_t<0, 128>(g);
}

}  // namespace nvfp4

// kernels.h -- internal launcher interface between the C ABI (api.cu) and the
// kernel translation units.  Not installed; the public interface is
// include/nvfp4.h.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

struct QuantArgs {
  const void* x;          // bf16 rows x cols, leading dimension ld
  int64_t rows, cols, ld;
  int layout;             // 0 row-wise, 1 transposed
  int mode;               // nvfp4_mode
  int rht_group;          // 0, 16, 32, 64, 128
  uint64_t seed;
  const float* amax;      // tensor amax (quantize)
  void* amax_accum;       // zeroed 32-bit word receiving the amax bits (pre-pass)
  uint8_t* codes;
  uint8_t* scales;
  float* gscale;
  cudaStream_t stream;
};

struct DequantArgs {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* gscale;
  int64_t vrows, vcols;
  int mode, rht_group;
  uint64_t seed;
  int inverse_rht;
  float* out;
  cudaStream_t stream;
};

struct RhtArgs {
  const void* in;
  int in_dtype;           // 0 bf16, 1 fp32
  int64_t rows, cols, ld;
  int layout, rht_group;
  uint64_t seed;
  int inverse;
  float* out;
  cudaStream_t stream;
};

cudaError_t launch_amax(const QuantArgs& a);
cudaError_t launch_quantize(const QuantArgs& a);

// The TMA-tiled kernels (quantize_tma.cu) take every shape they can tile;
// launch_amax / launch_quantize route there and fall back to the one-block-
// per-thread kernels for the rest (narrow or short tensors).
bool tma_path_applies(const QuantArgs& a);
cudaError_t launch_amax_tma(const QuantArgs& a);
cudaError_t launch_quantize_tma(const QuantArgs& a);

// With a rotation (g > 0) and both dimensions at least 128, the rotation runs
// on the tensor cores (rotate_mma.cu); launch_rotate_mma writes the rotated
// view as dense fp32 (the forward nvfp4_rht of a bf16 tensor).
bool mma_path_applies(const QuantArgs& a);
cudaError_t launch_amax_mma(const QuantArgs& a);
cudaError_t launch_quantize_mma(const QuantArgs& a);
cudaError_t launch_rotate_mma(const QuantArgs& a, float* zout);

// Both layouts' tensor amax from one read (rotate_mma.cu): row-wise view with
// rotation group g_r, transposed view with g_c (0 = no rotation).  amax_r and
// amax_c are zeroed 32-bit accumulators.  Applies where the single-layout
// tensor-core path does (both dimensions >= 128, 16-byte aligned rows).
// Tensors one both-layout launch can take at once (a group: the same rotation
// groups, modes and seed for every member).
constexpr int kMaxDualMembers = 4;

bool dual_mma_path_applies(const void* x, int64_t rows, int64_t cols, int64_t ld);
// Both-layout pre-pass of n (1 .. kMaxDualMembers) non-empty tensors whose row
// view is not rotated (g_r = 0), in one launch of the slot-ring kernel.
cudaError_t launch_amax_dual_ring(int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                                  const int64_t* ld, int g_r, int g_c, uint64_t seed, float* const* amax_r,
                                  float* const* amax_c, cudaStream_t stream);
cudaError_t launch_amax_dual_mma(const void* x, int64_t rows, int64_t cols, int64_t ld, int g_r, int g_c,
                                 uint64_t seed, float* amax_r, float* amax_c, cudaStream_t stream);
cudaError_t launch_dequantize(const DequantArgs& a);

// Both layouts' codes and scales from one read of X (rotate_mma.cu), given
// both tensor amaxes.  The fused kernel takes the mode pairs of a fully-NVFP4
// linear layer's operands: row view RTN without rotation + column view
// MS-EDEN with group g (the forward operands X, W re-quantized for the
// backward pass), and MS-EDEN with group g in both views (the output
// gradient dY); dual_quantize_fused says whether it applies.
struct DualQuantArgs {
  const void* x;
  int64_t rows, cols, ld;
  int mode_row, rht_group_row, mode_col, rht_group_col;
  uint64_t seed;
  const float* amax_row;
  const float* amax_col;
  uint8_t* codes_row;
  uint8_t* scales_row;
  float* gscale_row;
  uint8_t* codes_col;
  uint8_t* scales_col;
  float* gscale_col;
  int reverse;            // walk the tiles from the last one back
  cudaStream_t stream;
};
bool dual_quantize_fused(const DualQuantArgs& a);
cudaError_t launch_quantize_dual_mma(const DualQuantArgs& a);
// One launch for a[0 .. n-1] (n <= kMaxDualMembers, each non-empty and fused,
// all with a[0]'s modes, groups, seed, tile order and stream).
cudaError_t launch_quantize_dual_group(const DualQuantArgs* a, int n);

// D = gA gB A B^T from two quantizer outputs (gemm.cu); shapes checked by the
// caller: m, n multiples of 128, k of 256, 16-byte aligned codes, scales, D rows.
struct GemmArgs {
  const uint8_t* a_codes;   // m x k/2
  const uint8_t* a_scales;  // m x k/16
  const float* a_gscale;
  const uint8_t* b_codes;   // n x k/2
  const uint8_t* b_scales;  // n x k/16
  const float* b_gscale;
  int64_t m, n, k;
  int out_bf16;
  void* d;                  // m rows, leading dimension ldd (elements)
  int64_t ldd;
  cudaStream_t stream;
  int tile_n;               // 0: 256-column tiles when n % 256 == 0, else 128; 128 or 256 forces one
};
bool gemm_available();
cudaError_t launch_gemm(const GemmArgs& g);
cudaError_t launch_rht(const RhtArgs& a);
// Packed 3-bit storage (pack3.cu): `blocks` 16-element blocks of nibble codes
// (8 bytes each) <-> 6 bytes each; scales copied, or for MX (mx != 0) one
// byte per block pair.
cudaError_t launch_pack3(const uint8_t* codes, const uint8_t* scales, int64_t blocks, int mx, uint8_t* pcodes,
                         uint8_t* pscales, cudaStream_t stream);
cudaError_t launch_unpack3(const uint8_t* pcodes, const uint8_t* pscales, int64_t blocks, int mx, uint8_t* codes,
                           uint8_t* scales, cudaStream_t stream);
cudaError_t launch_encode_e2m1(const float* in, int64_t n, uint8_t* out, cudaStream_t stream);
cudaError_t launch_encode_e4m3(const float* in, int64_t n, int round_up, uint8_t* out, cudaStream_t stream);

}  // namespace nvfp4

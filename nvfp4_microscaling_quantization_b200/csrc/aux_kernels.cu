// aux_kernels.cu -- dequantization and the standalone rotation, for sm_100a.
//
// Both work on the quantized VIEW (vrows x vcols, blocks of 16 along a row):
// one thread per 16-element block, g/16 consecutive lanes per rotation group,
// the same butterfly order as the quantizer.
#include "kernels.h"
#include "nvfp4_device.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void store16(float* out, const float* v) {
  float4* o = reinterpret_cast<float4*>(out);
#pragma unroll
  for (int q = 0; q < 4; ++q) o[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// value(code, flag) * RN(E4M3(scale & 0x7F) * s_g), then the optional inverse rotation.
template <int G, bool INVERSE>
__global__ void __launch_bounds__(kThreads)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  const float* __restrict__ gscale, int64_t total_blocks, int mode, uint64_t seed,
                  float* __restrict__ out) {
  constexpr uint32_t kLanesPerGroup = G > 16 ? G / 16 : 1;
  const int64_t total_warps = (total_blocks + 31) & ~int64_t(31);
  const uint32_t lig = (threadIdx.x & 31u) & (kLanesPerGroup - 1u);
  uint32_t sign_bits = 0;
  if constexpr (INVERSE) sign_bits = rht_sign_bits(philox_key(seed), lig);
  const float s_g = *gscale;
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t b = int64_t(blockIdx.x) * kThreads + threadIdx.x; b < total_warps; b += stride) {
    const bool valid = b < total_blocks;
    float v[16];
    if (valid) {
      const uint2 c = *reinterpret_cast<const uint2*>(codes + b * 8);
      const uint32_t S = scales[b];
      // MXFP4 / MXFP3: UE8M0 scale 2^(S - 127) (S = 0: the subnormal
      // 2^-127); else RN(E4M3(S) * s_g)
      const bool mx = mode == kMXFP4 || mode == kMXFP3;
      const float d = mx ? __uint_as_float(S ? (S << 23) : 0x00400000u) : __fmul_rn(e4m3_decode(S & 0x7Fu), s_g);
      const bool flagged = (mode == kIF4 || mode == kIF3) && (S & 0x80u);
      if (flagged || mode == kNVINT4 || mode == kNVINT3) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t code = ((i < 8 ? c.x : c.y) >> (4 * (i & 7))) & 0xFu;
          const int k = (code & 8u) ? -static_cast<int>(code & 7u) : static_cast<int>(code & 7u);
          // IF4: RN(RN(k RN(6/7)) d); IF3: RN(RN(k RN(4/3)) d); NVINT4/3: RN(k d)
          const float lv = mode == kIF4 ? __fmul_rn(static_cast<float>(k), kIF4K2)
                           : (mode == kIF3 ? __fmul_rn(static_cast<float>(k), kIF3K2) : static_cast<float>(k));
          v[i] = __fmul_rn(lv, d);
        }
      } else if (mode == kNVFP3 || mode == kMXFP3 || mode == kIF3) {
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = __fmul_rn(e2m0_value(((i < 8 ? c.x : c.y) >> (4 * (i & 7))) & 0xFu), d);
      } else {
        e2m1x8_to_f32(c.x, v);
        e2m1x8_to_f32(c.y, v + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], d);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    if constexpr (INVERSE) rht_inverse<G>(v, sign_bits, lig);
    if (valid) store16(out + b * 16, v);
  }
}

// Rotation (or its inverse) of the view of `in` (bf16 or fp32), written as
// dense fp32.  A utility for checks, not the quantizer's path: the transposed
// view reads strided columns.
template <int G, bool INVERSE>
__global__ void __launch_bounds__(kThreads)
rht_kernel(const void* __restrict__ in, int in_dtype, int64_t rows, int64_t cols, int64_t ld,
           int layout, uint64_t seed, float* __restrict__ out) {
  constexpr uint32_t kLanesPerGroup = G / 16;
  const int64_t vrows = layout == 0 ? rows : cols;
  const int64_t vcols = layout == 0 ? cols : rows;
  const int64_t nb = vcols / 16;
  const int64_t total = vrows * nb;
  const int64_t total_warps = (total + 31) & ~int64_t(31);
  const uint32_t lig = (threadIdx.x & 31u) & (kLanesPerGroup - 1u);
  const uint32_t sign_bits = rht_sign_bits(philox_key(seed), lig);
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t b = int64_t(blockIdx.x) * kThreads + threadIdx.x; b < total_warps; b += stride) {
    const bool valid = b < total;
    float v[16];
    if (valid) {
      const int64_t vr = b / nb, vc0 = (b - vr * nb) * 16;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int64_t idx = layout == 0 ? vr * ld + vc0 + i : (vc0 + i) * ld + vr;
        v[i] = in_dtype == 0 ? __uint_as_float(uint32_t(static_cast<const uint16_t*>(in)[idx]) << 16)
                             : static_cast<const float*>(in)[idx];
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = 0.0f;
    }
    if constexpr (INVERSE) rht_inverse<G>(v, sign_bits, lig);
    else rht_forward<G>(v, sign_bits, lig);
    if (valid) store16(out + b * 16, v);
  }
}

// One code per byte, through the quantizer's own conversion helpers.
__global__ void __launch_bounds__(kThreads)
encode_e2m1_kernel(const float* __restrict__ in, int64_t n, uint8_t* __restrict__ out) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride) {
    float v[8] = {in[i], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    out[i] = static_cast<uint8_t>(clear_negative_zero(cvt_e2m1x8(v)) & 0xFu);
  }
}

__global__ void __launch_bounds__(kThreads)
encode_e4m3_kernel(const float* __restrict__ in, int64_t n, int round_up, uint8_t* __restrict__ out) {
  const int64_t stride = int64_t(gridDim.x) * kThreads;
  for (int64_t i = int64_t(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride)
    out[i] = static_cast<uint8_t>(round_up ? e4m3_ru_sat(in[i]) : e4m3_rne_sat(in[i]));
}

int grid_for(int64_t total_blocks) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (total_blocks + kThreads - 1) / kThreads;
  return static_cast<int>(need < int64_t(sms) * 8 ? need : int64_t(sms) * 8);
}

template <int G, bool INVERSE>
cudaError_t dequant_one(const DequantArgs& a) {
  const int64_t total = a.vrows * (a.vcols / 16);
  const int grid = grid_for(total);
  if (grid == 0) return cudaSuccess;
  dequantize_kernel<G, INVERSE><<<grid, kThreads, 0, a.stream>>>(a.codes, a.scales, a.gscale, total,
                                                                 a.mode, a.seed, a.out);
  return cudaGetLastError();
}

template <int G, bool INVERSE>
cudaError_t rht_one(const RhtArgs& a) {
  const int64_t vrows = a.layout == 0 ? a.rows : a.cols;
  const int64_t vcols = a.layout == 0 ? a.cols : a.rows;
  const int grid = grid_for(vrows * (vcols / 16));
  if (grid == 0) return cudaSuccess;
  rht_kernel<G, INVERSE><<<grid, kThreads, 0, a.stream>>>(a.in, a.in_dtype, a.rows, a.cols, a.ld,
                                                          a.layout, a.seed, a.out);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequantize(const DequantArgs& a) {
  if (!a.inverse_rht) return dequant_one<0, false>(a);
  switch (a.rht_group) {
    case 16: return dequant_one<16, true>(a);
    case 32: return dequant_one<32, true>(a);
    case 64: return dequant_one<64, true>(a);
    case 128: return dequant_one<128, true>(a);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_encode_e2m1(const float* in, int64_t n, uint8_t* out, cudaStream_t stream) {
  const int grid = grid_for(n);
  if (grid == 0) return cudaSuccess;
  encode_e2m1_kernel<<<grid, kThreads, 0, stream>>>(in, n, out);
  return cudaGetLastError();
}

cudaError_t launch_encode_e4m3(const float* in, int64_t n, int round_up, uint8_t* out, cudaStream_t stream) {
  const int grid = grid_for(n);
  if (grid == 0) return cudaSuccess;
  encode_e4m3_kernel<<<grid, kThreads, 0, stream>>>(in, n, round_up, out);
  return cudaGetLastError();
}

cudaError_t launch_rht(const RhtArgs& a) {
  if (!a.inverse && a.in_dtype == 0) {
    // the forward rotation of a bf16 tensor is the quantizer's own: on the
    // tensor cores whenever the quantizer would use them
    QuantArgs q{a.in, a.rows, a.cols, a.ld, a.layout, kRTN, a.rht_group, a.seed, nullptr, nullptr,
                nullptr, nullptr, nullptr, a.stream};
    if (mma_path_applies(q)) return launch_rotate_mma(q, a.out);
  }
  switch (a.rht_group * 2 + (a.inverse ? 1 : 0)) {
    case 32: return rht_one<16, false>(a);
    case 33: return rht_one<16, true>(a);
    case 64: return rht_one<32, false>(a);
    case 65: return rht_one<32, true>(a);
    case 128: return rht_one<64, false>(a);
    case 129: return rht_one<64, true>(a);
    case 256: return rht_one<128, false>(a);
    case 257: return rht_one<128, true>(a);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nvfp4

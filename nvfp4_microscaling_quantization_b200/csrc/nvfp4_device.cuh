// nvfp4_device.cuh -- device building blocks of the NVFP4 quantizer (sm_100a).
//
// Every floating-point step that decides a code or a scale is one IEEE
// binary32 operation with round-to-nearest-even: scalar steps through the
// __f*_rn intrinsics, two-lane steps through add/mul/fma .rn.f32x2 written in
// PTX with the rounding stated (an instruction with an explicit rounding
// modifier is never fused with another), and the library is built with
// -fmad=false.  The step order is the method's: rotate, block absmax, block
// scale, scale to the grid, round, pack.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace nvfp4 {

enum Mode {
  kRTN = 0, kSR = 1, kMSEDEN = 2, kIF4 = 3, k4over6 = 4, kScaleSearch = 5, kMXFP4 = 6, kNVINT4 = 7,
  kNVFP3 = 8, kNVINT3 = 9, kIF3 = 10, kMXFP3 = 11
};
template <int MODE>
__host__ __device__ constexpr bool is_mx() { return MODE == kMXFP4 || MODE == kMXFP3; }
template <int MODE>
__host__ __device__ constexpr bool is_3bit_e4m3() { return MODE == kNVFP3 || MODE == kNVINT3 || MODE == kIF3; }

// Scale search: the candidates are the E4M3 codes S0 + delta(t), t = 0 ..
// 18, around the absmax scale S0, visited nearest first (0, -1, +1, -2, ...),
// clamped to 0 .. 0x7E; a strictly lower error replaces the best so far.
constexpr int kSearchCandidates = 19;
__host__ __device__ constexpr int search_delta(int t) { return ((t + 1) / 2) * ((t & 1) ? -1 : 1); }
__device__ __forceinline__ uint32_t search_code(uint32_t s0, int t) {
  const int s = static_cast<int>(s0) + search_delta(t);
  return static_cast<uint32_t>(s < 0 ? 0 : (s > 0x7E ? 0x7E : s));
}

// ---------------------------------------------------------------------------
// Two-lane binary32 arithmetic (sm_100a f32x2): each lane is one IEEE RN
// operation.  The explicit .rn keeps a product from being fused into a
// following add, which would skip the product's rounding.
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

__device__ __forceinline__ unsigned long long pack2(float2 a) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a.x), "f"(a.y));
  return r;
}
__device__ __forceinline__ float2 unpack2(unsigned long long r) {
  float2 a;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a.x), "=f"(a.y) : "l"(r));
  return a;
}
__device__ __forceinline__ float2 add2_rn(float2 a, float2 b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
  return unpack2(d);
}
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
  return unpack2(d);
}
__device__ __forceinline__ float2 fma2_rn(float2 a, float2 b, float2 c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)), "l"(pack2(c)));
  return unpack2(d);
}
// a - b per lane: the negation is exact, so each lane is the one RN subtraction.
__device__ __forceinline__ float2 sub2_rn(float2 a, float2 b) { return add2_rn(a, f2(-b.x, -b.y)); }
// a + b and a - b lane by lane through the scalar intrinsics, for a sum
// whose operand b is a rounded product: the scalar adds are never merged with
// the multiplication that produced b.  (The packed add.rn.f32x2 is not safe
// here: a GPU parity test of IF4 found a packed product and sum contracted
// into one fused operation, skipping the product's rounding.)
__device__ __forceinline__ float2 sub2_after_mul(float2 a, float2 b) { return f2(__fsub_rn(a.x, b.x), __fsub_rn(a.y, b.y)); }
// RN(a b) per lane as a fused multiply-add whose addend is -0 held in a
// register the compiler cannot see through (nz, from ScaleCtx): exact, since
// x + (-0) = x for every x, zeros included, and a product formed this way is
// never merged with a sum that follows, so that sum can be the packed one.
__device__ __forceinline__ float2 mul2_unmerged(float2 a, float2 b, float nz) { return fma2_rn(a, b, f2(nz, nz)); }
// a - b per lane in one packed subtraction; b must not be a product that the
// compiler could merge into it (see mul2_unmerged).
__device__ __forceinline__ float2 sub2_packed(float2 a, float2 b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(pack2(a)), "l"(pack2(b)));
  return unpack2(d);
}

// max(|a|, |b|, |c|) in one three-input sm_100 max (exact; a NaN operand is
// ignored as by fmaxf).
__device__ __forceinline__ float absmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(fabsf(a)), "f"(fabsf(b)), "f"(fabsf(c)));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
// max of N non-negative values, as a tree of three-input maxima (short
// dependency chains for latency-bound reductions).
template <int N>
__device__ __forceinline__ float max_tree(const float (&m)[N]) {
  if constexpr (N == 1) {
    return m[0];
  } else if constexpr (N == 2) {
    return fmaxf(m[0], m[1]);
  } else {
    constexpr int M = (N + 2) / 3;
    float r[M];
#pragma unroll
    for (int i = 0; i < N / 3; ++i) r[i] = max3(m[3 * i], m[3 * i + 1], m[3 * i + 2]);
    if constexpr (N % 3 == 1) r[M - 1] = m[N - 1];
    if constexpr (N % 3 == 2) r[M - 1] = fmaxf(m[N - 2], m[N - 1]);
    return max_tree<M>(r);
  }
}
// max |v[i]| of N values as a tree.
template <int N>
__device__ __forceinline__ float absmax_tree(const float (&v)[N]) {
  constexpr int M = (N + 2) / 3;
  float r[M];
#pragma unroll
  for (int i = 0; i < N / 3; ++i) r[i] = absmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  if constexpr (N % 3 == 1) r[M - 1] = fabsf(v[N - 1]);
  if constexpr (N % 3 == 2) r[M - 1] = fmaxf(fabsf(v[N - 2]), fabsf(v[N - 1]));
  return max_tree<M>(r);
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
// as 1, 2, 3", SC'11): ten rounds of two 32x32->64 multiplications by the
// round multipliers, the high halves mixed with the other counter words and
// the key, the key advanced by the two Weyl increments between rounds.
struct PhiloxKey {
  uint32_t k0, k1;
};

__device__ __forceinline__ PhiloxKey philox_key(uint64_t seed) {
  return PhiloxKey{static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32)};
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, PhiloxKey key) {
  uint32_t k0 = key.k0, k1 = key.k1;
#pragma unroll
  for (int round = 0; round < 10; ++round) {
    // the two halves of each 32x32 -> 64-bit product as separate high and
    // low multiplications (the same bits; measured 5-7% faster for SR than
    // one widening multiplication)
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return c;
}

// Stream tags carried in counter word 2.
constexpr uint32_t kTagElement = 0;  // element stochastic rounding: 8 x 16-bit uniforms per call
constexpr uint32_t kTagBlock = 1;    // scale stochastic rounding: 8 x 16-bit uniforms per call
constexpr uint32_t kTagSigns = 2;    // RHT signs: 128 sign bits from call 0

__device__ __forceinline__ uint4 philox_call(PhiloxKey key, uint64_t call, uint32_t tag) {
  return philox4x32_10(
      make_uint4(static_cast<uint32_t>(call), static_cast<uint32_t>(call >> 32), tag, 0u), key);
}

__device__ __forceinline__ uint32_t word_of(const uint4& w, uint32_t i) {
  return i == 0 ? w.x : (i == 1 ? w.y : (i == 2 ? w.z : w.w));
}

// 16-bit draw i (0..7) of a call: word i/2, low half for even i, high for odd.
__device__ __forceinline__ uint32_t half_word(const uint4& w, uint32_t i) {
  return (word_of(w, i >> 1) >> ((i & 1u) * 16u)) & 0xFFFFu;
}

// k * 2^-16 for k < 2^16, exactly: k placed in the fraction of 1.0 minus 1.
__device__ __forceinline__ float uniform16(uint32_t k) {
  return __fsub_rn(__uint_as_float(0x3F800000u | (k << 7)), 1.0f);
}

// ---------------------------------------------------------------------------
// Format conversions through the sm_100a conversion instructions.
//
// E2M1: 4 pairs of floats -> 8 codes in one 32-bit word, element 2k in the low
// nibble of byte k.  The hardware rounds to nearest-even and saturates at 6;
// a negative value that rounds to zero comes back as 0x8 and is cleared by
// clear_negative_zero() so zero is always code 0.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// For each nibble: keep the sign bit only if the magnitude bits are nonzero.
__device__ __forceinline__ uint32_t clear_negative_zero(uint32_t w) {
  // mag + 7 carries into bit 3 of a nibble iff its magnitude is nonzero (and
  // never into the next nibble); the magnitude bits of w always pass
  const uint32_t carry = (w & 0x77777777u) + 0x77777777u;
  return w & (carry | 0x77777777u);
}

// 8 packed E2M1 codes -> 8 floats (exact: every grid value is an f16).
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float* v) {
  uint32_t h[4];
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "mov.b32 {q0, q1, q2, q3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, q0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, q1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, q2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, q3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __half2 p = *reinterpret_cast<__half2*>(&h[k]);
    v[2 * k] = __low2float(p);
    v[2 * k + 1] = __high2float(p);
  }
}

// E4M3 round-to-nearest-even with saturation at 448 (v >= 0).
__device__ __forceinline__ uint32_t e4m3_rne_sat(float v) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(0.0f), "f"(v));
  return out & 0xFFu;
}

// E4M3 code (0x00..0x7E) -> float, exact.
__device__ __forceinline__ float e4m3_decode(uint32_t code) {
  uint32_t h2;
  const uint16_t in = static_cast<uint16_t>(code & 0x7Fu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __low2float(*reinterpret_cast<__half2*>(&h2));
}

// Smallest E4M3 value >= v, capped at 448 (v >= 0).
__device__ __forceinline__ uint32_t e4m3_ru_sat(float v) {
  uint32_t s = e4m3_rne_sat(v);
  if (s < 0x7Eu && e4m3_decode(s) < v) ++s;
  return s;
}

// Stochastic rounding of t >= 0 onto E4M3 with a uniform U in [0, 1):
// neighbours lo <= t < hi, hi with probability (t - lo) / (hi - lo); t >= 448
// gives 448.  (t - lo) and the division by the power-of-two gap are exact.
// Written without branches: for t >= 448 the RNE code is 0x7E and the code
// above it (0x7F) decodes to NaN, so the comparison fails and 0x7E stays; for
// t = 0 the code is 0 and nothing rounds up.
__device__ __forceinline__ uint32_t e4m3_sr(float t, float U) {
  uint32_t lo = e4m3_rne_sat(t);
  lo = e4m3_decode(lo) > t ? lo - 1 : lo;
  const float l = e4m3_decode(lo);
  const float h = e4m3_decode(lo + 1);
  // U < (t - l) / (h - l)  <=>  U * (h - l) < t - l: h - l is a power of two, so
  // both products and the difference are exact and the comparison is the same.
  return __fmul_rn(U, __fsub_rn(h, l)) < __fsub_rn(t, l) ? lo + 1 : lo;
}

// bf16 pair (one 32-bit word) -> two floats.
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xFFFF0000u);
}

// ---------------------------------------------------------------------------
// Random Hadamard rotation of a g-group (g in 16..128) held as 16 consecutive
// elements per lane by g/16 consecutive lanes.  Butterfly order: h = 1, 2, 4,
// 8 inside the lane, then h = 16, 32, 64 across lanes (partner = lane ^ h/16):
// (u_i, u_{i+h}) <- (u_i + u_{i+h}, u_i - u_{i+h}).  Each sum is one RN
// addition, so the result matches a sequential butterfly in the same order.
__device__ __forceinline__ void fwht16_local(float* v) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i & h) continue;
      const float a = v[i], b = v[i + h];
      v[i] = __fadd_rn(a, b);
      v[i + h] = __fsub_rn(a, b);
    }
  }
}

template <int G>
__device__ __forceinline__ void fwht_cross_lanes(float* v, uint32_t lane_in_group) {
#pragma unroll
  for (int hl = 1; hl < G / 16; hl <<= 1) {
    const bool upper = (lane_in_group & hl) != 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float other = __shfl_xor_sync(0xFFFFFFFFu, v[i], hl);
      v[i] = upper ? __fsub_rn(other, v[i]) : __fadd_rn(v[i], other);
    }
  }
}

template <int G>
struct RhtConst;
template <> struct RhtConst<16> { static constexpr float c = 0.25f; };
template <> struct RhtConst<32> { static constexpr float c = 0x1.6a09e6p-3f; };  // RN(1/sqrt(32))
template <> struct RhtConst<64> { static constexpr float c = 0.125f; };
template <> struct RhtConst<128> { static constexpr float c = 0x1.6a09e6p-4f; }; // RN(1/sqrt(128))

// 16 sign bits of this lane's slice of the g-long sign vector.
__device__ __forceinline__ uint32_t rht_sign_bits(PhiloxKey key, uint32_t lane_in_group) {
  const uint4 w = philox_call(key, 0, kTagSigns);
  return (word_of(w, lane_in_group >> 1) >> ((lane_in_group & 1u) * 16u)) & 0xFFFFu;
}

template <int G>
__device__ __forceinline__ void rht_forward(float* v, uint32_t sign_bits, uint32_t lane_in_group) {
#pragma unroll
  for (int i = 0; i < 16; ++i)
    v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((sign_bits >> i) & 1u) << 31));
  fwht16_local(v);
  if constexpr (G > 16) fwht_cross_lanes<G>(v, lane_in_group);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __fmul_rn(v[i], RhtConst<G>::c);
}

template <int G>
__device__ __forceinline__ void rht_inverse(float* v, uint32_t sign_bits, uint32_t lane_in_group) {
  fwht16_local(v);
  if constexpr (G > 16) fwht_cross_lanes<G>(v, lane_in_group);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    v[i] = __fmul_rn(v[i], RhtConst<G>::c);
    v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((sign_bits >> i) & 1u) << 31));
  }
}

// ---------------------------------------------------------------------------
// Tensor scale: s_g = RN(A / (6 M)), M = 256 for MS-EDEN, 4/6 and scale
// search, else 448.
template <int MODE>
__device__ __forceinline__ float global_scale_of(float amax) {
  if constexpr (is_mx<MODE>()) return 1.0f;  // MXFP4 / MXFP3 have no tensor scale
  if constexpr (MODE == kNVINT4) return amax > 0.0f ? __fdiv_rn(amax, 3136.0f) : 1.0f;  // 7 x 448
  if constexpr (MODE == kNVFP3 || MODE == kIF3) return amax > 0.0f ? __fdiv_rn(amax, 1792.0f) : 1.0f;  // 4 x 448
  if constexpr (MODE == kNVINT3) return amax > 0.0f ? __fdiv_rn(amax, 1344.0f) : 1.0f;  // 3 x 448
  constexpr float six_m = (MODE == kMSEDEN || MODE == k4over6 || MODE == kScaleSearch) ? 1536.0f : 2688.0f;
  return amax > 0.0f ? __fdiv_rn(amax, six_m) : 1.0f;
}

// INT4 option of IF4: levels k in [-7, 7] standing for k * 6/7.
constexpr float kIF4K1 = 0x1.2aaaaap+0f;  // RN(7/6)
constexpr float kIF4K2 = 0x1.b6db6ep-1f;  // RN(6/7)
constexpr float kRoundMagic = 12582912.0f; // 1.5 * 2^23: RN(t + it) - it = RNE(t) for |t| < 2^22

// NVINT4 code of one scaled value y: k = clamp(RNE(y), -7, 7) as a
// sign-magnitude nibble (sign bit 3, |k| in bits 0..2, never -0), with no
// conversion instruction: s = RN(y + 1.5 2^23) rounds y at the units bit
// (ties to even, |y| < 2^22), s - 1.5 2^23 = RNE(y) exactly; |k| is the low
// mantissa bits of 2^23 + |k| and the sign is the sign of k.
__device__ __forceinline__ uint32_t int4_nibble(float y) {
  const float s = __fadd_rn(y, kRoundMagic);
  const float k = fminf(fmaxf(__fsub_rn(s, kRoundMagic), -7.0f), 7.0f);
  return (__float_as_uint(__fadd_rn(fabsf(k), 8388608.0f)) & 7u) | ((__float_as_uint(k) >> 28) & 8u);
}

// INT4 codes of eight values from the bits s_i of s = min(RN(|t_i| + 1.5
// 2^23), 1.5 2^23 + 7) (|t_i| < 2^22), whose low byte is |k_i| =
// min(RNE(|t_i|), 7), and a word whose bit 3 of nibble i holds the sign of
// element i wherever |k_i| > 0: the low bytes gathered into nibbles with byte
// permutes, the signs added, and a zero code cleared of its sign.
__device__ __forceinline__ uint32_t int_nibbles8(const uint32_t* s, uint32_t signs) {
  const uint32_t even = __byte_perm(__byte_perm(s[0], s[2], 0x0040u), __byte_perm(s[4], s[6], 0x4000u), 0x7610u);
  const uint32_t odd = __byte_perm(__byte_perm(s[1], s[3], 0x0040u), __byte_perm(s[5], s[7], 0x4000u), 0x7610u);
  return clear_negative_zero(even | (odd << 4) | (signs & 0x88888888u));
}
// The signs of eight floats in bit 3 of nibbles 0..7 (top bytes gathered).
__device__ __forceinline__ uint32_t sign_nibbles8(const float* y) {
  const uint32_t even = __byte_perm(__byte_perm(__float_as_uint(y[0]), __float_as_uint(y[2]), 0x0073u),
                                    __byte_perm(__float_as_uint(y[4]), __float_as_uint(y[6]), 0x7300u), 0x7610u);
  const uint32_t odd = __byte_perm(__byte_perm(__float_as_uint(y[1]), __float_as_uint(y[3]), 0x0073u),
                                   __byte_perm(__float_as_uint(y[5]), __float_as_uint(y[7]), 0x7300u), 0x7610u);
  return ((even >> 4) & 0x08080808u) | (odd & 0x80808080u);
}
// s = min(RN(|t| + 1.5 2^23), 1.5 2^23 + KMAX): RNE(|t|) clamped to KMAX
// (7 for INT4, 3 for INT3) in its low bits.
template <int KMAX = 7>
__device__ __forceinline__ float int_magnitude_sum(float t) {
  return fminf(__fadd_rn(fabsf(t), kRoundMagic), kRoundMagic + static_cast<float>(KMAX));
}

// 3-bit elements, stored in nibbles (sign bit 3, magnitude code bits 0..1).
// E2M0: magnitudes {0, 1, 2, 4}, nearest with ties to the even code (0.5 ->
// 0, 1.5 -> 2, 3 -> 2), saturating at 4; zero is code 0.  The rounding runs
// on the bits of a1 = min(max(|y|, RU(0.5 + |y|/2)), 4), with no compares:
// below 1, a1 = RU(0.5 + |y|/2) lies in [0.5, 1) and is above 0.75 iff
// |y| > 0.5 (0.75 is a float, so the upward rounding keeps the comparison
// exact); from 1 on, a1 = min(|y|, 4).  Adding 2^22 - 1 to the bits of a1,
// plus one when its biased exponent is odd, carries into the exponent field
// iff the mantissa is above one half, or exactly one half at an odd exponent:
// the tie 1.5 (exponent 127) goes up and 3 (128) down, both to the even code
// 2, and 0.75 (126, i.e. |y| = 0.5) down to code 0.  The exponent field of
// the result is 126 + code, and its power of two is 2^(code - 1).
__device__ __forceinline__ uint32_t e2m0_exponent_bits(float y) {
  const float a = fabsf(y);
  const float a1 = fminf(fmaxf(a, __fmaf_ru(a, 0.5f, 0.5f)), 4.0f);
  const uint32_t b = __float_as_uint(a1);
  return b + 0x3FFFFFu + ((b >> 23) & 1u);
}
// |E2M0 value| from e2m0_exponent_bits: the power of two p in {0.5, 1, 2, 4},
// then min(2p - 1, p) (exact), which is 0 for p = 0.5 (code 0) and p otherwise.
__device__ __forceinline__ float e2m0_magnitude(uint32_t t) {
  const float p = __uint_as_float(t & 0xFF800000u);
  return fminf(__fmaf_rn(p, 2.0f, -1.0f), p);
}
// E2M0 codes of eight values from their e2m0_exponent_bits t_i: code_i =
// (exponent field + 2) mod 4, which lands in bits 28..29 of 32 (t_i + 2^24)
// = 32 t_i + 2^29 with bits 30..31 clear (exponent fields 126..129); the sign
// of y_i goes into bit 31, the top nibbles are gathered with byte permutes,
// and a zero code drops its sign.
__device__ __forceinline__ uint32_t e2m0_nibbles8(const uint32_t* t, const float* y) {
  uint32_t v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = (t[i] * 32u + 0x20000000u) | (__float_as_uint(y[i]) & 0x80000000u);
  const uint32_t even = __byte_perm(__byte_perm(v[0], v[2], 0x0073u), __byte_perm(v[4], v[6], 0x7300u), 0x7610u);
  const uint32_t odd = __byte_perm(__byte_perm(v[1], v[3], 0x0073u), __byte_perm(v[5], v[7], 0x7300u), 0x7610u);
  return clear_negative_zero(((even >> 4) & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u));
}
// signed E2M0 value of a nibble: 2^(m - 1) for m = 1..3
__device__ __forceinline__ float e2m0_value(uint32_t c) {
  const uint32_t m = c & 3u;
  return m == 0u ? 0.0f : __uint_as_float(((126u + m) << 23) | ((c & 8u) << 28));
}
constexpr float kIF3K1 = 0.75f;            // RN(3/4)
constexpr float kIF3K2 = 0x1.555556p+0f;   // RN(4/3)

// Where the random draws of one 16-element block come from.
struct BlockRng {
  PhiloxKey key;
  uint64_t first_element;  // view linear index of element 0 of the block (a multiple of 16)
  uint64_t block;          // view linear block index
};

struct BlockOut {
  uint32_t lo, hi;  // 16 packed codes: lo = elements 0..7, hi = elements 8..15
  uint32_t scale;   // scale byte (bit 7 = the IF4 / IF3 integer flag)
};

// NVFP3 / NVINT3 / IF3 codes of one block of scaled values y under scale
// byte S: E2M0, INT3, or (IF3) the option with the lower squared error in the
// y domain (fmaf in element order, ties keep E2M0) with bit 7 set for INT3.
// INT3 levels k = clamp(RNE(t), -3, 3) come from int_magnitude_sum<3>, their
// signs from t's (NVINT3) or, for IF3, from the E2M0 codes: a nonzero level
// needs |y| 3/4 >= 1/2, so |y| > 1/2, where the E2M0 code is nonzero and
// carries the sign of y.  The errors use |y| - |v|, the same square as y - v.
template <int MODE>
__device__ __forceinline__ BlockOut block3_codes(const float* y, uint32_t S) {
  if constexpr (MODE == kNVINT3) {
    uint32_t s[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = __float_as_uint(int_magnitude_sum<3>(y[i]));
    return BlockOut{int_nibbles8(s, sign_nibbles8(y)), int_nibbles8(s + 8, sign_nibbles8(y + 8)), S};
  } else {
    uint32_t t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) t[i] = e2m0_exponent_bits(y[i]);
    const uint32_t f_lo = e2m0_nibbles8(t, y), f_hi = e2m0_nibbles8(t + 8, y + 8);
    if constexpr (MODE == kIF3) {
      uint32_t s[16];
      float eF = 0.0f, eI = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = fabsf(y[i]);
        const float dF = __fsub_rn(a, e2m0_magnitude(t[i]));
        eF = __fmaf_rn(dF, dF, eF);
        const float sI = int_magnitude_sum<3>(__fmul_rn(y[i], kIF3K1));
        s[i] = __float_as_uint(sI);
        const float dI = __fsub_rn(a, __fmul_rn(__fsub_rn(sI, kRoundMagic), kIF3K2));
        eI = __fmaf_rn(dI, dI, eI);
      }
      if (eI < eF) return BlockOut{int_nibbles8(s, f_lo), int_nibbles8(s + 8, f_hi), S | 0x80u};
    }
    return BlockOut{f_lo, f_hi, S};
  }
}


__device__ __forceinline__ float block_absmax(const float* z) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(z[i]));
  return a;
}

// RTN codes of 16 scaled values.
__device__ __forceinline__ void rtn_codes(const float* y, uint32_t& lo, uint32_t& hi) {
  lo = clear_negative_zero(cvt_e2m1x8(y));
  hi = clear_negative_zero(cvt_e2m1x8(y + 8));
}

// Stochastic rounding of eight scaled values y[0..7] with the eight 16-bit
// uniforms U_i = k_i * 2^-16 of one Philox call w (draw i = half i&1 of word
// i/2), done on the bits of the floats with no conversion instruction.
// a = min(|y|, 6) lies between grid neighbours l <= a < u and goes up iff
// U < (a - l) / (u - l).  For a in [1, 6] the grid keeps one mantissa bit, so
// the fraction is low22 / 2^22 (low22 = the 22 mantissa bits below it) and
// U < low22 / 2^22 iff 64k < low22 iff low22 + (2^22 - 1 - 64k) carries into
// the kept bit; the code index is then (bits >> 22) - 252.  For a in [0, 1)
// the grid {0, 0.5, 1} is that of 0.5 + a/2 on [0.5, 1] (one kept bit below
// 0.5), and 0.5 + a/2 rounded upward is exact for the decision: 64k * 2^-23
// lies on the 2^-23 grid that the upward rounding lands on, so a - l exceeds
// it iff the rounded value does.  a1 = max(a, RU(0.5 + a/2)) picks the right
// one of the two (0.5 + a/2 <= a iff a >= 1); taking the minimum with 6 last
// gives the same a1 (a NaN or a value above 6 ends at 6 either way).
// The sum is formed 64 times larger, modulo 2^32, so that the index lands in
// bits 28..30 with bit 31 clear: t = 64 bits(a1) + 64 (2^22 - 1 - 64k - 252
// 2^22) = 64 bits(a1) + 0x4FFFFFC0 - 4096 k.  The draw k is taken from its
// word by multiply-adds rather than shifts and masks (the integer multiplier
// has spare issue, the logic unit has not): for the high half k = word >> 16,
// and for the low half -4096 k = -4096 word + 2^28 (word >> 16).  The sign of
// y goes into bit 31, and the top nibbles of the eight results are gathered
// into one word with byte permutes; a code of magnitude 0 drops its sign.
__device__ __forceinline__ uint32_t sr_codes8(const float* y, const uint4& w) {
  uint32_t v[8];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const uint32_t word = word_of(w, static_cast<uint32_t>(m));  // draws 2m (low half), 2m+1 (high half)
    const uint32_t hi = word >> 16;
    const float ae = fabsf(y[2 * m]), ao = fabsf(y[2 * m + 1]);
    const float a1e = fminf(fmaxf(ae, __fmaf_ru(ae, 0.5f, 0.5f)), 6.0f);
    const float a1o = fminf(fmaxf(ao, __fmaf_ru(ao, 0.5f, 0.5f)), 6.0f);
    const uint32_t te = hi * 0x10000000u + (word * 0xFFFFF000u + (__float_as_uint(a1e) * 64u + 0x4FFFFFC0u));
    const uint32_t to = hi * 0xFFFFF000u + (__float_as_uint(a1o) * 64u + 0x4FFFFFC0u);
    v[2 * m] = (te & 0x7FFFFFFFu) | (__float_as_uint(y[2 * m]) & 0x80000000u);
    v[2 * m + 1] = (to & 0x7FFFFFFFu) | (__float_as_uint(y[2 * m + 1]) & 0x80000000u);
  }
  // byte m of `even` / `odd` = top byte of v[2m] / v[2m+1]
  const uint32_t even = __byte_perm(__byte_perm(v[0], v[2], 0x0073u), __byte_perm(v[4], v[6], 0x7300u), 0x7610u);
  const uint32_t odd = __byte_perm(__byte_perm(v[1], v[3], 0x0073u), __byte_perm(v[5], v[7], 0x7300u), 0x7610u);
  return clear_negative_zero(((even >> 4) & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u));
}

// Quantize one block of 16 (already rotated) values z under tensor scale s_g.
template <int MODE>
__device__ __forceinline__ BlockOut quantize_block(const float* z, float s_g, const BlockRng& rng) {
  BlockOut out{0u, 0u, 0u};
  const float a_b = block_absmax(z);

  if constexpr (MODE == k4over6) {
    uint32_t S[2], c_lo[2], c_hi[2];
    float err[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float m = k == 0 ? 6.0f : 4.0f;
      const float s_f = __fdiv_rn(a_b, __fmul_rn(m, s_g));
      S[k] = e4m3_rne_sat(s_f);
      const float d = __fmul_rn(e4m3_decode(S[k]), s_g);
      float e = 0.0f;
      if (d == 0.0f) {
        c_lo[k] = c_hi[k] = 0u;
#pragma unroll
        for (int i = 0; i < 16; ++i) e = __fmaf_rn(z[i], z[i], e);
      } else {
        const float r = __frcp_rn(d);
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(z[i], r);
        rtn_codes(y, c_lo[k], c_hi[k]);
        float v[16];
        e2m1x8_to_f32(c_lo[k], v);
        e2m1x8_to_f32(c_hi[k], v + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float diff = __fsub_rn(z[i], __fmul_rn(v[i], d));
          e = __fmaf_rn(diff, diff, e);
        }
      }
      err[k] = e;
    }
    const int pick = err[1] < err[0] ? 1 : 0;
    out.lo = c_lo[pick];
    out.hi = c_hi[pick];
    out.scale = S[pick];
    return out;
  } else if constexpr (is_3bit_e4m3<MODE>()) {
    const float m = MODE == kNVINT3 ? 3.0f : 4.0f;
    const uint32_t S = e4m3_rne_sat(__fdiv_rn(a_b, __fmul_rn(m, s_g)));
    const float d = __fmul_rn(e4m3_decode(S), s_g);
    out.scale = S;
    if (d == 0.0f) return out;
    const float r = __frcp_rn(d);
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(z[i], r);
    return block3_codes<MODE>(y, S);
  } else if constexpr (MODE == kNVINT4) {
    const uint32_t S = e4m3_rne_sat(__fdiv_rn(a_b, __fmul_rn(7.0f, s_g)));
    const float d = __fmul_rn(e4m3_decode(S), s_g);
    out.scale = S;
    if (d == 0.0f) return out;
    const float r = __frcp_rn(d);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t c = int4_nibble(__fmul_rn(z[i], r));
      if (i < 8) out.lo |= c << (4 * i);
      else out.hi |= c << (4 * (i - 8));
    }
    return out;
  } else if constexpr (MODE == kScaleSearch) {
    const uint32_t s0 = e4m3_rne_sat(__fdiv_rn(a_b, __fmul_rn(6.0f, s_g)));
    float best = __int_as_float(0x7F800000);  // +inf
#pragma unroll 1
    for (int t = 0; t < kSearchCandidates; ++t) {
      const uint32_t S = search_code(s0, t);
      const float d = __fmul_rn(e4m3_decode(S), s_g);
      uint32_t lo = 0u, hi = 0u;
      float e = 0.0f;
      if (d == 0.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) e = __fmaf_rn(z[i], z[i], e);
      } else {
        const float r = __frcp_rn(d);
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(z[i], r);
        rtn_codes(y, lo, hi);
        float v[16];
        e2m1x8_to_f32(lo, v);
        e2m1x8_to_f32(hi, v + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float diff = __fsub_rn(z[i], __fmul_rn(v[i], d));
          e = __fmaf_rn(diff, diff, e);
        }
      }
      if (e < best) {
        best = e;
        out.lo = lo;
        out.hi = hi;
        out.scale = S;
      }
    }
    return out;
  } else {
    const float s_f = __fdiv_rn(a_b, __fmul_rn(6.0f, s_g));
    const uint32_t S = MODE == kSR ? e4m3_ru_sat(s_f) : e4m3_rne_sat(s_f);
    const float d = __fmul_rn(e4m3_decode(S), s_g);
    out.scale = S;
    if (d == 0.0f) return out;
    const float r = __frcp_rn(d);
    float y[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = __fmul_rn(z[i], r);

    if constexpr (MODE == kRTN) {
      rtn_codes(y, out.lo, out.hi);
    } else if constexpr (MODE == kSR) {
      const uint64_t call0 = rng.first_element >> 3;
      out.lo = sr_codes8(y, philox_call(rng.key, call0, kTagElement));
      out.hi = sr_codes8(y + 8, philox_call(rng.key, call0 + 1, kTagElement));
    } else if constexpr (MODE == kMSEDEN) {
      rtn_codes(y, out.lo, out.hi);
      float v[16];
      e2m1x8_to_f32(out.lo, v);
      e2m1x8_to_f32(out.hi, v + 8);
      float num = 0.0f, den = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        num = __fmaf_rn(y[i], y[i], num);
        den = __fmaf_rn(y[i], v[i], den);
      }
      const float c = (num > 0.0f && den > 0.0f) ? __fdiv_rn(num, den) : 1.0f;
      const float t = __fmul_rn(e4m3_decode(S), c);
      const uint4 w = philox_call(rng.key, rng.block >> 3, kTagBlock);
      const float U = uniform16(half_word(w, static_cast<uint32_t>(rng.block & 7u)));
      out.scale = e4m3_sr(t, U);
    } else {  // kIF4
      uint32_t f_lo, f_hi;
      rtn_codes(y, f_lo, f_hi);
      float v[16];
      e2m1x8_to_f32(f_lo, v);
      e2m1x8_to_f32(f_hi, v + 8);
      float eF = 0.0f, eI = 0.0f;
      uint32_t i_lo = 0u, i_hi = 0u;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float dF = __fsub_rn(y[i], v[i]);
        eF = __fmaf_rn(dF, dF, eF);
        int k = __float2int_rn(__fmul_rn(y[i], kIF4K1));
        k = max(-7, min(7, k));
        const float dI = __fsub_rn(y[i], __fmul_rn(static_cast<float>(k), kIF4K2));
        eI = __fmaf_rn(dI, dI, eI);
        const uint32_t code = k == 0 ? 0u : (static_cast<uint32_t>(k < 0 ? -k : k) | (k < 0 ? 8u : 0u));
        if (i < 8) i_lo |= code << (4 * i);
        else i_hi |= code << (4 * (i - 8));
      }
      if (eI < eF) {
        out.lo = i_lo;
        out.hi = i_hi;
        out.scale = S | 0x80u;
      } else {
        out.lo = f_lo;
        out.hi = f_hi;
      }
    }
    return out;
  }
}

// ---------------------------------------------------------------------------
// Two blocks at once.  The tiled kernels hold their data as float2 pairs whose
// .x and .y belong to two different 16-element blocks (two blocks of a row, or
// the same rows of two columns), so every per-element step of two blocks is
// one packed f32x2 instruction.  Each lane of a packed operation is one
// binary32 RN operation, so the per-block results, including the sequential
// per-block dot products, are exactly those of quantize_block.
struct PairRng {
  PhiloxKey key;
  uint64_t elem_a, elem_b;  // view index of element 0 of block a / b (multiples of 16)
  uint32_t k_a, k_b;        // 16-bit scale draws of block a / b (MS-EDEN): U = k 2^-16
};

// Per-launch constants of the block-scale step: the tensor scale s_g, the
// divisors q6 = RN(6 s_g) and q4 = RN(4 s_g) of s_f = RN(absmax / q), and
// their round-to-nearest reciprocals for the division below.
struct ScaleCtx {
  float s_g, q6, q4, r6, r4;
  float nz;             // -0, derived from the amax loaded at run time (see mul2_unmerged)
  bool markstein;       // the reciprocal-based division is exact for every block
  const float4* tbl;    // per E4M3 code S: {dec(S), d = RN(dec(S) s_g), RN(1/d) or 0, 0}
};

template <int MODE>
__device__ __forceinline__ ScaleCtx make_scale_ctx(float amax) {
  ScaleCtx c;
  c.tbl = nullptr;
  c.s_g = global_scale_of<MODE>(amax);
  // the absmax divisor RN(m s_g), m = the element maximum: 6 (E2M1), 7
  // (NVINT4), 4 (E2M0: NVFP3, IF3), 3 (NVINT3)
  constexpr float m = MODE == kNVINT4 ? 7.0f
                      : (MODE == kNVFP3 || MODE == kIF3) ? 4.0f
                      : MODE == kNVINT3 ? 3.0f : 6.0f;
  c.q6 = __fmul_rn(m, c.s_g);
  c.q4 = __fmul_rn(4.0f, c.s_g);
  c.r6 = __frcp_rn(c.q6);
  c.r4 = __frcp_rn(c.q4);
  // With q in [2^-90, 2^100] the remainder below cannot underflow unless
  // a / q < 2^-12, where any value within an ulp gives the same (zero) E4M3
  // scale; outside that range the kernels divide with __fdiv_rn.
  c.markstein = c.q4 >= 0x1p-90f && c.q6 <= 0x1p100f;
  // -0 for every amax >= 0 (for a negative amax +0, which changes nothing:
  // RN(a b + 0) differs from RN(a b) only in the sign of a zero result, and
  // every code of magnitude zero is stored unsigned)
  c.nz = __uint_as_float((__float_as_uint(amax) & 0x80000000u) ^ 0x80000000u);
  return c;
}

// RN(a / q) for the two lanes, with r = RN(1/q): Markstein's correction
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990): t = RN(a r) is within
// an ulp of a/q, the remainder a - t q is exact in one fused multiply-add, and
// RN(t + (a - t q) r) is the correctly rounded quotient.
__device__ __forceinline__ float2 div2_by(float2 a, float q, float r, bool markstein) {
  if (!markstein) return f2(__fdiv_rn(a.x, q), __fdiv_rn(a.y, q));
  const float2 q2 = f2(q, q), r2 = f2(r, r);
  const float2 t = mul2_rn(a, r2);
  const float2 rem = fma2_rn(f2(-t.x, -t.y), q2, a);
  const float2 d = fma2_rn(rem, r2, t);
  // a quotient that overflows (an absmax far above the tensor amax given)
  // comes out NaN here and infinite from the division; both saturate the
  // E4M3 scale, and so does 1024
  return f2(fminf(d.x, 1024.0f), fminf(d.y, 1024.0f));
}


// E4M3 RNE of two non-negative floats in one conversion: .x -> bits 0..7, .y -> bits 8..15.
__device__ __forceinline__ uint32_t e4m3x2_rne_sat(float a, float b) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(out) : "f"(b), "f"(a));
  return out;
}

// Stochastic rounding of two t >= 0 onto E4M3 (the rule of e4m3_sr) with the
// 16-bit draws ka, kb (U = k 2^-16): bits 0..7 for t.x, 8..15 for t.y, each in
// 0..0x7E, on the bits of the floats.  a1 = min(max(t, RU(t/2 + 2^-7)), 448):
// below 2^-6, E4M3's subnormal range (spacing 2^-9), a1 = RU(t/2 + 2^-7) lies
// in [2^-7, 2^-6), whose three kept mantissa bits are floor(t / 2^-9) and whose
// 20 bits below hold the fraction rounded upward on their grid (exact for a
// comparison with the integer 16k); from 2^-6 on a1 = t, whose 20 bits below
// the kept three are the fraction of its E4M3 interval.  Either way the code
// is (exponent field << 3 | kept bits) - 960, and t goes up iff U < fraction
// iff 16k < low20 iff low20 + 2^20 - 1 - 16k carries into the kept bits; 448
// (0x7E, the largest finite code) has low20 = 0 and never goes up.
__device__ __forceinline__ uint32_t e4m3x2_sr(float2 t, uint32_t ka, uint32_t kb) {
  const float a = fminf(fmaxf(t.x, __fmaf_ru(t.x, 0.5f, 0x1p-7f)), 448.0f);
  const float b = fminf(fmaxf(t.y, __fmaf_ru(t.y, 0.5f, 0x1p-7f)), 448.0f);
  const uint32_t ca = ((__float_as_uint(a) + 0xFFFFFu - (ka << 4)) >> 20) - 960u;
  const uint32_t cb = ((__float_as_uint(b) + 0xFFFFFu - (kb << 4)) >> 20) - 960u;
  return ca | (cb << 8);
}

// Stochastic rounding of one block of 16 scaled values; elem = view index of element 0.
__device__ __forceinline__ void sr_block(const float (&y)[16], PhiloxKey key, uint64_t elem, uint32_t& lo,
                                         uint32_t& hi) {
  const uint64_t call0 = elem >> 3;
  lo = sr_codes8(y, philox_call(key, call0, kTagElement));
  hi = sr_codes8(y + 8, philox_call(key, call0 + 1, kTagElement));
}

// max |z| of each of the two blocks of a pair: one chain of three-input
// maxima per block (exact in any order; two live values).
__device__ __forceinline__ void absmax_pair(const float2 (&z)[16], float& aa, float& ab) {
  float a = absmax3(z[0].x, z[1].x, z[2].x), b = absmax3(z[0].y, z[1].y, z[2].y);
#pragma unroll
  for (int i = 3; i < 15; i += 2) {
    a = max3(a, fabsf(z[i].x), fabsf(z[i + 1].x));
    b = max3(b, fabsf(z[i].y), fabsf(z[i + 1].y));
  }
  aa = fmaxf(a, fabsf(z[15].x));
  ab = fmaxf(b, fabsf(z[15].y));
}

// The scale table of one launch: for every E4M3 code S (0x7F, never produced,
// decodes to NaN) dec(S), d = RN(dec(S) s_g) and RN(1/d) (0 when d = 0), the
// same values quantize_pair would compute per block.  Built by `n` threads
// of the CTA into shared memory; the caller synchronises before use.
__device__ __forceinline__ void build_scale_table(float4* tbl, float s_g, uint32_t tid, uint32_t n) {
  for (uint32_t S = tid; S < 128; S += n) {
    const float dS = e4m3_decode(S);
    const float d = __fmul_rn(dS, s_g);
    tbl[S] = make_float4(dS, d, d != 0.0f ? __frcp_rn(d) : 0.0f, 0.0f);
  }
}

// The scale constants of E4M3 code S: from the launch's table (TBL), or
// computed (the same values).
template <bool TBL>
__device__ __forceinline__ float4 scale_entry(const ScaleCtx& sc, uint32_t S) {
  if constexpr (TBL) {
    return sc.tbl[S];
  } else {
    const float dS = e4m3_decode(S);
    const float d = __fmul_rn(dS, sc.s_g);
    return make_float4(dS, d, d != 0.0f ? __frcp_rn(d) : 0.0f, 0.0f);
  }
}

// Quantize blocks a (z[i].x) and b (z[i].y) of one pair under the launch's
// ScaleCtx (with TBL its scale table must be built: sc.tbl), writing their
// codes and scales; the same results as quantize_block on each block.
template <int MODE, bool TBL = true>
__device__ __forceinline__ void quantize_pair(const float2 (&z)[16], const ScaleCtx& sc, const PairRng& rng,
                                              BlockOut& oa, BlockOut& ob) {
  float aa, ab;
  absmax_pair(z, aa, ab);

  if constexpr (MODE == k4over6) {
    uint32_t S[2], ca_lo[2], ca_hi[2], cb_lo[2], cb_hi[2];
    float2 err[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 sf = k == 0 ? div2_by(f2(aa, ab), sc.q6, sc.r6, sc.markstein)
                               : div2_by(f2(aa, ab), sc.q4, sc.r4, sc.markstein);
      S[k] = e4m3x2_rne_sat(sf.x, sf.y);
      const float4 ta = scale_entry<TBL>(sc, S[k] & 0xFFu), tb = scale_entry<TBL>(sc, (S[k] >> 8) & 0xFFu);
      const float2 d = f2(ta.y, tb.y);
      const float2 r = f2(ta.z, tb.z);
      float ya[16], yb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 y = mul2_rn(z[i], r);
        ya[i] = y.x;
        yb[i] = y.y;
      }
      rtn_codes(ya, ca_lo[k], ca_hi[k]);
      rtn_codes(yb, cb_lo[k], cb_hi[k]);
      float va[16], vb[16];
      e2m1x8_to_f32(ca_lo[k], va);
      e2m1x8_to_f32(ca_hi[k], va + 8);
      e2m1x8_to_f32(cb_lo[k], vb);
      e2m1x8_to_f32(cb_hi[k], vb + 8);
      float2 e = f2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 diff = sub2_packed(z[i], mul2_unmerged(f2(va[i], vb[i]), d, sc.nz));
        e = fma2_rn(diff, diff, e);
      }
      err[k] = e;
    }
    const bool pa = err[1].x < err[0].x, pb = err[1].y < err[0].y;
    oa.lo = pa ? ca_lo[1] : ca_lo[0];
    oa.hi = pa ? ca_hi[1] : ca_hi[0];
    oa.scale = (pa ? S[1] : S[0]) & 0xFFu;
    ob.lo = pb ? cb_lo[1] : cb_lo[0];
    ob.hi = pb ? cb_hi[1] : cb_hi[0];
    ob.scale = ((pb ? S[1] : S[0]) >> 8) & 0xFFu;
    return;
  } else if constexpr (is_3bit_e4m3<MODE>()) {
    // q6 holds RN(m s_g) for the mode's element maximum m (make_scale_ctx)
    const float2 sf = div2_by(f2(aa, ab), sc.q6, sc.r6, sc.markstein);
    const uint32_t S2 = e4m3x2_rne_sat(sf.x, sf.y);
    const uint32_t Sa = S2 & 0xFFu, Sb = S2 >> 8;
    const float4 ta = scale_entry<TBL>(sc, Sa), tb = scale_entry<TBL>(sc, Sb);
    const float2 r = f2(ta.z, tb.z);  // 0 for a zero scale: y = 0, codes 0, no flag
    float ya[16], yb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = mul2_rn(z[i], r);
      ya[i] = y.x;
      yb[i] = y.y;
    }
    oa = block3_codes<MODE>(ya, Sa);
    ob = block3_codes<MODE>(yb, Sb);
    return;
  } else if constexpr (MODE == kMXFP3) {
    // one 32-element group, as MXFP4 with E2M0 elements (E2M0's largest
    // value, 4, has exponent 2 as E2M1's 6 does: the same scale byte)
    const uint32_t f = __float_as_uint(fmaxf(aa, ab)) >> 23;
    const uint32_t byte = f > 2u ? f - 2u : 0u;
    const float inv = __uint_as_float((254u - byte) << 23);
    float ya[16], yb[16];
    uint32_t ta[16], tb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = mul2_rn(z[i], f2(inv, inv));
      ya[i] = y.x;
      yb[i] = y.y;
      ta[i] = e2m0_exponent_bits(y.x);
      tb[i] = e2m0_exponent_bits(y.y);
    }
    oa = BlockOut{e2m0_nibbles8(ta, ya), e2m0_nibbles8(ta + 8, ya + 8), byte};
    ob = BlockOut{e2m0_nibbles8(tb, yb), e2m0_nibbles8(tb + 8, yb + 8), byte};
    return;
  } else if constexpr (MODE == kNVINT4) {
    // q6 holds RN(7 s_g) for this mode (make_scale_ctx)
    const float2 sf = div2_by(f2(aa, ab), sc.q6, sc.r6, sc.markstein);
    const uint32_t S2 = e4m3x2_rne_sat(sf.x, sf.y);
    const uint32_t Sa = S2 & 0xFFu, Sb = S2 >> 8;
    const float4 ta = scale_entry<TBL>(sc, Sa), tb = scale_entry<TBL>(sc, Sb);
    const float2 r = f2(ta.z, tb.z);  // RN(1/d), 0 for a zero scale: y = 0, codes 0
    // k = clamp(RNE(y), -7, 7): |k| from int_magnitude_sum, the sign that of y
    float ya[16], yb[16];
    uint32_t sa[16], sb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = mul2_rn(z[i], r);
      ya[i] = y.x;
      yb[i] = y.y;
      sa[i] = __float_as_uint(int_magnitude_sum(y.x));
      sb[i] = __float_as_uint(int_magnitude_sum(y.y));
    }
    oa = BlockOut{int_nibbles8(sa, sign_nibbles8(ya)), int_nibbles8(sa + 8, sign_nibbles8(ya + 8)), Sa};
    ob = BlockOut{int_nibbles8(sb, sign_nibbles8(yb)), int_nibbles8(sb + 8, sign_nibbles8(yb + 8)), Sb};
    return;
  } else if constexpr (MODE == kMXFP4) {
    // The pair is one 32-element MXFP4 group (block a its first half, b its
    // second).  Shared exponent E = floor(log2 max|z|) - 2 clamped to
    // [-127, 127]: from the exponent field f of the group maximum, the scale
    // byte E + 127 = max(f - 2, 0) (f = 0 for zero and subnormal maxima, whose
    // E clamps to -127).  y = z * 2^-E is z / 2^E rounded once (2^-E is a
    // normal float for every E here); RTN codes saturate at 6.
    const uint32_t f = __float_as_uint(fmaxf(aa, ab)) >> 23;
    const uint32_t byte = f > 2u ? f - 2u : 0u;
    const float inv = __uint_as_float((254u - byte) << 23);
    const float2 inv2 = f2(inv, inv);
    float ya[16], yb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float2 y = mul2_rn(z[i], inv2);
      ya[i] = y.x;
      yb[i] = y.y;
    }
    rtn_codes(ya, oa.lo, oa.hi);
    rtn_codes(yb, ob.lo, ob.hi);
    oa.scale = byte;
    ob.scale = byte;
    return;
  } else if constexpr (MODE == kScaleSearch) {
    const float2 sf = div2_by(f2(aa, ab), sc.q6, sc.r6, sc.markstein);
    const uint32_t s02 = e4m3x2_rne_sat(sf.x, sf.y);
    const uint32_t s0a = s02 & 0xFFu, s0b = s02 >> 8;
    float2 best = f2(__int_as_float(0x7F800000), __int_as_float(0x7F800000));
    oa = BlockOut{0u, 0u, 0u};
    ob = BlockOut{0u, 0u, 0u};
#pragma unroll 1
    for (int t = 0; t < kSearchCandidates; ++t) {
      const uint32_t Sa = search_code(s0a, t), Sb = search_code(s0b, t);
      const float4 ta = scale_entry<TBL>(sc, Sa), tb = scale_entry<TBL>(sc, Sb);
      const float2 d = f2(ta.y, tb.y), r = f2(ta.z, tb.z);
      // a zero scale (d = 0, RN(1/d) tabulated as 0) gives y = 0, codes 0 and
      // the error sum of z^2, as the block with no scale
      float ya[16], yb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 y = mul2_rn(z[i], r);
        ya[i] = y.x;
        yb[i] = y.y;
      }
      uint32_t ca_lo, ca_hi, cb_lo, cb_hi;
      rtn_codes(ya, ca_lo, ca_hi);
      rtn_codes(yb, cb_lo, cb_hi);
      float va[16], vb[16];
      e2m1x8_to_f32(ca_lo, va);
      e2m1x8_to_f32(ca_hi, va + 8);
      e2m1x8_to_f32(cb_lo, vb);
      e2m1x8_to_f32(cb_hi, vb + 8);
      float2 e = f2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 diff = sub2_packed(z[i], mul2_unmerged(f2(va[i], vb[i]), d, sc.nz));
        e = fma2_rn(diff, diff, e);
      }
      if (e.x < best.x) {
        best.x = e.x;
        oa = BlockOut{ca_lo, ca_hi, Sa};
      }
      if (e.y < best.y) {
        best.y = e.y;
        ob = BlockOut{cb_lo, cb_hi, Sb};
      }
    }
    return;
  } else {
    const float2 sf = div2_by(f2(aa, ab), sc.q6, sc.r6, sc.markstein);
    uint32_t S2 = e4m3x2_rne_sat(sf.x, sf.y);
    uint32_t Sa = S2 & 0xFFu, Sb = S2 >> 8;
    float4 ta = scale_entry<TBL>(sc, Sa), tb = scale_entry<TBL>(sc, Sb);
    if constexpr (MODE == kSR) {
      if (Sa < 0x7Eu && ta.x < sf.x) ta = scale_entry<TBL>(sc, ++Sa);
      if (Sb < 0x7Eu && tb.x < sf.y) tb = scale_entry<TBL>(sc, ++Sb);
    }
    const float2 dS = f2(ta.x, tb.x);
    oa.scale = Sa;
    ob.scale = Sb;
    const float2 d = f2(ta.y, tb.y);
    const float2 r = f2(ta.z, tb.z);
    float ya[16], yb[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      // IF4 subtracts from y below: its product is kept unmerged
      const float2 y = MODE == kIF4 ? mul2_unmerged(z[i], r, sc.nz) : mul2_rn(z[i], r);
      ya[i] = y.x;
      yb[i] = y.y;
    }
    if constexpr (MODE == kRTN) {
      rtn_codes(ya, oa.lo, oa.hi);
      rtn_codes(yb, ob.lo, ob.hi);
    } else if constexpr (MODE == kSR) {
      sr_block(ya, rng.key, rng.elem_a, oa.lo, oa.hi);
      sr_block(yb, rng.key, rng.elem_b, ob.lo, ob.hi);
    } else if constexpr (MODE == kMSEDEN) {
      rtn_codes(ya, oa.lo, oa.hi);
      rtn_codes(yb, ob.lo, ob.hi);
      float va[16], vb[16];
      e2m1x8_to_f32(oa.lo, va);
      e2m1x8_to_f32(oa.hi, va + 8);
      e2m1x8_to_f32(ob.lo, vb);
      e2m1x8_to_f32(ob.hi, vb + 8);
      float2 num = f2(0.0f, 0.0f), den = f2(0.0f, 0.0f);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 y = f2(ya[i], yb[i]);
        num = fma2_rn(y, y, num);
        den = fma2_rn(y, f2(va[i], vb[i]), den);
      }
      const float qa = __fdiv_rn(num.x, den.x), qb = __fdiv_rn(num.y, den.y);
      const float ca = (num.x > 0.0f && den.x > 0.0f) ? qa : 1.0f;
      const float cb = (num.y > 0.0f && den.y > 0.0f) ? qb : 1.0f;
      const uint32_t S = e4m3x2_sr(mul2_rn(dS, f2(ca, cb)), rng.k_a, rng.k_b);
      oa.scale = S & 0xFFu;
      ob.scale = S >> 8;
    } else {  // kIF4
      uint32_t fa_lo, fa_hi, fb_lo, fb_hi;
      rtn_codes(ya, fa_lo, fa_hi);
      rtn_codes(yb, fb_lo, fb_hi);
      float va[16], vb[16];
      e2m1x8_to_f32(fa_lo, va);
      e2m1x8_to_f32(fa_hi, va + 8);
      e2m1x8_to_f32(fb_lo, vb);
      e2m1x8_to_f32(fb_hi, vb + 8);
      float2 eF = f2(0.0f, 0.0f), eI = f2(0.0f, 0.0f);
      uint32_t sa[16], sb[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 y = f2(ya[i], yb[i]);
        const float2 dF = sub2_packed(y, f2(va[i], vb[i]));
        eF = fma2_rn(dF, dF, eF);
        // the INT4 level k = clamp(RNE(y K1), -7, 7) through its magnitude
        // |k| = s - 1.5 2^23, s = RN(RN(min(|y|, 6) K1) + 1.5 2^23): RN(6 K1)
        // is 7 exactly and RN is monotone, so clamping |y| at 6 first clamps
        // the level at 7 and the two-lane sum needs no clamp of its own; and
        // |y| - |k| K2 = +-(y - k K2), the same square (k is 0 or has the
        // sign of y)
        const float2 yc = f2(fminf(fabsf(y.x), 6.0f), fminf(fabsf(y.y), 6.0f));
        const float2 s2 = add2_rn(mul2_unmerged(yc, f2(kIF4K1, kIF4K1), sc.nz), f2(kRoundMagic, kRoundMagic));
        sa[i] = __float_as_uint(s2.x);
        sb[i] = __float_as_uint(s2.y);
        const float2 vi = mul2_rn(sub2_rn(s2, f2(kRoundMagic, kRoundMagic)), f2(kIF4K2, kIF4K2));
        const float2 dI = f2(__fsub_rn(fabsf(y.x), vi.x), __fsub_rn(fabsf(y.y), vi.y));
        eI = fma2_rn(dI, dI, eI);
      }
      // signs: a nonzero level needs RN(|y| K1) > 1/2, so |y| > 3/8, where
      // the E2M1 code of y is nonzero and carries its sign
      const uint32_t ia_lo = int_nibbles8(sa, fa_lo), ia_hi = int_nibbles8(sa + 8, fa_hi);
      const uint32_t ib_lo = int_nibbles8(sb, fb_lo), ib_hi = int_nibbles8(sb + 8, fb_hi);
      const bool inta = eI.x < eF.x, intb = eI.y < eF.y;
      oa.lo = inta ? ia_lo : fa_lo;
      oa.hi = inta ? ia_hi : fa_hi;
      ob.lo = intb ? ib_lo : fb_lo;
      ob.hi = intb ? ib_hi : fb_hi;
      if (inta) oa.scale |= 0x80u;
      if (intb) ob.scale |= 0x80u;
    }
  }
}

// 16-bit scale draws of N consecutive view blocks b0 .. b0+N-1 (MS-EDEN):
// one Philox call when they lie in one group of eight, two otherwise.
template <int N>
__device__ __forceinline__ void block_draws(PhiloxKey key, uint64_t b0, uint32_t (&k)[N]) {
  const uint32_t first = static_cast<uint32_t>(b0 & 7u);
  const uint4 w0 = philox_call(key, b0 >> 3, kTagBlock);
  if (first + N <= 8) {
#pragma unroll
    for (int j = 0; j < N; ++j) k[j] = half_word(w0, first + j);
  } else {
    const uint4 w1 = philox_call(key, (b0 >> 3) + 1, kTagBlock);
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const uint32_t i = first + j;
      k[j] = i < 8 ? half_word(w0, i) : half_word(w1, i - 8);
    }
  }
}

}  // namespace nvfp4

/* CPU check of the bit-level code formation the quantization kernels use,
 * against the rules written from their definitions.
 *
 * (1) Stochastic rounding onto E2M1 (eight elements per 16-bit-uniform call).
 *     Rule: a = min(|y|, 6); l = the largest grid value <= a, u the next one
 *     (grid 0, 0.5, 1, 1.5, 2, 3, 4, 6); with U = k 2^-16 the magnitude goes
 *     up iff U < (a - l) / (u - l); code = sign(y) << 3 | index, and a code of
 *     magnitude 0 is 0.  Evaluated in binary64, where a - l and the quotient
 *     by the power-of-two gap are exact.
 *     Kernel form (restated): a1 = min(max(a, RU(0.5 a + 0.5)), 6); with
 *     the draws of a pair in one word (low half: even element, high half:
 *     odd) and h = word >> 16, t = 64 bits(a1) + 0x4FFFFFC0 + h 2^28 +
 *     word (2^32 - 4096) for the even element and t = 64 bits(a1) +
 *     0x4FFFFFC0 + h (2^32 - 4096) for the odd one (mod 2^32);
 *     v = (t & 0x7FFFFFFF) | (bits(y) & 0x80000000); the top nibbles of the
 *     eight v gathered into one word with byte permutes, then the sign of a
 *     zero magnitude cleared.
 * (2) INT4 and INT3 levels (NVINT4, IF4's integer option; NVINT3, IF3's).
 *     Rule: k = clamp(RNE(t), -K, K) (K = 7, 3) as a sign-magnitude nibble,
 *     never -0.
 *     Kernel form (restated): s = min(RN(|t| + 1.5 2^23), 1.5 2^23 + K); the
 *     low bytes of eight s gathered into nibbles with byte permutes, the
 *     signs of the eight t added from their top bytes, then the sign of a
 *     zero magnitude cleared.
 * (2b) IF4's INT4 level magnitude from y.
 *     Rule: |k| = |clamp(RNE(RN(y K1)), -7, 7)| with K1 = RN(7/6).
 *     Kernel form (restated): s = RN(RN(min(|y|, 6) K1) + 1.5 2^23), |k| =
 *     the low byte of s (no clamp on s: RN(6 K1) = 7).
 * (2c) Stochastic rounding onto E4M3 (MS-EDEN's corrected scale t >= 0).
 *     Rule: lo = the largest E4M3 value <= t (448 for t >= 448), hi the next;
 *     with U = k 2^-16 the code goes up iff U (hi - lo) < t - lo (binary64,
 *     exact).
 *     Kernel form (restated): a1 = min(max(t, RU(t/2 + 2^-7)), 448); code =
 *     ((bits(a1) + 2^20 - 1 - 16k) >> 20) - 960.
 * (3) E2M0 codes and magnitudes (NVFP3, MXFP3, IF3's E2M0 option).
 *     Rule: the nearest of {0, 1, 2, 4} to |y| (distances in binary64 from
 *     min(|y|, 8), exact), a tie going to the even code index (0.5 -> 0,
 *     1.5 -> 2, 3 -> 2); code = sign(y) << 3 | index, a zero index unsigned.
 *     Kernel form (restated): a1 = min(max(|y|, RU(0.5 |y| + 0.5)), 4);
 *     t = bits(a1) + 2^22 - 1 + ((bits(a1) >> 23) & 1); v = (32 t + 2^29) |
 *     (bits(y) & 0x80000000); the top nibbles of eight v gathered as for SR,
 *     then the sign of a zero index cleared; the magnitude is min(2p - 1, p)
 *     with p the float of bits t & 0xFF800000.
 *     Also checked: where RNE(RN(|y| 3/4)) >= 1 (a nonzero IF3 integer
 *     level) the E2M0 index is nonzero, so it carries the sign of y.
 * Byte permute: byte n of perm(x, y, s) is byte (nibble n of s) of the
 * eight bytes y:x (x bytes 0..3, y bytes 4..7).
 * Build: cc -O2 -ffp-contract=off -fno-fast-math -frounding-math, linked with
 * -lm (the upward-rounded fused multiply-add runs under FE_UPWARD). */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static uint32_t perm(uint32_t x, uint32_t y, uint32_t s) {
  const uint64_t b = ((uint64_t)y << 32) | x;
  uint32_t r = 0;
  for (int n = 0; n < 4; ++n) r |= (uint32_t)((b >> (8 * ((s >> (4 * n)) & 7u))) & 0xFFu) << (8 * n);
  return r;
}
static uint32_t clear_negative_zero(uint32_t w) {
  uint32_t out = 0;
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = (w >> (4 * i)) & 0xFu;
    out |= ((c & 7u) ? c : 0u) << (4 * i);
  }
  return out;
}
static float fma_up(float a, float b, float c) {
  const int old = fegetround();
  fesetround(FE_UPWARD);
  volatile float r = fmaf(a, b, c);
  fesetround(old);
  return r;
}

/* ------------------------------------------------------------------ SR */
static const double kGrid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static uint32_t sr_rule(float y, uint32_t k) {
  double a = fabs((double)y);
  if (!(a <= 6.0)) a = 6.0;
  int i = 0;
  while (i < 7 && kGrid[i + 1] <= a) ++i;
  uint32_t idx = (uint32_t)i;
  if (i < 7 && (double)k * 0x1p-16 < (a - kGrid[i]) / (kGrid[i + 1] - kGrid[i])) idx = (uint32_t)i + 1u;
  return idx == 0 ? 0u : (idx | (signbit(y) ? 8u : 0u));
}

/* the eight-element kernel form; k[i] = draw of element i, held as the
 * generator delivers it: word i/2, low half for even i, high for odd */
static uint32_t sr_kernel8(const float* y, const uint32_t* k) {
  uint32_t v[8];
  for (int m = 0; m < 4; ++m) {
    const uint32_t word = k[2 * m] | (k[2 * m + 1] << 16);
    const uint32_t h = word >> 16;
    for (int j = 0; j < 2; ++j) {
      const int i = 2 * m + j;
      const float a = fabsf(y[i]);
      const float a1 = fminf(fmaxf(a, fma_up(a, 0.5f, 0.5f)), 6.0f);
      const uint32_t base = to_bits(a1) * 64u + 0x4FFFFFC0u;
      const uint32_t t = j == 0 ? h * 0x10000000u + word * 0xFFFFF000u + base : h * 0xFFFFF000u + base;
      v[i] = (t & 0x7FFFFFFFu) | (to_bits(y[i]) & 0x80000000u);
    }
  }
  const uint32_t even = perm(perm(v[0], v[2], 0x0073u), perm(v[4], v[6], 0x7300u), 0x7610u);
  const uint32_t odd = perm(perm(v[1], v[3], 0x0073u), perm(v[5], v[7], 0x7300u), 0x7610u);
  return clear_negative_zero(((even >> 4) & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u));
}

/* The draws next to the decision point of y: k with k 2^-16 just below and
 * above (a - l)/(u - l), and the extremes. */
static int decision_draws(float y, uint32_t* out) {
  double a = fabs((double)y);
  if (!(a <= 6.0)) a = 6.0;
  int i = 0;
  while (i < 7 && kGrid[i + 1] <= a) ++i;
  const double f = i < 7 ? (a - kGrid[i]) / (kGrid[i + 1] - kGrid[i]) : 0.0;
  const int64_t c = (int64_t)floor(f * 65536.0);
  int n = 0;
  for (int64_t d = -2; d <= 2; ++d)
    if (c + d >= 0 && c + d <= 65535) out[n++] = (uint32_t)(c + d);
  out[n++] = 0;
  out[n++] = 65535;
  return n;
}

static uint64_t rng_state;
static uint64_t next64(void) {
  rng_state ^= rng_state << 13;
  rng_state ^= rng_state >> 7;
  rng_state ^= rng_state << 17;
  return rng_state;
}

/* Every finite bf16 value (both signs) at the draws next to its decision
 * point, each as element `slot` of an eight-element word whose other
 * elements are random; then `n_random` words of random binary32 values in
 * (-8, 8) with random draws.  Returns the number of elements whose code
 * differs from the rule; *checked receives the number compared. */
int64_t sr_check(int64_t n_random, int variant, int64_t* checked) {
  int64_t bad = 0, n = 0;
  rng_state = 0x9E3779B97F4A7C15ull;
  for (uint32_t h = 0; h < 65536u; ++h) {
    const float y0 = from_bits(h << 16);
    if (!isfinite(y0)) continue;
    uint32_t ks[8];
    const int nk = decision_draws(y0, ks);
    for (int j = 0; j < nk; ++j) {
      float y[8];
      uint32_t k[8];
      const int slot = (int)(next64() & 7u);
      for (int e = 0; e < 8; ++e) {
        y[e] = from_bits((uint32_t)next64() & 0xC0FFFFFFu);  /* |y| < 8 */
        k[e] = (uint32_t)next64() & 0xFFFFu;
      }
      y[slot] = y0;
      k[slot] = ks[j];
      uint32_t w = sr_kernel8(y, k);
      if (variant == 1) w ^= 1u << (4 * slot);  /* a planted mistake: one index bit flipped */
      for (int e = 0; e < 8; ++e) {
        ++n;
        bad += ((w >> (4 * e)) & 0xFu) != sr_rule(y[e], k[e]);
      }
    }
  }
  for (int64_t r = 0; r < n_random; ++r) {
    float y[8];
    uint32_t k[8];
    for (int e = 0; e < 8; ++e) {
      y[e] = from_bits((uint32_t)next64() & 0xC0FFFFFFu);
      k[e] = (uint32_t)next64() & 0xFFFFu;
    }
    /* below 1, where 0.5 + a/2 is inexact and its upward rounding decides:
     * one element of each word at a draw next to its decision point */
    if (r & 1) {
      uint32_t ks[8];
      const int slot = (int)(next64() & 7u);
      y[slot] = from_bits(((uint32_t)next64() & 0x807FFFFFu) | 0x3F000000u) * (float)((next64() & 1u) + 1u) * 0.5f;
      const int nk = decision_draws(y[slot], ks);
      k[slot] = ks[next64() % (uint64_t)nk];
    }
    const uint32_t w = sr_kernel8(y, k);
    for (int e = 0; e < 8; ++e) {
      ++n;
      bad += ((w >> (4 * e)) & 0xFu) != sr_rule(y[e], k[e]);
    }
  }
  *checked = n;
  return bad;
}

/* ------------------------------------------------------------ INT4, INT3 */
static uint32_t int_rule(float t, int kmax) {
  double k = nearbyint((double)t);  /* ties to even (default rounding mode) */
  if (k > kmax) k = kmax;
  if (k < -kmax) k = -kmax;
  const int ki = (int)k;
  return ki == 0 ? 0u : ((uint32_t)(ki < 0 ? -ki : ki) | (ki < 0 ? 8u : 0u));
}

static uint32_t int_kernel8(const float* t, int kmax) {
  const float magic = 12582912.0f;  /* 1.5 2^23 */
  uint32_t s[8];
  for (int i = 0; i < 8; ++i) s[i] = to_bits(fminf(fabsf(t[i]) + magic, magic + (float)kmax));
  const uint32_t even = perm(perm(s[0], s[2], 0x0040u), perm(s[4], s[6], 0x4000u), 0x7610u);
  const uint32_t odd = perm(perm(s[1], s[3], 0x0040u), perm(s[5], s[7], 0x4000u), 0x7610u);
  const uint32_t se = perm(perm(to_bits(t[0]), to_bits(t[2]), 0x0073u), perm(to_bits(t[4]), to_bits(t[6]), 0x7300u), 0x7610u);
  const uint32_t so = perm(perm(to_bits(t[1]), to_bits(t[3]), 0x0073u), perm(to_bits(t[5]), to_bits(t[7]), 0x7300u), 0x7610u);
  const uint32_t signs = ((se >> 4) & 0x08080808u) | (so & 0x80808080u);
  return clear_negative_zero(even | (odd << 4) | (signs & 0x88888888u));
}

/* Values t: every multiple of 1/4 in [-10, 10] (the ties x.5 among them, and
 * values past the clamp), their binary32 neighbours, every finite bf16 value
 * (at 2^22 and above RN(|t| + 1.5 2^23) is past the clamp as well), and
 * random binary32 values in (-16, 16); eight per word in order.  Returns the
 * number of elements whose nibble differs from the rule. */
static int64_t int_levels_check(int64_t n_random, int variant, int kmax, int64_t* checked) {
  int64_t bad = 0, n = 0;
  rng_state = 0xD1B54A32D192ED03ull;
  float vals[8];
  int nv = 0;
#define FLUSH()                                                              \
  do {                                                                       \
    uint32_t w = int_kernel8(vals, kmax);                                    \
    if (variant == 1) w ^= 4u;                                               \
    for (int e = 0; e < nv; ++e) {                                           \
      ++n;                                                                   \
      bad += ((w >> (4 * e)) & 0xFu) != int_rule(vals[e], kmax);            \
    }                                                                        \
    nv = 0;                                                                  \
  } while (0)
#define PUSH(x)                                                              \
  do {                                                                       \
    vals[nv++] = (x);                                                        \
    if (nv == 8) FLUSH();                                                    \
  } while (0)
  for (int q = -40; q <= 40; ++q) {
    const float t = (float)q * 0.25f;
    PUSH(t);
    PUSH(nextafterf(t, INFINITY));
    PUSH(nextafterf(t, -INFINITY));
  }
  for (uint32_t h = 0; h < 65536u; ++h) {
    const float t = from_bits(h << 16);
    if (isfinite(t)) PUSH(t);
  }
  for (int64_t r = 0; r < n_random; ++r) PUSH(from_bits((uint32_t)next64() & 0xC1FFFFFFu));
  if (nv) {
    while (nv < 8) vals[nv++] = 0.0f;
    FLUSH();
  }
#undef PUSH
#undef FLUSH
  *checked = n;
  return bad;
}

int64_t int4_check(int64_t n_random, int variant, int64_t* checked) {
  return int_levels_check(n_random, variant, 7, checked);
}
int64_t int3_check(int64_t n_random, int variant, int64_t* checked) {
  return int_levels_check(n_random, variant, 3, checked);
}

/* ------------------------------------------------------- IF4 level from y */
static const float kIF4K1 = 0x1.2aaaaap+0f; /* RN(7/6) */

static uint32_t if4_level_rule(float y) {
  volatile float t = y * kIF4K1;
  double k = nearbyint((double)t);
  if (k > 7.0) k = 7.0;
  if (k < -7.0) k = -7.0;
  return (uint32_t)fabs(k);
}

static uint32_t if4_level_kernel(float y) {
  volatile float t = fminf(fabsf(y), 6.0f) * kIF4K1;
  volatile float s = t + 12582912.0f;
  return to_bits(s) & 0xFFu;
}

/* Values y: every finite bf16 value, the points where RN(y K1) is a tie
 * (m + 1/2) / K1 with their binary32 neighbours, 6 and its neighbours, and
 * random binary32 values in (-16, 16).  Variant 1 drops the clamp at 6. */
int64_t if4_level_check(int64_t n_random, int variant, int64_t* checked) {
  int64_t bad = 0, n = 0;
  rng_state = 0x2545F4914F6CDD1Dull;
#define CHECK(yv)                                                            \
  do {                                                                       \
    const float y_ = (yv);                                                   \
    uint32_t got = if4_level_kernel(y_);                                     \
    if (variant == 1) {                                                      \
      volatile float t_ = fabsf(y_) * kIF4K1;                                \
      volatile float s_ = t_ + 12582912.0f;                                  \
      got = to_bits(s_) & 0xFFu;                                             \
    }                                                                        \
    ++n;                                                                     \
    bad += got != if4_level_rule(y_);                                        \
  } while (0)
  for (uint32_t h = 0; h < 65536u; ++h) {
    const float y = from_bits(h << 16);
    if (isfinite(y)) CHECK(y);
  }
  for (int m = -8; m <= 8; ++m) {
    const float y0 = (float)(((double)m + 0.5) / (double)kIF4K1);
    float y = y0;
    for (int d = 0; d < 4; ++d) y = nextafterf(y, -INFINITY);
    for (int d = 0; d < 9; ++d, y = nextafterf(y, INFINITY)) CHECK(y);
  }
  for (int sgn = 0; sgn < 2; ++sgn) {
    const float x = sgn ? -6.0f : 6.0f;
    CHECK(x);
    CHECK(nextafterf(x, INFINITY));
    CHECK(nextafterf(x, -INFINITY));
  }
  for (int64_t r = 0; r < n_random; ++r) CHECK(from_bits((uint32_t)next64() & 0xC1FFFFFFu));
#undef CHECK
  *checked = n;
  return bad;
}

/* ------------------------------------------------------------ E4M3 SR */
static double e4m3_value(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  return e == 0 ? m * 0x1p-9 : (1.0 + m / 8.0) * ldexp(1.0, (int)e - 7);
}

static uint32_t e4m3_sr_rule(float t, uint32_t k) {
  if (t >= 448.0f) return 0x7Eu;
  uint32_t lo = 0;
  while (lo + 1 < 0x7Fu && e4m3_value(lo + 1) <= (double)t) ++lo;
  const double l = e4m3_value(lo), h = e4m3_value(lo + 1);
  return (double)k * 0x1p-16 * (h - l) < (double)t - l ? lo + 1 : lo;
}

static uint32_t e4m3_sr_kernel(float t, uint32_t k) {
  const float a1 = fminf(fmaxf(t, fma_up(t, 0.5f, 0x1p-7f)), 448.0f);
  return ((to_bits(a1) + 0xFFFFFu - (k << 4)) >> 20) - 960u;
}

/* Values t: every E4M3 value and its binary32 neighbours, the decision point
 * lo + k 2^-16 (hi - lo) of every interval at a stride of draws with its
 * neighbours and the neighbouring draws, values past 448, and random binary32
 * values in [0, 2^10).  Variant 1 drops the upward rounding of t/2 + 2^-7. */
int64_t e4m3_sr_check(int64_t n_random, int variant, int64_t* checked) {
  int64_t bad = 0, n = 0;
  rng_state = 0x8C2F1E5A77D3B901ull;
#define CHECK(tv, kv)                                                        \
  do {                                                                       \
    const float t_ = (tv);                                                   \
    const uint32_t k_ = (kv);                                                \
    uint32_t got = e4m3_sr_kernel(t_, k_);                                   \
    if (variant == 1) {                                                      \
      volatile float h_ = t_ * 0.5f;                                         \
      volatile float g_ = h_ + 0x1p-7f;                                      \
      const float a_ = fminf(fmaxf(t_, g_), 448.0f);                         \
      got = ((to_bits(a_) + 0xFFFFFu - (k_ << 4)) >> 20) - 960u;             \
    }                                                                        \
    ++n;                                                                     \
    bad += got != e4m3_sr_rule(t_, k_);                                      \
  } while (0)
  for (uint32_t c = 0; c < 0x7Fu; ++c) {
    const float v = (float)e4m3_value(c);
    const float ts[3] = {v, nextafterf(v, INFINITY), c ? nextafterf(v, -INFINITY) : v};
    for (int i = 0; i < 3; ++i)
      for (uint32_t k = 0; k < 65536u; k += 251u) CHECK(ts[i], k);
  }
  for (uint32_t c = 0; c < 0x7Eu; ++c) {
    const double l = e4m3_value(c), h = e4m3_value(c + 1);
    for (uint32_t k = 1; k < 65535u; k += 97u) {
      const float t = (float)(l + k * 0x1p-16 * (h - l));
      const float ts[3] = {t, nextafterf(t, INFINITY), nextafterf(t, -INFINITY)};
      for (int i = 0; i < 3; ++i)
        for (int d = -1; d <= 1; ++d) CHECK(ts[i], (uint32_t)((int)k + d));
    }
  }
  for (float t = 448.0f; t < 1e30f; t *= 3.7f) CHECK(t, (uint32_t)(next64() & 0xFFFFu));
  for (int64_t r = 0; r < n_random; ++r)
    CHECK(from_bits((uint32_t)next64() & 0x447FFFFFu), (uint32_t)(next64() & 0xFFFFu));
#undef CHECK
  *checked = n;
  return bad;
}

/* ------------------------------------------------------------------ E2M0 */
static const double kE2m0[4] = {0.0, 1.0, 2.0, 4.0};

static uint32_t e2m0_rule(float y) {
  /* |y| capped at 8 (nearest value 4 either way) keeps the distances exact */
  const double a = fmin(fabs((double)y), 8.0);
  int best = 0;
  for (int c = 1; c < 4; ++c) {
    const double dc = fabs(a - kE2m0[c]), db = fabs(a - kE2m0[best]);
    if (dc < db || (dc == db && (c & 1) == 0)) best = c;
  }
  return best == 0 ? 0u : ((uint32_t)best | (signbit(y) ? 8u : 0u));
}

static uint32_t e2m0_t(float y) {
  const float a = fabsf(y);
  const float a1 = fminf(fmaxf(a, fma_up(a, 0.5f, 0.5f)), 4.0f);
  const uint32_t b = to_bits(a1);
  return b + 0x3FFFFFu + ((b >> 23) & 1u);
}

static float e2m0_magnitude(uint32_t t) {
  const float p = from_bits(t & 0xFF800000u);
  volatile float q = fmaf(p, 2.0f, -1.0f);
  return fminf(q, p);
}

static uint32_t e2m0_kernel8(const float* y) {
  uint32_t v[8];
  for (int i = 0; i < 8; ++i) v[i] = (e2m0_t(y[i]) * 32u + 0x20000000u) | (to_bits(y[i]) & 0x80000000u);
  const uint32_t even = perm(perm(v[0], v[2], 0x0073u), perm(v[4], v[6], 0x7300u), 0x7610u);
  const uint32_t odd = perm(perm(v[1], v[3], 0x0073u), perm(v[5], v[7], 0x7300u), 0x7610u);
  return clear_negative_zero(((even >> 4) & 0x0F0F0F0Fu) | (odd & 0xF0F0F0F0u));
}

/* Values y: every finite bf16 value, the thresholds 0.5, 1.5, 3 and the
 * saturation 4 with their binary32 neighbours (both signs), and random
 * binary32 values in (-16, 16); eight per word.  Counts the elements whose
 * code or magnitude differs from the rule, and those where a nonzero IF3
 * integer level meets a zero E2M0 index (variant 1 flips one code bit per
 * word, variant 2 takes the magnitude 0.5 for index 0). */
int64_t e2m0_check(int64_t n_random, int variant, int64_t* checked) {
  int64_t bad = 0, n = 0;
  rng_state = 0x94D049BB133111EBull;
  float vals[8];
  int nv = 0;
#define FLUSH()                                                              \
  do {                                                                       \
    uint32_t w = e2m0_kernel8(vals);                                         \
    if (variant == 1) w ^= 1u;                                               \
    for (int e = 0; e < nv; ++e) {                                           \
      const uint32_t want = e2m0_rule(vals[e]);                              \
      const uint32_t t = e2m0_t(vals[e]);                                    \
      const float mag = variant == 2 ? from_bits(t & 0xFF800000u) : e2m0_magnitude(t); \
      const float lvl = nearbyintf(fabsf(vals[e]) * 0.75f);                  \
      ++n;                                                                   \
      bad += ((w >> (4 * e)) & 0xFu) != want;                                \
      bad += (double)mag != kE2m0[want & 3u];                                \
      bad += lvl >= 1.0f && (want & 3u) == 0u;                               \
    }                                                                        \
    nv = 0;                                                                  \
  } while (0)
#define PUSH(x)                                                              \
  do {                                                                       \
    vals[nv++] = (x);                                                        \
    if (nv == 8) FLUSH();                                                    \
  } while (0)
  static const float edges[] = {0.0f, 0.5f, 0.75f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  for (int k = 0; k < (int)(sizeof(edges) / sizeof(edges[0])); ++k) {
    for (int sgn = 0; sgn < 2; ++sgn) {
      const float x = sgn ? -edges[k] : edges[k];
      PUSH(x);
      PUSH(nextafterf(x, INFINITY));
      PUSH(nextafterf(x, -INFINITY));
    }
  }
  for (uint32_t h = 0; h < 65536u; ++h) {
    const float y = from_bits(h << 16);
    if (isfinite(y)) PUSH(y);
  }
  for (int64_t r = 0; r < n_random; ++r) PUSH(from_bits((uint32_t)next64() & 0xC1FFFFFFu));
  if (nv) {
    while (nv < 8) vals[nv++] = 0.0f;
    FLUSH();
  }
#undef PUSH
#undef FLUSH
  *checked = n;
  return bad;
}

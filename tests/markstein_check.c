/* Exhaustive check, on the CPU, of the division the quantization kernels use
 * for the block scale s_f = RN(a / q), q = RN(m s_g): with r = RN(1/q),
 *
 *     t = RN(a r),  rem = fma(-t, q, a),  d = fma(rem, r, t)
 *
 * (P. Markstein, "Computation of elementary functions on the IBM RISC
 * System/6000 processor", IBM J. Res. Dev. 34(1), 1990: the remainder is exact
 * and one fused correction gives the correctly rounded quotient).  The kernel
 * sequence is restated here with C's fmaf (correctly rounded) and binary32
 * arithmetic, and compared bit for bit with the correctly rounded quotient
 * RN32(a / q), obtained as (float)((double)a / (double)q): a binary64 quotient
 * rounded again to binary32 is the correctly rounded binary32 quotient,
 * because 53 >= 2 * 24 + 2.
 *
 * Divisors: every binary32 significand q in [1, 2) (2^23 values); the result
 * is invariant under scaling a and q by powers of two while nothing
 * overflows or underflows, which the kernels ensure (they divide exactly
 * otherwise).  Dividends: for every E4M3 decision point B -- the E4M3 values
 * (where round-up changes code) and the midpoints between neighbours (where
 * round-to-nearest changes code), whose significands are the 16 values
 * 1 + j/16 -- the five binary32 numbers nearest B q (RN(B q) and two
 * neighbours each way), so every quotient that lands at or beside a scale
 * decision is covered; plus `extra` pseudo-random dividends per divisor.
 * Build: cc -O2 -ffp-contract=off -fno-fast-math, linked with -lm. */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* variant 0: the kernel sequence; variant 1: the product t = RN(a r) alone,
 * without the remainder correction (must differ somewhere: shows that the
 * comparison detects a wrong quotient). */
static float kernel_quotient(float a, float q, float r, int variant) {
  const float t = a * r;
  if (variant == 1) return t;
  const float rem = fmaf(-t, q, a);
  return fmaf(rem, r, t);
}

static int check_one(float a, float q, float r, int variant) {
  const float d = kernel_quotient(a, q, r, variant);
  const float exact = (float)((double)a / (double)q);
  return to_bits(d) != to_bits(exact);
}

/* Returns the number of (a, q) pairs where the kernel quotient differs from
 * RN32(a / q); *checked receives the number of pairs tried.  Divisor
 * significands i0 .. i1-1 (of 2^23). */
int64_t markstein_check(int64_t i0, int64_t i1, int extra, int variant, int64_t* checked, uint32_t* first_a,
                        uint32_t* first_q) {
  int64_t bad = 0, n = 0;
  uint64_t rng = 0x9E3779B97F4A7C15ull ^ (uint64_t)i0;
  for (int64_t i = i0; i < i1; ++i) {
    const float q = from_bits(0x3F800000u | (uint32_t)i);
    const float r = (float)(1.0 / (double)q); /* RN32(1/q): double rounding innocuous for division */
    for (int j = 0; j < 16; ++j) {
      const float B = 1.0f + (float)j / 16.0f;
      const float a0 = B * q; /* RN(B q): B has 5 significant bits, q 24 */
      const uint32_t ab = to_bits(a0);
      for (int k = -2; k <= 2; ++k) {
        const float a = from_bits(ab + (uint32_t)k);
        ++n;
        if (check_one(a, q, r, variant)) {
          if (bad == 0) { *first_a = to_bits(a); *first_q = to_bits(q); }
          ++bad;
        }
      }
    }
    for (int e = 0; e < extra; ++e) {
      rng ^= rng << 13; rng ^= rng >> 7; rng ^= rng << 17; /* xorshift64 */
      const float a = from_bits(0x3F800000u | (uint32_t)(rng & 0x7FFFFFu)) * ((rng >> 40) & 1 ? 2.0f : 1.0f);
      ++n;
      if (check_one(a, q, r, variant)) {
        if (bad == 0) { *first_a = to_bits(a); *first_q = to_bits(q); }
        ++bad;
      }
    }
  }
  *checked = n;
  return bad;
}

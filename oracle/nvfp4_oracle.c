/*
 * nvfp4_oracle.c -- plain, slow, single-threaded CPU oracle for block-scaled
 * NVFP4 quantization (RTN, SR, MS-EDEN, IF4, 4/6, with an optional random
 * Hadamard rotation).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the parity reference for the CUDA
 * library in nvfp4_microscaling_quantization_b200/csrc.  It shares no code,
 * header, table or constant generator with that library, and the library
 * never links, loads or calls it.  Only the tests, __graft_entry__.smoke()
 * and bench.py's CPU-baseline leg use it.
 *
 * Arithmetic: every floating-point step is one IEEE-754 binary32 operation
 * with round-to-nearest-even ("RN" below), compiled with -ffp-contract=off
 * and no fast-math, so the compiler never fuses or reorders it.  The only
 * fused operation is the explicit C99 fmaf() used for the per-block dot
 * products, which is itself a single correctly rounded operation.  binary32
 * is the precision the pages fix for the per-tensor scale (an FP32 scale per
 * tensor), and every integer decision (a 4-bit code, an 8-bit scale, the IF4
 * flag, the 4/6 choice) is taken in that precision on both sides.
 *
 * Sources (page title, then section / table / figure):
 *  [QII-abs]  "Quartet II: Accurate LLM Pre-Training in NVFP4 by Improved
 *             Unbiased Gradient Estimation", abstract (OpenAlex record).
 *  [QII-fwd]  "Quartet II: Fortschritte in der NVFP4-Vortrainierung fuer
 *             Grosse Sprachmodelle", section "Quantisierung im
 *             Vorwaertsdurchlauf".
 *  [QII-bwd]  same article, section "Quantisierung im Rueckwaertsdurchlauf";
 *             [QII-key] its list "Kerninnovationen von Quartet II".
 *  [PAL-intro] "Comparing INT4 and NVFP4 Palettes on Real Gradient Tensors",
 *             opening section (E2M1 value set, 16-element block, Hadamard).
 *  [PAL-corners] same post, section "The two corners, and what the palette
 *             does to them" (absmax scaling, stochastic rounding and its error).
 *  [PAL-16x16] same post, section "45 real tensors disagree" (16x16 RHT).
 *  [IF4-abs]  IF4 paper page (arXiv 2603.28765, "Adaptive Block-Scaled Data
 *             Types"), abstract; [IF4-F1] its Figure 1; [IF4-T1] its Table 1;
 *             [IF4-F3] its Figure 3.
 *  [IF4-T6]  the same page's 3-bit formats table (MXFP3, NVINT3, NVFP3, IF3:
 *             scale type, element type, group size, bits per value).
 *  [SS-abs]   the same IF4 paper page, its related-paper entry on ScaleSearch
 *             (abstract): block scales chosen by searching the scale's
 *             mantissa values for the lowest quantization error.
 *  [PHILOX]   Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy
 *             as 1, 2, 3", SC'11 -- the Philox4x32 bijection with 10 rounds.
 *
 * Where the pages leave a step open, the reading taken is stated at that step.
 * Parity status of every function here is pinned by tests in tests/ (see the
 * "pinned by" line of each function).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_SHAPE (-2)
#define ORC_ERR_UNSUPPORTED (-4)

/* modes and layouts: same numbering as the public C ABI (an interface, not
 * shared code). */
enum { ORC_RTN = 0, ORC_SR = 1, ORC_MS_EDEN = 2, ORC_IF4 = 3, ORC_4OVER6 = 4, ORC_SCALE_SEARCH = 5, ORC_MXFP4 = 6,
       ORC_NVINT4 = 7, ORC_NVFP3 = 8, ORC_NVINT3 = 9, ORC_IF3 = 10, ORC_MXFP3 = 11 };
enum { ORC_ROWWISE = 0, ORC_TRANSPOSED = 1 };

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 [PHILOX].  One call maps a 128-bit counter and a 64-bit key
 * to 128 random bits.  A round multiplies counter words 0 and 2 by the two
 * round multipliers (full 64-bit products), and builds the new counter from
 * the high halves xored with the other words and the key, and the low halves;
 * the key is bumped by the two Weyl constants between rounds.
 * Pinned by: tests/test_oracle_philox.py (cuRAND host generator). */
void oracle_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                          uint32_t out[4]) {
  const uint32_t mult0 = 0xD2511F53u, mult1 = 0xCD9E8D57u;
  const uint32_t weyl0 = 0x9E3779B9u, weyl1 = 0xBB67AE85u;
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t p0 = (uint64_t)mult0 * (uint64_t)c0;
    uint64_t p1 = (uint64_t)mult1 * (uint64_t)c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    k0 += weyl0;
    k1 += weyl1;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The three random streams of the method, each keyed by the seed
 * (key = seed low word, seed high word) and by a tag in counter word 2.
 * Reading (the pages name no generator): a counter-based generator keyed by
 * (seed, element or block index), so results are reproducible. */
static void philox_call(uint64_t seed, uint64_t call, uint32_t tag, uint32_t w[4]) {
  uint32_t ctr[4] = {(uint32_t)call, (uint32_t)(call >> 32), tag, 0u};
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  oracle_philox4x32_10(ctr, key, w);
}

/* Element stochastic-rounding uniform (tag 0): element e of the quantized
 * view (row-major linear index).  Call e/8 yields 8 uniforms of 16 bits:
 * word (e mod 8)/2, low half for even e, high half for odd e.  U = k * 2^-16. */
float oracle_uniform_element(uint64_t seed, uint64_t e) {
  uint32_t w[4];
  philox_call(seed, e >> 3, 0u, w);
  uint32_t word = w[(e & 7u) >> 1];
  uint32_t k = (word >> (16u * (uint32_t)(e & 1u))) & 0xFFFFu;
  return (float)k * 0x1p-16f; /* exact */
}

/* Scale stochastic-rounding uniform (tag 1): block b of the quantized view
 * (row-major linear block index).  Call b/8 yields 8 uniforms of 16 bits, laid
 * out like the element uniforms: word (b mod 8)/2, low half for even b, high
 * half for odd b.  U = k * 2^-16. */
float oracle_uniform_block(uint64_t seed, uint64_t b) {
  uint32_t w[4];
  philox_call(seed, b >> 3, 1u, w);
  uint32_t word = w[(b & 7u) >> 1];
  uint32_t k = (word >> (16u * (uint32_t)(b & 1u))) & 0xFFFFu;
  return (float)k * 0x1p-16f; /* exact */
}

/* Random Hadamard signs (tag 2): sigma_j for j < g (g <= 128) is -1 when bit
 * (j mod 32) of word (j/32) of call 0 is set.  One sign vector of length g is
 * shared by every group of the tensor (see oracle_rht_rows). */
float oracle_rht_sign(uint64_t seed, int j) {
  uint32_t w[4];
  philox_call(seed, (uint64_t)(j >> 7), 2u, w);
  uint32_t bit = (w[(j >> 5) & 3] >> (j & 31)) & 1u;
  return bit ? -1.0f : 1.0f;
}

/* ------------------------------------------------------------------------ */
/* E2M1 (FP4) grid [PAL-intro]: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
 * Reading for the bit layout (the pages give only the value set): a code is
 * sign (bit 3) and a 3-bit magnitude index into that list, which is the usual
 * 1-sign/2-exponent/1-mantissa layout with exponent bias 1. */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_decode(uint8_t code) {
  float m = E2M1_MAG[code & 7u];
  return (code & 8u) ? -m : m;
}

/* Round-to-nearest onto the E2M1 grid, ties to the even code (magnitude index
 * with bit 0 clear), saturating at 6; a zero magnitude is always code 0 (no
 * negative zero).  Reading: ties-to-even as in IEEE-754; saturation because
 * the forward pass is the biased, clipping corner [PAL-corners].
 * The thresholds are the midpoints between neighbouring grid values.
 * Pinned by: tests/test_oracle_formats.py (brute-force nearest grid value
 * over every finite bf16 pattern). */
uint8_t oracle_e2m1_rtn(float y) {
  float a = fabsf(y);
  uint8_t mag;
  if (a <= 0.25f) mag = 0;       /* tie 0.25 -> 0 (even)   */
  else if (a < 0.75f) mag = 1;   /* tie 0.75 -> 1.0 (even) */
  else if (a <= 1.25f) mag = 2;  /* tie 1.25 -> 1.0 (even) */
  else if (a < 1.75f) mag = 3;   /* tie 1.75 -> 2.0 (even) */
  else if (a <= 2.5f) mag = 4;   /* tie 2.5  -> 2.0 (even) */
  else if (a < 3.5f) mag = 5;    /* tie 3.5  -> 4.0 (even) */
  else if (a <= 5.0f) mag = 6;   /* tie 5.0  -> 4.0 (even) */
  else mag = 7;                  /* saturate at 6          */
  if (mag == 0) return 0;
  return (uint8_t)((y < 0.0f ? 8u : 0u) | mag);
}

/* Stochastic rounding onto the E2M1 grid [PAL-corners]: a magnitude between
 * neighbouring grid values l <= a < u rounds up with probability (a-l)/(u-l),
 * so the expectation is a.  Magnitudes above 6 are clamped to 6 first.  With
 * a uniform U, rounding up happens iff U < (a-l)/(u-l); that fraction is exact
 * in binary32 because u-l is a power of two and a-l is exact.
 * Pinned by: tests/test_oracle_modes.py (Monte-Carlo mean, closed-form error). */
uint8_t oracle_e2m1_sr(float y, float U) {
  float a = fabsf(y);
  if (a > 6.0f) a = 6.0f;
  int lo = 0;
  for (int k = 7; k >= 0; --k) {
    if (E2M1_MAG[k] <= a) { lo = k; break; }
  }
  int mag = lo;
  if (lo < 7) {
    float l = E2M1_MAG[lo], u = E2M1_MAG[lo + 1];
    float f = (a - l) / (u - l);
    if (U < f) mag = lo + 1;
  }
  if (mag == 0) return 0;
  return (uint8_t)((y < 0.0f ? 8u : 0u) | (uint8_t)mag);
}

/* ------------------------------------------------------------------------ */
/* E4M3 block scale [IF4-T1]: the NVFP4 scale is FP8 E4M3 with largest value
 * 448 (6 x 448 is the format maximum) and smallest 2^-9 (0.5 x 2^-9 is the
 * format minimum), i.e. exponent bias 7, 3 mantissa bits, subnormals, and
 * the all-ones pattern 0x7F reserved (not a finite value).  Only codes
 * 0x00..0x7E are produced. */
float oracle_e4m3_decode(uint8_t code) {
  int e = (code >> 3) & 15, m = code & 7;
  float mag;
  if (e == 0) mag = ldexpf((float)m, -9);            /* m/8 * 2^-6 */
  else mag = ldexpf((float)(8 + m), e - 10);         /* (1+m/8) * 2^(e-7) */
  return (code & 0x80u) ? -mag : mag;
}

/* Nearest E4M3 value to v >= 0, ties to the even code, saturating at 448:
 * a plain search over the 127 finite non-negative codes.
 * Pinned by: tests/test_oracle_formats.py (torch float8_e4m3fn conversion). */
uint8_t oracle_e4m3_rne_sat(float v) {
  if (!(v > 0.0f)) return 0;
  if (v >= 448.0f) return 0x7E;
  int best = 0;
  double best_d = fabs((double)v);
  for (int c = 1; c <= 0x7E; ++c) {
    double dist = fabs((double)v - (double)oracle_e4m3_decode((uint8_t)c));
    if (dist < best_d || (dist == best_d && (c & 1) == 0)) { best = c; best_d = dist; }
  }
  return (uint8_t)best;
}

/* Smallest E4M3 value >= v (v >= 0), capped at 448: the scale of the unbiased
 * corner must not let any element exceed the top grid value [PAL-corners].
 * Pinned by: tests/test_oracle_formats.py (brute force over the table). */
uint8_t oracle_e4m3_ru_sat(float v) {
  if (!(v > 0.0f)) return 0;
  for (int c = 0; c <= 0x7E; ++c)
    if (oracle_e4m3_decode((uint8_t)c) >= v) return (uint8_t)c;
  return 0x7E;
}

/* Stochastic rounding of t >= 0 onto E4M3: the two neighbouring values
 * lo <= t < hi, hi with probability (t-lo)/(hi-lo); t >= 448 gives 448.
 * This is how MS-EDEN folds its correction factor into the group scale
 * [QII-bwd]. */
uint8_t oracle_e4m3_sr(float t, float U) {
  if (!(t > 0.0f)) return 0;
  if (t >= 448.0f) return 0x7E;
  int lo = 0;
  for (int c = 0x7E; c >= 0; --c) {
    if (oracle_e4m3_decode((uint8_t)c) <= t) { lo = c; break; }
  }
  float l = oracle_e4m3_decode((uint8_t)lo);
  float h = oracle_e4m3_decode((uint8_t)(lo + 1));
  float f = (t - l) / (h - l); /* exact: h-l is a power of two */
  return (uint8_t)(U < f ? lo + 1 : lo);
}

/* ------------------------------------------------------------------------ */
/* Random Hadamard transform [PAL-intro], [PAL-16x16], [QII-bwd]:
 * z = c_g * H_g * (sigma o x) on every group of g consecutive elements of a
 * row, H_g the Sylvester Hadamard matrix, c_g = RN(1/sqrt(g)).  Computed as
 * the textbook fast Walsh-Hadamard butterfly: for h = 1, 2, 4, ..., g/2 and
 * every i with (i & h) == 0, (u_i, u_{i+h}) <- (u_i + u_{i+h}, u_i - u_{i+h}),
 * each sum one binary32 RN operation, then one RN multiply by c_g.
 * The inverse applies the same butterflies to z, multiplies by c_g, then by
 * sigma (H_g H_g = g I).
 * Reading: the sign vector has length g and is shared by every group, so the
 * two operands of a GEMM rotated along the same reduction dimension with the
 * same seed cancel the rotation.
 * Pinned by: tests/test_oracle_rht.py (scipy.linalg.hadamard, exact inverse
 * on small integers, norm preservation). */
float oracle_rht_scale(int g) {
  switch (g) {
    case 16: return 0.25f;
    case 32: return 0x1.6a09e6p-3f;  /* RN(1/sqrt(32)) */
    case 64: return 0.125f;
    case 128: return 0x1.6a09e6p-4f; /* RN(1/sqrt(128)) */
    default: return 0.0f;
  }
}

static int valid_group(int g) { return g == 16 || g == 32 || g == 64 || g == 128; }

static void rht_group_inplace(float* u, int g, const float* sigma, float c, int inverse) {
  if (!inverse)
    for (int j = 0; j < g; ++j) u[j] = sigma[j] * u[j]; /* exact sign flip */
  for (int h = 1; h < g; h <<= 1) {
    for (int i = 0; i < g; ++i) {
      if (i & h) continue;
      float a = u[i], b = u[i + h];
      u[i] = a + b;
      u[i + h] = a - b;
    }
  }
  for (int j = 0; j < g; ++j) u[j] = u[j] * c;
  if (inverse)
    for (int j = 0; j < g; ++j) u[j] = sigma[j] * u[j];
}

/* Rotate (or un-rotate) every g-group along the rows of a dense fp32 matrix
 * in[rows][cols] into out (may alias in).  cols must be a multiple of g. */
int oracle_rht_rows(const float* in, int64_t rows, int64_t cols, int g,
                    uint64_t seed, int inverse, float* out) {
  if (!valid_group(g)) return ORC_ERR_ARG;
  if (rows < 0 || cols < 0 || cols % g) return ORC_ERR_SHAPE;
  float sigma[128];
  for (int j = 0; j < g; ++j) sigma[j] = oracle_rht_sign(seed, j);
  float c = oracle_rht_scale(g);
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t s = 0; s < cols; s += g) {
      float u[128];
      for (int j = 0; j < g; ++j) u[j] = in[r * cols + s + j];
      rht_group_inplace(u, g, sigma, c, inverse);
      for (int j = 0; j < g; ++j) out[r * cols + s + j] = u[j];
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* The quantized view.  Row-wise: V = X (blocks of 16 along a row of X).
 * Transposed: V = X^T (blocks of 16 consecutive rows of one column of X,
 * output stored as X^T row-major).  The backward pass re-quantizes W and X
 * along the other dimension, which is why both views exist [QII-fwd]. */
static float bf16_to_f32(uint16_t h) {
  uint32_t bits = (uint32_t)h << 16;
  float f;
  memcpy(&f, &bits, 4);
  return f;
}

/* View row vr (length vc) of x as fp32, rotated when g > 0. */
static void load_view_row(const uint16_t* x, int64_t ld, int layout, int64_t vr,
                          int64_t vc, int g, const float* sigma, float c, float* row) {
  for (int64_t j = 0; j < vc; ++j)
    row[j] = bf16_to_f32(layout == ORC_ROWWISE ? x[vr * ld + j] : x[j * ld + vr]);
  if (g > 0)
    for (int64_t s = 0; s < vc; s += g) rht_group_inplace(row + s, g, sigma, c, 0);
}

static int check_quant_args(int64_t rows, int64_t cols, int64_t ld, int layout,
                            int mode, int g, int64_t* vr, int64_t* vc) {
  if (layout != ORC_ROWWISE && layout != ORC_TRANSPOSED) return ORC_ERR_ARG;
  if (mode < ORC_RTN || mode > ORC_MXFP3) return ORC_ERR_ARG;
  if (g != 0 && !valid_group(g)) return ORC_ERR_ARG;
  if (mode == ORC_MS_EDEN && g == 0) return ORC_ERR_UNSUPPORTED;
  if (rows < 0 || cols < 0 || ld < cols) return ORC_ERR_SHAPE;
  *vr = layout == ORC_ROWWISE ? rows : cols;
  *vc = layout == ORC_ROWWISE ? cols : rows;
  if (*vc % 16) return ORC_ERR_SHAPE;
  if ((mode == ORC_MXFP4 || mode == ORC_MXFP3) && *vc % 32) return ORC_ERR_SHAPE;
  if (g > 0 && *vc % g) return ORC_ERR_SHAPE;
  return ORC_OK;
}

/* Tensor amax A = max |z| over the whole (rotated) view [QII-fwd] "FP32
 * scale per tensor".  Streams one view row at a time. */
int oracle_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int layout,
                int g, uint64_t seed, float* amax_out) {
  int64_t vr, vc;
  int st = check_quant_args(rows, cols, ld, layout, ORC_RTN, g, &vr, &vc);
  if (st) return st;
  float sigma[128];
  for (int j = 0; j < g; ++j) sigma[j] = oracle_rht_sign(seed, j);
  float c = g ? oracle_rht_scale(g) : 0.0f;
  float* row = (float*)malloc(sizeof(float) * (size_t)(vc > 0 ? vc : 1));
  if (!row) return ORC_ERR_ARG;
  float A = 0.0f;
  for (int64_t r = 0; r < vr; ++r) {
    load_view_row(x, ld, layout, r, vc, g, sigma, c, row);
    for (int64_t j = 0; j < vc; ++j)
      if (fabsf(row[j]) > A) A = fabsf(row[j]);
  }
  free(row);
  *amax_out = A;
  return ORC_OK;
}

/* FP32 per-tensor scale s_g.  Reading ([QII-fwd] only says that each tensor
 * has an FP32 scale; [IF4-T1] gives the maxima 6 x 448 and, for 4/6, 6 x 256): the
 * tensor amax is mapped to the format maximum, s_g = RN(A / (6 M)) with
 * M = 448, or M = 256 for 4/6, MS-EDEN and scale search.  A zero tensor
 * gets s_g = 1.  Scale search takes 256 like 4/6, whose larger-scale option
 * it contains: its upper candidates then reach above the absmax scale before
 * the E4M3 maximum.
 * MS-EDEN takes the 4/6 cap for the same reason 4/6 does: its block scale is
 * later multiplied by a correction factor c, and the scale's stochastic
 * rounding must never saturate at 448 or it loses unbiasedness.  c stays
 * below 1.61: every element with a nonzero RTN value v has y/v <= 1.5, the
 * elements rounded to zero add at most 15 * 0.25^2 to <y, y>, and the block
 * maximum contributes at least 3 * 3 to <y, v>; so 256 * 1.61 < 448. */
float oracle_global_scale(float A, int mode) {
  if (mode == ORC_MXFP4) return 1.0f; /* MXFP4 has no tensor scale [IF4-T1] */
  if (mode == ORC_NVINT4) return A > 0.0f ? A / 3136.0f : 1.0f; /* NVINT4: 7 x 448 [IF4-T1] */
  if (mode == ORC_MXFP3) return 1.0f;
  /* 3-bit formats [IF4-T6]: the element maximum x 448 (E2M0: 4, INT3: 3) */
  if (mode == ORC_NVFP3 || mode == ORC_IF3) return A > 0.0f ? A / 1792.0f : 1.0f;
  if (mode == ORC_NVINT3) return A > 0.0f ? A / 1344.0f : 1.0f;
  float sixM = (mode == ORC_4OVER6 || mode == ORC_MS_EDEN || mode == ORC_SCALE_SEARCH) ? 1536.0f
                                                                                      : 2688.0f; /* exact */
  if (!(A > 0.0f)) return 1.0f;
  return A / sixM;
}

/* Scaled-INT4 constants of IF4.  Reading ([IF4-T1]: IF4's maximum is 6 x 448,
 * not NVINT4's 7 x 448; [IF4-abs]/[IF4-F1]: "scaled INT4" under the same E4M3
 * scale): the INT4 levels k in [-7, 7] stand for k * 6/7, so both options span
 * +-6 under one scale. */
static const float IF4_K1 = (float)(7.0 / 6.0); /* RN(7/6) */
static const float IF4_K2 = (float)(6.0 / 7.0); /* RN(6/7) */

void oracle_if4_constants(float* k1, float* k2) { *k1 = IF4_K1; *k2 = IF4_K2; }

static int int4_level(float y) {
  float t = y * IF4_K1;
  float k = nearbyintf(t); /* ties to even (default rounding mode) */
  if (k > 7.0f) k = 7.0f;
  if (k < -7.0f) k = -7.0f;
  return (int)k;
}
static uint8_t int4_code(int k) { return k == 0 ? 0 : (uint8_t)((k < 0 ? 8 : 0) | (k < 0 ? -k : k)); }
static float int4_value(int k) { return (float)k * IF4_K2; }

/* 3-bit elements [IF4-T6] (the page lists MXFP3 and NVFP3 with E2M0
 * elements, NVINT3 with INT3, IF3 with INT3 / E2M0).  Readings: E2M0 is the
 * E2M1 layout without the mantissa bit (bias 1, the zero exponent holding
 * only 0): magnitudes {0, 1, 2, 4}, round to nearest with ties to the even
 * code; INT3 is sign-magnitude, |k| <= 3.  A 3-bit code is stored in a
 * nibble: sign bit 3, magnitude code in bits 0..1 (bit 2 clear); zero is code
 * 0.  IF3's INT3 levels k stand for k * 4/3 under the shared scale, so both
 * options span +-4 (as IF4's k * 6/7 spans E2M1's +-6). */
static const float E2M0_MAG[4] = {0.0f, 1.0f, 2.0f, 4.0f};
static const float IF3_K1 = (float)(3.0 / 4.0); /* RN(3/4), exact */
static const float IF3_K2 = (float)(4.0 / 3.0); /* RN(4/3) */

static uint8_t e2m0_rtn(float y) {
  float a = fabsf(y);
  uint8_t m = (uint8_t)((a > 0.5f) + (a >= 1.5f) + (a > 3.0f)); /* ties 0.5, 1.5, 3 to codes 0, 2, 2 */
  return m == 0 ? 0 : (uint8_t)(m | (y < 0.0f ? 8u : 0u));
}
static float e2m0_decode(uint8_t c) {
  float v = E2M0_MAG[c & 3u];
  return (c & 8u) ? -v : v;
}
static int int3_level(float t) {
  float k = nearbyintf(t);
  if (k > 3.0f) k = 3.0f;
  if (k < -3.0f) k = -3.0f;
  return (int)k;
}

/* Quantize one 16-element block z[0..15] of view row vr, block column bc.
 * Writes 16 codes (one per element, low nibble) and returns the scale byte. */
static uint8_t quantize_block(const float* z, int mode, float s_g, uint64_t seed,
                              int64_t vr, int64_t vc, int64_t bc, uint8_t* code) {
  float a_b = 0.0f; /* block absmax [PAL-corners]: the absmax sets each block's scale */
  for (int i = 0; i < 16; ++i)
    if (fabsf(z[i]) > a_b) a_b = fabsf(z[i]);

  if (mode == ORC_MXFP3) {
    /* MXFP3 [IF4-T6]: as MXFP4 (32-element groups, UE8M0 shared exponent)
     * with E2M0 elements: E = floor(log2 max |x|) - 2 (2 = the exponent of
     * E2M0's largest value, 4), clamped to [-127, 127]; codes E2M0 RTN of
     * x / 2^E, saturating at 4. */
    const float* grp = (bc & 1) ? z - 16 : z;
    float a = 0.0f;
    for (int i = 0; i < 32; ++i)
      if (fabsf(grp[i]) > a) a = fabsf(grp[i]);
    int E = -127;
    if (a > 0.0f) {
      int e2;
      frexpf(a, &e2);
      E = e2 - 1 - 2;
      if (E < -127) E = -127;
      if (E > 127) E = 127;
    }
    float X = ldexpf(1.0f, E);
    for (int i = 0; i < 16; ++i) code[i] = e2m0_rtn(z[i] / X);
    return (uint8_t)(E + 127);
  }
  if (mode == ORC_NVFP3 || mode == ORC_NVINT3 || mode == ORC_IF3) {
    /* NVFP3 / NVINT3 / IF3 [IF4-T6]: NVFP4's steps with the 3-bit grids, the
     * block absmax mapped to the element maximum m (4 for E2M0 and IF3, 3
     * for INT3): S = E4M3_RNE(RN(a_b / RN(m s_g))), d = RN(dec(S) s_g),
     * y = RN(z RN(1/d)).  IF3 keeps the option with the lower squared error
     * in the y domain (fmaf in element order; ties keep E2M0) and sets bit 7
     * of the scale for INT3, as IF4 does. */
    float m = mode == ORC_NVINT3 ? 3.0f : 4.0f;
    float q = m * s_g;
    uint8_t S3 = oracle_e4m3_rne_sat(a_b / q);
    float d3 = oracle_e4m3_decode(S3) * s_g;
    if (d3 == 0.0f) {
      memset(code, 0, 16);
      return S3;
    }
    float r3 = 1.0f / d3;
    uint8_t cf[16], ci[16];
    float eF = 0.0f, eI = 0.0f;
    for (int i = 0; i < 16; ++i) {
      float y = z[i] * r3;
      if (mode == ORC_NVINT3) {
        code[i] = int4_code(int3_level(y));
        continue;
      }
      cf[i] = e2m0_rtn(y);
      if (mode == ORC_NVFP3) {
        code[i] = cf[i];
        continue;
      }
      float dF = y - e2m0_decode(cf[i]);
      eF = fmaf(dF, dF, eF);
      int k = int3_level(y * IF3_K1);
      ci[i] = int4_code(k);
      float dI = y - (float)k * IF3_K2;
      eI = fmaf(dI, dI, eI);
    }
    if (mode == ORC_IF3) {
      if (eI < eF) {
        memcpy(code, ci, 16);
        return (uint8_t)(S3 | 0x80u);
      }
      memcpy(code, cf, 16);
    }
    return S3;
  }
  if (mode == ORC_NVINT4) {
    /* NVINT4 [IF4-T1]: 16-element blocks, E4M3 scale, INT4 values, maximum
     * 7 x 448, minimum 1 x 2^-9.  Reading: as NVFP4 with the integer grid
     * k in [-7, 7] in place of E2M1: s_g = RN(A / (7 448)) (set above),
     * S = E4M3_RNE(RN(a_b / RN(7 s_g))), d = RN(dec(S) s_g),
     * k = clamp(RNE(RN(z RN(1/d))), -7, 7), stored as IF4's INT4 nibble
     * (sign bit 3, |k| in bits 0..2), value RN(k d). */
    float q7 = 7.0f * s_g;
    uint8_t S7 = oracle_e4m3_rne_sat(a_b / q7);
    float d7 = oracle_e4m3_decode(S7) * s_g;
    if (d7 == 0.0f) {
      memset(code, 0, 16);
      return S7;
    }
    float r7 = 1.0f / d7;
    for (int i = 0; i < 16; ++i) {
      float k = nearbyintf(z[i] * r7); /* ties to even (default rounding mode) */
      if (k > 7.0f) k = 7.0f;
      if (k < -7.0f) k = -7.0f;
      code[i] = int4_code((int)k);
    }
    return S7;
  }

  if (mode == ORC_MXFP4) {
    /* MXFP4 [IF4-T1]: 32-element groups, one UE8M0 (power of two) scale, E2M1
     * values, no tensor scale; maximum 6 x 2^127, minimum 0.5 x 2^-127.
     * Reading (the pages give only that row; the scale rule is that of the
     * OCP Microscaling specification, whose format the row names): the
     * shared exponent is E = floor(log2(max |x| over the group)) - 2 (2 = the
     * exponent of E2M1's largest value), clamped to [-127, 127] (-127 for an
     * all-zero group); the elements are x / 2^E rounded to nearest E2M1, ties
     * to even, saturating at 6.  The scale byte is E + 127, stored for both
     * 16-element halves of the group, so every mode has one scale per 16
     * elements.  This block is the half (bc & 1) of its group. */
    const float* grp = (bc & 1) ? z - 16 : z;
    float a = 0.0f;
    for (int i = 0; i < 32; ++i)
      if (fabsf(grp[i]) > a) a = fabsf(grp[i]);
    int E = -127;
    if (a > 0.0f) {
      int e2;
      frexpf(a, &e2); /* a = m 2^e2, m in [0.5, 1): floor(log2 a) = e2 - 1 */
      E = e2 - 1 - 2;
      if (E < -127) E = -127;
      if (E > 127) E = 127;
    }
    float X = ldexpf(1.0f, E);
    for (int i = 0; i < 16; ++i) code[i] = oracle_e2m1_rtn(z[i] / X);
    return (uint8_t)(E + 127);
  }

  if (mode == ORC_4OVER6) {
    /* 4/6 [QII-fwd] "Four Over Six", [IF4-T1] scale maximum 256.  Reading:
     * map the block absmax to 6 and to 4, keep the scale with the lower
     * squared error in the original domain; ties keep 6. */
    uint8_t Sc[2];
    float err[2];
    uint8_t cc[2][16];
    const float m[2] = {6.0f, 4.0f};
    for (int k = 0; k < 2; ++k) {
      float q = m[k] * s_g;
      float s_f = a_b / q;
      Sc[k] = oracle_e4m3_rne_sat(s_f);
      float d = oracle_e4m3_decode(Sc[k]) * s_g;
      float e = 0.0f;
      if (d == 0.0f) {
        for (int i = 0; i < 16; ++i) { cc[k][i] = 0; e = fmaf(z[i], z[i], e); }
      } else {
        float r = 1.0f / d;
        for (int i = 0; i < 16; ++i) {
          float y = z[i] * r;
          cc[k][i] = oracle_e2m1_rtn(y);
          float deq = oracle_e2m1_decode(cc[k][i]) * d;
          float diff = z[i] - deq;
          e = fmaf(diff, diff, e);
        }
      }
      err[k] = e;
    }
    int pick = err[1] < err[0] ? 1 : 0;
    memcpy(code, cc[pick], 16);
    return Sc[pick];
  }

  if (mode == ORC_SCALE_SEARCH) {
    /* Scale search [PAL-corners]: the low-error corner tries 19 candidate
     * scales per block with round-to-nearest and keeps the one with the
     * least error; [SS-abs]: a search over the microscale's mantissa values
     * for the lowest quantization error.
     * Reading: the candidates are the 19 E4M3 codes S0 - 9 .. S0 + 9 around
     * the absmax scale S0 = E4M3_RNE(RN(a_b / RN(6 s_g))) (E4M3 codes are
     * ordered like their values, so a code step is one mantissa step),
     * clamped to 0 .. 0x7E and visited in the order S0, S0 - 1, S0 + 1,
     * S0 - 2, ...; each is scored as 4/6 scores its two (RTN codes, squared
     * error in the original domain, fmaf in element order); only a strictly
     * lower error replaces the best so far, so ties keep the candidate
     * nearest S0, and S0 first. */
    float q0 = 6.0f * s_g;
    int S0 = oracle_e4m3_rne_sat(a_b / q0);
    uint8_t best_S = 0, cc[16];
    float best_e = INFINITY;
    for (int t = 0; t < 19; ++t) {
      int delta = ((t + 1) / 2) * ((t & 1) ? -1 : 1);
      int Sc = S0 + delta;
      if (Sc < 0) Sc = 0;
      if (Sc > 0x7E) Sc = 0x7E;
      float d = oracle_e4m3_decode((uint8_t)Sc) * s_g;
      float e = 0.0f;
      if (d == 0.0f) {
        for (int i = 0; i < 16; ++i) { cc[i] = 0; e = fmaf(z[i], z[i], e); }
      } else {
        float r = 1.0f / d;
        for (int i = 0; i < 16; ++i) {
          cc[i] = oracle_e2m1_rtn(z[i] * r);
          float diff = z[i] - oracle_e2m1_decode(cc[i]) * d;
          e = fmaf(diff, diff, e);
        }
      }
      if (e < best_e) {
        best_e = e;
        best_S = (uint8_t)Sc;
        memcpy(code, cc, 16);
      }
    }
    return best_S;
  }

  float q = 6.0f * s_g;
  float s_f = a_b / q;
  uint8_t S = mode == ORC_SR ? oracle_e4m3_ru_sat(s_f) : oracle_e4m3_rne_sat(s_f);
  float d = oracle_e4m3_decode(S) * s_g;
  if (d == 0.0f) {
    memset(code, 0, 16);
    return S; /* S == 0 here for supported inputs */
  }
  float r = 1.0f / d;
  float y[16];
  for (int i = 0; i < 16; ++i) y[i] = z[i] * r;

  if (mode == ORC_RTN) {
    for (int i = 0; i < 16; ++i) code[i] = oracle_e2m1_rtn(y[i]);
    return S;
  }
  if (mode == ORC_SR) {
    for (int i = 0; i < 16; ++i) {
      uint64_t e = (uint64_t)vr * (uint64_t)vc + (uint64_t)(bc * 16 + i);
      code[i] = oracle_e2m1_sr(y[i], oracle_uniform_element(seed, e));
    }
    return S;
  }
  if (mode == ORC_MS_EDEN) {
    /* MS-EDEN [QII-abs], [QII-key], [QII-bwd]: the element values are rounded
     * deterministically (RTN); the EDEN correction factor
     * c = <z, z> / <z, Q(z)> is folded into the group scale by stochastic
     * rounding of the scale, which moves the randomness from the FP4 values
     * onto the microscale.  Reading: one factor per 16-element block (the
     * "group scale"), computed in the y = z/d domain where the common factor
     * d cancels from the ratio; both dot products accumulate in element order
     * with fmaf starting from zero. */
    float num = 0.0f, den = 0.0f;
    for (int i = 0; i < 16; ++i) {
      code[i] = oracle_e2m1_rtn(y[i]);
      float v = oracle_e2m1_decode(code[i]);
      num = fmaf(y[i], y[i], num);
      den = fmaf(y[i], v, den);
    }
    float c = (num > 0.0f && den > 0.0f) ? num / den : 1.0f;
    float t = oracle_e4m3_decode(S) * c;
    uint64_t b = (uint64_t)vr * (uint64_t)(vc / 16) + (uint64_t)bc;
    return oracle_e4m3_sr(t, oracle_uniform_block(seed, b));
  }
  /* IF4 [IF4-abs], [IF4-F1], [IF4-F3]: quantize the block both to FP4 and to
   * scaled INT4 under the same scale, keep the option with the lower squared
   * error (ties keep FP4) and flag INT4 in the scale's sign bit.  Reading:
   * flag 1 = INT4 (an all-FP4 IF4 tensor is then byte-identical to NVFP4);
   * INT4 nibble = sign bit 3, |k| in bits 0..2; error in the y domain, which
   * ranks the two options as the original domain does since they share d. */
  uint8_t cf[16], ci[16];
  float eF = 0.0f, eI = 0.0f;
  for (int i = 0; i < 16; ++i) {
    cf[i] = oracle_e2m1_rtn(y[i]);
    float dF = y[i] - oracle_e2m1_decode(cf[i]);
    eF = fmaf(dF, dF, eF);
    int k = int4_level(y[i]);
    ci[i] = int4_code(k);
    float dI = y[i] - int4_value(k);
    eI = fmaf(dI, dI, eI);
  }
  if (eI < eF) {
    memcpy(code, ci, 16);
    return (uint8_t)(S | 0x80u);
  }
  memcpy(code, cf, 16);
  return S;
}

/* Quantize view rows [row_begin, row_end) of x (bf16, rows x cols, leading
 * dimension ld, row-major) into codes (view_rows x view_cols/2 bytes, the
 * full output array: only the given rows are written), scales (view_rows x
 * view_cols/16 bytes) and *global_scale.  amax_in (host, nullable) replaces
 * the tensor amax.  Codes pack element 2k in the low nibble of byte k of a
 * row and element 2k+1 in the high nibble. */
int oracle_quantize_rows(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                         int layout, int mode, int g, uint64_t seed, const float* amax_in,
                         int64_t row_begin, int64_t row_end, uint8_t* codes,
                         uint8_t* scales, float* global_scale) {
  int64_t vr, vc;
  int st = check_quant_args(rows, cols, ld, layout, mode, g, &vr, &vc);
  if (st) return st;
  if (row_begin < 0 || row_end > vr || row_begin > row_end) return ORC_ERR_ARG;
  float A;
  if (amax_in) A = *amax_in;
  else if ((st = oracle_amax(x, rows, cols, ld, layout, g, seed, &A))) return st;
  float s_g = oracle_global_scale(A, mode);
  *global_scale = s_g;

  float sigma[128];
  for (int j = 0; j < g; ++j) sigma[j] = oracle_rht_sign(seed, j);
  float c = g ? oracle_rht_scale(g) : 0.0f;
  float* row = (float*)malloc(sizeof(float) * (size_t)(vc > 0 ? vc : 1));
  if (!row) return ORC_ERR_ARG;
  for (int64_t r = row_begin; r < row_end; ++r) {
    load_view_row(x, ld, layout, r, vc, g, sigma, c, row);
    for (int64_t bc = 0; bc < vc / 16; ++bc) {
      uint8_t code[16];
      uint8_t S = quantize_block(row + bc * 16, mode, s_g, seed, r, vc, bc, code);
      scales[r * (vc / 16) + bc] = S;
      for (int k = 0; k < 8; ++k)
        codes[r * (vc / 2) + bc * 8 + k] = (uint8_t)(code[2 * k] | (code[2 * k + 1] << 4));
    }
  }
  free(row);
  return ORC_OK;
}

int oracle_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int layout,
                    int mode, int g, uint64_t seed, const float* amax_in, uint8_t* codes,
                    uint8_t* scales, float* global_scale) {
  int64_t vr = layout == ORC_TRANSPOSED ? cols : rows;
  return oracle_quantize_rows(x, rows, cols, ld, layout, mode, g, seed, amax_in, 0, vr,
                              codes, scales, global_scale);
}

/* Dequantize a quantized view (view_rows x view_cols) to fp32:
 * value(code, flag) * RN(dec(S & 0x7F) * s_g), then, when inverse_rht is set,
 * the inverse rotation along the rows.  value is the E2M1 value, or for an
 * IF4 block with the flag set, the scaled-INT4 value RN(k * RN(6/7)). */
int oracle_dequantize(const uint8_t* codes, const uint8_t* scales, float s_g,
                      int64_t vr, int64_t vc, int mode, int g, uint64_t seed,
                      int inverse_rht, float* out) {
  if (mode < ORC_RTN || mode > ORC_MXFP3) return ORC_ERR_ARG;
  if (g != 0 && !valid_group(g)) return ORC_ERR_ARG;
  if (vr < 0 || vc < 0 || vc % 16 || (g && vc % g)) return ORC_ERR_SHAPE;
  if ((mode == ORC_MXFP4 || mode == ORC_MXFP3) && vc % 32) return ORC_ERR_SHAPE;
  if (inverse_rht && g == 0) return ORC_ERR_ARG;
  for (int64_t r = 0; r < vr; ++r) {
    for (int64_t j = 0; j < vc; ++j) {
      uint8_t S = scales[r * (vc / 16) + j / 16];
      uint8_t byte = codes[r * (vc / 2) + j / 2];
      uint8_t code = (j & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
      int flagged = (mode == ORC_IF4 || mode == ORC_IF3) && (S & 0x80u);
      int integer = flagged || mode == ORC_NVINT4 || mode == ORC_NVINT3;
      int e2m0 = mode == ORC_NVFP3 || mode == ORC_MXFP3 || (mode == ORC_IF3 && !flagged);
      float d = (mode == ORC_MXFP4 || mode == ORC_MXFP3)
                    ? ldexpf(1.0f, (int)S - 127) /* UE8M0: 2^(S - 127) */
                    : oracle_e4m3_decode((uint8_t)(S & 0x7Fu)) * s_g;
      float v;
      if (integer) {
        int k = (int)(code & 7u);
        k = (code & 8u) ? -k : k;
        v = mode == ORC_IF4 ? int4_value(k) : (mode == ORC_IF3 ? (float)k * IF3_K2 : (float)k);
      } else if (e2m0) {
        v = e2m0_decode(code);
      } else {
        v = oracle_e2m1_decode(code);
      }
      out[r * vc + j] = v * d;
    }
  }
  if (inverse_rht) return oracle_rht_rows(out, vr, vc, g, seed, 1, out);
  return ORC_OK;
}

/* The rotated view z (view_rows x view_cols fp32) of a bf16 matrix, forward
 * only: what the quantizer sees before the block absmax. */
int oracle_rht_view(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int layout,
                    int g, uint64_t seed, float* out) {
  int64_t vr, vc;
  int st = check_quant_args(rows, cols, ld, layout, ORC_RTN, g, &vr, &vc);
  if (st) return st;
  if (g == 0) return ORC_ERR_ARG;
  float sigma[128];
  for (int j = 0; j < g; ++j) sigma[j] = oracle_rht_sign(seed, j);
  float c = oracle_rht_scale(g);
  for (int64_t r = 0; r < vr; ++r) load_view_row(x, ld, layout, r, vc, g, sigma, c, out + r * vc);
  return ORC_OK;
}

/* Array forms of the two codecs, for exhaustive comparisons. */
void oracle_e2m1_rtn_array(const float* in, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_rtn(in[i]);
}

void oracle_e4m3_array(const float* in, int64_t n, int round_up, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = round_up ? oracle_e4m3_ru_sat(in[i]) : oracle_e4m3_rne_sat(in[i]);
}

/* Packed storage of the 3-bit formats (a storage layout, this library's
 * reading; [IF4-T6] fixes only the bits per value: 3 bits per element plus
 * the scale, 3.5 for NVFP3 / NVINT3 / IF3 and 3.25 for MXFP3).  Element j of
 * block b of a view row: its nibble code (sign bit 3, magnitude bits 0..1) is
 * written as the 3-bit value sign * 4 + magnitude at bit 3 (j mod 16) of the
 * block's 6 bytes, least significant bit first, one bit at a time.  Scales:
 * copied, or for MXFP3 (mx != 0) the byte of every even block only. */
void oracle_pack3(const uint8_t* codes, const uint8_t* scales, int64_t vr, int64_t vc, int mx,
                  uint8_t* packed, uint8_t* packed_scales) {
  const int64_t nb = vc / 16;
  for (int64_t r = 0; r < vr; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      uint8_t* dst = packed + (r * nb + b) * 6;
      for (int k = 0; k < 6; ++k) dst[k] = 0;
      for (int j = 0; j < 16; ++j) {
        const int64_t e = b * 16 + j;
        const uint8_t byte = codes[r * (vc / 2) + e / 2];
        const uint8_t nib = (e % 2) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
        const unsigned v3 = (unsigned)(nib & 3u) + ((nib & 8u) ? 4u : 0u);
        for (int t = 0; t < 3; ++t) {
          const int bit = 3 * j + t;
          if ((v3 >> t) & 1u) dst[bit / 8] = (uint8_t)(dst[bit / 8] | (1u << (bit % 8)));
        }
      }
      if (!mx) packed_scales[r * nb + b] = scales[r * nb + b];
      else if (b % 2 == 0) packed_scales[r * (nb / 2) + b / 2] = scales[r * nb + b];
    }
  }
}

void oracle_unpack3(const uint8_t* packed, const uint8_t* packed_scales, int64_t vr, int64_t vc, int mx,
                    uint8_t* codes, uint8_t* scales) {
  const int64_t nb = vc / 16;
  for (int64_t r = 0; r < vr; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint8_t* src = packed + (r * nb + b) * 6;
      for (int j = 0; j < 16; ++j) {
        unsigned v3 = 0;
        for (int t = 0; t < 3; ++t) {
          const int bit = 3 * j + t;
          v3 |= (unsigned)((src[bit / 8] >> (bit % 8)) & 1u) << t;
        }
        const uint8_t nib = (uint8_t)((v3 & 3u) | ((v3 & 4u) ? 8u : 0u));
        const int64_t e = b * 16 + j;
        uint8_t* byte = &codes[r * (vc / 2) + e / 2];
        *byte = (e % 2) ? (uint8_t)((*byte & 15u) | (nib << 4)) : (uint8_t)((*byte & 0xF0u) | nib);
      }
      scales[r * nb + b] = mx ? packed_scales[r * (nb / 2) + b / 2] : packed_scales[r * nb + b];
    }
  }
}

/* Quantize an already rotated view z with a given tensor amax: steps 2 onward
 * of oracle_quantize_rows, for checking a quantizer on rotated values it
 * computed itself.  z holds the vr view rows row0 .. row0+vr-1 (vc fp32 each,
 * dense); the random streams are indexed by the full view's element and block
 * numbers, so a slice of rows gives those rows of the full result. */
int oracle_quantize_rotated(const float* z, int64_t row0, int64_t vr, int64_t vc, int mode,
                            uint64_t seed, float amax, uint8_t* codes, uint8_t* scales,
                            float* global_scale) {
  if (mode < ORC_RTN || mode > ORC_MXFP3) return ORC_ERR_ARG;
  if (row0 < 0 || vr < 0 || vc < 0 || vc % 16 || ((mode == ORC_MXFP4 || mode == ORC_MXFP3) && vc % 32)) return ORC_ERR_SHAPE;
  float s_g = oracle_global_scale(amax, mode);
  *global_scale = s_g;
  for (int64_t r = 0; r < vr; ++r) {
    for (int64_t bc = 0; bc < vc / 16; ++bc) {
      uint8_t code[16];
      uint8_t S = quantize_block(z + r * vc + bc * 16, mode, s_g, seed, row0 + r, vc, bc, code);
      scales[r * (vc / 16) + bc] = S;
      for (int k = 0; k < 8; ++k)
        codes[r * (vc / 2) + bc * 8 + k] = (uint8_t)(code[2 * k] | (code[2 * k + 1] << 4));
    }
  }
  return ORC_OK;
}

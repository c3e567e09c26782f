/*
 * nvfp4.h -- C ABI of libnvfp4.so: block-scaled NVFP4 quantization of bf16
 * training tensors on NVIDIA B200 (sm_100a).
 *
 * The method (sources named by page title and section):
 *  - One FP8 E4M3 scale per 16 consecutive elements and one FP32 scale per
 *    tensor; values rounded to nearest onto E2M1 (FP4) for the forward pass,
 *    with the optional "Four Over Six" block scale choice.  Quartet II article
 *    (mind-verse.de), section "Quantisierung im Vorwaertsdurchlauf".
 *  - E2M1 values {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}, 16-element
 *    blocks, a random Hadamard rotation before quantizing.  "Comparing INT4
 *    and NVFP4 Palettes on Real Gradient Tensors", opening section.
 *  - Unbiased stochastic rounding with an absmax scale that never clips.
 *    Same post, section "The two corners, and what the palette does to them".
 *  - MS-EDEN: deterministic rounding after a randomized Hadamard rotation,
 *    with an EDEN correction factor folded into the group scale by stochastic
 *    rounding.  Quartet II abstract (OpenAlex record) and article, section
 *    "Quantisierung im Rueckwaertsdurchlauf" and list "Kerninnovationen".
 *  - IF4: per 16-element block, the lower-error of FP4 and scaled INT4 under
 *    the same E4M3 scale, flagged in the scale's sign bit.  IF4 paper page
 *    (arXiv 2603.28765), abstract, Figure 1, Table 1, Figure 3.
 *  - The other block-scaled formats of that page (Table 1: MXFP4, NVINT4;
 *    the 3-bit table: NVFP3, NVINT3, IF3, MXFP3) and scale search (the
 *    palettes post's low-error corner, the page's ScaleSearch entry): see
 *    nvfp4_mode.
 *  - nvfp4_gemm multiplies two quantized operands on the block-scaled tensor
 *    cores (Quartet II abstract: NVFP4 in Blackwell hardware).
 *
 * Conventions shared by every entry point:
 *  - Pointers are DEVICE pointers unless stated otherwise.  The library
 *    allocates nothing and keeps no state between calls; every buffer is
 *    owned by the caller and must stay valid until the stream work finishes.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and returns without synchronising the host.  Arguments are
 *    checked on the host before anything is launched: a failed check returns
 *    a negative nvfp4_status and enqueues nothing.  A failed launch returns
 *    NVFP4_ERR_CUDA.  Faults during execution surface at the caller's next
 *    synchronisation.
 *  - x is bf16, row-major, rows x cols, leading dimension ld (elements,
 *    ld >= cols).  The quantized VIEW is V = X (NVFP4_ROWWISE: blocks of 16
 *    along a row of X) or V = X^T (NVFP4_TRANSPOSED: blocks of 16 down a
 *    column of X, output stored as X^T row-major).  The view has vrows x vcols
 *    = rows x cols (row-wise) or cols x rows (transposed).
 *  - codes: vrows x vcols/2 bytes; byte k of a row holds element 2k in its
 *    low nibble and element 2k+1 in its high nibble.  An E2M1 code is sign
 *    (bit 3) and a magnitude index (bits 0..2) into {0,.5,1,1.5,2,3,4,6}; an
 *    INT4 code (IF4 blocks flagged INT4, NVINT4) is sign (bit 3) and |k|
 *    (bits 0..2), value k * 6/7 (IF4) or k (NVINT4); the 3-bit codes use
 *    bits 0..1 for the magnitude.  Zero is always code 0.
 *  - scales: vrows x vcols/16 bytes, E4M3 (bias 7, max 448, min 2^-9), or
 *    UE8M0 for MXFP4 / MXFP3 (the 32-element group's byte in both halves);
 *    for IF4 and IF3, bit 7 set means the block holds integer codes.
 *  - global_scale: one float s_g; an element decodes to
 *    value(code) * RN(E4M3(scale & 0x7F) * s_g).
 *  - rht_group g in {0 (no rotation), 16, 32, 64, 128}: the random Hadamard
 *    rotation c_g H_g diag(sigma) applied to every g consecutive elements
 *    along a view row, sigma = g random signs drawn from `seed` (one sign
 *    vector shared by every group), c_g = RN(1/sqrt(g)).
 *  - seed keys every random draw (element rounding, scale rounding, signs)
 *    through Philox4x32-10 keyed by (seed, element or block index), so a
 *    result is a pure function of (input, arguments, seed).
 *  - Inputs must be finite; a nonzero tensor amax must be at least 2^-96.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = -1, /* null pointer, unknown enum value, bad group */
  NVFP4_ERR_SHAPE = -2,       /* block dimension not a multiple of 16 or of g; ld < cols */
  NVFP4_ERR_ALIGNMENT = -3,   /* x not 16-byte aligned, ld not a multiple of 8, ... */
  NVFP4_ERR_UNSUPPORTED = -4, /* valid but unsupported combination (MS-EDEN without RHT) */
  NVFP4_ERR_WORKSPACE = -5,   /* workspace missing or smaller than nvfp4_workspace_bytes */
  NVFP4_ERR_CUDA = -6         /* a CUDA call or kernel launch failed */
} nvfp4_status;

typedef enum { NVFP4_ROWWISE = 0, NVFP4_TRANSPOSED = 1 } nvfp4_layout;

typedef enum {
  NVFP4_RTN = 0,     /* round to nearest, tensor amax -> 6 x 448 */
  NVFP4_SR = 1,      /* stochastic rounding, block scale rounded up, amax -> 6 x 448 */
  NVFP4_MS_EDEN = 2, /* RTN codes + EDEN-corrected, stochastically rounded scale; needs g > 0; amax -> 6 x 256 */
  NVFP4_IF4 = 3,     /* per block FP4 or scaled INT4 (flag in scale bit 7), amax -> 6 x 448 */
  NVFP4_4OVER6 = 4,  /* per block scale mapping the absmax to 6 or to 4, amax -> 6 x 256 */
  NVFP4_SCALE_SEARCH = 5, /* per block the best of 19 E4M3 scales around the absmax scale (lowest
                             squared error, RTN codes; palettes post, "The two corners, and what
                             the palette does to them"; the ScaleSearch entry of the IF4 paper
                             page), amax -> 6 x 256 */
  NVFP4_MXFP4 = 6,   /* MXFP4 (IF4 paper page, Table 1): groups of 32 view elements with one
                        UE8M0 scale 2^E, E = floor(log2 max|z|) - 2 clamped to [-127, 127], RTN
                        E2M1 values of z / 2^E; no tensor scale (global_scale = 1, amax_in and
                        the workspace unused); the scale byte E + 127 is stored for each
                        16-element half of a group; needs vcols % 32 == 0 and a view of at least
                        one tile of the tiled kernels (else NVFP4_ERR_UNSUPPORTED) */
  NVFP4_NVINT4 = 7,  /* NVINT4 (IF4 paper page, Table 1): E4M3 block scale mapping the absmax to
                        7, INT4 levels k = clamp(RNE(z / d), -7, 7) stored as sign-magnitude
                        nibbles (as IF4's INT4 option, value k d), amax -> 7 x 448 */
  /* 3-bit formats (IF4 paper page, the 3-bit table), codes held in nibbles
   * (sign bit 3, magnitude code bits 0..1): E2M0 magnitudes {0, 1, 2, 4}
   * (nearest, ties to the even code), INT3 levels |k| <= 3. */
  NVFP4_NVFP3 = 8,   /* E4M3 block scale mapping the absmax to 4, E2M0 values, amax -> 4 x 448 */
  NVFP4_NVINT3 = 9,  /* E4M3 block scale mapping the absmax to 3, INT3 levels, amax -> 3 x 448 */
  NVFP4_IF3 = 10,    /* per block E2M0 or INT3 levels k standing for k 4/3 under one E4M3 scale
                        (lower squared error, bit 7 of the scale = INT3), amax -> 4 x 448 */
  NVFP4_MXFP3 = 11   /* as NVFP4_MXFP4 with E2M0 values (same shape rules) */
} nvfp4_mode;

/* Bytes of device workspace nvfp4_quantize needs when amax_in is NULL (the
 * tensor amax is then computed in a pre-pass into the workspace).  Returns 0
 * for invalid arguments. */
NVFP4_API size_t nvfp4_workspace_bytes(int64_t rows, int64_t cols, int layout, int mode, int rht_group);

/* Tensor amax of the (rotated) view: *amax_out = max |z| over the whole view,
 * z the view rotated by the RHT when rht_group > 0.  This is the pre-pass of
 * nvfp4_quantize, exposed so a caller can compute the amax once (or take it
 * from a producer) and pass it as amax_in.  amax_out: one device float,
 * overwritten.  Source: the FP32 per-tensor scale of the Quartet II article,
 * section "Quantisierung im Vorwaertsdurchlauf". */
NVFP4_API int nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout,
               int rht_group, uint64_t seed, float* amax_out, void* stream);

/* Both layouts' tensor amax from one read of x: *amax_row = nvfp4_amax of the
 * row-wise view with rotation group rht_group_row, *amax_col = nvfp4_amax of
 * the transposed view with rht_group_col (either may be 0), same seed; the
 * two values equal those of the two single calls bit for bit.  A fully-NVFP4
 * linear layer quantizes each of W, X and dY in both orientations (forward
 * along one dimension, backward along the other: Quartet II article, section
 * "Quantisierung im Vorwaertsdurchlauf", W and X re-quantized for the
 * backward pass), so reading the tensor once for both pre-passes halves
 * their HBM traffic.  Shape rules: those of nvfp4_amax for each layout
 * (cols a multiple of 16 and of rht_group_row, rows a multiple of 16 and of
 * rht_group_col, cols a multiple of 8).  amax_row, amax_col: device floats,
 * overwritten.  Tensors too small for the fused kernel run as two pre-passes. */
NVFP4_API int nvfp4_amax_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int rht_group_row,
                              int rht_group_col, uint64_t seed, float* amax_row, float* amax_col,
                              void* stream);

/* The largest n the group calls below take. */
#define NVFP4_MAX_GROUP 64

/* nvfp4_amax_dual for n tensors at once (1 <= n <= NVFP4_MAX_GROUP): member i
 * is (x[i], rows[i], cols[i], ld[i]) with outputs amax_row[i], amax_col[i];
 * the rotation groups and the seed are common to all.  The results are those
 * of n nvfp4_amax_dual calls bit for bit.  A linear layer's forward operands
 * X and W are both measured before their quantization (Quartet II article,
 * section "Quantisierung im Vorwaertsdurchlauf"); with an unrotated row view
 * (rht_group_row = 0) up to four members share one launch, which walks all
 * their tiles with one persistent grid (one ramp and one tail instead of
 * one per tensor).  x, rows, cols, ld, amax_row, amax_col: host arrays of n
 * entries (the tensors and outputs they point to are device memory).
 * Checks: every member as nvfp4_amax_dual, all before any launch. */
NVFP4_API int nvfp4_amax_dual_group(int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                                    const int64_t* ld, int rht_group_row, int rht_group_col, uint64_t seed,
                                    float* const* amax_row, float* const* amax_col, void* stream);

/* Quantize x to packed E2M1/INT4 codes, E4M3 block scales and the FP32
 * tensor scale, in the given layout and mode (see the conventions above).
 *  amax_in:   device float holding the tensor amax of the (rotated) view, or
 *             NULL to compute it in a pre-pass (needs the workspace).  The
 *             tensor scale is s_g = RN(amax / (6 M)), M = 448 (RTN, SR, IF4)
 *             or 256 (MS-EDEN, 4/6, scale search); RN(amax / (7 x 448)) for
 *             NVINT4; 1 for MXFP4; s_g = 1 for a zero amax.
 *  codes, scales, global_scale: outputs (sizes above); global_scale is one
 *             device float.
 *  workspace: device memory of at least nvfp4_workspace_bytes(...) bytes when
 *             amax_in is NULL, 16-byte aligned; may be NULL otherwise.
 * Shapes: vcols must be a multiple of 16 and of rht_group; for the
 * transposed layout cols must also be a multiple of 8.  Alignment: x 16-byte
 * aligned, ld a multiple of 8, codes 8-byte aligned. */
NVFP4_API int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout,
                   int mode, int rht_group, uint64_t seed, const float* amax_in,
                   uint8_t* codes, uint8_t* scales, float* global_scale, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Both layouts' quantization of x from one read of it: the outputs of
 *   nvfp4_quantize(x, ..., NVFP4_ROWWISE, mode_row, rht_group_row, seed, amax_row, codes_row, scales_row, gscale_row)
 *   nvfp4_quantize(x, ..., NVFP4_TRANSPOSED, mode_col, rht_group_col, seed, amax_col, codes_col, scales_col, gscale_col)
 * bit for bit.  A fully-NVFP4 linear layer needs W, X and dY quantized along
 * both dimensions (Quartet II article, section "Quantisierung im
 * Vorwaertsdurchlauf": W and X are re-quantized for the backward pass; section
 * "Quantisierung im Rueckwaertsdurchlauf": dY enters both backward GEMMs), so
 * one kernel that reads each tile once and writes both views saves a full
 * read of the tensor.  The fused kernel takes the pairs such a layer uses --
 * row-wise RTN without rotation with transposed MS-EDEN (group g), and MS-EDEN
 * with the same group g in both layouts, g in {16, 32, 64, 128} -- on tensors
 * of at least 128 x 128; any other pair (and smaller tensors) runs as the two
 * single-layout calls, with the same results.
 *  amax_row, amax_col: device floats holding the two views' tensor amaxes
 *             (nvfp4_amax_dual gives both from one read); required, except
 *             for the MX modes, which have no tensor scale.
 *  codes_row, scales_row, gscale_row: the row-wise view's outputs (rows x
 *             cols/2, rows x cols/16 bytes, one float); codes_col, scales_col,
 *             gscale_col: the transposed view's (cols x rows/2, cols x rows/16,
 *             one float).  Caller-owned device memory; the two sets must not
 *             overlap.
 * Shape and alignment rules: those of nvfp4_quantize for each layout.
 * Errors as nvfp4_quantize; nothing is launched when a check fails. */
NVFP4_API int nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int mode_row,
                                  int rht_group_row, int mode_col, int rht_group_col, uint64_t seed,
                                  const float* amax_row, const float* amax_col, uint8_t* codes_row,
                                  uint8_t* scales_row, float* gscale_row, uint8_t* codes_col,
                                  uint8_t* scales_col, float* gscale_col, void* stream);

/* nvfp4_quantize_dual for n tensors at once (1 <= n <= NVFP4_MAX_GROUP):
 * member i is (x[i], rows[i], cols[i], ld[i]) with amaxes amax_row[i],
 * amax_col[i] and outputs codes_row[i], scales_row[i], gscale_row[i],
 * codes_col[i], scales_col[i], gscale_col[i]; the modes, rotation groups and
 * seed are common to all.  The results are those of n nvfp4_quantize_dual
 * calls bit for bit.  Members on the fused path (see nvfp4_quantize_dual)
 * share one launch, up to four at a time -- a linear layer's forward operands
 * X and W, both quantized in both layouts (Quartet II article, section
 * "Quantisierung im Vorwaertsdurchlauf"), in one pass with one ramp and one
 * tail; the others run as their single calls.  All pointer arguments are
 * host arrays of n entries (pointing to device memory); entries of the MX
 * modes' amax arrays may be NULL.  Checks: every member as
 * nvfp4_quantize_dual, all before any launch. */
NVFP4_API int nvfp4_quantize_dual_group(int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                                        const int64_t* ld, int mode_row, int rht_group_row, int mode_col,
                                        int rht_group_col, uint64_t seed, const float* const* amax_row,
                                        const float* const* amax_col, uint8_t* const* codes_row,
                                        uint8_t* const* scales_row, float* const* gscale_row,
                                        uint8_t* const* codes_col, uint8_t* const* scales_col,
                                        float* const* gscale_col, void* stream);

/* Decode a quantized view (vrows x vcols) back to fp32:
 * out[r][j] = value(code, flag) * RN(E4M3(scale & 0x7F) * s_g), and, when
 * inverse_rht != 0 (needs rht_group > 0 and the seed used to quantize), the
 * inverse rotation along each row.  value is the E2M1 value, or for an IF4
 * block with bit 7 of its scale set, RN(k * RN(6/7)); for NVINT4 the integer
 * k itself; for MXFP4 the scale factor is 2^(scale - 127) instead (no s_g).  out: vrows x vcols
 * dense fp32, 16-byte aligned.  global_scale: device float. */
NVFP4_API int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                     int64_t vrows, int64_t vcols, int mode, int rht_group, uint64_t seed,
                     int inverse_rht, float* out, void* stream);

typedef enum { NVFP4_OUT_F32 = 0, NVFP4_OUT_BF16 = 1 } nvfp4_out_dtype;

/* NVFP4 GEMM on the block-scaled tensor cores, consuming two quantizer
 * outputs as they are:
 *   D[i][j] = RN(gA * gB) * sum_k qA[i][k] SA[i][k/16] qB[j][k] SB[j][k/16]
 * with q the E2M1 values and S the E4M3 block scales; the sum is accumulated
 * in fp32 by the tensor cores, the product with RN(gA * gB) is one fp32
 * multiply, then the store rounds to out_dtype (RN).  A is the m x k view
 * quantized along k (nvfp4_quantize row-wise on an m x k tensor, or
 * transposed on a k x m one), B likewise n x k; so Y = X W^T, dX = dY W and
 * dW = dY^T X of a fully-NVFP4 linear layer are each one call (Quartet II
 * record, abstract: NVFP4 is supported in hardware by Blackwell GPUs, the
 * authors' kernels run linear layers up to 4.2x faster than BF16; the
 * article's sections "Quantisierung im Vorwaertsdurchlauf" and "...
 * Rueckwaertsdurchlauf" for which operand is quantized along which
 * dimension).  The scales must be plain E4M3 (modes RTN, SR, MS-EDEN, 4/6,
 * scale search):
 * an IF4 scale carries the INT4 flag in bit 7, which the tensor cores do not
 * interpret, so IF4 outputs are not valid operands.  Two operands rotated along k with
 * the same seed and group give the product of the unrotated ones up to the
 * quantization error (the rotation is orthogonal up to the rounding of its
 * constant).
 *  a_codes: m x k/2 bytes, a_scales: m x k/16 bytes, a_gscale: device float;
 *  b_codes, b_scales, b_gscale: the same for n x k.  All device memory, owned
 *  by the caller, read only.
 *  d: m rows of n values (fp32 or bf16 per out_dtype), row stride ldd
 *  elements, overwritten.
 * Shapes: m and n multiples of 128, k a positive multiple of 256, ldd >= n
 * (NVFP4_ERR_SHAPE); m or n zero is a no-op.  Alignment: codes and scales
 * 16-byte aligned, d 16-byte aligned with ldd a multiple of 4 (fp32) or 8
 * (bf16) (NVFP4_ERR_ALIGNMENT).  Asynchronous on `stream`; a kernel whose
 * internal waits time out (a broken device) writes NaN to D[0][0]. */
NVFP4_API int nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_gscale,
                         const uint8_t* b_codes, const uint8_t* b_scales, const float* b_gscale, int64_t m,
                         int64_t n, int64_t k, int out_dtype, void* d, int64_t ldd, void* stream);

/* The random Hadamard rotation of the view, as fp32: out (vrows x vcols,
 * dense, 16-byte aligned) = the view of `in` with every rht_group-long piece
 * of a row rotated (inverse == 0) or un-rotated (inverse != 0).  in_dtype 0 =
 * bf16, 1 = fp32 (then ld counts fp32 elements and must be a multiple of 4).
 * Source: randomized Hadamard rotation, Quartet II article section
 * "Quantisierung im Rueckwaertsdurchlauf"; 16x16 rotation in the palettes
 * post, section "45 real tensors disagree". */
NVFP4_API int nvfp4_rht(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld, int layout,
              int rht_group, uint64_t seed, int inverse, float* out, void* stream);

/* nvfp4_quantize for callers that cannot give the library any device memory
 * beyond their tensors.  The paper has no counterpart to this entry point.
 *
 * nvfp4_quantize needs a workspace when it computes the tensor amax itself
 * (amax_in == NULL).  Some callers cannot provide one: an engine plugin that
 * is handed only its input and output buffers, or a process whose framework
 * has reserved all device memory in its own caching pool, where a fresh
 * cudaMalloc would fail or stall the host until the device is idle.  This
 * variant takes the same arguments minus the workspace and uses instead a
 * fixed 256-byte array of device memory compiled into the library (every GPU
 * that loads the library keeps those bytes until the process exits).  It
 * allocates nothing and calls no allocating routine.
 *  - The first call in a CUDA context looks up that array's device address
 *    (with the device current) and keeps it for that context; make that
 *    first call before any stream capture.  A context created again on the
 *    same device (after cudaDeviceReset) gets a fresh lookup, never the old
 *    address.
 *  - All calls on a device share the one array.  Each call clears the part
 *    that must start at zero on its own stream, but two calls that overlap
 *    on the GPU (different streams, or different host threads) race on it
 *    and may produce wrong tensor scales: serialise them.
 *  - A call whose workspace need (nvfp4_workspace_bytes) exceeds 256 bytes is
 *    rejected with NVFP4_ERR_WORKSPACE; with amax_in supplied no scratch is
 *    used at all.
 * Results are identical to nvfp4_quantize's for the same arguments. */
NVFP4_API int nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                     int layout, int mode, int rht_group, uint64_t seed,
                                     const float* amax_in, uint8_t* codes, uint8_t* scales,
                                     float* global_scale, void* stream);

/* Element and scale codecs of the quantizer, exposed on their own.
 * nvfp4_encode_e2m1: out[i] = E2M1 code (low nibble, one code per byte) of
 * in[i] rounded to nearest, ties to the even code, saturating at +-6, zero
 * always code 0 -- the rounding every RTN, MS-EDEN, IF4 and 4/6 element goes
 * through.  nvfp4_encode_e4m3: out[i] = E4M3 code of in[i] >= 0 rounded to
 * nearest-even (round_up == 0) or up to the next E4M3 value (round_up != 0),
 * saturating at 448 -- the block-scale rounding.  in: n device floats (finite;
 * non-negative for E4M3), out: n device bytes.  Sources: E2M1 value set, the
 * palettes post, opening section; E4M3 range, IF4 paper page, Table 1. */
NVFP4_API int nvfp4_encode_e2m1(const float* in, int64_t n, uint8_t* out, void* stream);
NVFP4_API int nvfp4_encode_e4m3(const float* in, int64_t n, int round_up, uint8_t* out, void* stream);

/* Packed storage of the 3-bit formats (IF4 paper page, the 3-bit formats
 * table: 3.5 bits per value for NVFP3, NVINT3 and IF3 -- 3-bit elements and
 * an 8-bit scale per 16 -- and 3.25 for MXFP3 -- one 8-bit scale per 32).
 * nvfp4_quantize holds a 3-bit code in a nibble (sign bit 3, magnitude code
 * bits 0..1, bit 2 clear); nvfp4_pack3 keeps 3 bits of it: the 16 codes of a
 * block in 6 bytes, element i in bits 3i .. 3i+2 of the block's 48-bit
 * little-endian field (bit 3i+2 the sign, bits 3i .. 3i+1 the magnitude code).
 *  codes, scales:   a quantized view as nvfp4_quantize writes it for `mode`
 *                   (vrows x vcols/2 and vrows x vcols/16 bytes);
 *  packed_codes:    vrows x (vcols/16) x 6 bytes, 2-byte aligned;
 *  packed_scales:   vrows x vcols/16 bytes (E4M3 modes), or vrows x vcols/32
 *                   (NVFP4_MXFP3: the group's byte once).
 * nvfp4_unpack3 restores codes and scales exactly (the MXFP3 byte in both
 * halves of its group).  mode: NVFP4_NVFP3, NVFP4_NVINT3, NVFP4_IF3 or
 * NVFP4_MXFP3 (others: NVFP4_ERR_UNSUPPORTED).  vcols: a multiple of 16 (32
 * for MXFP3).  Nibbles with bit 2 set (never produced by the 3-bit modes) do
 * not survive the packing.  The layout is this library's reading: the pages
 * give the bits per value, not a bit order. */
NVFP4_API int nvfp4_pack3(const uint8_t* codes, const uint8_t* scales, int64_t vrows, int64_t vcols, int mode,
                          uint8_t* packed_codes, uint8_t* packed_scales, void* stream);
NVFP4_API int nvfp4_unpack3(const uint8_t* packed_codes, const uint8_t* packed_scales, int64_t vrows,
                            int64_t vcols, int mode, uint8_t* codes, uint8_t* scales, void* stream);

/* Static string naming a status code (never NULL). */
NVFP4_API const char* nvfp4_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */

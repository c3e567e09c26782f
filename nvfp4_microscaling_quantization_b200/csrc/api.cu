// api.cu -- the C ABI of libnvfp4.so (declared in include/nvfp4.h):
// argument checks on the host, then kernel launches on the caller's stream.
#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"
#include "nvfp4.h"

namespace {

constexpr size_t kWorkspaceBytes = 256;  // one 32-bit amax accumulator, padded

bool valid_group(int g) { return g == 0 || g == 16 || g == 32 || g == 64 || g == 128; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Checks shared by quantize and amax.  On success fills the view shape.
// An empty tensor (rows or cols zero) may come with NULL data pointers and any
// ld; nothing is read or written for it except the tensor scale.
int check_tensor(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout, int rht_group,
                 int64_t* vrows, int64_t* vcols) {
  if (layout != NVFP4_ROWWISE && layout != NVFP4_TRANSPOSED) return NVFP4_ERR_INVALID_ARG;
  if (!valid_group(rht_group)) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0) return NVFP4_ERR_SHAPE;
  *vrows = layout == NVFP4_ROWWISE ? rows : cols;
  *vcols = layout == NVFP4_ROWWISE ? cols : rows;
  if (*vcols % 16) return NVFP4_ERR_SHAPE;
  if (rht_group && *vcols % rht_group) return NVFP4_ERR_SHAPE;
  if (layout == NVFP4_TRANSPOSED && cols % 8) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!x) return NVFP4_ERR_INVALID_ARG;
  if (ld < cols) return NVFP4_ERR_SHAPE;
  if (!aligned(x, 16) || ld % 8) return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

int from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

}  // namespace

extern "C" {

size_t nvfp4_workspace_bytes(int64_t rows, int64_t cols, int layout, int mode, int rht_group) {
  if (rows < 0 || cols < 0 || (layout != 0 && layout != 1) || mode < 0 || mode > NVFP4_MXFP3 ||
      !valid_group(rht_group))
    return 0;
  return kWorkspaceBytes;
}

int nvfp4_amax(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout, int rht_group,
               uint64_t seed, float* amax_out, void* stream) {
  int64_t vr, vc;
  int st = check_tensor(x, rows, cols, ld, layout, rht_group, &vr, &vc);
  if (st) return st;
  if (!amax_out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(amax_out, 4)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = from_cuda(cudaMemsetAsync(amax_out, 0, sizeof(float), s)))) return st;
  nvfp4::QuantArgs a{x, rows, cols, ld, layout, NVFP4_RTN, rht_group, seed, nullptr, amax_out,
                     nullptr, nullptr, nullptr, s};
  return from_cuda(nvfp4::launch_amax(a));
}

int nvfp4_amax_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int rht_group_row,
                    int rht_group_col, uint64_t seed, float* amax_row, float* amax_col, void* stream) {
  return nvfp4_amax_dual_group(1, &x, &rows, &cols, &ld, rht_group_row, rht_group_col, seed, &amax_row, &amax_col,
                               stream);
}

int nvfp4_amax_dual_group(int n, const void* const* x, const int64_t* rows, const int64_t* cols, const int64_t* ld,
                          int rht_group_row, int rht_group_col, uint64_t seed, float* const* amax_row,
                          float* const* amax_col, void* stream) {
  if (n < 1 || n > NVFP4_MAX_GROUP || !x || !rows || !cols || !ld || !amax_row || !amax_col)
    return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    int64_t vr, vc;
    int st = check_tensor(x[i], rows[i], cols[i], ld[i], NVFP4_ROWWISE, rht_group_row, &vr, &vc);
    if (st) return st;
    if ((st = check_tensor(x[i], rows[i], cols[i], ld[i], NVFP4_TRANSPOSED, rht_group_col, &vr, &vc))) return st;
    if (!amax_row[i] || !amax_col[i]) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(amax_row[i], 4) || !aligned(amax_col[i], 4)) return NVFP4_ERR_ALIGNMENT;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int st;
  for (int i = 0; i < n; ++i) {
    if ((st = from_cuda(cudaMemsetAsync(amax_row[i], 0, sizeof(float), s)))) return st;
    if ((st = from_cuda(cudaMemsetAsync(amax_col[i], 0, sizeof(float), s)))) return st;
  }
  // members with an unrotated row view go through the slot-ring kernel, up to
  // kMaxDualMembers of them in one launch; the rest one by one
  const void* gx[nvfp4::kMaxDualMembers];
  int64_t gr[nvfp4::kMaxDualMembers], gc[nvfp4::kMaxDualMembers], gl[nvfp4::kMaxDualMembers];
  float *ga[nvfp4::kMaxDualMembers], *gb[nvfp4::kMaxDualMembers];
  int m = 0;
  for (int i = 0; i < n; ++i) {
    const bool empty = rows[i] == 0 || cols[i] == 0;
    if (empty) continue;
    if (nvfp4::dual_mma_path_applies(x[i], rows[i], cols[i], ld[i])) {
      if (rht_group_row == 0) {
        gx[m] = x[i], gr[m] = rows[i], gc[m] = cols[i], gl[m] = ld[i], ga[m] = amax_row[i], gb[m] = amax_col[i];
        if (++m == nvfp4::kMaxDualMembers) {
          if ((st = from_cuda(nvfp4::launch_amax_dual_ring(m, gx, gr, gc, gl, rht_group_row, rht_group_col, seed,
                                                           ga, gb, s))))
            return st;
          m = 0;
        }
        continue;
      }
      if ((st = from_cuda(nvfp4::launch_amax_dual_mma(x[i], rows[i], cols[i], ld[i], rht_group_row, rht_group_col,
                                                      seed, amax_row[i], amax_col[i], s))))
        return st;
      continue;
    }
    nvfp4::QuantArgs a{x[i], rows[i], cols[i], ld[i], NVFP4_ROWWISE, NVFP4_RTN, rht_group_row, seed, nullptr,
                       amax_row[i], nullptr, nullptr, nullptr, s};
    if ((st = from_cuda(nvfp4::launch_amax(a)))) return st;
    a.layout = NVFP4_TRANSPOSED;
    a.rht_group = rht_group_col;
    a.amax_accum = amax_col[i];
    if ((st = from_cuda(nvfp4::launch_amax(a)))) return st;
  }
  if (m > 0)
    return from_cuda(nvfp4::launch_amax_dual_ring(m, gx, gr, gc, gl, rht_group_row, rht_group_col, seed, ga, gb, s));
  return NVFP4_OK;
}

int nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld, int layout, int mode,
                   int rht_group, uint64_t seed, const float* amax_in, uint8_t* codes,
                   uint8_t* scales, float* global_scale, void* workspace, size_t workspace_bytes,
                   void* stream) {
  int64_t vr, vc;
  int st = check_tensor(x, rows, cols, ld, layout, rht_group, &vr, &vc);
  if (st) return st;
  if (mode < NVFP4_RTN || mode > NVFP4_MXFP3) return NVFP4_ERR_INVALID_ARG;
  if (mode == NVFP4_MS_EDEN && rht_group == 0) return NVFP4_ERR_UNSUPPORTED;
  const bool mx = mode == NVFP4_MXFP4 || mode == NVFP4_MXFP3;
  if (mx && vc % 32) return NVFP4_ERR_SHAPE;
  const bool empty = vr == 0 || vc == 0;
  if (!global_scale || (!empty && (!codes || !scales))) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 8) || !aligned(global_scale, 4)) return NVFP4_ERR_ALIGNMENT;
  if (amax_in && !aligned(amax_in, 4)) return NVFP4_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mx) {
    // no tensor amax: amax_in and the workspace are not used; the kernels
    // read one float from amax (ignored), so they get the output scalar
    nvfp4::QuantArgs m{x, rows, cols, ld, layout, mode, rht_group, seed, global_scale, nullptr,
                       codes, scales, global_scale, s};
    if (!empty && !nvfp4::mma_path_applies(m) && !nvfp4::tma_path_applies(m)) return NVFP4_ERR_UNSUPPORTED;
    return from_cuda(nvfp4::launch_quantize(m));
  }
  if (!amax_in) {
    if (!workspace || workspace_bytes < kWorkspaceBytes) return NVFP4_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return NVFP4_ERR_ALIGNMENT;
  }
  nvfp4::QuantArgs a{x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, nullptr,
                     codes, scales, global_scale, s};
  if (!amax_in) {
    if ((st = from_cuda(cudaMemsetAsync(workspace, 0, sizeof(float), s)))) return st;
    a.amax_accum = workspace;
    if ((st = from_cuda(nvfp4::launch_amax(a)))) return st;
    a.amax = static_cast<const float*>(workspace);
  }
  return from_cuda(nvfp4::launch_quantize(a));
}

int nvfp4_quantize_dual(const void* x, int64_t rows, int64_t cols, int64_t ld, int mode_row, int rht_group_row,
                        int mode_col, int rht_group_col, uint64_t seed, const float* amax_row, const float* amax_col,
                        uint8_t* codes_row, uint8_t* scales_row, float* gscale_row, uint8_t* codes_col,
                        uint8_t* scales_col, float* gscale_col, void* stream) {
  return nvfp4_quantize_dual_group(1, &x, &rows, &cols, &ld, mode_row, rht_group_row, mode_col, rht_group_col, seed,
                                   &amax_row, &amax_col, &codes_row, &scales_row, &gscale_row, &codes_col,
                                   &scales_col, &gscale_col, stream);
}

int nvfp4_quantize_dual_group(int n, const void* const* x, const int64_t* rows, const int64_t* cols,
                              const int64_t* ld, int mode_row, int rht_group_row, int mode_col, int rht_group_col,
                              uint64_t seed, const float* const* amax_row, const float* const* amax_col,
                              uint8_t* const* codes_row, uint8_t* const* scales_row, float* const* gscale_row,
                              uint8_t* const* codes_col, uint8_t* const* scales_col, float* const* gscale_col,
                              void* stream) {
  if (n < 1 || n > NVFP4_MAX_GROUP || !x || !rows || !cols || !ld || !amax_row || !amax_col || !codes_row ||
      !scales_row || !gscale_row || !codes_col || !scales_col || !gscale_col)
    return NVFP4_ERR_INVALID_ARG;
  for (int m : {mode_row, mode_col})
    if (m < NVFP4_RTN || m > NVFP4_MXFP3) return NVFP4_ERR_INVALID_ARG;
  if ((mode_row == NVFP4_MS_EDEN && rht_group_row == 0) || (mode_col == NVFP4_MS_EDEN && rht_group_col == 0))
    return NVFP4_ERR_UNSUPPORTED;
  const bool mx_r = mode_row == NVFP4_MXFP4 || mode_row == NVFP4_MXFP3;
  const bool mx_c = mode_col == NVFP4_MXFP4 || mode_col == NVFP4_MXFP3;
  for (int i = 0; i < n; ++i) {
    int64_t vr, vc;
    int st = check_tensor(x[i], rows[i], cols[i], ld[i], NVFP4_ROWWISE, rht_group_row, &vr, &vc);
    if (st) return st;
    if ((st = check_tensor(x[i], rows[i], cols[i], ld[i], NVFP4_TRANSPOSED, rht_group_col, &vr, &vc))) return st;
    if ((mx_r && cols[i] % 32) || (mx_c && rows[i] % 32)) return NVFP4_ERR_SHAPE;
    const bool empty = rows[i] == 0 || cols[i] == 0;
    if (!gscale_row[i] || !gscale_col[i]) return NVFP4_ERR_INVALID_ARG;
    if (!empty && (!codes_row[i] || !scales_row[i] || !codes_col[i] || !scales_col[i])) return NVFP4_ERR_INVALID_ARG;
    if ((!mx_r && !amax_row[i]) || (!mx_c && !amax_col[i])) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(codes_row[i], 8) || !aligned(codes_col[i], 8) || !aligned(gscale_row[i], 4) ||
        !aligned(gscale_col[i], 4))
      return NVFP4_ERR_ALIGNMENT;
    if ((amax_row[i] && !aligned(amax_row[i], 4)) || (amax_col[i] && !aligned(amax_col[i], 4)))
      return NVFP4_ERR_ALIGNMENT;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int st;
  // members on the fused path: up to kMaxDualMembers of them in one launch
  nvfp4::DualQuantArgs grp[nvfp4::kMaxDualMembers];
  int m = 0;
  for (int i = 0; i < n; ++i) {
    const bool empty = rows[i] == 0 || cols[i] == 0;
    nvfp4::DualQuantArgs d{x[i], rows[i], cols[i], ld[i], mode_row, rht_group_row, mode_col, rht_group_col, seed,
                           amax_row[i], amax_col[i], codes_row[i], scales_row[i], gscale_row[i], codes_col[i],
                           scales_col[i], gscale_col[i], 1, s};
    if (!empty && nvfp4::dual_quantize_fused(d)) {
      grp[m] = d;
      if (++m == nvfp4::kMaxDualMembers) {
        if ((st = from_cuda(nvfp4::launch_quantize_dual_group(grp, m)))) return st;
        m = 0;
      }
      continue;
    }
    // any other pair: the two single-layout launches (MX modes read no amax:
    // their kernels are given the output scalar, as nvfp4_quantize does)
    nvfp4::QuantArgs a{x[i], rows[i], cols[i], ld[i], NVFP4_ROWWISE, mode_row, rht_group_row, seed,
                       mx_r ? gscale_row[i] : amax_row[i], nullptr, codes_row[i], scales_row[i], gscale_row[i], s};
    if (!empty && mx_r && !nvfp4::mma_path_applies(a) && !nvfp4::tma_path_applies(a)) return NVFP4_ERR_UNSUPPORTED;
    if ((st = from_cuda(nvfp4::launch_quantize(a)))) return st;
    nvfp4::QuantArgs b{x[i], rows[i], cols[i], ld[i], NVFP4_TRANSPOSED, mode_col, rht_group_col, seed,
                       mx_c ? gscale_col[i] : amax_col[i], nullptr, codes_col[i], scales_col[i], gscale_col[i], s};
    if (!empty && mx_c && !nvfp4::mma_path_applies(b) && !nvfp4::tma_path_applies(b)) return NVFP4_ERR_UNSUPPORTED;
    if ((st = from_cuda(nvfp4::launch_quantize(b)))) return st;
  }
  if (m > 0) return from_cuda(nvfp4::launch_quantize_dual_group(grp, m));
  return NVFP4_OK;
}

int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                     int64_t vrows, int64_t vcols, int mode, int rht_group, uint64_t seed,
                     int inverse_rht, float* out, void* stream) {
  if (!codes || !scales || !global_scale || !out) return NVFP4_ERR_INVALID_ARG;
  if (mode < NVFP4_RTN || mode > NVFP4_MXFP3 || !valid_group(rht_group)) return NVFP4_ERR_INVALID_ARG;
  if ((mode == NVFP4_MXFP4 || mode == NVFP4_MXFP3) && vcols % 32) return NVFP4_ERR_SHAPE;
  if (inverse_rht && rht_group == 0) return NVFP4_ERR_INVALID_ARG;
  if (vrows < 0 || vcols < 0 || vcols % 16 || (rht_group && vcols % rht_group)) return NVFP4_ERR_SHAPE;
  if (!aligned(codes, 8) || !aligned(out, 16) || !aligned(global_scale, 4)) return NVFP4_ERR_ALIGNMENT;
  nvfp4::DequantArgs a{codes, scales, global_scale, vrows, vcols, mode, rht_group, seed,
                       inverse_rht ? 1 : 0, out, static_cast<cudaStream_t>(stream)};
  return from_cuda(nvfp4::launch_dequantize(a));
}

int nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_gscale, const uint8_t* b_codes,
               const uint8_t* b_scales, const float* b_gscale, int64_t m, int64_t n, int64_t k, int out_dtype,
               void* d, int64_t ldd, void* stream) {
  if (out_dtype != NVFP4_OUT_F32 && out_dtype != NVFP4_OUT_BF16) return NVFP4_ERR_INVALID_ARG;
  if (m < 0 || n < 0 || k < 0 || m % 128 || n % 128 || k % 256 || ldd < n) return NVFP4_ERR_SHAPE;
  if (m == 0 || n == 0) return NVFP4_OK;
  if (!d || !a_gscale || !b_gscale) return NVFP4_ERR_INVALID_ARG;
  if (k == 0) return NVFP4_ERR_SHAPE;
  if (!a_codes || !a_scales || !b_codes || !b_scales) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) || !aligned(b_scales, 16) ||
      !aligned(a_gscale, 4) || !aligned(b_gscale, 4) || !aligned(d, 16) ||
      ldd % (out_dtype == NVFP4_OUT_F32 ? 4 : 8))
    return NVFP4_ERR_ALIGNMENT;
  if (!nvfp4::gemm_available()) return NVFP4_ERR_CUDA;
  nvfp4::GemmArgs g{a_codes, a_scales, a_gscale, b_codes, b_scales, b_gscale, m, n, k,
                    out_dtype == NVFP4_OUT_BF16 ? 1 : 0, d, ldd, static_cast<cudaStream_t>(stream)};
  return from_cuda(nvfp4::launch_gemm(g));
}

int nvfp4_rht(const void* in, int in_dtype, int64_t rows, int64_t cols, int64_t ld, int layout,
              int rht_group, uint64_t seed, int inverse, float* out, void* stream) {
  if (!in || !out) return NVFP4_ERR_INVALID_ARG;
  if (in_dtype != 0 && in_dtype != 1) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_ROWWISE && layout != NVFP4_TRANSPOSED) return NVFP4_ERR_INVALID_ARG;
  if (rht_group == 0 || !valid_group(rht_group)) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols || ld < 1) return NVFP4_ERR_SHAPE;
  const int64_t vcols = layout == NVFP4_ROWWISE ? cols : rows;
  if (vcols % 16 || vcols % rht_group) return NVFP4_ERR_SHAPE;
  if (!aligned(in, in_dtype == 0 ? 2 : 4) || !aligned(out, 16)) return NVFP4_ERR_ALIGNMENT;
  nvfp4::RhtArgs a{in, in_dtype, rows, cols, ld, layout, rht_group, seed, inverse ? 1 : 0, out,
                   static_cast<cudaStream_t>(stream)};
  return from_cuda(nvfp4::launch_rht(a));
}

int nvfp4_encode_e2m1(const float* in, int64_t n, uint8_t* out, void* stream) {
  if (!in || !out) return NVFP4_ERR_INVALID_ARG;
  if (n < 0) return NVFP4_ERR_SHAPE;
  if (!aligned(in, 4)) return NVFP4_ERR_ALIGNMENT;
  return from_cuda(nvfp4::launch_encode_e2m1(in, n, out, static_cast<cudaStream_t>(stream)));
}

int nvfp4_encode_e4m3(const float* in, int64_t n, int round_up, uint8_t* out, void* stream) {
  if (!in || !out) return NVFP4_ERR_INVALID_ARG;
  if (n < 0) return NVFP4_ERR_SHAPE;
  if (!aligned(in, 4)) return NVFP4_ERR_ALIGNMENT;
  return from_cuda(nvfp4::launch_encode_e4m3(in, n, round_up, out, static_cast<cudaStream_t>(stream)));
}

namespace {
int check_pack3(const void* a, const void* b, const void* c, const void* d, int64_t vrows, int64_t vcols, int mode) {
  if (mode != NVFP4_NVFP3 && mode != NVFP4_NVINT3 && mode != NVFP4_IF3 && mode != NVFP4_MXFP3)
    return NVFP4_ERR_UNSUPPORTED;
  if (vrows < 0 || vcols < 0 || vcols % (mode == NVFP4_MXFP3 ? 32 : 16)) return NVFP4_ERR_SHAPE;
  if (vrows == 0 || vcols == 0) return NVFP4_OK;
  if (!a || !b || !c || !d) return NVFP4_ERR_INVALID_ARG;
  return NVFP4_OK;
}
}  // namespace

int nvfp4_pack3(const uint8_t* codes, const uint8_t* scales, int64_t vrows, int64_t vcols, int mode,
                uint8_t* packed_codes, uint8_t* packed_scales, void* stream) {
  int st = check_pack3(codes, scales, packed_codes, packed_scales, vrows, vcols, mode);
  if (st || vrows == 0 || vcols == 0) return st;
  if (!aligned(codes, 8) || !aligned(packed_codes, 2)) return NVFP4_ERR_ALIGNMENT;
  return from_cuda(nvfp4::launch_pack3(codes, scales, vrows * (vcols / 16), mode == NVFP4_MXFP3, packed_codes,
                                       packed_scales, static_cast<cudaStream_t>(stream)));
}

int nvfp4_unpack3(const uint8_t* packed_codes, const uint8_t* packed_scales, int64_t vrows, int64_t vcols, int mode,
                  uint8_t* codes, uint8_t* scales, void* stream) {
  int st = check_pack3(packed_codes, packed_scales, codes, scales, vrows, vcols, mode);
  if (st || vrows == 0 || vcols == 0) return st;
  if (!aligned(codes, 8) || !aligned(packed_codes, 2)) return NVFP4_ERR_ALIGNMENT;
  return from_cuda(nvfp4::launch_unpack3(packed_codes, packed_scales, vrows * (vcols / 16), mode == NVFP4_MXFP3,
                                         codes, scales, static_cast<cudaStream_t>(stream)));
}

const char* nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_SHAPE: return "NVFP4_ERR_SHAPE";
    case NVFP4_ERR_ALIGNMENT: return "NVFP4_ERR_ALIGNMENT";
    case NVFP4_ERR_UNSUPPORTED: return "NVFP4_ERR_UNSUPPORTED";
    case NVFP4_ERR_WORKSPACE: return "NVFP4_ERR_WORKSPACE";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
    default: return "NVFP4_UNKNOWN_STATUS";
  }
}

}  // extern "C"

"""Block-scaled NVFP4 quantization of bf16 training tensors on B200 (sm_100a).

The kernels and the C ABI live in libnvfp4.so (sources in csrc/, interface in
include/nvfp4.h); `binding` is the ctypes layer over it and `workloads` the
seeded synthetic inputs.  Importing the package does not load the library;
the first call through `binding` does, and raises if it is missing.
"""
from . import workloads  # noqa: F401
from .binding import (  # noqa: F401
    FOUR_OVER_SIX, IF3, IF4, MS_EDEN, MXFP3, MXFP4, NVFP3, NVINT3, NVINT4, ROWWISE, RTN, SCALE_SEARCH, SR,
    TRANSPOSED, Nvfp4Error, amax, amax_dual, amax_dual_group,
    dequantize, encode_e2m1, encode_e4m3, gemm, lib, nvfp4_amax, nvfp4_dequantize, nvfp4_encode_e2m1,
    nvfp4_encode_e4m3, nvfp4_gemm, nvfp4_quantize, nvfp4_quantize_dual, nvfp4_rht, nvfp4_status_string, nvfp4_workspace_bytes,
    nvfp4_amax_dual_group, nvfp4_quantize_dual_group, quantize, quantize_dual, quantize_dual_group, rht, view_shape)

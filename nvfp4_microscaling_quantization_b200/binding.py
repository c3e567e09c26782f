"""Thin Python binding of libnvfp4.so (argument marshalling only).

The functions named like the C ABI (nvfp4_quantize, nvfp4_dequantize, nvfp4_rht,
nvfp4_amax, nvfp4_gemm, nvfp4_workspace_bytes, nvfp4_status_string) take raw device
pointers and sizes exactly as include/nvfp4.h declares them.  The tensor-level
helpers (quantize, dequantize, rht, amax, gemm) take torch CUDA tensors, allocate the
outputs with torch (device memory is the only thing torch provides here) and
call the same entry points on the current CUDA stream.  Every step of the
computation runs in the library's kernels; there is no CPU path.  If the
library has not been built, every call raises.
"""
import ctypes
import os
from typing import Optional, Tuple

import torch

ROWWISE, TRANSPOSED = 0, 1
RTN, SR, MS_EDEN, IF4, FOUR_OVER_SIX, SCALE_SEARCH, MXFP4, NVINT4 = 0, 1, 2, 3, 4, 5, 6, 7
NVFP3, NVINT3, IF3, MXFP3 = 8, 9, 10, 11

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libnvfp4.so")

_lib = None


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {nvfp4_status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """The loaded libnvfp4.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libnvfp4.so not found at {LIB_PATH}; build it with "
                "`python -m nvfp4_microscaling_quantization_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        P, i64, u64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_size_t
        L.nvfp4_workspace_bytes.argtypes = [i64, i64, i32, i32, i32]
        L.nvfp4_workspace_bytes.restype = sz
        L.nvfp4_amax.argtypes = [P, i64, i64, i64, i32, i32, u64, P, P]
        L.nvfp4_amax.restype = i32
        L.nvfp4_amax_dual.argtypes = [P, i64, i64, i64, i32, i32, u64, P, P, P]
        L.nvfp4_amax_dual.restype = i32
        L.nvfp4_quantize.argtypes = [P, i64, i64, i64, i32, i32, i32, u64, P, P, P, P, P, sz, P]
        L.nvfp4_quantize.restype = i32
        L.nvfp4_quantize_dual.argtypes = [P, i64, i64, i64, i32, i32, i32, i32, u64, P, P, P, P, P, P, P, P, P]
        L.nvfp4_quantize_dual.restype = i32
        PP, I64P = ctypes.POINTER(P), ctypes.POINTER(i64)
        L.nvfp4_amax_dual_group.argtypes = [i32, PP, I64P, I64P, I64P, i32, i32, u64, PP, PP, P]
        L.nvfp4_amax_dual_group.restype = i32
        L.nvfp4_quantize_dual_group.argtypes = [i32, PP, I64P, I64P, I64P, i32, i32, i32, i32, u64,
                                                PP, PP, PP, PP, PP, PP, PP, PP, P]
        L.nvfp4_quantize_dual_group.restype = i32
        L.nvfp4_dequantize.argtypes = [P, P, P, i64, i64, i32, i32, u64, i32, P, P]
        L.nvfp4_dequantize.restype = i32
        L.nvfp4_rht.argtypes = [P, i32, i64, i64, i64, i32, i32, u64, i32, P, P]
        L.nvfp4_rht.restype = i32
        L.nvfp4_encode_e2m1.argtypes = [P, i64, P, P]
        L.nvfp4_encode_e2m1.restype = i32
        L.nvfp4_encode_e4m3.argtypes = [P, i64, i32, P, P]
        L.nvfp4_encode_e4m3.restype = i32
        L.nvfp4_quantize_noalloc.argtypes = [P, i64, i64, i64, i32, i32, i32, u64, P, P, P, P, P]
        L.nvfp4_quantize_noalloc.restype = i32
        L.nvfp4_gemm.argtypes = [P, P, P, P, P, P, i64, i64, i64, i32, P, i64, P]
        L.nvfp4_gemm.restype = i32
        L.nvfp4_pack3.argtypes = [P, P, i64, i64, i32, P, P, P]
        L.nvfp4_pack3.restype = i32
        L.nvfp4_unpack3.argtypes = [P, P, i64, i64, i32, P, P, P]
        L.nvfp4_unpack3.restype = i32
        L.nvfp4_status_string.argtypes = [i32]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


# --------------------------------------------------------------------------- raw C ABI
def nvfp4_status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()


def nvfp4_workspace_bytes(rows, cols, layout, mode, rht_group) -> int:
    return lib().nvfp4_workspace_bytes(rows, cols, layout, mode, rht_group)


def nvfp4_amax(x, rows, cols, ld, layout, rht_group, seed, amax_out, stream) -> int:
    return lib().nvfp4_amax(x, rows, cols, ld, layout, rht_group, seed, amax_out, stream)


def nvfp4_amax_dual(x, rows, cols, ld, rht_group_row, rht_group_col, seed, amax_row, amax_col, stream) -> int:
    return lib().nvfp4_amax_dual(x, rows, cols, ld, rht_group_row, rht_group_col, seed, amax_row, amax_col,
                                 stream)


def nvfp4_amax_dual_group(n, x, rows, cols, ld, rht_group_row, rht_group_col, seed, amax_row, amax_col,
                          stream) -> int:
    """x, amax_row, amax_col: ctypes arrays of n pointers; rows, cols, ld: of n int64."""
    return lib().nvfp4_amax_dual_group(n, x, rows, cols, ld, rht_group_row, rht_group_col, seed, amax_row,
                                       amax_col, stream)


def nvfp4_quantize_dual_group(n, x, rows, cols, ld, mode_row, rht_group_row, mode_col, rht_group_col, seed,
                              amax_row, amax_col, codes_row, scales_row, gscale_row, codes_col, scales_col,
                              gscale_col, stream) -> int:
    """Pointer arguments: ctypes arrays of n pointers; rows, cols, ld: of n int64."""
    return lib().nvfp4_quantize_dual_group(n, x, rows, cols, ld, mode_row, rht_group_row, mode_col, rht_group_col,
                                           seed, amax_row, amax_col, codes_row, scales_row, gscale_row, codes_col,
                                           scales_col, gscale_col, stream)


def nvfp4_quantize(x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, codes, scales,
                   global_scale, workspace, workspace_bytes, stream) -> int:
    return lib().nvfp4_quantize(x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, codes,
                                scales, global_scale, workspace, workspace_bytes, stream)


def nvfp4_quantize_dual(x, rows, cols, ld, mode_row, rht_group_row, mode_col, rht_group_col, seed, amax_row,
                        amax_col, codes_row, scales_row, gscale_row, codes_col, scales_col, gscale_col,
                        stream) -> int:
    return lib().nvfp4_quantize_dual(x, rows, cols, ld, mode_row, rht_group_row, mode_col, rht_group_col, seed,
                                     amax_row, amax_col, codes_row, scales_row, gscale_row, codes_col, scales_col,
                                     gscale_col, stream)


def nvfp4_dequantize(codes, scales, global_scale, vrows, vcols, mode, rht_group, seed, inverse_rht,
                     out, stream) -> int:
    return lib().nvfp4_dequantize(codes, scales, global_scale, vrows, vcols, mode, rht_group, seed,
                                  inverse_rht, out, stream)


def nvfp4_rht(x, in_dtype, rows, cols, ld, layout, rht_group, seed, inverse, out, stream) -> int:
    return lib().nvfp4_rht(x, in_dtype, rows, cols, ld, layout, rht_group, seed, inverse, out, stream)


def nvfp4_quantize_noalloc(x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, codes, scales,
                           global_scale, stream) -> int:
    return lib().nvfp4_quantize_noalloc(x, rows, cols, ld, layout, mode, rht_group, seed, amax_in, codes,
                                        scales, global_scale, stream)


def nvfp4_gemm(a_codes, a_scales, a_gscale, b_codes, b_scales, b_gscale, m, n, k, out_dtype, d, ldd,
               stream) -> int:
    return lib().nvfp4_gemm(a_codes, a_scales, a_gscale, b_codes, b_scales, b_gscale, m, n, k, out_dtype, d,
                            ldd, stream)


def nvfp4_pack3(codes, scales, vrows, vcols, mode, packed_codes, packed_scales, stream) -> int:
    return lib().nvfp4_pack3(codes, scales, vrows, vcols, mode, packed_codes, packed_scales, stream)


def nvfp4_unpack3(packed_codes, packed_scales, vrows, vcols, mode, codes, scales, stream) -> int:
    return lib().nvfp4_unpack3(packed_codes, packed_scales, vrows, vcols, mode, codes, scales, stream)


def nvfp4_encode_e2m1(x, n, out, stream) -> int:
    return lib().nvfp4_encode_e2m1(x, n, out, stream)


def nvfp4_encode_e4m3(x, n, round_up, out, stream) -> int:
    return lib().nvfp4_encode_e4m3(x, n, round_up, out, stream)


# ----------------------------------------------------------------------- tensor helpers
def _stream_handle(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _matrix(x: torch.Tensor, dtype) -> Tuple[int, int, int]:
    if not x.is_cuda:
        raise ValueError("nvfp4 works on CUDA tensors only")
    if x.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {x.dtype}")
    if x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    rows, cols = x.shape
    return rows, cols, max(x.stride(0), cols, 1)


def view_shape(rows: int, cols: int, layout: int) -> Tuple[int, int]:
    return (rows, cols) if layout == ROWWISE else (cols, rows)


def _check(status: int, what: str):
    if status != 0:
        raise Nvfp4Error(status, what)


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def amax(x: torch.Tensor, layout: int = ROWWISE, rht_group: int = 0, seed: int = 0,
         out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    rows, cols, ld = _matrix(x, torch.bfloat16)
    out = torch.empty(1, dtype=torch.float32, device=x.device) if out is None else out
    _check(nvfp4_amax(_p(x), rows, cols, ld, layout, rht_group, seed, _p(out), _stream_handle(stream)),
           "nvfp4_amax")
    return out


def amax_dual(x: torch.Tensor, rht_group_row: int = 0, rht_group_col: int = 0, seed: int = 0,
              stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(amax of the row-wise view, amax of the transposed view) from one read of x."""
    rows, cols, ld = _matrix(x, torch.bfloat16)
    out = torch.empty(2, dtype=torch.float32, device=x.device)
    _check(nvfp4_amax_dual(_p(x), rows, cols, ld, rht_group_row, rht_group_col, seed, _p(out[0:1]),
                           _p(out[1:2]), _stream_handle(stream)), "nvfp4_amax_dual")
    return out[0:1], out[1:2]


def alloc_outputs(rows: int, cols: int, layout: int, device) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    vr, vc = view_shape(rows, cols, layout)
    codes = torch.empty((vr, vc // 2), dtype=torch.uint8, device=device)
    scales = torch.empty((vr, vc // 16), dtype=torch.uint8, device=device)
    gscale = torch.empty(1, dtype=torch.float32, device=device)
    return codes, scales, gscale


def quantize(x: torch.Tensor, layout: int = ROWWISE, mode: int = RTN, rht_group: int = 0, seed: int = 0,
             amax_in: Optional[torch.Tensor] = None, out=None, workspace: Optional[torch.Tensor] = None,
             stream=None):
    """Quantize a bf16 CUDA matrix; returns (codes, scales, global_scale) device tensors."""
    rows, cols, ld = _matrix(x, torch.bfloat16)
    codes, scales, gscale = alloc_outputs(rows, cols, layout, x.device) if out is None else out
    ws_bytes = 0
    if amax_in is None:
        ws_bytes = nvfp4_workspace_bytes(rows, cols, layout, mode, rht_group)
        if workspace is None:
            workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device)
    st = nvfp4_quantize(_p(x), rows, cols, ld, layout, mode, rht_group, seed, _p(amax_in), _p(codes),
                        _p(scales), _p(gscale), _p(workspace) if amax_in is None else None,
                        workspace.numel() if (amax_in is None and workspace is not None) else 0,
                        _stream_handle(stream))
    _check(st, "nvfp4_quantize")
    return codes, scales, gscale


def quantize_dual(x: torch.Tensor, mode_row: int, rht_group_row: int, mode_col: int, rht_group_col: int,
                  seed: int = 0, amax_row: Optional[torch.Tensor] = None, amax_col: Optional[torch.Tensor] = None,
                  out_row=None, out_col=None, stream=None):
    """Both layouts of a bf16 CUDA matrix from one read (nvfp4_quantize_dual);
    returns ((codes, scales, gscale) row-wise, (codes, scales, gscale)
    transposed).  Without amax_row / amax_col both tensor amaxes come from one
    nvfp4_amax_dual pre-pass on the same stream."""
    rows, cols, ld = _matrix(x, torch.bfloat16)
    if amax_row is None or amax_col is None:
        amax_row, amax_col = amax_dual(x, rht_group_row, rht_group_col, seed, stream=stream)
    r = alloc_outputs(rows, cols, ROWWISE, x.device) if out_row is None else out_row
    c = alloc_outputs(rows, cols, TRANSPOSED, x.device) if out_col is None else out_col
    _check(nvfp4_quantize_dual(_p(x), rows, cols, ld, mode_row, rht_group_row, mode_col, rht_group_col, seed,
                               _p(amax_row), _p(amax_col), _p(r[0]), _p(r[1]), _p(r[2]), _p(c[0]), _p(c[1]),
                               _p(c[2]), _stream_handle(stream)), "nvfp4_quantize_dual")
    return r, c


def _ptrs(ts):
    return (ctypes.c_void_p * len(ts))(*[(t.data_ptr() if t is not None else None) for t in ts])


def _i64s(vals):
    return (ctypes.c_int64 * len(vals))(*vals)


def amax_dual_group(xs, rht_group_row: int = 0, rht_group_col: int = 0, seed: int = 0, stream=None):
    """amax_dual of every tensor of xs (nvfp4_amax_dual_group): a list of
    (amax of the row-wise view, amax of the transposed view) pairs."""
    shapes = [_matrix(x, torch.bfloat16) for x in xs]
    outs = [torch.empty(2, dtype=torch.float32, device=x.device) for x in xs]
    n = len(xs)
    _check(nvfp4_amax_dual_group(n, _ptrs(xs), _i64s([s[0] for s in shapes]), _i64s([s[1] for s in shapes]),
                                 _i64s([s[2] for s in shapes]), rht_group_row, rht_group_col, seed,
                                 _ptrs([o[0:1] for o in outs]), _ptrs([o[1:2] for o in outs]),
                                 _stream_handle(stream)), "nvfp4_amax_dual_group")
    return [(o[0:1], o[1:2]) for o in outs]


def quantize_dual_group(xs, mode_row: int, rht_group_row: int, mode_col: int, rht_group_col: int, seed: int = 0,
                        amaxes=None, outs=None, stream=None):
    """quantize_dual of every tensor of xs (nvfp4_quantize_dual_group);
    amaxes: a list of (amax_row, amax_col) pairs (from amax_dual_group when
    None); returns a list of (row-wise outputs, transposed outputs)."""
    shapes = [_matrix(x, torch.bfloat16) for x in xs]
    if amaxes is None:
        amaxes = amax_dual_group(xs, rht_group_row, rht_group_col, seed, stream=stream)
    if outs is None:
        outs = [(alloc_outputs(r, c, ROWWISE, x.device), alloc_outputs(r, c, TRANSPOSED, x.device))
                for x, (r, c, _) in zip(xs, shapes)]
    n = len(xs)
    _check(nvfp4_quantize_dual_group(
        n, _ptrs(xs), _i64s([s[0] for s in shapes]), _i64s([s[1] for s in shapes]), _i64s([s[2] for s in shapes]),
        mode_row, rht_group_row, mode_col, rht_group_col, seed, _ptrs([a[0] for a in amaxes]),
        _ptrs([a[1] for a in amaxes]), _ptrs([o[0][0] for o in outs]), _ptrs([o[0][1] for o in outs]),
        _ptrs([o[0][2] for o in outs]), _ptrs([o[1][0] for o in outs]), _ptrs([o[1][1] for o in outs]),
        _ptrs([o[1][2] for o in outs]), _stream_handle(stream)), "nvfp4_quantize_dual_group")
    return outs


def dequantize(codes: torch.Tensor, scales: torch.Tensor, gscale: torch.Tensor, mode: int = RTN,
               rht_group: int = 0, seed: int = 0, inverse_rht: bool = False, stream=None) -> torch.Tensor:
    vr, half = codes.shape
    vc = 2 * half
    out = torch.empty((vr, vc), dtype=torch.float32, device=codes.device)
    _check(nvfp4_dequantize(_p(codes), _p(scales), _p(gscale), vr, vc, mode, rht_group, seed,
                            int(inverse_rht), _p(out), _stream_handle(stream)), "nvfp4_dequantize")
    return out


def rht(x: torch.Tensor, layout: int = ROWWISE, rht_group: int = 128, seed: int = 0, inverse: bool = False,
        stream=None) -> torch.Tensor:
    if x.dtype == torch.bfloat16:
        dt = 0
    elif x.dtype == torch.float32:
        dt = 1
    else:
        raise TypeError("rht takes bf16 or fp32")
    rows, cols, ld = _matrix(x, x.dtype)
    vr, vc = view_shape(rows, cols, layout)
    out = torch.empty((vr, vc), dtype=torch.float32, device=x.device)
    _check(nvfp4_rht(_p(x), dt, rows, cols, ld, layout, rht_group, seed, int(inverse), _p(out),
                     _stream_handle(stream)), "nvfp4_rht")
    return out


def pack3(codes: torch.Tensor, scales: torch.Tensor, mode: int, stream=None):
    """Packed 3-bit storage of a quantized view (NVFP3, NVINT3, IF3, MXFP3):
    returns (packed codes [vrows, vcols/16 * 6], packed scales [vrows, vcols/16],
    or [vrows, vcols/32] for MXFP3)."""
    vr, vc = codes.shape[0], 2 * codes.shape[1]
    pc = torch.empty((vr, vc // 16 * 6), dtype=torch.uint8, device=codes.device)
    ps = torch.empty((vr, vc // (32 if mode == MXFP3 else 16)), dtype=torch.uint8, device=codes.device)
    _check(nvfp4_pack3(_p(codes), _p(scales), vr, vc, mode, _p(pc), _p(ps), _stream_handle(stream)), "nvfp4_pack3")
    return pc, ps


def unpack3(packed_codes: torch.Tensor, packed_scales: torch.Tensor, vcols: int, mode: int, stream=None):
    """Inverse of pack3: (codes [vrows, vcols/2], scales [vrows, vcols/16])."""
    vr = packed_codes.shape[0]
    codes = torch.empty((vr, vcols // 2), dtype=torch.uint8, device=packed_codes.device)
    scales = torch.empty((vr, vcols // 16), dtype=torch.uint8, device=packed_codes.device)
    _check(nvfp4_unpack3(_p(packed_codes), _p(packed_scales), vr, vcols, mode, _p(codes), _p(scales),
                         _stream_handle(stream)), "nvfp4_unpack3")
    return codes, scales


def encode_e2m1(x: torch.Tensor, stream=None) -> torch.Tensor:
    """E2M1 code (one per byte) of every float of a CUDA fp32 tensor."""
    if not x.is_cuda or x.dtype != torch.float32:
        raise TypeError("encode_e2m1 takes a CUDA float32 tensor")
    x = x.contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(nvfp4_encode_e2m1(_p(x), x.numel(), _p(out), _stream_handle(stream)), "nvfp4_encode_e2m1")
    return out


def encode_e4m3(x: torch.Tensor, round_up: bool = False, stream=None) -> torch.Tensor:
    """E4M3 code of every non-negative float of a CUDA fp32 tensor (RNE or round-up, saturating)."""
    if not x.is_cuda or x.dtype != torch.float32:
        raise TypeError("encode_e4m3 takes a CUDA float32 tensor")
    x = x.contiguous()
    out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(nvfp4_encode_e4m3(_p(x), x.numel(), int(round_up), _p(out), _stream_handle(stream)),
           "nvfp4_encode_e4m3")
    return out


OUT_F32, OUT_BF16 = 0, 1


def gemm(a, b, out_dtype=torch.float32, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """D = gA gB A B^T on the block-scaled tensor cores.

    a, b: (codes, scales, global_scale) device tensors as quantize returns them,
    for an m x k and an n x k view quantized along k (RTN, SR, MS-EDEN or 4/6).
    Returns D [m, n] in out_dtype (torch.float32 or torch.bfloat16), or writes
    `out` (m rows, row stride out.stride(0)).
    """
    (ac, asc, ag), (bc, bsc, bg) = a, b
    m, k = ac.shape[0], 2 * ac.shape[1]
    n = bc.shape[0]
    if 2 * bc.shape[1] != k:
        raise ValueError(f"operands disagree on k: {k} and {2 * bc.shape[1]}")
    for t in (ac, asc, ag, bc, bsc, bg):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("gemm operands must be contiguous CUDA tensors")
    if out is None:
        out = torch.empty(m, n, dtype=out_dtype, device=ac.device)
    if out.dtype not in (torch.float32, torch.bfloat16) or out.stride(1) != 1 or tuple(out.shape) != (m, n):
        raise ValueError("out must be an m x n float32 or bfloat16 tensor with unit column stride")
    st = nvfp4_gemm(ctypes.c_void_p(ac.data_ptr()), ctypes.c_void_p(asc.data_ptr()), ctypes.c_void_p(ag.data_ptr()),
                    ctypes.c_void_p(bc.data_ptr()), ctypes.c_void_p(bsc.data_ptr()), ctypes.c_void_p(bg.data_ptr()),
                    m, n, k, OUT_BF16 if out.dtype == torch.bfloat16 else OUT_F32,
                    ctypes.c_void_p(out.data_ptr()), out.stride(0), _stream_handle(stream))
    if st:
        raise Nvfp4Error(st, "nvfp4_gemm")
    return out

"""CPU oracle for block-scaled NVFP4 quantization -- TEST INFRASTRUCTURE ONLY.

A ctypes wrapper over oracle/nvfp4_oracle.c (plain C99, binary32 round-to-
nearest-even, no contraction).  Only tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py may import this package; the CUDA library and its
Python binding never do.

Every function takes and returns numpy arrays on the host.
"""
import ctypes
import os

import numpy as np

from . import build as _build

ROWWISE, TRANSPOSED = 0, 1
RTN, SR, MS_EDEN, IF4, FOUR_OVER_SIX, SCALE_SEARCH, MXFP4, NVINT4 = 0, 1, 2, 3, 4, 5, 6, 7
NVFP3, NVINT3, IF3, MXFP3 = 8, 9, 10, 11

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        _declare(_lib)
    return _lib


def _declare(L):
    P = ctypes.c_void_p
    i64, u64, i32, f32 = ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_float
    L.oracle_philox4x32_10.argtypes = [P, P, P]
    L.oracle_philox4x32_10.restype = None
    L.oracle_uniform_element.argtypes = [u64, u64]
    L.oracle_uniform_element.restype = f32
    L.oracle_uniform_block.argtypes = [u64, u64]
    L.oracle_uniform_block.restype = f32
    L.oracle_rht_sign.argtypes = [u64, i32]
    L.oracle_rht_sign.restype = f32
    L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e2m1_decode.restype = f32
    L.oracle_e2m1_rtn.argtypes = [f32]
    L.oracle_e2m1_rtn.restype = ctypes.c_uint8
    L.oracle_e2m1_sr.argtypes = [f32, f32]
    L.oracle_e2m1_sr.restype = ctypes.c_uint8
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = f32
    L.oracle_e4m3_rne_sat.argtypes = [f32]
    L.oracle_e4m3_rne_sat.restype = ctypes.c_uint8
    L.oracle_e4m3_ru_sat.argtypes = [f32]
    L.oracle_e4m3_ru_sat.restype = ctypes.c_uint8
    L.oracle_e4m3_sr.argtypes = [f32, f32]
    L.oracle_e4m3_sr.restype = ctypes.c_uint8
    L.oracle_rht_scale.argtypes = [i32]
    L.oracle_rht_scale.restype = f32
    L.oracle_rht_rows.argtypes = [P, i64, i64, i32, u64, i32, P]
    L.oracle_rht_rows.restype = i32
    L.oracle_amax.argtypes = [P, i64, i64, i64, i32, i32, u64, P]
    L.oracle_amax.restype = i32
    L.oracle_global_scale.argtypes = [f32, i32]
    L.oracle_global_scale.restype = f32
    L.oracle_quantize_rows.argtypes = [P, i64, i64, i64, i32, i32, i32, u64, P, i64, i64, P, P, P]
    L.oracle_quantize_rows.restype = i32
    L.oracle_quantize.argtypes = [P, i64, i64, i64, i32, i32, i32, u64, P, P, P, P]
    L.oracle_quantize.restype = i32
    L.oracle_dequantize.argtypes = [P, P, f32, i64, i64, i32, i32, u64, i32, P]
    L.oracle_dequantize.restype = i32
    L.oracle_rht_view.argtypes = [P, i64, i64, i64, i32, i32, u64, P]
    L.oracle_rht_view.restype = i32
    L.oracle_if4_constants.argtypes = [P, P]
    L.oracle_if4_constants.restype = None
    L.oracle_quantize_rotated.argtypes = [P, i64, i64, i64, i32, u64, f32, P, P, P]
    L.oracle_quantize_rotated.restype = i32
    L.oracle_e2m1_rtn_array.argtypes = [P, i64, P]
    L.oracle_e2m1_rtn_array.restype = None
    L.oracle_e4m3_array.argtypes = [P, i64, i32, P]
    L.oracle_e4m3_array.restype = None
    L.oracle_pack3.argtypes = [P, P, i64, i64, i32, P, P]
    L.oracle_pack3.restype = None
    L.oracle_unpack3.argtypes = [P, P, i64, i64, i32, P, P]
    L.oracle_unpack3.restype = None


class OracleError(RuntimeError):
    pass


def _check(st):
    if st != 0:
        raise OracleError(f"oracle status {st}")


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_bf16_bits(x):
    """Accept a uint16 array of bf16 bit patterns (2-D, row-major, may have ld > cols)."""
    x = np.asarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle takes bf16 as uint16 bit patterns")
    return x


def view_shape(rows, cols, layout):
    return (rows, cols) if layout == ROWWISE else (cols, rows)


def philox(ctr, key):
    c = np.ascontiguousarray(ctr, dtype=np.uint32)
    k = np.ascontiguousarray(key, dtype=np.uint32)
    out = np.zeros(4, dtype=np.uint32)
    lib().oracle_philox4x32_10(_ptr(c), _ptr(k), _ptr(out))
    return out


def uniform_element(seed, e):
    return lib().oracle_uniform_element(seed, e)


def uniform_block(seed, b):
    return lib().oracle_uniform_block(seed, b)


def rht_signs(seed, g):
    return np.array([lib().oracle_rht_sign(seed, j) for j in range(g)], dtype=np.float32)


def rht_scale(g):
    return lib().oracle_rht_scale(g)


def e2m1_rtn(y):
    return lib().oracle_e2m1_rtn(float(y))


def e2m1_sr(y, u):
    return lib().oracle_e2m1_sr(float(y), float(u))


def e2m1_decode(code):
    return lib().oracle_e2m1_decode(int(code))


def e2m1_rtn_array(v):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e2m1_rtn_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_array(v, round_up=False):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().oracle_e4m3_array(_ptr(v), v.size, int(round_up), _ptr(out))
    return out


def e4m3_decode(code):
    return lib().oracle_e4m3_decode(int(code))


def e4m3_rne_sat(v):
    return lib().oracle_e4m3_rne_sat(float(v))


def e4m3_ru_sat(v):
    return lib().oracle_e4m3_ru_sat(float(v))


def e4m3_sr(t, u):
    return lib().oracle_e4m3_sr(float(t), float(u))


def if4_constants():
    k = np.zeros(2, dtype=np.float32)
    lib().oracle_if4_constants(_ptr(k[0:1]), _ptr(k[1:2]))
    return float(k[0]), float(k[1])


def global_scale(amax, mode):
    return lib().oracle_global_scale(float(amax), mode)


def rht_rows(v, g, seed, inverse=False):
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    out = np.empty_like(v)
    _check(lib().oracle_rht_rows(_ptr(v), rows, cols, g, seed, int(inverse), _ptr(out)))
    return out


def rht_view(x_bits, layout, g, seed, cols=None):
    x = _as_bf16_bits(x_bits)
    rows, ld = x.shape
    cols = ld if cols is None else cols
    vr, vc = view_shape(rows, cols, layout)
    out = np.empty((vr, vc), dtype=np.float32)
    _check(lib().oracle_rht_view(_ptr(np.ascontiguousarray(x)), rows, cols, ld, layout, g, seed,
                                 _ptr(out)))
    return out


def amax(x_bits, layout, g, seed, cols=None):
    x = np.ascontiguousarray(_as_bf16_bits(x_bits))
    rows, ld = x.shape
    cols = ld if cols is None else cols
    a = np.zeros(1, dtype=np.float32)
    _check(lib().oracle_amax(_ptr(x), rows, cols, ld, layout, g, seed, _ptr(a)))
    return float(a[0])


def quantize(x_bits, layout, mode, g, seed, amax_in=None, cols=None, row_range=None):
    """Returns (codes uint8 [vr, vc/2], scales uint8 [vr, vc/16], global_scale float).

    x_bits: uint16 [rows, ld] bf16 patterns; cols (<= ld) is the logical width.
    row_range: optional (begin, end) of view rows to compute; other rows stay 0.
    """
    x = np.ascontiguousarray(_as_bf16_bits(x_bits))
    rows, ld = x.shape
    cols = ld if cols is None else cols
    vr, vc = view_shape(rows, cols, layout)
    codes = np.zeros((vr, vc // 2), dtype=np.uint8)
    scales = np.zeros((vr, max(vc // 16, 0)), dtype=np.uint8)
    gs = np.zeros(1, dtype=np.float32)
    a = None if amax_in is None else np.array([amax_in], dtype=np.float32)
    b, e = (0, vr) if row_range is None else row_range
    _check(lib().oracle_quantize_rows(_ptr(x), rows, cols, ld, layout, mode, g, seed,
                                      None if a is None else _ptr(a), b, e, _ptr(codes),
                                      _ptr(scales), _ptr(gs)))
    return codes, scales, float(gs[0])


def quantize_rotated(z, mode, seed, amax, row0=0):
    """Quantize an already rotated fp32 view z [vr, vc] with the given tensor amax.

    z holds view rows row0 .. row0+vr-1 of the full view; the random streams
    follow the full view's element and block numbers."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    vr, vc = z.shape
    codes = np.zeros((vr, vc // 2), dtype=np.uint8)
    scales = np.zeros((vr, vc // 16), dtype=np.uint8)
    gs = np.zeros(1, dtype=np.float32)
    _check(lib().oracle_quantize_rotated(_ptr(z), row0, vr, vc, mode, seed, float(amax), _ptr(codes), _ptr(scales),
                                         _ptr(gs)))
    return codes, scales, float(gs[0])


def dequantize(codes, scales, gscale, mode, g, seed, inverse_rht=False):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    vr, half = codes.shape
    vc = half * 2
    out = np.empty((vr, vc), dtype=np.float32)
    _check(lib().oracle_dequantize(_ptr(codes), _ptr(scales), float(gscale), vr, vc, mode, g,
                                   seed, int(inverse_rht), _ptr(out)))
    return out


def pack3(codes, scales, mode):
    """Packed 3-bit storage of a quantized view (NVFP3, NVINT3, IF3, MXFP3):
    (packed codes [vr, vc/16 * 6], packed scales [vr, vc/16] or [vr, vc/32] for MXFP3)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    vr, vc = codes.shape[0], codes.shape[1] * 2
    mx = int(mode == MXFP3)
    pc = np.zeros((vr, vc // 16 * 6), dtype=np.uint8)
    ps = np.zeros((vr, vc // (32 if mx else 16)), dtype=np.uint8)
    lib().oracle_pack3(_ptr(codes), _ptr(scales), vr, vc, mx, _ptr(pc), _ptr(ps))
    return pc, ps


def unpack3(packed, packed_scales, vcols, mode):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    packed_scales = np.ascontiguousarray(packed_scales, dtype=np.uint8)
    vr = packed.shape[0]
    codes = np.zeros((vr, vcols // 2), dtype=np.uint8)
    scales = np.zeros((vr, vcols // 16), dtype=np.uint8)
    lib().oracle_unpack3(_ptr(packed), _ptr(packed_scales), vr, vcols, int(mode == MXFP3), _ptr(codes), _ptr(scales))
    return codes, scales


def unpack_codes(codes):
    """Split packed bytes into one 4-bit code per element (low nibble first)."""
    codes = np.asarray(codes, dtype=np.uint8)
    out = np.empty(codes.shape[:-1] + (codes.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = codes & 15
    out[..., 1::2] = codes >> 4
    return out


def _gemm_operand_ints(codes, scales, rows=None):
    """Dequantized operand times 2^10, as exact int64: every E2M1 value is a
    multiple of 1/2 and every E4M3 value a multiple of 2^-9, so q * dec(S) is a
    multiple of 2^-10 below 6 * 448 < 2^12."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    if rows is not None:
        codes, scales = codes[rows], scales[rows]
    if np.any(scales >= 0x7F):
        raise ValueError("GEMM operands take finite plain E4M3 scales (bit 7 clear, not 0x7F)")
    q2 = np.array([round(2.0 * e2m1_decode(c)) for c in range(16)], dtype=np.int64)       # 2 * value
    s9 = np.array([round(512.0 * e4m3_decode(s)) if s != 0x7F else 0 for s in range(128)], dtype=np.int64)
    q = q2[unpack_codes(codes)]
    s = np.repeat(s9[scales], 16, axis=-1)
    return q * s


def gemm(a_codes, a_scales, a_gscale, b_codes, b_scales, b_gscale, a_rows=None, b_rows=None):
    """The NVFP4 GEMM on two quantized operands (A: m x k view, B: n x k view,
    both quantized along k), as float64:

        D[i][j] = RN32(gA * gB) * sum_k qA[i][k] SA[i][k/16] qB[j][k] SB[j][k/16]

    (Quartet II record, abstract: NVFP4 GEMMs run in Blackwell hardware;
    Quartet II article, sections "Quantisierung im Vorwaertsdurchlauf" and
    "... Rueckwaertsdurchlauf": every GEMM operand is quantized along the
    reduction dimension).  The sum is exact: each operand element times 2^10
    is an integer below 2^22, so a product is below 2^44 and a sum of up to
    2^19 products stays below 2^63 in int64.  The one product with the tensor
    scales is rounded to float64.  a_rows / b_rows select rows of A / B (then
    D is len(a_rows) x len(b_rows)).
    """
    ai = _gemm_operand_ints(a_codes, a_scales, a_rows)
    bi = _gemm_operand_ints(b_codes, b_scales, b_rows)
    if ai.shape[1] != bi.shape[1]:
        raise ValueError("operands disagree on k")
    if ai.shape[1] > (1 << 19):
        raise ValueError("k above 2^19: the int64 sum could overflow")
    s = ai @ bi.T
    gab = float(np.float32(np.float32(a_gscale) * np.float32(b_gscale)))
    return s.astype(np.float64) * (2.0 ** -20) * gab

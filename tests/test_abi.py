"""The C-ABI library loads, exports every symbol include/nvfp4.h declares, and
rejects bad arguments on the host before anything is launched.

CPU-only: every call below fails one of the library's host-side checks, so no
CUDA call is reached and no device pointer is ever dereferenced.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

OK, INVALID, SHAPE, ALIGN, UNSUPPORTED, WORKSPACE, CUDA = 0, -1, -2, -3, -4, -5, -6
FAKE = 0x100000  # 16-byte aligned, never dereferenced: each call fails a check first


@pytest.fixture(scope="module")
def N():
    from nvfp4_microscaling_quantization_b200 import binding, build
    build.build()
    binding.lib()
    return binding


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ["nvfp4_quantize", "nvfp4_dequantize", "nvfp4_rht", "nvfp4_amax", "nvfp4_workspace_bytes",
              "nvfp4_status_string", "nvfp4_encode_e2m1", "nvfp4_encode_e4m3", "nvfp4_quantize_noalloc",
              "nvfp4_amax_dual", "nvfp4_gemm", "nvfp4_quantize_dual", "nvfp4_pack3", "nvfp4_unpack3",
              "nvfp4_amax_dual_group", "nvfp4_quantize_dual_group"]:
        assert n in names


def test_library_exports_every_declared_symbol(N):
    lib = N.lib()
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_nothing_else_exported(N):
    """Only the C ABI is visible (the kernels and helpers are hidden)."""
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", N.LIB_PATH], capture_output=True, text=True).stdout
    exported = sorted({l.split()[-1] for l in out.splitlines() if " T " in l})
    assert exported == declared_symbols()


def test_status_strings(N):
    for st, name in [(OK, "NVFP4_OK"), (INVALID, "NVFP4_ERR_INVALID_ARG"), (SHAPE, "NVFP4_ERR_SHAPE"),
                     (ALIGN, "NVFP4_ERR_ALIGNMENT"), (UNSUPPORTED, "NVFP4_ERR_UNSUPPORTED"),
                     (WORKSPACE, "NVFP4_ERR_WORKSPACE"), (CUDA, "NVFP4_ERR_CUDA")]:
        assert N.nvfp4_status_string(st) == name
    assert N.nvfp4_status_string(12345) == "NVFP4_UNKNOWN_STATUS"


def test_workspace_bytes(N):
    assert N.nvfp4_workspace_bytes(4096, 4096, 0, 2, 128) == 256
    assert N.nvfp4_workspace_bytes(4096, 4096, 2, 2, 128) == 0
    assert N.nvfp4_workspace_bytes(4096, 4096, 0, 12, 128) == 0
    assert N.nvfp4_workspace_bytes(4096, 4096, 0, 0, 48) == 0


def q(N, x=FAKE, rows=64, cols=64, ld=64, layout=0, mode=0, g=0, amax=None, codes=FAKE + 0x1000,
      scales=FAKE + 0x2000, gs=FAKE + 0x3000, ws=None, ws_bytes=0):
    return N.nvfp4_quantize(x, rows, cols, ld, layout, mode, g, 0, amax, codes, scales, gs, ws, ws_bytes, None)


def test_quantize_rejects(N):
    assert q(N, x=None) == INVALID
    assert q(N, x=None, rows=0) == WORKSPACE     # an empty tensor may have no data pointer
    assert q(N, x=None, rows=0, gs=None) == INVALID
    assert q(N, layout=2) == INVALID
    assert q(N, g=48) == INVALID
    assert q(N, mode=12) == INVALID
    assert q(N, mode=6, cols=48, ld=48) == SHAPE          # MXFP4: whole 32-element groups
    assert q(N, mode=6, rows=8, cols=64) == UNSUPPORTED   # MXFP4: below one tile of the tiled kernels
    assert q(N, mode=11, cols=48, ld=48) == SHAPE         # MXFP3 likewise
    assert q(N, mode=11, rows=8, cols=64) == UNSUPPORTED
    assert q(N, cols=40, ld=40) == SHAPE            # row-wise blocks need cols % 16 == 0
    assert q(N, rows=40, layout=1) == SHAPE         # transposed blocks need rows % 16 == 0
    assert q(N, cols=64, g=128) == SHAPE            # rotation group must divide the block dimension
    assert q(N, rows=-1) == SHAPE
    assert q(N, ld=32) == SHAPE                     # ld < cols
    assert q(N, rows=64, cols=4, ld=8, layout=1) == SHAPE  # transposed needs cols % 8 == 0
    assert q(N, x=FAKE + 8) == ALIGN                # x not 16-byte aligned
    assert q(N, ld=68) == ALIGN                     # ld not a multiple of 8
    assert q(N, mode=2, g=0) == UNSUPPORTED         # MS-EDEN needs the rotation
    assert q(N, codes=None) == INVALID
    assert q(N, scales=None) == INVALID
    assert q(N, gs=None) == INVALID
    assert q(N, codes=FAKE + 4) == ALIGN
    assert q(N) == WORKSPACE                        # no amax_in and no workspace
    assert q(N, ws=FAKE + 0x4000, ws_bytes=8) == WORKSPACE
    assert q(N, ws=FAKE + 0x4008, ws_bytes=256) == ALIGN


def test_noalloc_rejects_like_quantize(N):
    nq = N.nvfp4_quantize_noalloc
    assert nq(FAKE, 64, 64, 64, 2, 0, 0, 0, None, FAKE, FAKE, FAKE, None) == INVALID   # layout
    assert nq(FAKE, 64, 64, 64, 0, 0, 48, 0, None, FAKE, FAKE, FAKE, None) == INVALID  # group
    assert nq(FAKE, 64, 64, 64, 0, 12, 0, 0, None, FAKE, FAKE, FAKE, None) == INVALID  # mode


def qd(N, x=FAKE, rows=256, cols=256, ld=256, mr=0, gr=0, mc=2, gc=128, ar=FAKE, ac=FAKE, outs=None):
    o = outs if outs is not None else (FAKE + 0x1000, FAKE + 0x2000, FAKE + 0x3000, FAKE + 0x4000, FAKE + 0x5000,
                                       FAKE + 0x6000)
    return N.nvfp4_quantize_dual(x, rows, cols, ld, mr, gr, mc, gc, 0, ar, ac, *o, None)


def test_quantize_dual_rejects(N):
    assert qd(N, x=None) == INVALID
    assert qd(N, mr=12) == INVALID
    assert qd(N, gr=48) == INVALID
    assert qd(N, mr=2, gr=0) == UNSUPPORTED          # MS-EDEN needs the rotation, in either view
    assert qd(N, mc=2, gc=0) == UNSUPPORTED
    assert qd(N, cols=40, ld=40) == SHAPE            # row view: cols % 16
    assert qd(N, rows=40) == SHAPE                   # column view: rows % 16
    assert qd(N, rows=64, gc=128) == SHAPE           # column view: rows % g
    assert qd(N, mc=6, gc=0, rows=48) == SHAPE       # MXFP4 column view: whole 32-element groups
    assert qd(N, ar=None) == INVALID                 # the row view's amax is required (not an MX mode)
    assert qd(N, ac=None) == INVALID
    assert qd(N, outs=(None, FAKE, FAKE, FAKE, FAKE, FAKE)) == INVALID
    assert qd(N, outs=(FAKE, FAKE, FAKE, FAKE, FAKE, None)) == INVALID
    assert qd(N, outs=(FAKE + 4, FAKE, FAKE, FAKE, FAKE, FAKE)) == ALIGN
    assert qd(N, x=FAKE + 8) == ALIGN
    assert qd(N, ar=FAKE + 2) == ALIGN


def _group_args(n, shapes, amax=True):
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    ptrs = lambda vals: (P * n)(*vals)  # noqa: E731
    return dict(x=ptrs([FAKE + 0x10000 * i for i in range(n)]), rows=(I64 * n)(*[s[0] for s in shapes]),
                cols=(I64 * n)(*[s[1] for s in shapes]), ld=(I64 * n)(*[s[1] for s in shapes]),
                a=ptrs([FAKE + 0x100 * i if amax else None for i in range(n)]),
                o=[ptrs([FAKE + 0x1000 * (j + 1) + 0x40 * i for i in range(n)]) for j in range(6)])


def test_group_calls_reject(N):
    """The group calls check every member as the single calls do, before any
    launch: a bad second member fails the whole call."""
    good = (256, 256)
    g = _group_args(2, [good, good])
    ag = lambda n, g, gr=0, gc=128: N.nvfp4_amax_dual_group(n, g["x"], g["rows"], g["cols"], g["ld"], gr, gc, 0,  # noqa: E731
                                                            g["a"], g["a"], None)
    assert ag(0, g) == INVALID                      # no members
    assert ag(65, g) == INVALID                     # more than NVFP4_MAX_GROUP
    assert N.nvfp4_amax_dual_group(2, None, g["rows"], g["cols"], g["ld"], 0, 128, 0, g["a"], g["a"], None) == INVALID
    assert ag(2, g, gc=48) == INVALID               # rotation group
    bad = _group_args(2, [good, (256, 40)])         # second member: cols not a multiple of 16
    assert ag(2, bad) == SHAPE
    noamax = _group_args(2, [good, good], amax=False)
    assert ag(2, noamax) == INVALID                 # outputs required

    def qg(n, g, mr=0, gr=0, mc=2, gc=128):
        o = g["o"]
        return N.nvfp4_quantize_dual_group(n, g["x"], g["rows"], g["cols"], g["ld"], mr, gr, mc, gc, 0, g["a"],
                                           g["a"], o[0], o[1], o[2], o[3], o[4], o[5], None)
    assert qg(0, g) == INVALID
    assert qg(65, g) == INVALID
    assert qg(2, g, mr=12) == INVALID               # mode
    assert qg(2, g, mr=2, gr=0) == UNSUPPORTED      # MS-EDEN needs the rotation
    assert qg(2, bad) == SHAPE
    assert qg(2, noamax) == INVALID                 # the row view's amax is required (not an MX mode)
    mis = _group_args(2, [good, good])
    mis["o"][0] = (ctypes.c_void_p * 2)(FAKE, FAKE + 4)  # second member's codes not 8-byte aligned
    assert qg(2, mis) == ALIGN


def test_pack3_rejects(N):
    p, u = N.nvfp4_pack3, N.nvfp4_unpack3
    assert p(FAKE, FAKE, 4, 64, 0, FAKE, FAKE, None) == UNSUPPORTED      # RTN is not a 3-bit mode
    assert p(FAKE, FAKE, 4, 40, 8, FAKE, FAKE, None) == SHAPE            # vcols % 16
    assert p(FAKE, FAKE, 4, 48, 11, FAKE, FAKE, None) == SHAPE           # MXFP3: vcols % 32
    assert p(None, FAKE, 4, 64, 8, FAKE, FAKE, None) == INVALID
    assert p(FAKE, FAKE, 0, 64, 8, None, None, None) == OK               # empty: nothing touched
    assert p(FAKE + 4, FAKE, 4, 64, 8, FAKE, FAKE, None) == ALIGN        # codes 8-byte aligned
    assert p(FAKE, FAKE, 4, 64, 8, FAKE + 1, FAKE, None) == ALIGN        # packed codes 2-byte aligned
    assert u(FAKE, FAKE, 4, 64, 9, None, FAKE, None) == INVALID
    assert u(FAKE, FAKE, 4, 64, 3, FAKE, FAKE, None) == UNSUPPORTED


def test_other_entry_points_reject(N):
    assert N.nvfp4_amax(None, 64, 64, 64, 0, 0, 0, FAKE, None) == INVALID
    assert N.nvfp4_amax(FAKE, 64, 64, 64, 0, 0, 0, None, None) == INVALID
    assert N.nvfp4_amax(FAKE, 64, 40, 40, 0, 0, 0, FAKE, None) == SHAPE
    ad = N.nvfp4_amax_dual
    assert ad(None, 64, 64, 64, 0, 0, 0, FAKE, FAKE, None) == INVALID
    assert ad(FAKE, 64, 64, 64, 0, 0, 0, FAKE, None, None) == INVALID
    assert ad(FAKE, 64, 64, 64, 48, 0, 0, FAKE, FAKE, None) == INVALID   # group
    assert ad(FAKE, 64, 40, 40, 0, 0, 0, FAKE, FAKE, None) == SHAPE      # row view: cols % 16
    assert ad(FAKE, 40, 64, 64, 0, 0, 0, FAKE, FAKE, None) == SHAPE      # column view: rows % 16
    assert ad(FAKE, 64, 64, 64, 0, 128, 0, FAKE, FAKE, None) == SHAPE    # column view: rows % g
    assert ad(FAKE, 64, 64, 64, 0, 0, 0, FAKE + 2, FAKE, None) == ALIGN
    d = N.nvfp4_dequantize
    assert d(None, FAKE, FAKE, 4, 64, 0, 0, 0, 0, FAKE, None) == INVALID
    assert d(FAKE, FAKE, FAKE, 4, 64, 0, 0, 0, 1, FAKE, None) == INVALID  # inverse without rotation
    assert d(FAKE, FAKE, FAKE, 4, 40, 0, 0, 0, 0, FAKE, None) == SHAPE
    assert d(FAKE, FAKE, FAKE, 4, 64, 12, 0, 0, 0, FAKE, None) == INVALID
    assert d(FAKE, FAKE, FAKE, 4, 64, 0, 0, 0, 0, FAKE + 4, None) == ALIGN
    r = N.nvfp4_rht
    assert r(FAKE, 0, 64, 64, 64, 0, 0, 0, 0, FAKE, None) == INVALID      # group 0
    assert r(FAKE, 2, 64, 64, 64, 0, 16, 0, 0, FAKE, None) == INVALID     # dtype
    assert r(FAKE, 0, 64, 48, 48, 0, 32, 0, 0, FAKE, None) == SHAPE
    assert r(FAKE + 1, 0, 64, 64, 64, 0, 16, 0, 0, FAKE, None) == ALIGN
    assert N.nvfp4_encode_e2m1(None, 4, FAKE, None) == INVALID
    assert N.nvfp4_encode_e2m1(FAKE, -1, FAKE, None) == SHAPE
    assert N.nvfp4_encode_e4m3(FAKE + 2, 4, 0, FAKE, None) == ALIGN
    g = N.nvfp4_gemm
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert g(*ok, 128, 128, 256, 2, FAKE, 128, None) == INVALID        # output dtype
    assert g(*ok, 100, 128, 256, 0, FAKE, 128, None) == SHAPE          # m % 128
    assert g(*ok, 128, 130, 256, 0, FAKE, 130, None) == SHAPE          # n % 128
    assert g(*ok, 128, 128, 320, 0, FAKE, 128, None) == SHAPE          # k % 256
    assert g(*ok, 128, 128, 0, 0, FAKE, 128, None) == SHAPE            # k = 0
    assert g(*ok, 128, 128, 256, 0, FAKE, 64, None) == SHAPE           # ldd < n
    assert g(*ok, 0, 128, 256, 0, None, 128, None) == OK               # empty: nothing touched
    assert g(None, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 128, 256, 0, FAKE, 128, None) == INVALID
    assert g(*ok, 128, 128, 256, 0, None, 128, None) == INVALID
    assert g(FAKE + 8, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 128, 256, 0, FAKE, 128, None) == ALIGN
    assert g(*ok, 128, 128, 256, 0, FAKE, 130, None) == ALIGN          # fp32 rows: ldd % 4
    assert g(*ok, 128, 128, 256, 1, FAKE, 132, None) == ALIGN          # bf16 rows: ldd % 8


def test_binding_refuses_cpu_tensors(N):
    import torch
    with pytest.raises(ValueError):
        N.quantize(torch.zeros(16, 16, dtype=torch.bfloat16))


def test_mode_numbers_agree_everywhere(N):
    """The nvfp4_mode values of include/nvfp4.h are the binding's, the
    workloads module's and the oracle's (each side defines them itself)."""
    import oracle
    from nvfp4_microscaling_quantization_b200 import workloads as W
    text = open(HEADER).read()
    enum = dict((name, int(v)) for name, v in re.findall(r"NVFP4_([A-Z0-9_]+) = (\d+)", text))
    names = {"RTN": "RTN", "SR": "SR", "MS_EDEN": "MS_EDEN", "IF4": "IF4", "4OVER6": "FOUR_OVER_SIX",
             "SCALE_SEARCH": "SCALE_SEARCH", "MXFP4": "MXFP4", "NVINT4": "NVINT4", "NVFP3": "NVFP3",
             "NVINT3": "NVINT3", "IF3": "IF3", "MXFP3": "MXFP3"}
    for c_name, py_name in names.items():
        v = enum[c_name]
        assert getattr(N, py_name) == v and getattr(W, py_name) == v and getattr(oracle, py_name) == v, c_name
    assert set(W.MODE_NAMES) == set(enum[c] for c in names)

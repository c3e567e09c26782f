"""The block-scale division of the quantization kernels, pinned on the CPU.

The kernels compute s_f = RN(absmax / q) (q = RN(m s_g), m the element
maximum 3, 4, 6 or 7) not with a division but with the round-to-nearest
reciprocal r = RN(1/q) and Markstein's remainder correction:
t = RN(a r), rem = fma(-t, q, a), s_f = fma(rem, r, t).  This test restates
that sequence in C (tests/markstein_check.c) and compares it, bit for bit, with
the correctly rounded quotient for every binary32 divisor significand (2^23
divisors, so every q any m and tensor scale can produce, up to a power of two)
at the five dividends nearest each E4M3 decision point B q (the E4M3 values and
the midpoints between them), plus random dividends.  No difference is
allowed: the block scales of every mode are then those of an exact division.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker():
    d = tempfile.mkdtemp(prefix="markstein_")
    so = os.path.join(d, "markstein_check.so")
    subprocess.run(["cc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                    os.path.join(HERE, "markstein_check.c"), "-o", so, "-lm"], check=True)
    L = ctypes.CDLL(so)
    L.markstein_check.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int64),
                                  ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
    L.markstein_check.restype = ctypes.c_int64
    return L


def _run(L, i0, i1, extra, variant=0):
    n = ctypes.c_int64(0)
    fa, fq = ctypes.c_uint32(0), ctypes.c_uint32(0)
    bad = L.markstein_check(i0, i1, extra, variant, ctypes.byref(n), ctypes.byref(fa), ctypes.byref(fq))
    return bad, n.value, fa.value, fq.value


def test_uncorrected_product_is_caught(checker):
    """The comparison has teeth: the product RN(a RN(1/q)) without the
    remainder correction differs from the exact quotient on many pairs."""
    bad, n, _, _ = _run(checker, 0, 1 << 16, 0, variant=1)
    assert n == (1 << 16) * 16 * 5 and bad > 1000


def test_every_divisor_significand(checker):
    bad, n, fa, fq = _run(checker, 0, 1 << 23, 2)
    assert n == (1 << 23) * (16 * 5 + 2)
    assert bad == 0, f"{bad} quotients differ from RN(a/q); first a=0x{fa:08x} q=0x{fq:08x}"

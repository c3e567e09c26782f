"""The kernels' bit-level formation of codes, pinned on the CPU.

Stochastic rounding onto E2M1 and onto E4M3 (MS-EDEN's scale), the INT4
levels of NVINT4 and IF4, the INT3
levels of NVINT3 and IF3, and the E2M0 codes of NVFP3, MXFP3 and IF3 are
formed in the kernels without conversion instructions: integer sums on the
bits of the floats, and byte permutes that gather eight elements' nibbles
into one code word.  tests/code_bits_check.c restates those sequences in C
and compares every element, bit for bit, with the rules written from their
definitions: stochastic rounding goes up iff U < (a - l)/(u - l) (the
palettes post, "The two corners, and what the palette does to them"), the
INT4 level is clamp(RNE(t), -7, 7) as a sign-magnitude nibble (IF4 paper
page, Table 1 and Figure 3), the INT3 level clamp(RNE(t), -3, 3), and E2M0
the nearest of {0, 1, 2, 4} with ties to the even code (the same page's
3-bit formats table lists E2M0 and INT3 elements).  Inputs: every finite
bf16 value at the draws next to its decision point and at the extremes, in
random word slots, plus random binary32 values; the ties, clamp edges and
signed zeros of the integer levels and of E2M0.  No difference is allowed.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker():
    d = tempfile.mkdtemp(prefix="code_bits_")
    so = os.path.join(d, "code_bits_check.so")
    subprocess.run(["cc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-frounding-math", "-fPIC", "-shared",
                    os.path.join(HERE, "code_bits_check.c"), "-o", so, "-lm"], check=True)
    L = ctypes.CDLL(so)
    for fn in (L.sr_check, L.int4_check, L.int3_check, L.e2m0_check, L.if4_level_check, L.e4m3_sr_check):
        fn.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)]
        fn.restype = ctypes.c_int64
    return L


def _run(fn, n_random, variant=0):
    n = ctypes.c_int64(0)
    bad = fn(n_random, variant, ctypes.byref(n))
    return bad, n.value


def test_planted_mistakes_are_caught(checker):
    """The comparisons have teeth: one flipped code bit per word is found."""
    bad, n = _run(checker.sr_check, 0, variant=1)
    assert bad > 100000 and n > 0
    bad, n = _run(checker.int4_check, 0, variant=1)
    assert bad > 1000 and n > 0
    bad, n = _run(checker.int3_check, 0, variant=1)
    assert bad > 1000 and n > 0
    bad, n = _run(checker.e2m0_check, 0, variant=1)
    assert bad > 1000 and n > 0
    bad, n = _run(checker.e2m0_check, 0, variant=2)  # magnitude 0.5 kept for index 0
    assert bad > 1000 and n > 0
    bad, n = _run(checker.if4_level_check, 1 << 16, variant=1)  # no clamp of |y| at 6
    assert bad > 1000 and n > 0
    bad, n = _run(checker.e4m3_sr_check, 1 << 16, variant=1)  # t/2 + 2^-7 rounded to nearest
    assert bad > 100 and n > 0


def test_stochastic_rounding_codes(checker):
    bad, n = _run(checker.sr_check, 1 << 18)
    assert n > 3_000_000
    assert bad == 0, f"{bad} of {n} stochastic-rounding codes differ from the rule"


def test_int4_level_codes(checker):
    bad, n = _run(checker.int4_check, 1 << 20)
    assert n > 1_000_000
    assert bad == 0, f"{bad} of {n} INT4 nibbles differ from the rule"


def test_int3_level_codes(checker):
    bad, n = _run(checker.int3_check, 1 << 20)
    assert n > 1_000_000
    assert bad == 0, f"{bad} of {n} INT3 nibbles differ from the rule"


def test_e2m0_codes_and_magnitudes(checker):
    bad, n = _run(checker.e2m0_check, 1 << 20)
    assert n > 1_000_000
    assert bad == 0, f"{bad} of {n} E2M0 codes, magnitudes or IF3 sign sources differ from the rule"


def test_if4_integer_level_from_y(checker):
    bad, n = _run(checker.if4_level_check, 1 << 20)
    assert n > 1_000_000
    assert bad == 0, f"{bad} of {n} IF4 integer levels differ from clamp(RNE(RN(y K1)), -7, 7)"


def test_e4m3_stochastic_scale_rounding(checker):
    bad, n = _run(checker.e4m3_sr_check, 1 << 20)
    assert n > 1_000_000
    assert bad == 0, f"{bad} of {n} stochastically rounded E4M3 scales differ from the rule"

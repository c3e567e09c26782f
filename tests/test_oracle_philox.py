"""Pins the oracle's Philox4x32-10 and its three random streams to cuRAND.

cuRAND's *host* generator (CURAND_RNG_PSEUDO_PHILOX4_32_10, created with
curandCreateGeneratorHost, so no GPU is needed) is an independent
implementation of the SC'11 Philox4x32-10 bijection.  With seed s it emits
4-word block j = philox(counter = (j // 65536 as a 64-bit value split into
words 0 and 1, j % 65536, 0), key = (s low word, s high word)), and
curandSetGeneratorOffset(4 j) starts the stream at block j.  That mapping lets
the test reach every counter word the method uses: words 0/1 (the call index),
word 2 (the stream tag) and both key words (the seed).
"""
import ctypes
import os

import numpy as np
import pytest

CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161


def _curand():
    for path in ("/usr/local/cuda/lib64/libcurand.so", "libcurand.so", "libcurand.so.10"):
        try:
            return ctypes.CDLL(path)
        except OSError:
            continue
    pytest.skip("libcurand not available")


def curand_block(lib, seed, block):
    gen = ctypes.c_void_p()
    assert lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) == 0
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        assert lib.curandSetGeneratorOffset(gen, ctypes.c_ulonglong(4 * block)) == 0
        out = np.zeros(4, dtype=np.uint32)
        assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(4)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    return out


def counter_of_block(block):
    call, sub = divmod(block, 65536)
    return [call & 0xFFFFFFFF, call >> 32, sub, 0]


SEEDS = [0, 1, 7, 0xDEADBEEF12345678, (1 << 64) - 1]
BLOCKS = [0, 1, 2, 3, 65535, 65536 * 5 + 2, (1 << 48) + 1, (3 << 48) + 65536 * 77 + 1]


@pytest.mark.parametrize("seed", SEEDS)
def test_philox_matches_curand(orc, seed):
    lib = _curand()
    key = [seed & 0xFFFFFFFF, seed >> 32]
    for block in BLOCKS:
        ref = curand_block(lib, seed, block)
        got = orc.philox(counter_of_block(block), key)
        assert list(got) == list(ref), (seed, block)


def test_streams_follow_their_counters(orc):
    """Element (tag 0), block (tag 1) and sign (tag 2) draws are the stated words of cuRAND blocks."""
    lib = _curand()
    seed = 0x0123456789ABCDEF
    # element e -> call e>>3, tag 0 -> cuRAND block (e>>3)*65536 + 0
    for e in [0, 1, 5, 7, 8, 1023, 123457]:
        w = curand_block(lib, seed, (e >> 3) * 65536 + 0)
        word = int(w[(e & 7) >> 1])
        k = (word >> (16 * (e & 1))) & 0xFFFF
        assert orc.uniform_element(seed, e) == k / 65536.0
    # block b -> call b>>3, tag 1, 16-bit halves like the element draws
    for b in [0, 1, 2, 3, 4, 7, 8, 999, 77777]:
        w = curand_block(lib, seed, (b >> 3) * 65536 + 1)
        word = int(w[(b & 7) >> 1])
        k = (word >> (16 * (b & 1))) & 0xFFFF
        assert orc.uniform_block(seed, b) == k / 65536.0
    # sign j -> call 0, tag 2
    w = curand_block(lib, seed, 2)
    signs = orc.rht_signs(seed, 128)
    for j in range(128):
        bit = (int(w[j >> 5]) >> (j & 31)) & 1
        assert signs[j] == (-1.0 if bit else 1.0)


def test_signs_depend_on_seed_and_are_balanced(orc):
    s0, s1 = orc.rht_signs(0, 128), orc.rht_signs(1, 128)
    assert not np.array_equal(s0, s1)
    # 128 fair coin flips: |sum| > 48 has probability ~ 2e-5
    for s in (s0, s1):
        assert abs(float(s.sum())) < 48

"""The multi-process oracle driver (oracle/pool.py) assembles exactly the
single-process oracle's results: the tensor amax, the rotated view, and the
codes, scales and tensor scale of every layout, on shapes whose row ranges
split unevenly."""
import numpy as np
import pytest
import torch

import oracle
from oracle.pool import OraclePool
from nvfp4_microscaling_quantization_b200 import workloads as W


@pytest.fixture(scope="module")
def pool():
    with OraclePool(workers=3) as p:
        yield p


def _x(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return W.bf16_bits(torch.randn(rows, cols, generator=g).to(torch.bfloat16))


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
@pytest.mark.parametrize("mode,g", [(W.RTN, 0), (W.SR, 128), (W.MS_EDEN, 64), (W.IF4, 0), (W.FOUR_OVER_SIX, 32)])
def test_pool_matches_oracle(pool, layout, mode, g):
    xb = _x(256, 384, 7 + mode)
    seed = 11
    a = oracle.amax(xb, layout, g, seed)
    assert pool.amax(xb, layout, g, seed) == a
    exp = oracle.quantize(xb, layout, mode, g, seed, amax_in=a)
    got = pool.quantize(xb, layout, mode, g, seed, a)
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1]) and got[2] == exp[2]
    if g:
        z = oracle.rht_view(xb, layout, g, seed)
        zp = pool.rht_view(xb, layout, g, seed)
        assert np.array_equal(z.view(np.uint32), zp.view(np.uint32))
        exp_r = oracle.quantize_rotated(z, mode, seed, a)
        got_r = pool.quantize_rotated(zp, mode, seed, a)
        assert np.array_equal(got_r[0], exp_r[0]) and np.array_equal(got_r[1], exp_r[1])


def test_pool_shared_input(pool):
    xb = _x(128, 256, 4)
    h = pool.put(xb)
    a = oracle.amax(xb, W.TRANSPOSED, 64, 2)
    assert pool.amax(h, W.TRANSPOSED, 64, 2) == a
    exp = oracle.quantize(xb, W.TRANSPOSED, W.MS_EDEN, 64, 2, amax_in=a)
    got = pool.quantize(h, W.TRANSPOSED, W.MS_EDEN, 64, 2, a)
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1])
    assert np.array_equal(pool.rht_view(h, W.TRANSPOSED, 64, 2), oracle.rht_view(xb, W.TRANSPOSED, 64, 2))


def test_pool_row_range(pool):
    xb = _x(96, 256, 3)
    a = oracle.amax(xb, W.ROWWISE, 0, 5)
    exp = oracle.quantize(xb, W.ROWWISE, W.RTN, 0, 5, amax_in=a, row_range=(10, 77))
    got = pool.quantize(xb, W.ROWWISE, W.RTN, 0, 5, a, row_range=(10, 77))
    assert np.array_equal(got[0], exp[0]) and np.array_equal(got[1], exp[1])

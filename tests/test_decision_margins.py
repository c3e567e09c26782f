"""The rule that explains end-to-end differences of rotated quantizations
(tests/decision_margins.py), checked on the CPU with the oracle: a difference
caused by moving a value across a rounding point by one ulp is explained; a
difference planted in the oracle's output away from every rounding point is
not."""
import numpy as np
import pytest

import oracle
from decision_margins import explain

SEED = 9


def _z(rows=4, cols=64, seed=1):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((rows, cols)).astype(np.float32)


def _diffs(mode, zo, zg, amax):
    co, so, gs = oracle.quantize_rotated(zo, mode, SEED, amax)
    cg, sg, _ = oracle.quantize_rotated(zg, mode, SEED, amax)
    return oracle.unpack_codes(co) != oracle.unpack_codes(cg), so != sg, gs


def _explain_block(mode, zo, zg, gs, cd, sd, r, b, glen=16):
    vc = zo.shape[1]
    c0 = b * glen
    return explain(mode, zo[r, c0:c0 + glen], zg[r, c0:c0 + glen], gs, SEED, r * vc + c0, r * (vc // 16) + c0 // 16,
                   cd[r, c0:c0 + glen], bool(sd[r, c0 // 16:(c0 + glen) // 16].any()))


def _place_on_threshold(zo, amax, mode, r, b, i, y_target):
    """Set element i of block b of row r so that its scaled value is y_target
    (the block maximum stays the same)."""
    _, so, gs = oracle.quantize_rotated(zo, mode, SEED, amax)
    S = so[r, b] & 0x7F
    d = np.float32(np.float32(oracle.e4m3_decode(S)) * np.float32(gs))
    zo[r, 16 * b + i] = np.float32(y_target) * d
    return d


@pytest.mark.parametrize("mode,threshold", [(oracle.RTN, 1.25), (oracle.MS_EDEN, 2.5), (oracle.IF4, 0.75),
                                            (oracle.NVINT4, 2.5), (oracle.NVFP3, 1.5)])
def test_one_ulp_across_a_rounding_point_is_explained(mode, threshold):
    zo = _z()
    zo[:, 16 * 1] = 9.0  # a fixed block maximum in block 1 of every row
    amax = float(np.abs(zo).max())
    r, b, i = 2, 1, 5
    _place_on_threshold(zo, amax, mode, r, b, i, threshold)
    found = False
    for step in (1, -1, 2, -2):
        zg = zo.copy()
        zg[r, 16 * b + i] = np.nextafter(zo[r, 16 * b + i], np.float32(np.inf) * step, dtype=np.float32)
        if step in (2, -2):
            zg[r, 16 * b + i] = np.nextafter(zg[r, 16 * b + i], np.float32(np.inf) * step, dtype=np.float32)
        cd, sd, gs = _diffs(mode, zo, zg, amax)
        if cd.any() or sd.any():
            found = True
            for rr, bb in np.argwhere(cd.reshape(cd.shape[0], -1, 16).any(axis=2) | sd):
                ok, why = _explain_block(mode, zo, zg, gs, cd, sd, rr, bb)
                assert ok, why
    assert found, "moving the value across the rounding point changed nothing"


def _perturbed(zo, ulps, seed):
    """zo moved by up to `ulps` fp32 ulps per element (a rotation's rounding noise)."""
    rng = np.random.default_rng(seed)
    steps = rng.integers(-ulps, ulps + 1, size=zo.shape)
    out = zo.copy()
    for k in range(1, ulps + 1):
        up, down = steps >= k, steps <= -k
        out[up] = np.nextafter(out[up], np.float32(np.inf), dtype=np.float32)
        out[down] = np.nextafter(out[down], np.float32(-np.inf), dtype=np.float32)
    return out


@pytest.mark.parametrize("mode", [oracle.RTN, oracle.SR, oracle.MS_EDEN, oracle.IF4, oracle.FOUR_OVER_SIX,
                                  oracle.NVINT4, oracle.IF3])
def test_planted_code_is_not_explained(mode):
    from decision_margins import element_thresholds
    zo = _z(seed=3)
    zg = _perturbed(zo, 3, seed=5)
    amax = float(np.abs(zo).max())
    co, so, gs = oracle.quantize_rotated(zo, mode, SEED, amax)
    nib = oracle.unpack_codes(co)
    # the element of block (1, 2) farthest from every rounding point of the
    # mode: flip a magnitude bit of its code in a copy of the oracle's output
    r, b = 1, 2
    d = np.float32(np.float32(oracle.e4m3_decode(so[r, b] & 0x7F)) * np.float32(gs))
    y = np.abs(zo[r, 16 * b:16 * b + 16].astype(np.float64) / d)
    dist = np.full(16, np.inf)
    for t in element_thresholds(mode):
        dist = np.minimum(dist, np.abs(y[:, None] - np.asarray(t)[None, :]).min(axis=1))
    i = int(np.argmax(dist))
    assert dist[i] > 0.05
    cg = nib.copy()
    cg[r, 16 * b + i] ^= 1
    cd = cg != nib
    sd = np.zeros_like(so, dtype=bool)
    ok, why = _explain_block(mode, zo, zg, gs, cd, sd, r, b)
    assert not ok, f"a planted code was explained: {why}"


@pytest.mark.parametrize("mode", [oracle.RTN, oracle.MS_EDEN, oracle.NVINT4])
def test_planted_scale_is_not_explained(mode):
    zo = _z(seed=4)
    zg = zo.copy()
    zg[0, 0] = np.nextafter(zg[0, 0], np.float32(np.inf), dtype=np.float32)   # a tiny rotation difference
    amax = float(np.abs(zo).max())
    _, so, gs = oracle.quantize_rotated(zo, mode, SEED, amax)
    cd = np.zeros((zo.shape[0], zo.shape[1]), dtype=bool)
    sd = np.zeros_like(so, dtype=bool)
    sd[0, 0] = True
    ok, why = _explain_block(mode, zo, zg, gs, cd, sd, 0, 0)
    # the planted scale is explained only if block 0 happens to sit at a decision point
    if ok:
        assert "near" in why or "within" in why
    sd2 = np.zeros_like(so, dtype=bool)
    sd2[2, 1] = True
    ok2, why2 = _explain_block(mode, zo, zo.copy(), gs, cd, sd2, 2, 1)
    assert not ok2, f"a scale difference with identical rotated values was explained: {why2}"

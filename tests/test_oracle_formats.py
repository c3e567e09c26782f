"""Pins the oracle's E2M1 and E4M3 codecs and its constants.

E2M1 value set {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6}: "Comparing INT4 and
NVFP4 Palettes on Real Gradient Tensors", opening section.
E4M3 scale range (max 448, min 2^-9, read off 6 x 448 and 0.5 x 2^-9): IF4
paper page (arXiv 2603.28765), Table 1.

Independent references used here: brute-force nearest search written from the
value set, torch's float8_e4m3fn conversion (a library routine), and exact
rational arithmetic (fractions.Fraction).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def nearest_code(y):
    """Nearest signed grid value by exhaustive search, ties to the even magnitude index."""
    a = abs(Fraction(y))
    best, best_d = 0, None
    for k, m in enumerate(GRID):
        d = abs(a - Fraction(m))
        if best_d is None or d < best_d or (d == best_d and k % 2 == 0):
            best, best_d = k, d
    if best == 0:
        return 0
    return (8 if y < 0 else 0) | best


def all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


def test_e2m1_grid_values(orc):
    for code in range(16):
        mag = GRID[code & 7]
        assert orc.e2m1_decode(code) == (-mag if code & 8 else mag)


def test_e2m1_rtn_exhaustive_bf16(orc):
    """Every finite bf16 value rounds to the nearest grid value (ties to even code, +0 for zero)."""
    vals = all_finite_bf16()
    # exact search is slow in Fraction; use exact float64 arithmetic on the magnitudes, which
    # is exact here (differences of bf16 values and grid values fit in 53 bits or are far
    # from any tie), and check ties with Fraction.
    a = np.abs(vals.astype(np.float64))
    dist = np.abs(a[:, None] - np.array(GRID)[None, :])
    best = np.argmin(dist, axis=1)
    dmin = dist[np.arange(len(a)), best]
    tie = (dist == dmin[:, None]).sum(axis=1) > 1
    got = np.array([orc.e2m1_rtn(float(v)) for v in vals], dtype=np.int64)
    exp = np.where(best == 0, 0, np.where(vals < 0, 8, 0) | best)
    nt = ~tie
    assert np.array_equal(got[nt], exp[nt])
    for v, g in zip(vals[tie], got[tie]):
        assert g == nearest_code(float(v)), v
    assert tie.sum() >= 14  # the 7 midpoints, both signs, are bf16 values


def test_e2m1_rtn_fp32_neighbourhoods(orc):
    """fp32 values within 64 ulps of every midpoint and grid value, both signs."""
    pts = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] + GRID[1:] + [6.5, 7.0, 1e30]
    for p in pts:
        base = np.float32(p).view(np.uint32).astype(np.int64)
        for off in range(-64, 65):
            v = np.array([base + off], dtype=np.uint32).view(np.float32)[0]
            for s in (1.0, -1.0):
                y = float(np.float32(s * v))
                assert orc.e2m1_rtn(y) == nearest_code(y), y


def test_e4m3_decode_matches_torch(orc):
    for code in range(0x7F):
        t = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item()
        assert orc.e4m3_decode(code) == t, code
    assert orc.e4m3_decode(0x7E) == 448.0
    assert orc.e4m3_decode(0x01) == 2.0 ** -9
    assert orc.e4m3_decode(0x08) == 2.0 ** -6  # smallest normal


def _torch_e4m3(vals):
    t = torch.from_numpy(np.asarray(vals, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def _e4m3_sample_points():
    table = np.array([float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float())
                      for c in range(0x7F)], dtype=np.float64)
    mids = (table[1:] + table[:-1]) / 2
    centres = np.concatenate([table[1:], mids, [2.0 ** -10, 2.0 ** -11, 448.0, 460.0]])
    pts = []
    for p in centres:
        base = np.float32(p).view(np.uint32).astype(np.int64)
        pts.append(np.arange(base - 8, base + 9, dtype=np.int64))
    bits = np.concatenate(pts).astype(np.uint32)
    rng = np.random.default_rng(0)
    rand = np.exp2(rng.uniform(-14, np.log2(463.0), 50000)).astype(np.float32)
    return np.concatenate([bits.view(np.float32), rand]), table


def test_e4m3_rne_matches_torch(orc):
    """RNE onto E4M3 agrees with torch's float8_e4m3fn conversion below the overflow point."""
    vals, _ = _e4m3_sample_points()
    vals = vals[(vals > 0) & (vals < 464.0)]
    ref = _torch_e4m3(vals)
    got = np.array([orc.e4m3_rne_sat(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_saturates(orc):
    for v in [448.0, 449.0, 464.0, 500.0, 1e6, 3e38]:
        assert orc.e4m3_rne_sat(v) == 0x7E
        assert orc.e4m3_ru_sat(v) == 0x7E
    assert orc.e4m3_rne_sat(0.0) == 0 and orc.e4m3_ru_sat(0.0) == 0


def test_e4m3_round_up_brute_force(orc):
    vals, table = _e4m3_sample_points()
    vals = vals[(vals > 0) & (vals <= 448.0)]
    for v in vals[::7]:
        exp = int(np.argmax(table >= float(v)))
        assert orc.e4m3_ru_sat(float(v)) == exp, v
        assert table[exp] >= v and (exp == 0 or table[exp - 1] < v)


def test_e4m3_sr_brackets_and_is_unbiased(orc):
    _, table = _e4m3_sample_points()
    rng = np.random.default_rng(1)
    for t in [2.0 ** -10, 0.3, 1.0, 1.03, 7.77, 100.1, 447.0]:
        t32 = float(np.float32(t))
        lo = int(np.searchsorted(table, t32, side="right") - 1)
        us = (np.arange(4096) + 0.5) / 4096.0  # a uniform grid of U values
        codes = np.array([orc.e4m3_sr(t32, float(np.float32(u))) for u in us])
        assert set(np.unique(codes)).issubset({lo, lo + 1})
        mean = np.mean(table[codes])
        assert abs(mean - t32) <= (table[lo + 1] - table[lo]) / 4096 + 1e-12
    assert orc.e4m3_sr(448.0, 0.0) == 0x7E and orc.e4m3_sr(1000.0, 0.9) == 0x7E
    assert orc.e4m3_sr(1.0, 0.999) == 0x38  # exactly representable: never moves
    del rng


def f32_nearest(q: Fraction) -> float:
    """Round a positive rational to the nearest binary32 (ties even), by exhaustive neighbour check."""
    f = np.float32(float(q))
    cands = [np.nextafter(f, np.float32(0)), f, np.nextafter(f, np.float32(np.inf))]
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - q), int(np.float32(c).view(np.uint32)) & 1))
    return float(best)


def isqrt_fraction(g, digits=60):
    # 1/sqrt(g) to ~60 decimal digits via integer square root
    scale = 10 ** digits
    from math import isqrt
    return Fraction(scale, isqrt(g * scale * scale))


@pytest.mark.parametrize("g", [16, 32, 64, 128])
def test_rht_scale_constant(orc, g):
    c = orc.rht_scale(g)
    assert c == f32_nearest(isqrt_fraction(g))


def test_global_scale(orc):
    """M = 448 (6 x 448, IF4 page Table 1), M = 256 for 4/6 (6 x 256) and for MS-EDEN (headroom)."""
    assert orc.global_scale(0.0, 0) == 1.0
    assert orc.global_scale(2688.0, 0) == 1.0
    assert orc.global_scale(1536.0, 4) == 1.0
    for a in [1e-3, 0.37, 5.0, 123.0]:
        for mode, six_m in [(0, 2688), (1, 2688), (2, 1536), (3, 2688), (4, 1536)]:
            assert orc.global_scale(a, mode) == f32_nearest(Fraction(float(np.float32(a))) / six_m)


def test_if4_constants(orc):
    k1, k2 = orc.if4_constants()
    assert k1 == f32_nearest(Fraction(7, 6))
    assert k2 == f32_nearest(Fraction(6, 7))

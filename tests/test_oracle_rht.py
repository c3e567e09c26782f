"""Pins the oracle's random Hadamard transform.

The rotation is z = c_g H_g (sigma o x) per group of g elements along a row,
with H_g the Sylvester Hadamard matrix ("Comparing INT4 and NVFP4 Palettes on
Real Gradient Tensors": a random Hadamard rotation before quantizing, 16x16 in
section "45 real tensors disagree"; Quartet II article, section
"Quantisierung im Rueckwaertsdurchlauf": randomized Hadamard rotations).

Independent references: scipy.linalg.hadamard (Sylvester construction),
H H^T = g I, the exact inverse on small integers, and the fp64 product.
"""
import numpy as np
import pytest
import scipy.linalg

GROUPS = [16, 32, 64, 128]


@pytest.mark.parametrize("g", GROUPS)
def test_rotation_of_unit_vectors_is_scaled_hadamard(orc, g):
    """Row j of the identity maps to c_g * sigma_j * H[j, :] exactly (H symmetric)."""
    seed = 11
    eye = np.eye(g, dtype=np.float32)
    z = orc.rht_rows(eye, g, seed)
    H = scipy.linalg.hadamard(g).astype(np.float64)
    sigma = orc.rht_signs(seed, g).astype(np.float64)
    c = orc.rht_scale(g)
    expect = (c * sigma[:, None] * H).astype(np.float32)
    assert np.array_equal(z, expect)
    # and H H^T = g I for the matrix the transform applies
    Hm = (z.astype(np.float64) / c) * sigma[:, None]
    assert np.array_equal(Hm @ Hm.T, g * np.eye(g))


@pytest.mark.parametrize("g", GROUPS)
def test_rotation_matches_fp64_product(orc, g):
    rng = np.random.default_rng(g)
    rows, cols = 8, 4 * g
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[0, :g] *= 1e3  # one group with a large dynamic range
    seed = 12345
    z = orc.rht_rows(x, g, seed).astype(np.float64)
    H = scipy.linalg.hadamard(g).astype(np.float64)
    sigma = orc.rht_signs(seed, g).astype(np.float64)
    c = float(orc.rht_scale(g))
    for r in range(rows):
        for s in range(0, cols, g):
            xg = x[r, s:s + g].astype(np.float64)
            ref = c * (H @ (sigma * xg))
            bound = (np.log2(g) + 2) * 2.0 ** -24 * c * np.abs(xg).sum()
            assert np.max(np.abs(z[r, s:s + g] - ref)) <= bound


@pytest.mark.parametrize("g", [16, 64])
def test_inverse_is_exact_on_small_integers(orc, g):
    """c_g is a power of two for g = 16, 64, so forward + inverse is exact on small integers."""
    rng = np.random.default_rng(3)
    x = rng.integers(-8, 9, size=(4, 2 * g)).astype(np.float32)
    z = orc.rht_rows(x, g, 99)
    back = orc.rht_rows(z, g, 99, inverse=True)
    assert np.array_equal(back, x)


@pytest.mark.parametrize("g", GROUPS)
def test_inverse_and_norm(orc, g):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((16, 2 * g)).astype(np.float32)
    z = orc.rht_rows(x, g, 7)
    back = orc.rht_rows(z, g, 7, inverse=True)
    assert np.max(np.abs(back - x)) <= 4 * np.log2(g) * 2.0 ** -24 * np.abs(x).max() * np.sqrt(g)
    n0 = np.linalg.norm(x.astype(np.float64), axis=1)
    n1 = np.linalg.norm(z.astype(np.float64), axis=1)
    assert np.allclose(n0, n1, rtol=4e-6)


def test_rotation_spreads_an_outlier(orc):
    """A single spike spreads to equal magnitudes across its group (the outlier-spreading role)."""
    x = np.zeros((1, 128), dtype=np.float32)
    x[0, 17] = 64.0
    z = orc.rht_rows(x, 128, 1)
    assert np.allclose(np.abs(z), 64.0 * orc.rht_scale(128))


def test_view_rotation_transposed_equals_rowwise_of_transpose(orc):
    rng = np.random.default_rng(8)
    import torch
    x = torch.from_numpy(rng.standard_normal((256, 48)).astype(np.float32)).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    bits_t = x.t().contiguous().view(torch.int16).numpy().view(np.uint16)
    zt = orc.rht_view(bits, 1, 128, 5)
    zr = orc.rht_view(bits_t, 0, 128, 5)
    assert np.array_equal(zt, zr)

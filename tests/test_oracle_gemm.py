"""Pins of the oracle's NVFP4 GEMM against what the pages and arithmetic fix.

- brute force in exact rational arithmetic on a tiny case, with E2M1 values
  from the value set of the palettes post ("Comparing INT4 and NVFP4 Palettes
  on Real Gradient Tensors", opening section) and E4M3 values decoded by
  torch's float8_e4m3fn (a decoder independent of the oracle's);
- a lossless round trip: inputs on the E2M1 grid under power-of-two scales
  quantize (RTN) without error, so the GEMM of their quantizations is X W^T
  exactly, computed here by numpy from X and W themselves;
- operand-order invariants: swapping A and B transposes D, scaling one tensor
  scale by 2 scales D by 2;
- operands rotated with the same seed multiply to X W^T within the
  quantization error; with different seeds they do not.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import workloads as W

E2M1_MAG = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
            Fraction(6)]


def e2m1_value(code):
    v = E2M1_MAG[code & 7]
    return -v if code & 8 else v


def e4m3_value(code):
    t = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    return Fraction(float(t.item()))


def test_gemm_brute_force_tiny():
    m, n, k = 3, 2, 64
    ac, asc = W.gemm_operand(m, k, 11)
    bc, bsc = W.gemm_operand(n, k, 12)
    ac, asc, bc, bsc = (t.numpy() for t in (ac, asc, bc, bsc))
    ga, gb = np.float32(0.75), np.float32(2.0 ** -7)
    got = oracle.gemm(ac, asc, ga, bc, bsc, gb)
    gab = Fraction(float(np.float32(ga * gb)))
    for i in range(m):
        for j in range(n):
            s = Fraction(0)
            for kk in range(k):
                qa = e2m1_value((int(ac[i, kk // 2]) >> (4 * (kk & 1))) & 15)
                qb = e2m1_value((int(bc[j, kk // 2]) >> (4 * (kk & 1))) & 15)
                s += qa * e4m3_value(int(asc[i, kk // 16])) * qb * e4m3_value(int(bsc[j, kk // 16]))
            assert got[i, j] == float(s * gab), (i, j)


def _grid_tensor(rows, k, rng, s_exp):
    """Values on the E2M1 grid times a per-block E4M3 power of two times 2^s_exp,
    with one block per tensor holding 6 * 448 * 2^s_exp (so the tensor scale is
    exactly 2^s_exp) and every block holding a +-6 (so each block scale is
    exactly its power of two)."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mag = grid[rng.integers(0, 8, (rows, k))]
    sign = np.where(rng.random((rows, k)) < 0.5, -1.0, 1.0)
    v = (mag * sign).reshape(rows, k // 16, 16)
    v[:, :, 0] = 6.0 * np.where(rng.random((rows, k // 16)) < 0.5, -1.0, 1.0)
    e = rng.integers(-6, 8, (rows, k // 16)).astype(np.float64)
    e[0, 0] = np.log2(448.0 / 1.75)  # 448 = 1.75 * 2^8: the block holding the tensor maximum
    blk = np.where(e == e[0, 0], 448.0, 2.0 ** e)
    x = v * blk[:, :, None] * 2.0 ** s_exp
    return x.reshape(rows, k)


def test_gemm_lossless_round_trip_is_exact_product():
    rng = np.random.default_rng(5)
    m, n, k = 32, 48, 256
    x = _grid_tensor(m, k, rng, -12)
    w = _grid_tensor(n, k, rng, -10)
    xb = W.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    wb = W.bf16_bits(torch.from_numpy(w).to(torch.bfloat16))
    assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).double().numpy(), x)  # bf16-exact inputs
    qa = oracle.quantize(xb, oracle.ROWWISE, oracle.RTN, 0, 0)
    qb = oracle.quantize(wb, oracle.ROWWISE, oracle.RTN, 0, 0)
    assert qa[2] == 2.0 ** -12 and qb[2] == 2.0 ** -10
    assert np.array_equal(oracle.dequantize(*qa, oracle.RTN, 0, 0).astype(np.float64), x)
    got = oracle.gemm(*qa, *qb)
    assert np.array_equal(got, x @ w.T)


def test_gemm_operand_swap_and_scale():
    m, n, k = 16, 24, 512
    ac, asc = (t.numpy() for t in W.gemm_operand(m, k, 21))
    bc, bsc = (t.numpy() for t in W.gemm_operand(n, k, 22))
    d = oracle.gemm(ac, asc, 1.0, bc, bsc, 1.0)
    assert np.array_equal(oracle.gemm(bc, bsc, 1.0, ac, asc, 1.0), d.T)
    assert np.array_equal(oracle.gemm(ac, asc, 2.0, bc, bsc, 1.0), 2.0 * d)
    rows = [3, 0, 7]
    assert np.array_equal(oracle.gemm(ac, asc, 1.0, bc, bsc, 1.0, a_rows=rows), d[rows])


def test_gemm_rejects_if4_scales():
    ac, asc = (t.numpy() for t in W.gemm_operand(4, 32, 1))
    asc = asc.copy()
    asc[0, 0] |= 0x80
    with pytest.raises(ValueError):
        oracle.gemm(ac, asc, 1.0, ac, asc, 1.0)


def test_gemm_of_rotated_operands_cancels_the_rotation():
    """Two operands rotated along k with the same seed (one sign vector shared
    by every group and both operands) multiply to X W^T up to the quantization
    error, because c_g H_g diag(sigma) is orthogonal up to the rounding of c_g
    (Quartet II article, "Quantisierung im Vorwaertsdurchlauf": rotations
    along the microscaling groups; the shared sign vector is the reading that
    makes them cancel).  With different seeds the rotations do not cancel and
    the product is unrelated to X W^T."""
    gen = torch.Generator().manual_seed(3)
    x = torch.randn(128, 1024, generator=gen).to(torch.bfloat16)
    w = (torch.randn(96, 1024, generator=gen) * 0.02).to(torch.bfloat16)
    exact = x.double().numpy() @ w.double().numpy().T
    xb, wb = W.bf16_bits(x), W.bf16_bits(w)

    def rel(seed_x, seed_w, mode, g):
        qa = oracle.quantize(xb, oracle.ROWWISE, mode, g, seed_x)
        qb = oracle.quantize(wb, oracle.ROWWISE, mode, g, seed_w)
        d = oracle.gemm(*qa, *qb)
        return np.linalg.norm(d - exact) / np.linalg.norm(exact)

    plain = rel(5, 5, oracle.RTN, 0)
    same = rel(5, 5, oracle.MS_EDEN, 128)
    other = rel(5, 6, oracle.MS_EDEN, 128)
    print(f"\nrelative Frobenius error of the GEMM: RTN {plain:.4f}, MS-EDEN same seed {same:.4f}, "
          f"different seeds {other:.3f}")
    # each operand carries ~9.5% relative RMS quantization error (NVFP4 MSE
    # 9e-3 per unit variance), so a dot product of two carries ~sqrt(2) x 9.5%
    assert plain < 0.2 and same < 1.2 * plain
    assert other > 0.9

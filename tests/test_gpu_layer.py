"""The fully-NVFP4 linear layer assembled from the library's calls, as bench.py
times it: X [T, d_in], W [d_out, d_in], dY [T, d_out], each quantized in both
layouts from one read (nvfp4_amax_dual + nvfp4_quantize_dual: RTN row-wise +
MS-EDEN transposed for X and W, MS-EDEN both ways for dY, one seed, 128-point
rotations), then Y = X W^T, dX = dY W, dW = dY^T X on the block-scaled tensor
cores (nvfp4_gemm).

Each GEMM equals the oracle GEMM of the same quantized operands within the
GEMM tolerance (the oracle sums exactly), and each output is the exact product
of the unquantized tensors up to the quantization error: the backward GEMMs
pair operands rotated along their reduction dimension with the same signs, so
the rotations cancel (Quartet II article, sections "Quantisierung im
Vorwaertsdurchlauf" and "... Rueckwaertsdurchlauf")."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

pytestmark = pytest.mark.gpu

GEMM_TOL = 2.0 ** -12


def _np(t):
    return t.cpu().numpy()


def _check_gemm(d, a, b):
    (ac, asc, ag), (bc, bsc, bg) = a, b
    ref = oracle.gemm(_np(ac), _np(asc), float(ag.item()), _np(bc), _np(bsc), float(bg.item()))
    ai = np.abs(oracle._gemm_operand_ints(_np(ac), _np(asc))).astype(np.float64)
    bi = np.abs(oracle._gemm_operand_ints(_np(bc), _np(bsc))).astype(np.float64)
    gab = float(np.float32(np.float32(ag.item()) * np.float32(bg.item())))
    l1 = (ai @ bi.T) * 2.0 ** -20 * gab
    got = d.float().cpu().numpy().astype(np.float64)
    # bf16 output: the fp32 result within the tolerance, then one bf16 rounding
    assert np.all(np.abs(got - ref) <= GEMM_TOL * l1 + 2.0 ** -8 * np.abs(ref) + 1e-30)
    return got


@pytest.mark.parametrize("tokens,d_in,d_out", [(1024, 512, 768), (2048, 1024, 512)])
def test_linear_layer(tokens, d_in, d_out):
    g = torch.Generator().manual_seed(tokens + d_in + d_out)
    x = torch.randn(tokens, d_in, generator=g).to(torch.bfloat16).cuda()
    w = (torch.randn(d_out, d_in, generator=g) * 0.02).to(torch.bfloat16).cuda()
    dy = (torch.randn(tokens, d_out, generator=g) * 1e-3).to(torch.bfloat16).cuda()
    seed, grp = 21, 128
    xr, xc = N.quantize_dual(x, W.RTN, 0, W.MS_EDEN, grp, seed)
    wr, wc = N.quantize_dual(w, W.RTN, 0, W.MS_EDEN, grp, seed)
    dyr, dyc = N.quantize_dual(dy, W.MS_EDEN, grp, W.MS_EDEN, grp, seed)
    y = N.gemm(xr, wr, torch.bfloat16)
    dx = N.gemm(dyr, wc, torch.bfloat16)
    dw = N.gemm(dyc, xc, torch.bfloat16)
    torch.cuda.synchronize()
    assert y.shape == (tokens, d_out) and dx.shape == (tokens, d_in) and dw.shape == (d_out, d_in)
    got = {"Y": _check_gemm(y, xr, wr), "dX": _check_gemm(dx, dyr, wc), "dW": _check_gemm(dw, dyc, xc)}
    xf, wf, dyf = (t.double().cpu().numpy() for t in (x, w, dy))
    exact = {"Y": xf @ wf.T, "dX": dyf @ wf, "dW": dyf.T @ xf}
    for name in got:
        rel = np.linalg.norm(got[name] - exact[name]) / np.linalg.norm(exact[name])
        # NVFP4 quantization of both operands: ~0.1 relative error; a rotation
        # that did not cancel would give ~1.4
        assert rel < 0.3, (name, rel)

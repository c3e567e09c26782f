"""GPU parity of the NVFP4 GEMM (nvfp4_gemm through the C ABI) against the
oracle GEMM, which sums the products exactly.

Exact cases: operands whose partial sums are all multiples of 2^-4 below 2^20
(E4M3 scales that are powers of two in [1/2, 4] with k = 512, or every scale
1 with k = 4096, tensor scales powers of two): fp32 accumulation is exact in
any order, so D must equal the oracle's bit for bit.  They pin the operand
layout and swizzle, the order along K, the placement of every scale factor,
the tile loop and the output layout.

General cases (any finite scales): the tensor cores accumulate in fp32 in an
order of their own, so |D - D_oracle| <= GEMM_TOL * RN(gA gB) * sum_k |terms|
per output; the largest normalized error seen is printed.

End to end: X and W quantized on the GPU, their GEMM against the oracle GEMM
of the oracle's own quantization of the same inputs (the codes of the two
quantizations are compared first).  At the full size of the MLP up-projection
step (Y = X W^T, 16384 x 14336 x 4096, bf16 output as bench.py times it),
sampled rows and columns of D against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import bits

pytestmark = pytest.mark.gpu

GEMM_TOL = 2.0 ** -12
POW2_SCALES = [0x30, 0x38, 0x40, 0x48]  # E4M3 0.5, 1, 2, 4
ONE = [0x38]


def _operand(rows, k, seed, scale_codes=None):
    c, s = W.gemm_operand(rows, k, seed, scale_codes)
    return c, s


def _dev(arr):
    return torch.from_numpy(np.ascontiguousarray(arr)).to("cuda")


def _gpu_gemm(a, b, ga, gb, out_dtype=torch.float32):
    """a, b: (codes, scales) numpy operands; D on the GPU, returned as float64 numpy."""
    ta = (_dev(a[0]), _dev(a[1]), torch.tensor([ga], dtype=torch.float32, device="cuda"))
    tb = (_dev(b[0]), _dev(b[1]), torch.tensor([gb], dtype=torch.float32, device="cuda"))
    d = N.gemm(ta, tb, out_dtype)
    torch.cuda.synchronize()
    return d.float().cpu().numpy().astype(np.float64)


def _l1(a, b, ga, gb, a_rows=None, b_rows=None):
    """RN(gA gB) * sum_k |terms| per output, from the oracle's exact operand values."""
    ai = np.abs(oracle._gemm_operand_ints(a[0], a[1], a_rows)).astype(np.float64)
    bi = np.abs(oracle._gemm_operand_ints(b[0], b[1], b_rows)).astype(np.float64)
    return (ai @ bi.T) * 2.0 ** -20 * float(np.float32(np.float32(ga) * np.float32(gb)))


WORST = [0.0]


def _check_tol(got, ref, l1, tol=GEMM_TOL):
    err = np.abs(got - ref) / np.maximum(l1, np.finfo(np.float64).tiny)
    WORST[0] = max(WORST[0], float(err.max()))
    print(f"max |D - D_oracle| / (gab sum |terms|) = {err.max():.3e}")
    assert err.max() <= tol, err.max()


@pytest.mark.parametrize("m,n,k,scales,seed", [
    (128, 128, 512, POW2_SCALES, 1),      # one tile
    (256, 384, 512, POW2_SCALES, 2),      # 2 x 3 tiles
    (128, 256, 4096, ONE, 3),             # 16 K tiles: the stage ring wraps
    (2048, 2560, 512, POW2_SCALES, 4),    # 320 tiles: more than one per CTA, both accumulators
])
def test_gemm_exact_cases(m, n, k, scales, seed):
    a = tuple(t.numpy() for t in _operand(m, k, 100 + seed, scales))
    b = tuple(t.numpy() for t in _operand(n, k, 200 + seed, scales))
    ga, gb = 2.0 ** -3, 2.0 ** 5
    ref = oracle.gemm(a[0], a[1], ga, b[0], b[1], gb)
    got = _gpu_gemm(a, b, ga, gb)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]


@pytest.mark.parametrize("m,n,k,seed", [(128, 128, 256, 5), (384, 256, 2048, 6), (1024, 1152, 1024, 7)])
def test_gemm_general_scales(m, n, k, seed):
    a = tuple(t.numpy() for t in _operand(m, k, 300 + seed))
    b = tuple(t.numpy() for t in _operand(n, k, 400 + seed))
    ga, gb = 0.0123, 3.5
    ref = oracle.gemm(a[0], a[1], ga, b[0], b[1], gb)
    got = _gpu_gemm(a, b, ga, gb)
    _check_tol(got, ref, _l1(a, b, ga, gb))


def test_gemm_bf16_output():
    m, n, k = 256, 256, 1024
    a = tuple(t.numpy() for t in _operand(m, k, 501))
    b = tuple(t.numpy() for t in _operand(n, k, 502))
    ref = oracle.gemm(a[0], a[1], 1.0, b[0], b[1], 1.0)
    got = _gpu_gemm(a, b, 1.0, 1.0, torch.bfloat16)
    # the fp32 result within the tolerance, then one bf16 rounding (half an ulp, 2^-9 relative)
    l1 = _l1(a, b, 1.0, 1.0)
    assert np.all(np.abs(got - ref) <= GEMM_TOL * l1 + 2.0 ** -8 * np.abs(ref) + 1e-30)


# Output row pitches: 32-byte aligned rows take the 32-byte store path, rows
# aligned to 16 bytes only take the 16-byte one.
@pytest.mark.parametrize("dtype,extra", [(torch.float32, 64), (torch.float32, 4), (torch.bfloat16, 8)])
def test_gemm_output_row_stride(dtype, extra):
    m, n, k = 128, 256, 512
    a = tuple(t.to("cuda") for t in _operand(m, k, 601, POW2_SCALES))
    b = tuple(t.to("cuda") for t in _operand(n, k, 602, POW2_SCALES))
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    big = torch.full((m, n + extra), 7.0, dtype=dtype, device="cuda")
    N.gemm((a[0], a[1], one), (b[0], b[1], one), out=big[:, :n])
    torch.cuda.synchronize()
    ref = oracle.gemm(a[0].cpu().numpy(), a[1].cpu().numpy(), 1.0, b[0].cpu().numpy(), b[1].cpu().numpy(), 1.0)
    # exact in fp32 (power-of-two scales); bf16 D is that value rounded to nearest even
    want = torch.from_numpy(ref.astype(np.float32)).to(dtype).float().numpy().astype(np.float64)
    assert np.array_equal(big[:, :n].float().cpu().numpy().astype(np.float64), want)
    assert torch.all(big[:, n:] == 7.0)  # columns past n untouched


@pytest.mark.parametrize("mode,g", [(W.RTN, 0), (W.FOUR_OVER_SIX, 0), (W.MS_EDEN, 128)])
def test_gemm_of_quantized_tensors(mode, g):
    """Y = X W^T from X (256 x 1024) and W (384 x 1024) quantized along k."""
    gen = torch.Generator().manual_seed(77)
    x = (torch.randn(256, 1024, generator=gen)).to(torch.bfloat16)
    w = (torch.randn(384, 1024, generator=gen) * 0.02).to(torch.bfloat16)
    seed = 9
    qa = N.quantize(x.cuda(), W.ROWWISE, mode, g, seed)
    qb = N.quantize(w.cuda(), W.ROWWISE, mode, g, seed)
    d = N.gemm(qa, qb)
    torch.cuda.synchronize()
    oa = oracle.quantize(bits(x), W.ROWWISE, mode, g, seed)
    ob = oracle.quantize(bits(w), W.ROWWISE, mode, g, seed)
    assert np.array_equal(qa[0].cpu().numpy(), oa[0]) and np.array_equal(qa[1].cpu().numpy(), oa[1])
    assert np.array_equal(qb[0].cpu().numpy(), ob[0]) and np.array_equal(qb[1].cpu().numpy(), ob[1])
    ref = oracle.gemm(*oa, *ob)
    _check_tol(d.cpu().numpy().astype(np.float64), ref, _l1((oa[0], oa[1]), (ob[0], ob[1]), oa[2], ob[2]))


def test_gemm_full_size_forward_sampled():
    """Y = X W^T of the MLP up-projection step: X 16384 x 4096 N(0,1), W 14336 x
    4096 N(0, 0.02^2), both RTN row-wise, bf16 output; 24 x 24 sampled outputs."""
    wl = W.mlp_up()
    t = wl.tensors(device="cuda")
    x, w = t["x"], t["w"]
    qa = N.quantize(x, W.ROWWISE, W.RTN, 0, wl.seed)
    qb = N.quantize(w, W.ROWWISE, W.RTN, 0, wl.seed)
    d = N.gemm(qa, qb, torch.bfloat16)
    torch.cuda.synchronize()
    rng = np.random.default_rng(2024)
    ra = np.unique(np.concatenate([[0, x.shape[0] - 1], rng.integers(0, x.shape[0], 22)]))
    rb = np.unique(np.concatenate([[0, w.shape[0] - 1], rng.integers(0, w.shape[0], 22)]))
    xb, wb = bits(x.cpu()), bits(w.cpu())
    ax = oracle.amax(xb, W.ROWWISE, 0, wl.seed)
    aw = oracle.amax(wb, W.ROWWISE, 0, wl.seed)
    oa = [oracle.quantize(xb[r:r + 1], W.ROWWISE, W.RTN, 0, wl.seed, amax_in=ax) for r in ra]
    ob = [oracle.quantize(wb[r:r + 1], W.ROWWISE, W.RTN, 0, wl.seed, amax_in=aw) for r in rb]
    ac, asc = np.concatenate([o[0] for o in oa]), np.concatenate([o[1] for o in oa])
    bc, bsc = np.concatenate([o[0] for o in ob]), np.concatenate([o[1] for o in ob])
    assert np.array_equal(qa[0][torch.from_numpy(ra).cuda()].cpu().numpy(), ac)
    assert np.array_equal(qb[0][torch.from_numpy(rb).cuda()].cpu().numpy(), bc)
    ga, gb = oa[0][2], ob[0][2]
    ref = oracle.gemm(ac, asc, ga, bc, bsc, gb)
    got = d[torch.from_numpy(ra).cuda()][:, torch.from_numpy(rb).cuda()].float().cpu().numpy().astype(np.float64)
    l1 = _l1((ac, asc), (bc, bsc), ga, gb)
    err = np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)
    assert np.all(err <= GEMM_TOL * l1), (err / l1).max()

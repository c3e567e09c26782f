"""nvfp4_quantize_dual: both layouts from one read, through the C ABI.

Its outputs must equal, bit for bit, those of the two single-layout
nvfp4_quantize calls given the same tensor amaxes (the single-layout calls are
themselves parity-tested against the oracle), on the mode pairs the fused
kernel takes (RTN row-wise without rotation + MS-EDEN transposed, MS-EDEN both
ways; every rotation group), on ragged shapes, padded rows and tensors with
several tiles per CTA; the other pairs run as two single launches and must
match too.  On the 256x256 workload the fused outputs are also compared with
the oracle directly."""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import assert_same, bits, to_device

pytestmark = pytest.mark.gpu


def _host(t):
    return t[0].cpu().numpy(), t[1].cpu().numpy(), float(t[2].item())


def _dual_vs_single(x, mode_r, g_r, mode_c, g_c, seed):
    a_r, a_c = N.amax_dual(x, g_r, g_c, seed)
    row, col = N.quantize_dual(x, mode_r, g_r, mode_c, g_c, seed, amax_row=a_r, amax_col=a_c)
    srow = N.quantize(x, W.ROWWISE, mode_r, g_r, seed, amax_in=a_r)
    scol = N.quantize(x, W.TRANSPOSED, mode_c, g_c, seed, amax_in=a_c)
    torch.cuda.synchronize()
    what = f"shape={tuple(x.shape)} ld={x.stride(0)} row=({mode_r},{g_r}) col=({mode_c},{g_c})"
    assert_same(_host(row), _host(srow), what + " row-wise")
    assert_same(_host(col), _host(scol), what + " transposed")
    return row, col


FUSED = [(W.RTN, 0, W.MS_EDEN, g) for g in (16, 32, 64, 128)] + [(W.MS_EDEN, g, W.MS_EDEN, g) for g in (16, 32, 64, 128)]


@pytest.mark.parametrize("mode_r,g_r,mode_c,g_c", FUSED)
@pytest.mark.parametrize("shape,pad", [((256, 256), 0), ((384, 640), 0), ((512, 384), 8), ((4096, 4096), 0)])
def test_dual_equals_single(mode_r, g_r, mode_c, g_c, shape, pad):
    rows, cols = shape
    g = torch.Generator().manual_seed(rows * 7 + cols + g_c)
    x = to_device((torch.randn(rows, cols, generator=g) * 0.3).to(torch.bfloat16), pad)
    _dual_vs_single(x, mode_r, g_r, mode_c, g_c, seed=1234 + g_c)


@pytest.mark.parametrize("mode_r,g_r,mode_c,g_c", [(W.RTN, 0, W.MS_EDEN, 16), (W.MS_EDEN, 16, W.MS_EDEN, 16)])
def test_dual_ragged_tiles(mode_r, g_r, mode_c, g_c):
    # rows and cols not multiples of the 128 x 128 tile: partial tiles at both edges
    g = torch.Generator().manual_seed(5)
    x = to_device((torch.randn(400, 272, generator=g) * 2.0).to(torch.bfloat16))
    _dual_vs_single(x, mode_r, g_r, mode_c, g_c, seed=77)


@pytest.mark.parametrize("mode_r,g_r,mode_c,g_c", [(W.SR, 128, W.IF4, 0), (W.RTN, 0, W.RTN, 0),
                                                   (W.MS_EDEN, 64, W.MS_EDEN, 128), (W.MXFP4, 0, W.MXFP4, 32)])
def test_dual_other_pairs(mode_r, g_r, mode_c, g_c):
    g = torch.Generator().manual_seed(9)
    x = to_device(torch.randn(256, 384, generator=g).to(torch.bfloat16))
    _dual_vs_single(x, mode_r, g_r, mode_c, g_c, seed=3)


def test_dual_small_tensor_falls_back():
    g = torch.Generator().manual_seed(2)
    x = to_device(torch.randn(64, 96, generator=g).to(torch.bfloat16))
    _dual_vs_single(x, W.RTN, 0, W.MS_EDEN, 16, seed=8)


def test_dual_against_oracle():
    wl = W.small()
    x_cpu = wl.tensors()["x"]
    xb = bits(x_cpu)
    x = x_cpu.cuda()
    seed = wl.seed
    for mode_r, g_r, mode_c, g_c in [(W.RTN, 0, W.MS_EDEN, 128), (W.MS_EDEN, 128, W.MS_EDEN, 128)]:
        a_r, a_c = N.amax_dual(x, g_r, g_c, seed)
        row, col = N.quantize_dual(x, mode_r, g_r, mode_c, g_c, seed, amax_row=a_r, amax_col=a_c)
        torch.cuda.synchronize()
        for layout, mode, grp, out, a in ((W.ROWWISE, mode_r, g_r, row, a_r), (W.TRANSPOSED, mode_c, g_c, col, a_c)):
            got = _host(out)
            if grp == 0:
                exp = oracle.quantize(xb, layout, mode, grp, seed)
            else:
                z = N.rht(x, layout, grp, seed).cpu().numpy()
                exp = oracle.quantize_rotated(z, mode, seed, a.item())
            assert_same(got, exp, f"layout={layout} mode={mode} g={grp}")


def test_dual_empty():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    a = torch.zeros(1, dtype=torch.float32, device="cuda")
    row, col = N.quantize_dual(x, W.RTN, 0, W.MS_EDEN, 128, 0, amax_row=a, amax_col=a)
    torch.cuda.synchronize()
    assert row[0].numel() == 0 and col[0].numel() == 0
    assert float(row[2].item()) == 1.0 and float(col[2].item()) == 1.0


# ---------------------------------------------------------------- groups
def _f32bits(t):
    return t.detach().cpu().numpy().astype(np.float32).view(np.uint32)


def _members(shapes, seed, pad=0):
    g = torch.Generator().manual_seed(seed)
    return [to_device((torch.randn(r, c, generator=g) * (0.1 + i)).to(torch.bfloat16), pad if i % 2 else 0)
            for i, (r, c) in enumerate(shapes)]


# Members of different shapes (ragged tiles, a padded row pitch, one too small
# for the fused kernel, one empty), more of them than one launch takes.
GROUP_SHAPES = [(384, 256), (256, 640), (400, 272), (64, 96), (0, 128), (512, 384)]


@pytest.mark.parametrize("g_r,g_c", [(0, 128), (0, 16), (128, 128)])
def test_amax_dual_group_equals_single_calls(g_r, g_c):
    shapes = [(r, c) for r, c in GROUP_SHAPES if (r % g_c == 0 or r == 0) and (g_r == 0 or c % g_r == 0)]
    xs = _members(shapes, 11, pad=8)
    got = N.amax_dual_group(xs, g_r, g_c, seed=5)
    for x, (ar, ac) in zip(xs, got):
        wr, wc = N.amax_dual(x, g_r, g_c, seed=5)
        torch.cuda.synchronize()
        what = f"shape={tuple(x.shape)} groups=({g_r},{g_c})"
        assert np.array_equal(_f32bits(ar), _f32bits(wr)), what + " row view"
        assert np.array_equal(_f32bits(ac), _f32bits(wc)), what + " column view"


@pytest.mark.parametrize("mode_r,g_r,mode_c,g_c", [(W.RTN, 0, W.MS_EDEN, 128), (W.MS_EDEN, 128, W.MS_EDEN, 128),
                                                   (W.RTN, 0, W.MS_EDEN, 16), (W.SR, 0, W.IF4, 0)])
def test_quantize_dual_group_equals_single_calls(mode_r, g_r, mode_c, g_c):
    gc = g_c if g_c else 16
    shapes = [(r, c) for r, c in GROUP_SHAPES if (r % gc == 0 or r == 0) and (g_r == 0 or c % g_r == 0)]
    xs = _members(shapes, 12, pad=8)
    amaxes = N.amax_dual_group(xs, g_r, g_c, seed=6)
    outs = N.quantize_dual_group(xs, mode_r, g_r, mode_c, g_c, seed=6, amaxes=amaxes)
    for x, (ar, ac), (row, col) in zip(xs, amaxes, outs):
        wrow, wcol = N.quantize_dual(x, mode_r, g_r, mode_c, g_c, seed=6, amax_row=ar, amax_col=ac)
        torch.cuda.synchronize()
        what = f"shape={tuple(x.shape)} row=({mode_r},{g_r}) col=({mode_c},{g_c})"
        assert_same(_host(row), _host(wrow), what + " row-wise")
        assert_same(_host(col), _host(wcol), what + " transposed")


def test_group_of_the_mlp_forward_operands():
    """X and W of the MLP up-projection workload in one group: the step's
    forward pair, at full size."""
    wl = W.mlp_up()
    t = wl.tensors(torch.device("cuda"))
    xs = [t["x"], t["w"]]
    amaxes = N.amax_dual_group(xs, 0, 128, wl.seed)
    outs = N.quantize_dual_group(xs, W.RTN, 0, W.MS_EDEN, 128, wl.seed, amaxes=amaxes)
    for x, (ar, ac), (row, col) in zip(xs, amaxes, outs):
        wr, wc = N.amax_dual(x, 0, 128, wl.seed)
        wrow, wcol = N.quantize_dual(x, W.RTN, 0, W.MS_EDEN, 128, wl.seed, amax_row=wr, amax_col=wc)
        torch.cuda.synchronize()
        assert np.array_equal(_f32bits(ar), _f32bits(wr)) and np.array_equal(_f32bits(ac), _f32bits(wc))
        for got, want in ((row, wrow), (col, wcol)):
            assert torch.equal(got[0], want[0]) and torch.equal(got[1], want[1])
            assert np.array_equal(_f32bits(got[2]), _f32bits(want[2]))

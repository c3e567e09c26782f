"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (the same C-ABI call on the same shapes), on sampled output rows.  The
tensors are drawn on the GPU and copied to the host for the oracle.

For each call the oracle computes the tensor amax over the whole tensor, then
only the sampled view rows (the first, the last and randomly drawn ones).

Without the rotation the GPU's rows must equal the oracle's bit for bit, and
so must the FP32 tensor scale.  With the rotation the four-part comparison of
gpu_helpers is applied to the sampled rows: the rotated values within the
tolerance, the GPU pre-pass amax equal to max |z| of the GPU's own rotation
(over the whole tensor) and within the tolerance of the oracle's, the sampled
rows of the GPU's quantization bit-exact against the oracle quantizing the
GPU's own rotated rows, and the end-to-end difference (both sides given the
oracle's amax) confined to blocks with differing rotated values and at most
1e-5 of the sampled outputs.
"""
import zlib

import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import ROT_TOL, assert_same, bits, check_rotation, end_to_end_mismatch, record_mismatch

pytestmark = pytest.mark.gpu

N_SAMPLED_ROWS = 12


def _view_row_bits(xb, layout, r):
    """bf16 patterns whose (single-row) view is view row r of the full tensor."""
    return xb[r:r + 1] if layout == W.ROWWISE else np.ascontiguousarray(xb[:, r:r + 1])


def _check_call(wl, call, x, xb):
    rows, cols = x.shape
    vr, vc = N.view_shape(rows, cols, call.layout)
    g, seed, mode, layout = call.rht_group, wl.seed, call.mode, call.layout
    rng = np.random.default_rng(zlib.crc32(call.name.encode()))
    sample = sorted(set([0, vr - 1] + list(rng.integers(0, vr, N_SAMPLED_ROWS - 2))))
    a_orc = oracle.amax(xb, layout, g, seed)

    codes, scales, gs = N.quantize(x, layout, mode, g, seed)
    torch.cuda.synchronize()
    codes_h, scales_h, gs_h = codes.cpu().numpy(), scales.cpu().numpy(), float(gs.item())
    del codes, scales, gs

    if g == 0:
        assert gs_h == oracle.global_scale(a_orc, mode), call.name
        for r in sample:
            oc, osc, _ = oracle.quantize(xb, layout, mode, g, seed, amax_in=a_orc, row_range=(r, r + 1))
            assert np.array_equal(codes_h[r], oc[r]), (call.name, r, int(np.sum(codes_h[r] != oc[r])))
            assert np.array_equal(scales_h[r], osc[r]), (call.name, r, int(np.sum(scales_h[r] != osc[r])))
        return

    z = N.rht(x, layout, g, seed)
    a_gpu = N.amax(x, layout, g, seed).item()
    a_own = z.abs().max().item()
    z_rows = z[sample].cpu().numpy()
    del z
    assert a_gpu == a_own, (call.name, a_gpu, a_own)
    assert abs(a_gpu - a_orc) <= ROT_TOL * a_orc, (call.name, a_gpu, a_orc)
    assert gs_h == oracle.global_scale(a_gpu, mode), call.name

    amax_t = torch.tensor([a_orc], dtype=torch.float32, device="cuda")
    codes_e, scales_e, gs_e = N.quantize(x, layout, mode, g, seed, amax_in=amax_t)
    torch.cuda.synchronize()
    codes_e, scales_e, gs_e = codes_e.cpu().numpy(), scales_e.cpu().numpy(), float(gs_e.item())

    n_codes_bad = n_scales_bad = 0
    for i, r in enumerate(sample):
        what = f"{call.name} view row {r}"
        zg = z_rows[i:i + 1]
        zo = oracle.rht_view(_view_row_bits(xb, layout, r), layout, g, seed)
        check_rotation(zg, zo, g, what)
        oc, osc, og = oracle.quantize_rotated(zg, mode, seed, a_gpu, row0=r)
        assert_same((codes_h[r:r + 1], scales_h[r:r + 1], gs_h), (oc, osc, og), what + " (on the GPU's rotation)")
        oc, osc, og = oracle.quantize(xb, layout, mode, g, seed, amax_in=a_orc, row_range=(r, r + 1))
        nc, ns = end_to_end_mismatch((codes_e[r:r + 1], scales_e[r:r + 1], gs_e),
                                     (oc[r:r + 1], osc[r:r + 1], og), zg, zo, what)
        n_codes_bad += nc
        n_scales_bad += ns
    record_mismatch(n_codes_bad, len(sample) * vc, n_scales_bad, len(sample) * vc // 16, call.name)


def _check_workload(wl):
    tensors = wl.tensors("cuda")
    host = {k: bits(v) for k, v in tensors.items()}
    for call in wl.calls:
        _check_call(wl, call, tensors[call.tensor], host[call.tensor])


@pytest.mark.parametrize("name", ["weight", "gradient", "activation", "mlp_up"])
def test_full_size_sampled(name):
    _check_workload(W.ALL[name]())


def test_full_size_dual_pre_pass():
    """The dual pre-pass bench.py runs (one read per tensor) gives, at the MLP
    workload's full sizes, the two single-layout tensor amaxes bit for bit."""
    wl = W.mlp_up()
    tensors = wl.tensors("cuda")
    for name in ("x", "w", "dy"):
        calls = [c for c in wl.calls if c.tensor == name]
        row = next(c for c in calls if c.layout == W.ROWWISE)
        col = next(c for c in calls if c.layout == W.TRANSPOSED)
        x = tensors[name]
        a_row, a_col = N.amax_dual(x, row.rht_group, col.rht_group, wl.seed)
        s_row = N.amax(x, W.ROWWISE, row.rht_group, wl.seed)
        s_col = N.amax(x, W.TRANSPOSED, col.rht_group, wl.seed)
        torch.cuda.synchronize()
        assert a_row.item() == s_row.item(), name
        assert a_col.item() == s_col.item(), name

"""GPU parity at the workloads' full sizes, whole tensors, in the launch
configuration bench.py times (the same C-ABI calls on the same shapes).

The tensors are drawn on the GPU and copied to the host; the oracle runs over
ranges of view rows in worker processes (oracle/pool.py), which assembles
exactly its single-process result.  For every call of the weight (4096x4096),
gradient (8192x4096), activation (16384x8192) and MLP up-projection
(X 16384x4096, W 14336x4096, dY 16384x14336) workloads, every output is
compared:

without the rotation, the GPU's codes, scales and FP32 tensor scale equal the
oracle's bit for bit (the GPU computes the tensor amax itself; it must equal
the oracle's exactly);

with the rotation, the four-part comparison of gpu_helpers over the whole
view: every rotated value within the tolerance; the GPU pre-pass amax equal
to max |z| of the GPU's own rotation and within the tolerance of the
oracle's; the GPU's codes, scales and tensor scale bit-exact against the
oracle quantizing the GPU's own rotated view; and end to end (both sides
given the oracle's amax) every differing scale group explained by the
rotation's rounding, at most 1e-5 of the codes and of the scales differing.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.pool import OraclePool
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import (MISMATCH_MAX, ROT_TOL, assert_same, bits, check_rotation, end_to_end_mismatch,
                         record_mismatch)

pytestmark = pytest.mark.gpu

CHUNK_ROWS = 2048


@pytest.fixture(scope="module")
def pool():
    with OraclePool() as p:
        yield p


def _host(t):
    return t.cpu().numpy()


def _check_call(pool, wl, call, x, xb):
    rows, cols = x.shape
    vr, vc = N.view_shape(rows, cols, call.layout)
    g, seed, mode, layout = call.rht_group, wl.seed, call.mode, call.layout
    name = call.name
    mx = mode in (W.MXFP4, W.MXFP3)
    a_orc = 0.0 if mx else pool.amax(xb, layout, g, seed)

    codes, scales, gs = N.quantize(x, layout, mode, g, seed)
    torch.cuda.synchronize()
    got = (_host(codes), _host(scales), float(gs.item()))
    del codes, scales, gs

    if g == 0:
        exp = pool.quantize(xb, layout, mode, g, seed, a_orc)
        assert_same(got, exp, name)
        return

    z_dev = N.rht(x, layout, g, seed)
    a_gpu = 0.0 if mx else N.amax(x, layout, g, seed).item()
    a_own = z_dev.abs().max().item()
    z_gpu = _host(z_dev)
    del z_dev
    if not mx:
        assert a_gpu == a_own, (name, a_gpu, a_own)
        assert abs(a_gpu - a_orc) <= ROT_TOL * a_orc, (name, a_gpu, a_orc)
    z_orc = pool.rht_view(xb, layout, g, seed)
    for r0 in range(0, vr, CHUNK_ROWS):
        check_rotation(z_gpu[r0:r0 + CHUNK_ROWS], z_orc[r0:r0 + CHUNK_ROWS], g, f"{name} rows {r0}..")

    # every step after the rotation, exactly, on the GPU's own rotated view
    assert_same(got, pool.quantize_rotated(z_gpu, mode, seed, a_gpu), name + " (on the GPU's rotation)")

    # end to end against the oracle from x, both sides given the oracle's amax
    amax_t = torch.tensor([a_orc], dtype=torch.float32, device="cuda")
    codes_e, scales_e, gs_e = N.quantize(x, layout, mode, g, seed, amax_in=None if mx else amax_t)
    torch.cuda.synchronize()
    gpu_e = (_host(codes_e), _host(scales_e), float(gs_e.item()))
    del codes_e, scales_e, gs_e
    orc_e = pool.quantize(xb, layout, mode, g, seed, a_orc)
    n_codes, n_scales = vr * vc, vr * vc // 16
    diff_codes = int((oracle.unpack_codes(gpu_e[0]) != oracle.unpack_codes(orc_e[0])).sum())
    diff_scales = int((gpu_e[1] != orc_e[1]).sum())
    assert diff_codes <= MISMATCH_MAX * n_codes and diff_scales <= MISMATCH_MAX * n_scales, \
        (name, diff_codes, diff_scales)
    nc = ns = 0
    for r0 in range(0, vr, CHUNK_ROWS):
        r1 = min(vr, r0 + CHUNK_ROWS)
        c, s = end_to_end_mismatch((gpu_e[0][r0:r1], gpu_e[1][r0:r1], gpu_e[2]),
                                   (orc_e[0][r0:r1], orc_e[1][r0:r1], orc_e[2]),
                                   z_gpu[r0:r1], z_orc[r0:r1], f"{name} rows {r0}..", mode=mode, seed=seed, row0=r0)
        nc += c
        ns += s
    record_mismatch(nc, n_codes, ns, n_scales, name)
    print(f"{name}: whole view {vr}x{vc}: {nc} of {n_codes} codes and {ns} of {n_scales} scales differ end to end")


def _check_workload(pool, wl):
    tensors = wl.tensors("cuda")
    host = {k: pool.put(bits(v)) for k, v in tensors.items()}   # each tensor written once for the workers
    for call in wl.calls:
        _check_call(pool, wl, call, tensors[call.tensor], host[call.tensor])


@pytest.mark.parametrize("name", ["weight", "gradient", "activation", "mlp_up"])
def test_full_size_whole_tensors(pool, name):
    _check_workload(pool, W.ALL[name]())


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

"""Helpers shared by the GPU parity tests: run one call through the C ABI and
through the oracle on the same seeded input, and compare element by element.

Without the rotation (g = 0) every output is compared bit for bit.

With the rotation (g > 0) the kernels may sum the Hadamard products in another
order than the oracle's butterfly (the tensor-core kernels accumulate in fp32
in hardware order), so the comparison follows the tolerance stated for the
rotated modes, in four parts:

1. rotation: every rotated value within ROT_TOL of the oracle's relative to
   its own magnitude, or within an absolute floor of ROT_FLOOR_ULPS fp32 ulps
   of the largest magnitude of its g-group (for values that are small by
   cancellation);
2. tensor amax: the GPU pre-pass equals max |z| of the GPU's own rotated view
   exactly, and the oracle's amax within ROT_TOL;
3. quantization: the GPU's codes, scales and tensor scale equal, bit for bit,
   the oracle quantizing the GPU's own rotated view (so every step after the
   rotation is pinned exactly);
4. end to end: with one tensor amax for both sides, the GPU's codes and scales
   against the oracle's from x; every differing scale group must be explained
   by the rotation's rounding (one of the oracle's decisions in it lies within
   the bound propagated from the group's |z_gpu - z_orc| of a threshold:
   decision_margins), and the differing fraction of codes and of scales must
   be at most MISMATCH_MAX.  The counts are accumulated and printed at the end
   of the session.
"""
import numpy as np
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

ROT_TOL = 1e-5
MISMATCH_MAX = 1e-5

# end-to-end differences of the rotated modes: [codes differing, codes, scales differing, scales]
ROTATED_MISMATCH = [0, 0, 0, 0]


def bits(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits(t.cpu())


def to_device(x_cpu: torch.Tensor, ld_pad: int = 0) -> torch.Tensor:
    """Copy a bf16 CPU matrix to the GPU, optionally inside a wider (ld = cols + pad) buffer."""
    rows, cols = x_cpu.shape
    if ld_pad == 0:
        return x_cpu.cuda()
    buf = torch.zeros((rows, cols + ld_pad), dtype=torch.bfloat16, device="cuda")
    buf[:, :cols] = x_cpu.cuda()
    return buf[:, :cols]


def gpu_quantize(x_dev, layout, mode, g, seed, amax=None):
    amax_t = None if amax is None else torch.tensor([amax], dtype=torch.float32, device="cuda")
    codes, scales, gs = N.quantize(x_dev, layout, mode, g, seed, amax_in=amax_t)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), float(gs.item())


def mismatch_report(name, got, exp):
    bad = np.argwhere(got != exp)
    if len(bad) == 0:
        return ""
    i = tuple(bad[0])
    return f"{name}: {len(bad)} of {got.size} differ, first at {i}: got {got[i]:#x} expected {exp[i]:#x}"


def assert_same(gpu, orc, what=""):
    gc, gsc, gg = gpu
    oc, osc, og = orc
    msgs = [m for m in (mismatch_report("codes", gc, oc), mismatch_report("scales", gsc, osc)) if m]
    if gg != og and not (np.isnan(gg) and np.isnan(og)):
        msgs.append(f"global scale {gg!r} vs {og!r}")
    assert not msgs, what + ": " + "; ".join(msgs)


ROT_FLOOR_ULPS = 32
# the largest rotation difference seen, in ulps of the group maximum and as a
# fraction of the value itself (values above the floor): [ulps, relative]
ROTATION_WORST = [0.0, 0.0]


def check_rotation(z_gpu, z_orc, g, what=""):
    """Every rotated value within ROT_TOL of its own magnitude, or within an
    absolute floor of ROT_FLOOR_ULPS ulps of its g-group's largest magnitude.

    The floor covers values that are small because of cancellation: the
    oracle's butterfly and the tensor cores sum the same g exact products
    (bf16 x +-1) in different orders in fp32, and each rounding is relative to
    a partial sum, which can be as large as the group's largest value."""
    assert z_gpu.shape == z_orc.shape, what
    if z_gpu.size == 0:
        return
    vr, vc = z_orc.shape
    zo = z_orc.astype(np.float64).reshape(vr, vc // g, g)
    diff = np.abs(z_gpu.astype(np.float64).reshape(vr, vc // g, g) - zo)
    gmax = np.abs(zo).max(axis=2, keepdims=True)
    ulp = np.spacing(gmax.astype(np.float32)).astype(np.float64)  # one fp32 ulp of the group maximum
    floor = ROT_FLOOR_ULPS * ulp
    bad = diff > np.maximum(ROT_TOL * np.abs(zo), floor)
    nz = gmax > 0
    if nz.any():
        ROTATION_WORST[0] = max(ROTATION_WORST[0], float((diff / np.where(nz, ulp, 1.0)).max()))
        above = diff > floor
        if above.any():
            ROTATION_WORST[1] = max(ROTATION_WORST[1], float((diff[above] / np.abs(zo)[above]).max()))
    assert not bad.any(), f"{what}: {int(bad.sum())} rotated values outside the tolerance, worst " \
                          f"{float((diff / np.maximum(np.abs(zo), 1e-300)).max()):.3e} relative"


def gpu_rotation(x_dev, layout, g, seed):
    z = N.rht(x_dev, layout, g, seed)
    torch.cuda.synchronize()
    return z.cpu().numpy()


def end_to_end_mismatch(gpu, orc, z_gpu, z_orc, what="", mode=None, seed=0, row0=0):
    """Differences between the GPU's result and the oracle's from x (same tensor
    amax).  Every differing scale group must be explained by the rotation's
    rounding: one of the oracle's decisions in it lies within the bound
    propagated from the group's |z_gpu - z_orc| of a decision threshold
    (decision_margins).  Returns the differing (codes, scales) counts."""
    from decision_margins import MXFP3, MXFP4, explain
    gc, gsc, gg = gpu
    oc, osc, og = orc
    assert gg == og, f"{what}: global scale {gg!r} vs {og!r}"
    code_diff = oracle.unpack_codes(gc) != oracle.unpack_codes(oc)
    scale_diff = gsc != osc
    vr, vc = code_diff.shape
    n_codes, n_scales = int(code_diff.sum()), int(scale_diff.sum())
    if n_codes == 0 and n_scales == 0:
        return 0, 0
    assert mode is not None, f"{what}: differences found and no mode given to explain them"
    glen = 32 if mode in (MXFP4, MXFP3) else 16
    group_diff = code_diff.reshape(vr, vc // glen, glen).any(axis=2) | \
        scale_diff.reshape(vr, vc // glen, glen // 16).any(axis=2)
    for r, gi in np.argwhere(group_diff):
        c0 = gi * glen
        ok, why = explain(mode, z_orc[r, c0:c0 + glen], z_gpu[r, c0:c0 + glen], og, seed,
                          (row0 + r) * vc + c0, (row0 + r) * (vc // 16) + c0 // 16,
                          code_diff[r, c0:c0 + glen], bool(scale_diff[r, c0 // 16:(c0 + glen) // 16].any()))
        assert ok, f"{what}: view row {row0 + r}, elements {c0}..{c0 + glen - 1}: {why}"
    return n_codes, n_scales


def record_mismatch(n_codes_bad, n_codes, n_scales_bad, n_scales, what=""):
    ROTATED_MISMATCH[0] += n_codes_bad
    ROTATED_MISMATCH[1] += n_codes
    ROTATED_MISMATCH[2] += n_scales_bad
    ROTATED_MISMATCH[3] += n_scales
    if n_codes:
        assert n_codes_bad <= MISMATCH_MAX * n_codes, f"{what}: {n_codes_bad} of {n_codes} codes differ"
        assert n_scales_bad <= MISMATCH_MAX * n_scales, f"{what}: {n_scales_bad} of {n_scales} scales differ"


def compare_rotated_call(x_cpu, layout, mode, g, seed, ld_pad=0, amax=None):
    what = f"layout={layout} mode={mode} g={g} shape={tuple(x_cpu.shape)} ld_pad={ld_pad}"
    x_dev = to_device(x_cpu, ld_pad)
    xb = bits(x_cpu)
    z_gpu = gpu_rotation(x_dev, layout, g, seed)
    z_orc = oracle.rht_view(xb, layout, g, seed)
    check_rotation(z_gpu, z_orc, g, what)

    a_orc = oracle.amax(xb, layout, g, seed) if amax is None else amax
    if amax is None:
        a_gpu = N.amax(x_dev, layout, g, seed).item()
        a_own = float(np.abs(z_gpu).max()) if z_gpu.size else 0.0
        assert a_gpu == a_own, f"{what}: amax {a_gpu!r} is not max |z| = {a_own!r}"
        assert abs(a_gpu - a_orc) <= ROT_TOL * a_orc, f"{what}: amax {a_gpu!r} vs oracle {a_orc!r}"
    else:
        a_gpu = amax

    gpu = gpu_quantize(x_dev, layout, mode, g, seed, amax)
    assert_same(gpu, oracle.quantize_rotated(z_gpu, mode, seed, a_gpu), what + " (on the GPU's rotation)")

    gpu_same_amax = gpu if a_gpu == a_orc else gpu_quantize(x_dev, layout, mode, g, seed, a_orc)
    orc = oracle.quantize(xb, layout, mode, g, seed, amax_in=a_orc)
    nc, ns = end_to_end_mismatch(gpu_same_amax, orc, z_gpu, z_orc, what, mode=mode, seed=seed)
    record_mismatch(nc, z_orc.size, ns, z_orc.size // 16, what)
    return gpu


def compare_call(x_cpu, layout, mode, g, seed, ld_pad=0, amax=None):
    if g:
        return compare_rotated_call(x_cpu, layout, mode, g, seed, ld_pad, amax)
    x_dev = to_device(x_cpu, ld_pad)
    gpu = gpu_quantize(x_dev, layout, mode, g, seed, amax)
    orc = oracle.quantize(bits(x_cpu), layout, mode, g, seed, amax_in=amax)
    assert_same(gpu, orc, f"layout={layout} mode={mode} g={g} shape={tuple(x_cpu.shape)} ld_pad={ld_pad}")
    return gpu

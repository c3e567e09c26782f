"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on the same seeded inputs.

Without the rotation every mode is compared bit-exactly in codes, scales
(with the IF4 flag bit) and the FP32 tensor scale.  With the rotation the
comparison is the four-part one of gpu_helpers: rotated values within 1e-5 of
the oracle's, the quantization of the GPU's own rotated values bit-exact, and
the end-to-end difference from the oracle confined to blocks whose rotated
values differ, at most 1e-5 of the outputs.
"""
import numpy as np
import pytest
import torch

import oracle
from nvfp4_microscaling_quantization_b200 import binding as N
from nvfp4_microscaling_quantization_b200 import workloads as W

from gpu_helpers import (ROT_TOL, assert_same, bits, check_rotation, compare_call, gpu_quantize, gpu_rotation,
                         to_device)

pytestmark = pytest.mark.gpu

MODES = [W.RTN, W.SR, W.MS_EDEN, W.IF4, W.FOUR_OVER_SIX, W.SCALE_SEARCH, W.MXFP4, W.NVINT4, W.NVFP3, W.NVINT3, W.IF3,
         W.MXFP3]
GROUPS = [0, 16, 32, 64, 128]


@pytest.fixture(scope="module")
def small_x():
    return W.small().tensors()["x"]


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
@pytest.mark.parametrize("g", GROUPS)
@pytest.mark.parametrize("mode", MODES)
def test_small_workload_all_modes(small_x, mode, g, layout):
    """256x256 N(0,1), seed 0 -- every mode, rotation group and layout."""
    if mode == W.MS_EDEN and g == 0:
        pytest.skip("MS-EDEN needs the rotation")
    compare_call(small_x, layout, mode, g, 0)


def test_small_workload_calls(small_x):
    wl = W.small()
    for c in wl.calls:
        compare_call(small_x, c.layout, c.mode, c.rht_group, wl.seed)


RAGGED = [
    # rows, cols, ld_pad, layout, mode, g
    (37, 48, 0, W.ROWWISE, W.RTN, 16),
    (37, 48, 8, W.ROWWISE, W.SR, 16),
    (1, 128, 0, W.ROWWISE, W.MS_EDEN, 128),
    (3, 384, 8, W.ROWWISE, W.IF4, 128),
    (5, 16, 0, W.ROWWISE, W.FOUR_OVER_SIX, 0),
    (129, 4096 + 128, 0, W.ROWWISE, W.MS_EDEN, 128),
    (48, 72, 0, W.TRANSPOSED, W.RTN, 16),          # ragged column tile
    (144, 8, 0, W.TRANSPOSED, W.MS_EDEN, 16),      # ragged row tile
    (256, 200, 8, W.TRANSPOSED, W.SR, 128),        # padded ld, ragged columns
    (640, 384, 0, W.TRANSPOSED, W.MS_EDEN, 128),   # 5 x 6 tiles
    (96, 64, 0, W.TRANSPOSED, W.IF4, 32),
    (32, 24, 0, W.TRANSPOSED, W.FOUR_OVER_SIX, 0),
    (1024, 8, 16, W.TRANSPOSED, W.MS_EDEN, 64),
    # shapes the tiled (TMA) kernels take, with partial row and column tiles
    (40, 176, 8, W.ROWWISE, W.RTN, 16),
    (40, 176, 8, W.ROWWISE, W.MS_EDEN, 16),        # odd blocks per row: scale uniforms straddle calls
    (16, 80, 0, W.ROWWISE, W.SR, 16),
    (19, 96, 0, W.ROWWISE, W.FOUR_OVER_SIX, 32),
    (33, 1536, 0, W.ROWWISE, W.IF4, 128),
    (176, 136, 0, W.TRANSPOSED, W.RTN, 16),
    (208, 72, 8, W.TRANSPOSED, W.IF4, 0),          # odd scale pitch: byte stores
    (208, 72, 8, W.TRANSPOSED, W.MS_EDEN, 16),
    (384, 192, 0, W.TRANSPOSED, W.SR, 64),
    (256, 64, 0, W.TRANSPOSED, W.FOUR_OVER_SIX, 128),
    (1280, 640, 0, W.TRANSPOSED, W.MS_EDEN, 128),
    # scale search on each path: one-block kernels, TMA tiles (with and
    # without rotation), tensor-core tiles
    (37, 48, 0, W.ROWWISE, W.SCALE_SEARCH, 0),
    (40, 176, 8, W.ROWWISE, W.SCALE_SEARCH, 16),
    (208, 72, 8, W.TRANSPOSED, W.SCALE_SEARCH, 0),
    (640, 384, 0, W.TRANSPOSED, W.SCALE_SEARCH, 128),
    (384, 1152, 0, W.ROWWISE, W.SCALE_SEARCH, 128),
    # MXFP4 (32-element groups = the tiled kernels' block pairs): TMA tiles
    # with partial row and column tiles, with and without rotation, and
    # tensor-core tiles
    (40, 192, 8, W.ROWWISE, W.MXFP4, 16),
    (19, 1056, 0, W.ROWWISE, W.MXFP4, 0),
    (224, 72, 8, W.TRANSPOSED, W.MXFP4, 0),
    (640, 384, 0, W.TRANSPOSED, W.MXFP4, 128),
    (384, 1152, 0, W.ROWWISE, W.MXFP4, 128),
    # NVINT4 on each path: one-block kernels, TMA tiles, tensor-core tiles
    (37, 48, 8, W.ROWWISE, W.NVINT4, 0),
    (48, 72, 0, W.TRANSPOSED, W.NVINT4, 16),
    (40, 176, 8, W.ROWWISE, W.NVINT4, 16),
    (208, 72, 8, W.TRANSPOSED, W.NVINT4, 0),
    (640, 384, 0, W.TRANSPOSED, W.NVINT4, 128),
    # 3-bit formats on each path
    (37, 48, 8, W.ROWWISE, W.NVFP3, 16),
    (48, 72, 0, W.TRANSPOSED, W.IF3, 0),
    (5, 16, 0, W.ROWWISE, W.NVINT3, 0),
    (40, 176, 8, W.ROWWISE, W.IF3, 16),
    (208, 72, 8, W.TRANSPOSED, W.NVINT3, 0),
    (19, 1056, 0, W.ROWWISE, W.MXFP3, 0),
    (640, 384, 0, W.TRANSPOSED, W.IF3, 128),
    (384, 1152, 0, W.ROWWISE, W.MXFP3, 128),
    (256, 64, 0, W.TRANSPOSED, W.NVFP3, 128),
]


@pytest.mark.parametrize("rows,cols,ld_pad,layout,mode,g", RAGGED)
def test_ragged_shapes(rows, cols, ld_pad, layout, mode, g):
    gen = torch.Generator().manual_seed(rows * 1000 + cols)
    x = (torch.randn((rows, cols), generator=gen) * 3.0).to(torch.bfloat16)
    compare_call(x, layout, mode, g, 1234, ld_pad=ld_pad)


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
def test_empty_tensor(layout):
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda") if layout == W.ROWWISE else \
        torch.zeros((64, 0), dtype=torch.bfloat16, device="cuda")
    codes, scales, gs = N.quantize(x, layout, W.RTN, 0, 0)
    torch.cuda.synchronize()
    assert codes.numel() == 0 and scales.numel() == 0 and gs.item() == 1.0


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
@pytest.mark.parametrize("g", GROUPS)
def test_amax_matches_oracle(layout, g):
    x = W.gradient(rows=512, cols=384).tensors()["g"]
    got = N.amax(x.cuda(), layout, g, 77).item()
    exp = oracle.amax(bits(x), layout, g, 77)
    if g == 0:
        assert got == exp
    else:
        # max |z| of the GPU's own rotation exactly, the oracle's within the rotation tolerance
        assert got == float(np.abs(gpu_rotation(x.cuda(), layout, g, 77)).max())
        assert abs(got - exp) <= ROT_TOL * exp


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
def test_prepass_equals_supplied_amax(layout):
    x = W.gradient(rows=512, cols=384).tensors()["g"]
    xd = x.cuda()
    a = N.amax(xd, layout, 128, 5).item()
    for mode in (W.MS_EDEN, W.SR):
        assert_same(gpu_quantize(xd, layout, mode, 128, 5), gpu_quantize(xd, layout, mode, 128, 5, amax=a))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("g", [0, 32, 128])
def test_dequantize_parity(mode, g):
    if mode == W.MS_EDEN and g == 0:
        pytest.skip("MS-EDEN needs the rotation")
    x = W.activation(rows=64, cols=512).tensors()["a"]
    codes, scales, gs = oracle.quantize(bits(x), W.ROWWISE, mode, g, 9)
    c, s = torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda()
    gst = torch.tensor([gs], dtype=torch.float32, device="cuda")
    for inverse in ([False, True] if g else [False]):
        got = N.dequantize(c, s, gst, mode, g, 9, inverse_rht=inverse).cpu().numpy()
        exp = oracle.dequantize(codes, scales, gs, mode, g, 9, inverse_rht=inverse)
        assert np.array_equal(got.view(np.uint32), exp.view(np.uint32)), (mode, g, inverse)


@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
@pytest.mark.parametrize("g", [16, 32, 64, 128])
@pytest.mark.parametrize("shape", [(256, 384), (96, 384), (256, 112)])
def test_rotation_parity(layout, g, shape):
    """Forward rotation of bf16 (tensor cores where the quantizer uses them, the
    shuffle butterfly on smaller tensors) within the tolerance; the inverse on
    fp32 input follows the oracle's butterfly and is bit-exact."""
    rows, cols = shape
    if layout == W.TRANSPOSED and rows % g:
        rows = (rows + g - 1) // g * g
    if layout == W.ROWWISE and cols % g:
        pytest.skip("row length not a multiple of the group")
    x = W.gradient(rows=rows, cols=cols).tensors()["g"]
    got = gpu_rotation(x.cuda(), layout, g, 31)
    exp = oracle.rht_view(bits(x), layout, g, 31)
    check_rotation(got, exp, g, f"g={g} layout={layout}")
    print(f"\nrotation g={g} layout={layout} {shape}: bit-identical fraction "
          f"{np.mean(got.view(np.uint32) == exp.view(np.uint32)):.4f}")
    # inverse on fp32 input
    back = N.rht(torch.from_numpy(exp).cuda(), W.ROWWISE, g, 31, inverse=True).cpu().numpy()
    exp_back = oracle.rht_rows(exp, g, 31, inverse=True)
    assert np.array_equal(back.view(np.uint32), exp_back.view(np.uint32))


EDGE_MODES = [(W.RTN, 0), (W.SR, 0), (W.MS_EDEN, 16), (W.IF4, 0), (W.FOUR_OVER_SIX, 0), (W.IF4, 128),
              (W.SR, 128), (W.SCALE_SEARCH, 0), (W.MXFP4, 0), (W.NVINT4, 0), (W.NVFP3, 0), (W.NVINT3, 0),
              (W.IF3, 0), (W.MXFP3, 0)]


def _edge_tensors():
    out = {}
    out["zeros"] = torch.zeros((128, 256), dtype=torch.bfloat16)
    g = torch.Generator().manual_seed(3)
    x = torch.randn((128, 256), generator=g)
    x[17, 33] = 1e30  # one huge outlier: every other block lands on subnormal or zero scales
    out["outlier"] = x.to(torch.bfloat16)
    y = torch.ones((128, 256)) * 0.37
    y[::2] *= -1
    out["all_equal_blocks"] = y.to(torch.bfloat16)
    z = torch.randn((128, 256), generator=g)
    z[0, 0] = 3.389e38   # near the bf16 maximum
    z[1, 1] = -3.389e38
    out["bf16_max"] = z.to(torch.bfloat16)
    t = torch.randn((128, 256), generator=g) * 1e-20
    out["tiny"] = t.to(torch.bfloat16)
    s = torch.randn((128, 256), generator=g)
    s[:, 128:] *= 1e-4   # blocks far below the tensor max: subnormal E4M3 scales
    out["subnormal_scales"] = s.to(torch.bfloat16)
    return out


@pytest.mark.parametrize("name", list(_edge_tensors().keys()))
@pytest.mark.parametrize("mode,g", EDGE_MODES)
@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
def test_edge_cases(name, mode, g, layout):
    if name == "bf16_max" and g:
        pytest.skip("rotating values near the bf16 maximum overflows binary32 (out of the input domain)")
    x = _edge_tensors()[name]
    compare_call(x, layout, mode, g, 2024)


def test_exhaustive_bf16_rtn_path():
    """Every bf16 value of magnitude <= 6 goes through the quantizer with y = z exactly.

    Each block is [6, v1..v15]; amax_in = 10.5 gives s_g = 2^-8, every block scale
    is 256 and d = 1, so the codes are the E2M1 rounding of the bf16 values."""
    b = np.arange(1 << 16, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    vals = f[np.isfinite(f) & (np.abs(f) <= 6.0)]
    n = (len(vals) + 14) // 15
    vals = np.concatenate([vals, np.zeros(n * 15 - len(vals), dtype=np.float32)]).reshape(n, 15)
    blocks = np.concatenate([np.full((n, 1), 6.0, dtype=np.float32), vals], axis=1)
    rows = (n + 7) // 8
    pad = np.zeros((rows * 8 - n, 16), dtype=np.float32)
    mat = np.concatenate([blocks, pad]).reshape(rows, 128)
    x = torch.from_numpy(mat).to(torch.bfloat16)
    for mode in (W.RTN, W.SR, W.IF4, W.FOUR_OVER_SIX, W.SCALE_SEARCH, W.MXFP4, W.NVINT4, W.NVFP3, W.NVINT3, W.IF3,
                 W.MXFP3):
        gpu = compare_call(x, W.ROWWISE, mode, 0, 7, amax=10.5)
        if mode == W.RTN:
            assert gpu[2] == 2.0 ** -8
            assert np.all(gpu[1][:n // 8] == 0x78)  # scale 256


SATURATING_MODES = [(W.RTN, 0), (W.SR, 0), (W.MS_EDEN, 16), (W.MS_EDEN, 128), (W.IF4, 0), (W.IF4, 128),
                    (W.FOUR_OVER_SIX, 0), (W.SR, 128), (W.SCALE_SEARCH, 0), (W.NVINT4, 0), (W.NVFP3, 0),
                    (W.NVINT3, 0), (W.IF3, 0), (W.IF3, 128)]


@pytest.mark.parametrize("mode,g", SATURATING_MODES)
@pytest.mark.parametrize("layout", [W.ROWWISE, W.TRANSPOSED])
def test_amax_far_below_the_tensor_maximum(mode, g, layout):
    """A supplied tensor amax 1/64 of the true one: most block scales saturate at
    448 and the scaled values run far past every grid, so the saturation of
    E2M1 at 6, of E2M0 at 4, the clamps of the integer levels at 7 and 3, and
    MS-EDEN's corrected scale at 448 all decide codes."""
    gen = torch.Generator().manual_seed(41)
    x = (torch.randn((128, 256), generator=gen) * 3.0).to(torch.bfloat16)
    amax = float(x.float().abs().max()) / 64.0
    gpu = compare_call(x, layout, mode, g, 77, amax=amax)
    if mode not in (W.SCALE_SEARCH, W.FOUR_OVER_SIX):
        assert np.mean((np.asarray(gpu[1]) & 0x7F) == 0x7E) > 0.5  # most scales saturated at 448


def _neighbourhood(centres, radius):
    out = []
    for c in centres:
        base = int(np.float32(c).view(np.uint32))
        out.append(np.arange(max(base - radius, 0), base + radius + 1, dtype=np.int64))
    return np.unique(np.concatenate(out)).astype(np.uint32)


def test_e2m1_conversion_near_every_boundary():
    """The hardware E2M1 conversion agrees with the oracle's rounding on every fp32
    within 2^15 ulps of each threshold and grid value, both signs, and on a stride
    sweep of all finite fp32 patterns."""
    centres = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 1e-38]
    pos = _neighbourhood(centres, 1 << 15)
    sweep = np.arange(0, 1 << 32, 257, dtype=np.uint64).astype(np.uint32)
    bits_all = np.concatenate([pos, pos | np.uint32(0x80000000), sweep, np.array([0, 0x80000000], np.uint32)])
    v = bits_all.view(np.float32)
    v = v[np.isfinite(v)]
    got = N.encode_e2m1(torch.from_numpy(v).cuda()).cpu().numpy()
    exp = oracle.e2m1_rtn_array(v)
    bad = np.flatnonzero(got != exp)
    assert len(bad) == 0, f"{len(bad)} differ, e.g. {v[bad[:5]]} got {got[bad[:5]]} expected {exp[bad[:5]]}"


@pytest.mark.parametrize("round_up", [False, True])
def test_e4m3_conversion_near_every_boundary(round_up):
    table = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], dtype=np.float64)
    centres = list(table[1:]) + list((table[1:] + table[:-1]) / 2) + [2.0 ** -10, 464.0, 480.0]
    pos = _neighbourhood(centres, 1 << 10)
    sweep = np.arange(0, 0x7F800000, 131, dtype=np.uint64).astype(np.uint32)
    v = np.concatenate([pos, sweep]).view(np.float32)
    v = v[np.isfinite(v) & (v >= 0)]
    got = N.encode_e4m3(torch.from_numpy(v).cuda(), round_up=round_up).cpu().numpy()
    exp = oracle.e4m3_array(v, round_up=round_up)
    bad = np.flatnonzero(got != exp)
    assert len(bad) == 0, f"{len(bad)} differ, e.g. {v[bad[:5]]} got {got[bad[:5]]} expected {exp[bad[:5]]}"


def test_determinism_and_seeds():
    x = W.gradient(rows=256, cols=256).tensors()["g"].cuda()
    a = gpu_quantize(x, W.ROWWISE, W.SR, 128, 1)
    b = gpu_quantize(x, W.ROWWISE, W.SR, 128, 1)
    c = gpu_quantize(x, W.ROWWISE, W.SR, 128, 2)
    assert_same(a, b)
    assert not np.array_equal(a[0], c[0])
    e1 = gpu_quantize(x, W.TRANSPOSED, W.MS_EDEN, 128, 1)
    e2 = gpu_quantize(x, W.TRANSPOSED, W.MS_EDEN, 128, 1 << 40)
    assert not np.array_equal(e1[1], e2[1])


def test_side_stream_matches_default_stream():
    x = W.small().tensors()["x"].cuda()
    ref = gpu_quantize(x, W.TRANSPOSED, W.MS_EDEN, 128, 3)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        codes, scales, gs = N.quantize(x, W.TRANSPOSED, W.MS_EDEN, 128, 3, stream=s)
    s.synchronize()
    assert_same(ref, (codes.cpu().numpy(), scales.cpu().numpy(), float(gs.item())))


@pytest.mark.parametrize("layout,mode,g", [(W.ROWWISE, W.MS_EDEN, 128), (W.TRANSPOSED, W.SR, 32),
                                           (W.ROWWISE, W.RTN, 0), (W.TRANSPOSED, W.FOUR_OVER_SIX, 0)])
def test_outputs_at_8_byte_offsets(layout, mode, g):
    """Code and scale buffers that are only 8- (codes) or 1-byte (scales) aligned, as the ABI allows."""
    import ctypes
    x = W.gradient(rows=256, cols=512).tensors()["g"]
    xd = x.cuda()
    rows, cols = x.shape
    vr, vc = N.view_shape(rows, cols, layout)
    cbuf = torch.zeros(vr * vc // 2 + 64, dtype=torch.uint8, device="cuda")
    sbuf = torch.zeros(vr * vc // 16 + 64, dtype=torch.uint8, device="cuda")
    gs = torch.zeros(1, dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    P = ctypes.c_void_p
    st = N.nvfp4_quantize(P(xd.data_ptr()), rows, cols, cols, layout, mode, g, 21, None,
                          P(cbuf.data_ptr() + 8), P(sbuf.data_ptr() + 1), P(gs.data_ptr()), P(ws.data_ptr()), 256,
                          P(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    got_c = cbuf[8:8 + vr * vc // 2].cpu().numpy().reshape(vr, vc // 2)
    got_s = sbuf[1:1 + vr * vc // 16].cpu().numpy().reshape(vr, vc // 16)
    # the same call into aligned buffers (itself compared with the oracle by the other tests)
    assert_same((got_c, got_s, float(gs.item())), gpu_quantize(xd, layout, mode, g, 21))
    if g == 0:
        assert_same((got_c, got_s, float(gs.item())), oracle.quantize(bits(x), layout, mode, g, 21))


def test_if4_int4_rounding_ties():
    """IF4 blocks that take the scaled-INT4 option and hold y = 3.0, whose
    RN(y * RN(7/6)) is exactly 3.5: the level is RNE(3.5) = 4 only if the
    product is rounded before the level is (a fused multiply-add would give 3).

    amax_in = 10.5 gives s_g = 2^-8; with a 6.0 in every block the block scale
    is 256 and d = 1, so y = x.  The other values sit near the INT4 levels
    k * 6/7 so that the INT4 option wins."""
    levels = np.array([k * 6.0 / 7.0 for k in range(-7, 8)], dtype=np.float32)
    rng = np.random.default_rng(17)
    rows, cols = 64, 256
    blocks = rng.choice(levels, size=(rows * cols // 16, 16)).astype(np.float32)
    blocks[:, 0] = 6.0
    pos = 1 + rng.integers(0, 15, len(blocks))
    blocks[np.arange(len(blocks)), pos] = np.where(rng.random(len(blocks)) < 0.5, 3.0, -3.0)
    x = torch.from_numpy(blocks.reshape(rows, cols)).to(torch.bfloat16)
    gpu = compare_call(x, W.ROWWISE, W.IF4, 0, 5, amax=10.5)
    flagged = int(np.sum(gpu[1] >= 0x80))
    assert flagged > len(blocks) // 2, f"only {flagged} of {len(blocks)} blocks took the INT4 option"


@pytest.mark.parametrize("shape,g_row,g_col", [
    ((256, 384), 128, 128), ((640, 384), 0, 128), ((384, 1280), 128, 0), ((512, 512), 16, 64),
    ((256, 256), 0, 0), ((1280, 896), 32, 128),
    ((96, 256), 32, 32),      # below one tensor-core tile: two single pre-passes
    ((384, 19328), 128, 128),  # 453 tiles: CTAs with odd and even tile counts, several tile pairs each
    ((1280, 896), 64, 64),
])
def test_amax_dual_equals_two_single_passes(shape, g_row, g_col):
    """nvfp4_amax_dual (both layouts from one read) gives the two single-layout
    pre-passes' values bit for bit, and the oracle's within the rotation tolerance."""
    rows, cols = shape
    x = W.gradient(rows=rows, cols=cols).tensors()["g"]
    xd = x.cuda()
    a_row, a_col = N.amax_dual(xd, g_row, g_col, 41)
    s_row = N.amax(xd, W.ROWWISE, g_row, 41)
    s_col = N.amax(xd, W.TRANSPOSED, g_col, 41)
    torch.cuda.synchronize()
    assert a_row.item() == s_row.item() and a_col.item() == s_col.item()
    for layout, g, got in ((W.ROWWISE, g_row, a_row.item()), (W.TRANSPOSED, g_col, a_col.item())):
        exp = oracle.amax(bits(x), layout, g, 41)
        if g == 0:
            assert got == exp
        else:
            assert abs(got - exp) <= ROT_TOL * exp

"""Pins the oracle's quantization modes to what the pages and the mathematics fix.

* SR is unbiased when nothing clips, with error E[(y-l)(u-y)] per value
  ("Comparing INT4 and NVFP4 Palettes on Real Gradient Tensors", section "The
  two corners, and what the palette does to them"): Monte-Carlo mean within 4
  sigma, and the empirical error equals the closed form.
* MS-EDEN is unbiased in expectation and has lower error than SR (Quartet II
  abstract: "more than 2x lower quantization error than SR"; article list
  "Kerninnovationen"): Monte-Carlo mean within 4 sigma after the inverse
  rotation, and the MSE ordering RTN < MS-EDEN < SR on Gaussian data.
* IF4 keeps the lower-error option of FP4 and scaled INT4 and flags INT4 in
  the scale's sign bit (IF4 paper page, abstract, Figure 1 and Figure 3).
* 4/6 keeps the lower-error of the two block scales (Quartet II article,
  "Quantisierung im Vorwaertsdurchlauf"; IF4 page Table 1, scale max 256).
* Scale search keeps the lowest-error of the 19 E4M3 codes around the absmax
  scale (palettes post, "The two corners, and what the palette does to
  them"; the ScaleSearch entry of the IF4 page): checked against a search
  recomputed with torch's E4M3 decoder and a brute-force E2M1 rounding, and
  per block no worse than 4/6, whose two scales are among its candidates.
* MXFP4 (IF4 page, Table 1: groups of 32, UE8M0 scale, max 6 x 2^127, min
  0.5 x 2^-127): shared exponent floor(log2 amax) - 2 recomputed with numpy's
  frexp, codes by brute-force nearest E2M1 of x / 2^E, a lossless round trip.
* NVINT4 (IF4 page, Table 1: E4M3 scale, INT4 values, max 7 x 448): integer
  levels by brute-force nearest integer (ties to even) of the scaled value,
  and a lossless round trip.
* 3-bit formats (IF4 page, 3-bit table: MXFP3, NVINT3, NVFP3, IF3): E2M0 and
  INT3 rounding by brute force over every bf16 value in range, IF3 keeping
  the lower-error option, MXFP3's shared exponent.
* Table 1's MSE column (NVFP4 9.0, NVINT4 7.4, 4/6 7.5, IF4 6.2, MXFP4 13.2,
  x1e-3) on standard normal data, within 2% (tests/golden/if4_table1_mse.txt).
* Structural properties: transposed view = row-wise quantization of X^T,
  leading dimension, amax_in, zero tensor and zero blocks, nibble order.
"""
import numpy as np
import pytest
import torch

from nvfp4_microscaling_quantization_b200 import workloads as W

ROW, TR = 0, 1
RTN, SR, EDEN, IF4, FO6, SS, MX, NI4 = 0, 1, 2, 3, 4, 5, 6, 7
NF3, NI3, IF3M, MX3 = 8, 9, 10, 11
E2M0 = np.array([0.0, 1.0, 2.0, 4.0])
GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def bits_of(t):
    return W.bf16_bits(t)


def bf16(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def f32(a):
    return np.float32(a)


def deq(orc, codes, scales, gs, mode, g, seed, inverse=False):
    return orc.dequantize(codes, scales, gs, mode, g, seed, inverse_rht=inverse).astype(np.float64)


# ----------------------------------------------------------------------------- SR
def test_sr_monte_carlo_unbiased_and_closed_form_error(orc):
    """4096 identical rows: same scales, independent uniforms per row (element index)."""
    rng = np.random.default_rng(0)
    row = bf16(rng.standard_normal(256))
    T = 4096
    x = row[None, :].repeat(T, 1)
    codes, scales, gs = orc.quantize(bits_of(x), ROW, SR, 0, 42)
    assert np.all(scales == scales[0:1])  # every row gets the same block scales
    q = deq(orc, codes, scales, gs, SR, 0, 42)
    xv = row.float().numpy().astype(np.float64)
    # closed form per element: d^2 (y-l)(u-y) with y the scaled value
    d = np.array([np.float32(orc.e4m3_decode(s)) * np.float32(gs) for s in scales[0]], dtype=np.float32)
    dd = np.repeat(d, 16)
    r = (np.float32(1.0) / dd).astype(np.float32)
    y = np.abs((xv.astype(np.float32) * r).astype(np.float32)).astype(np.float64)
    y = np.minimum(y, 6.0)
    lo = GRID[np.searchsorted(GRID, y, side="right") - 1]
    hi = GRID[np.minimum(np.searchsorted(GRID, y, side="right"), 7)]
    var = dd.astype(np.float64) ** 2 * (y - lo) * (hi - y)
    mean = q.mean(axis=0)
    sd = np.sqrt(var / T)
    z = np.abs(mean - xv) / np.maximum(sd, 1e-30)
    z[var == 0] = 0.0
    assert np.all(np.abs(mean - xv)[var == 0] < 1e-6 * np.abs(xv).max())  # exact values stay exact
    # unbiased: every element within 4 sigma (+ the 2^-16 resolution of the uniforms)
    slack = dd.astype(np.float64) * (hi - lo) * 2.0 ** -16
    assert np.all(np.abs(mean - xv) <= 4 * sd + slack)
    # empirical MSE equals the closed form within its sampling error
    emp = ((q - xv[None, :]) ** 2).mean(axis=0).sum()
    assert abs(emp - var.sum()) <= 0.05 * var.sum()


def test_sr_never_exceeds_block_range(orc):
    """Round-up scales: |Q(x)| <= block absmax rounded up, never clipped."""
    rng = np.random.default_rng(1)
    x = bf16(rng.standard_t(3, size=(64, 256)))
    codes, scales, gs = orc.quantize(bits_of(x), ROW, SR, 0, 3)
    q = deq(orc, codes, scales, gs, SR, 0, 3)
    xv = x.float().numpy().astype(np.float64)
    d = np.vectorize(lambda s: np.float32(orc.e4m3_decode(int(s))) * np.float32(gs))(scales).astype(np.float64)
    assert np.all(np.abs(q) <= 6 * np.repeat(d, 16, axis=1) * (1 + 1e-6))
    # the block's largest element is never rounded away from its interval
    assert np.all(np.abs(q - xv) <= np.repeat(d, 16, axis=1) * 2.0 + 1e-12)


# ------------------------------------------------------------------------- MS-EDEN
def _eden_trials(orc, x_row, T, g=128):
    bits = bits_of(x_row[None, :])
    outs = []
    for s in range(T):
        seed = 1000 + s
        codes, scales, gs = orc.quantize(bits, ROW, EDEN, g, seed)
        outs.append(deq(orc, codes, scales, gs, EDEN, g, seed, inverse=True)[0])
    return np.array(outs)


def test_ms_eden_monte_carlo_unbiased(orc):
    rng = np.random.default_rng(2)
    x = bf16(rng.standard_normal(256))
    xv = x.float().numpy().astype(np.float64)
    T = 3000
    q = _eden_trials(orc, x, T)
    mean = q.mean(axis=0)
    sd = q.std(axis=0, ddof=1) / np.sqrt(T)
    z = (mean - xv) / sd
    # 4-sigma per element, and the whole vector's chi-square within 4 sigma of its mean
    assert np.max(np.abs(z)) < 4.0 + 0.5  # 256 elements: max |N(0,1)| rarely exceeds 4
    n = len(z)
    assert abs(np.sum(z ** 2) - n) < 4 * np.sqrt(2 * n)


def _mse(orc, x, mode, g, seeds):
    bits = bits_of(x)
    xv = x.float().numpy().astype(np.float64)
    tot = 0.0
    for s in seeds:
        codes, scales, gs = orc.quantize(bits, ROW, mode, g, s)
        q = deq(orc, codes, scales, gs, mode, g, s, inverse=g > 0)
        tot += np.mean((q - xv) ** 2)
    return tot / len(seeds)


def test_mse_ordering_rtn_eden_sr(orc):
    """RTN < MS-EDEN < SR on N(0,1) blocks, all with the 128-point RHT; SR/EDEN reported."""
    rng = np.random.default_rng(4)
    x = bf16(rng.standard_normal((64, 512)))
    seeds = list(range(8))
    m_rtn = _mse(orc, x, RTN, 128, seeds)
    m_eden = _mse(orc, x, EDEN, 128, seeds)
    m_sr = _mse(orc, x, SR, 128, seeds)
    print(f"\nMSE  RTN {m_rtn:.5f}  MS-EDEN {m_eden:.5f}  SR {m_sr:.5f}  SR/EDEN {m_sr / m_eden:.2f}")
    assert m_rtn < m_eden < m_sr
    assert m_sr / m_eden > 1.5  # the pages claim "more than 2x"; the ratio is reported above


def test_ms_eden_codes_are_rtn_codes(orc):
    """Randomness lives only on the scale: codes equal RTN's (same view, same block scale choice)."""
    rng = np.random.default_rng(5)
    x = bf16(rng.standard_normal((32, 256)))
    # MS-EDEN maps the amax to 6 x 256 and RTN to 6 x 448: amax 4 and 7 give the same s_g
    c_e, s_e, g_e = orc.quantize(bits_of(x), ROW, EDEN, 128, 9, amax_in=4.0)
    c_r, s_r, g_r = orc.quantize(bits_of(x), ROW, RTN, 128, 9, amax_in=7.0)
    assert g_e == g_r
    assert np.array_equal(c_e, c_r)
    # scales differ from RTN's by at most one E4M3 step after the correction (c near 1)
    se = np.vectorize(lambda s: orc.e4m3_decode(int(s)))(s_e)
    sr = np.vectorize(lambda s: orc.e4m3_decode(int(s)))(s_r)
    assert np.all(np.abs(se / sr - 1) < 0.3)
    assert np.mean(s_e != s_r) > 0.05


# --------------------------------------------------------------------------- IF4
def _block_views(orc, x_bits, layout, mode, g, seed):
    codes, scales, gs = orc.quantize(x_bits, layout, mode, g, seed)
    z = orc.rht_view(x_bits, layout, g, seed) if g else \
        torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    if layout == TR and not g:
        z = np.ascontiguousarray(z.T)
    return codes, scales, gs, z.astype(np.float32)


@pytest.mark.parametrize("g", [0, 128])
def test_if4_picks_lower_error_option(orc, g):
    wl = W.activation(rows=32, cols=512)
    a = wl.tensors()["a"]
    bits = bits_of(a)
    codes, scales, gs, z = _block_views(orc, bits, ROW, IF4, g, 3)
    k1, k2 = orc.if4_constants()
    cu = orc.unpack_codes(codes)
    n_int = 0
    for r in range(z.shape[0]):
        for b in range(z.shape[1] // 16):
            S = int(scales[r, b])
            d = f32(f32(orc.e4m3_decode(S & 0x7F)) * f32(gs))
            if d == 0:
                continue
            y = (z[r, 16 * b:16 * b + 16] * f32(f32(1.0) / d)).astype(np.float32)
            fp = np.array([orc.e2m1_decode(orc.e2m1_rtn(float(v))) for v in y], dtype=np.float64)
            k = np.clip(np.round((y * f32(k1)).astype(np.float32)), -7, 7)
            it = (k * f32(k2)).astype(np.float32).astype(np.float64)
            e_fp = np.sum((y - fp) ** 2)
            e_int = np.sum((y - it) ** 2)
            flag = bool(S & 0x80)
            n_int += flag
            chosen, other = (e_int, e_fp) if flag else (e_fp, e_int)
            assert chosen <= other * (1 + 1e-5) + 1e-12, (r, b)
            # codes are those of the chosen option
            c = cu[r, 16 * b:16 * b + 16]
            if flag:
                kk = np.where(c & 8, -(c & 7).astype(int), (c & 7).astype(int))
                assert np.array_equal(kk, k.astype(int))
            else:
                assert np.allclose([orc.e2m1_decode(int(v)) for v in c], fp)
    print(f"\nIF4 g={g}: INT4 picked for {n_int} of {z.size // 16} blocks")


def test_if4_fp4_blocks_equal_rtn(orc):
    """An IF4 block with the flag clear is byte-identical to RTN NVFP4 (flag 1 = INT4 reading)."""
    wl = W.activation(rows=64, cols=256)
    bits = bits_of(wl.tensors()["a"])
    c_i, s_i, g_i = orc.quantize(bits, ROW, IF4, 0, 3)
    c_r, s_r, g_r = orc.quantize(bits, ROW, RTN, 0, 3)
    assert g_i == g_r
    fp = (s_i & 0x80) == 0
    assert np.array_equal(s_i[fp], s_r[fp])
    assert np.array_equal((s_i & 0x7F), s_r)
    cb_i = orc.unpack_codes(c_i).reshape(c_i.shape[0], -1, 16)
    cb_r = orc.unpack_codes(c_r).reshape(c_r.shape[0], -1, 16)
    assert np.array_equal(cb_i[fp], cb_r[fp])
    assert 0 < np.mean(~fp) < 1


def test_if4_rht_raises_int4_share(orc):
    """Reported: the share of INT4 blocks with and without the rotation (IF4 page, Figure 5)."""
    wl = W.activation(rows=64, cols=1024)
    bits = bits_of(wl.tensors()["a"])
    _, s0, _ = orc.quantize(bits, ROW, IF4, 0, 3)
    _, s1, _ = orc.quantize(bits, ROW, IF4, 128, 3)
    f0, f1 = np.mean(s0 >= 0x80), np.mean(s1 >= 0x80)
    print(f"\nIF4 INT4 share: no RHT {f0:.3f}, RHT {f1:.3f}")
    assert f1 > f0


# --------------------------------------------------------------------------- 4/6
def test_four_over_six_picks_lower_error(orc):
    wl = W.weight(rows=32, cols=512)
    bits = bits_of(wl.tensors()["w"])
    codes, scales, gs, z = _block_views(orc, bits, ROW, FO6, 0, 1)
    A = np.abs(z).max()
    assert gs == orc.global_scale(A, FO6)
    cand = {}
    for r in range(z.shape[0]):
        for b in range(z.shape[1] // 16):
            zb = z[r, 16 * b:16 * b + 16]
            ab = f32(np.abs(zb).max())
            errs, Ss = [], []
            for m in (6.0, 4.0):
                S = orc.e4m3_rne_sat(f32(ab / f32(f32(m) * f32(gs))))
                d = f32(f32(orc.e4m3_decode(S)) * f32(gs))
                y = (zb * f32(f32(1.0) / d)).astype(np.float32)
                v = np.array([orc.e2m1_decode(orc.e2m1_rtn(float(t))) for t in y], dtype=np.float32)
                errs.append(np.sum((zb.astype(np.float64) - (v * d).astype(np.float32)) ** 2))
                Ss.append(S)
            S = int(scales[r, b])
            assert S in Ss
            chosen = errs[Ss.index(S)] if Ss[0] != Ss[1] else errs[0]
            assert chosen <= min(errs) * (1 + 1e-5) + 1e-30
            cand[(r, b)] = Ss.index(S)
    frac4 = np.mean([v == 1 for v in cand.values()])
    print(f"\n4/6: scale-to-4 chosen for {frac4:.3f} of blocks")
    assert 0 < frac4 < 1


def test_four_over_six_not_worse_than_rtn(orc):
    wl = W.weight(rows=64, cols=1024)
    x = wl.tensors()["w"]
    m_rtn = _mse(orc, x, RTN, 0, [0])
    m_46 = _mse(orc, x, FO6, 0, [0])
    print(f"\nweight-like MSE: RTN {m_rtn:.3e}  4/6 {m_46:.3e}")
    assert m_46 <= m_rtn


# ------------------------------------------------------------------ scale search
def _e4m3_value(code):
    return np.float32(torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).float().item())


def _e2m1_rtn_value(y):
    """Nearest E2M1 grid value to y (float32), ties to the even code index (brute force)."""
    a = min(abs(float(y)), 6.0)
    dist = np.abs(GRID - a)
    best = np.flatnonzero(dist == dist.min())
    i = best[0] if len(best) == 1 else best[best % 2 == 0][0]
    return np.float32(-GRID[i] if y < 0 else GRID[i])


def test_scale_search_picks_lowest_of_19(orc):
    wl = W.weight(rows=8, cols=256)
    bits = bits_of(wl.tensors()["w"])
    codes, scales, gs, z = _block_views(orc, bits, ROW, SS, 0, 1)
    assert gs == orc.global_scale(np.abs(z).max(), FO6)  # tensor scale M = 256, as 4/6
    cu = orc.unpack_codes(codes)
    moved = 0
    for r in range(z.shape[0]):
        for b in range(z.shape[1] // 16):
            zb = z[r, 16 * b:16 * b + 16]
            ab = f32(np.abs(zb).max())
            S0 = orc.e4m3_rne_sat(f32(ab / f32(f32(6.0) * f32(gs))))
            errs = {}
            for delta in range(-9, 10):
                Sc = min(max(S0 + delta, 0), 0x7E)
                d = f32(_e4m3_value(Sc) * f32(gs))
                if d == 0:
                    errs[Sc] = float(np.sum(zb.astype(np.float64) ** 2))
                    continue
                y = (zb * f32(f32(1.0) / d)).astype(np.float32)
                v = np.array([_e2m1_rtn_value(t) for t in y], dtype=np.float32)
                errs[Sc] = float(np.sum((zb.astype(np.float64) - (v * d).astype(np.float32)) ** 2))
            S = int(scales[r, b])
            assert S in errs, (r, b)
            assert errs[S] <= min(errs.values()) * (1 + 1e-5) + 1e-30, (r, b)
            d = f32(_e4m3_value(S) * f32(gs))
            if d > 0:  # codes are the RTN codes under the chosen scale
                y = (zb * f32(f32(1.0) / d)).astype(np.float32)
                vals = np.array([orc.e2m1_decode(int(c)) for c in cu[r, 16 * b:16 * b + 16]], dtype=np.float32)
                assert np.array_equal(vals, np.array([_e2m1_rtn_value(t) for t in y], dtype=np.float32))
            moved += S != S0
    print(f"\nscale search: scale moved off the absmax scale in {moved} of {len(scales.flat)} blocks")
    assert moved > 0


def test_scale_search_no_worse_than_four_over_six_per_block(orc):
    wl = W.weight(rows=64, cols=512)
    bits = bits_of(wl.tensors()["w"])
    z = bits_of(wl.tensors()["w"])
    z = torch.from_numpy(z.view(np.int16)).view(torch.bfloat16).double().numpy()
    errs = {}
    for mode in (FO6, SS):
        c, s, gs = orc.quantize(bits, ROW, mode, 0, 1)
        dq = deq(orc, c, s, gs, mode, 0, 1)
        errs[mode] = ((z - dq) ** 2).reshape(z.shape[0], -1, 16).sum(-1)
    assert np.all(errs[SS] <= errs[FO6] * (1 + 1e-6) + 1e-30)
    m_rtn = _mse(orc, wl.tensors()["w"], RTN, 0, [0])
    m_46, m_ss = errs[FO6].sum() / z.size, errs[SS].sum() / z.size
    print(f"\nweight-like MSE: RTN {m_rtn:.3e}  4/6 {m_46:.3e}  scale search {m_ss:.3e} "
          f"({100 * (1 - m_ss / m_rtn):.1f}% below RTN)")
    assert m_ss <= m_46 <= m_rtn


# ------------------------------------------------------------------------ MXFP4
def _rtn_grid_index(a):
    """Brute-force nearest E2M1 magnitude index of |a| <= 6 (ties to the even index)."""
    dist = np.abs(GRID - min(abs(float(a)), 6.0))
    best = np.flatnonzero(dist == dist.min())
    return int(best[0] if len(best) == 1 else best[best % 2 == 0][0])


def test_mxfp4_shared_exponent_and_codes(orc):
    rng = np.random.default_rng(12)
    rows, cols = 6, 256
    x = rng.standard_normal((rows, cols)) * 2.0 ** rng.integers(-30, 30, (rows, cols // 32)).repeat(32, 1)
    x[0, :32] = 0.0                       # an all-zero group
    x[1, 32:64] = 1e-39                   # subnormal-only group in binary32 (bf16 keeps it)
    xb = bf16(x)
    codes, scales, gs = orc.quantize(bits_of(xb), ROW, MX, 0, 0)
    assert gs == 1.0
    xv = xb.float().numpy()
    cu = orc.unpack_codes(codes)
    for r in range(rows):
        for gi in range(cols // 32):
            grp = xv[r, 32 * gi:32 * gi + 32].astype(np.float64)
            a = np.abs(grp).max()
            E = -127 if a == 0 else int(np.clip(np.frexp(a)[1] - 1 - 2, -127, 127))
            assert scales[r, 2 * gi] == scales[r, 2 * gi + 1] == E + 127, (r, gi)
            y = grp / 2.0 ** E
            for i in range(32):
                k = _rtn_grid_index(y[i])
                exp = 0 if k == 0 else (k | (8 if y[i] < 0 else 0))
                assert cu[r, 32 * gi + i] == exp, (r, gi, i)


def test_mxfp4_lossless_round_trip(orc):
    rng = np.random.default_rng(13)
    rows, cols = 8, 512
    v = GRID[rng.integers(0, 8, (rows, cols))] * np.where(rng.random((rows, cols)) < 0.5, -1.0, 1.0)
    v = v.reshape(rows, cols // 32, 32)
    v[:, :, 0] = np.where(rng.random((rows, cols // 32)) < 0.5, 4.0, 6.0)  # group max in [4, 6]
    e = rng.integers(-40, 40, (rows, cols // 32))
    x = (v * 2.0 ** e[:, :, None]).reshape(rows, cols)
    xb = bf16(x)
    assert np.array_equal(xb.double().numpy(), x)
    codes, scales, gs = orc.quantize(bits_of(xb), ROW, MX, 0, 0)
    assert np.array_equal(scales[:, ::2].astype(int), e + 127)
    assert np.array_equal(deq(orc, codes, scales, gs, MX, 0, 0), x)


def test_mxfp4_mse_above_nvfp4_on_gaussian(orc):
    """Table 1 (IF4 page) orders MXFP4's MSE above NVFP4's (13.2 vs 9.0, x1e-3); reported."""
    rng = np.random.default_rng(14)
    x = bf16(rng.standard_normal((128, 1024)))
    m_mx = _mse(orc, x, MX, 0, [0])
    m_nv = _mse(orc, x, RTN, 0, [0])
    print(f"\nN(0,1) MSE: NVFP4 {m_nv * 1e3:.2f}e-3  MXFP4 {m_mx * 1e3:.2f}e-3  ratio {m_mx / m_nv:.2f} "
          f"(Table 1: 9.0, 13.2, ratio 1.47)")
    assert m_mx > m_nv


def test_nvint4_levels_and_round_trip(orc):
    rng = np.random.default_rng(21)
    x = bf16(rng.standard_normal((16, 256)) * 3.0)
    codes, scales, gs = orc.quantize(bits_of(x), ROW, NI4, 0, 0)
    xv = x.float().numpy()
    assert gs == np.float32(np.float32(np.abs(xv).max()) / np.float32(3136.0))
    cu = orc.unpack_codes(codes)
    for r in range(xv.shape[0]):
        for b in range(xv.shape[1] // 16):
            zb = xv[r, 16 * b:16 * b + 16]
            S = orc.e4m3_rne_sat(f32(f32(np.abs(zb).max()) / f32(f32(7.0) * f32(gs))))
            assert scales[r, b] == S
            d = f32(_e4m3_value(S) * f32(gs))
            y = (zb * f32(f32(1.0) / d)).astype(np.float64)
            k = np.clip(np.round(y), -7, 7)          # numpy rounds half to even
            c = cu[r, 16 * b:16 * b + 16]
            kk = np.where(c & 8, -(c & 7).astype(int), (c & 7).astype(int))
            assert np.array_equal(kk, k.astype(int)), (r, b)
            assert np.all(c != 8)                     # zero is code 0
    # integers under a power-of-two scale quantize exactly: blocks holding +-7,
    # tensor max 7 * 448 * 2^-10 so that s_g = 2^-10 and every block scale is
    # an exact power of two
    k = rng.integers(-7, 8, (8, 256)).astype(np.float64).reshape(8, 16, 16)
    k[:, :, 0] = 7.0
    e = rng.integers(-6, 8, (8, 16)).astype(np.float64)
    e[0, 0] = 0
    blk = 2.0 ** e
    blk[0, 0] = 448.0
    xx = (k * blk[:, :, None] * 2.0 ** -10).reshape(8, 256)
    xb = bf16(xx)
    c2, s2, g2 = orc.quantize(bits_of(xb), ROW, NI4, 0, 0)
    assert g2 == 2.0 ** -10
    assert np.array_equal(deq(orc, c2, s2, g2, NI4, 0, 0), xx)


def _nearest_even(levels, t):
    """Nearest of the magnitudes `levels` to |t| (ties to the even index), with t's sign."""
    dist = np.abs(levels - min(abs(t), levels[-1]))
    best = np.flatnonzero(dist == dist.min())
    idx = int(best[0] if len(best) == 1 else best[best % 2 == 0][0])
    return -levels[idx] if t < 0 else levels[idx]


def _all_bf16_up_to(limit):
    b = np.arange(1 << 16, dtype=np.uint32)
    f = (b << 16).view(np.float32)
    return f[np.isfinite(f) & (np.abs(f) <= limit)]


def _unit_scale_blocks(vals, head):
    """Blocks [head, v1..v15] (the head sets every block scale), 8 blocks a row."""
    n = (len(vals) + 14) // 15
    v = np.concatenate([vals, np.zeros(n * 15 - len(vals), dtype=np.float32)]).reshape(n, 15)
    blocks = np.concatenate([np.full((n, 1), head, dtype=np.float32), v], axis=1)
    rows = (n + 7) // 8
    blocks = np.concatenate([blocks, np.zeros((rows * 8 - n, 16), dtype=np.float32)])
    return blocks.reshape(rows, 128), v


@pytest.mark.parametrize("mode,head,amax,levels,even", [
    (NF3, 4.0, 7.0, E2M0, True),          # s_g = 7 / 1792 = 2^-8, block scale 256, d = 1
    (NI3, 3.0, 5.25, np.array([0.0, 1.0, 2.0, 3.0]), True),  # s_g = 5.25 / 1344 = 2^-8
])
def test_3bit_grids_brute_force(orc, mode, head, amax, levels, even):
    """Every bf16 value up to the grid maximum under a block scale of exactly 1:
    the code is the nearest grid level (ties to the even level index, the
    E2M0 code / the integer), sign in bit 3, zero as code 0."""
    vals = _all_bf16_up_to(levels[-1])
    mat, v = _unit_scale_blocks(vals, head)
    codes, scales, gs = orc.quantize(bits_of(bf16(mat)), ROW, mode, 0, 0, amax_in=amax)
    assert gs == 2.0 ** -8 and np.all(scales[:len(v) // 8] == 0x78)   # E4M3 256
    cu = orc.unpack_codes(codes).reshape(-1, 16)[:len(v), 1:]
    for i in range(len(v)):
        for j in range(15):
            a = abs(float(v[i, j]))
            dist = np.abs(levels - a)
            best = np.flatnonzero(dist == dist.min())
            idx = int(best[0] if len(best) == 1 else best[best % 2 == 0][0])
            exp = 0 if idx == 0 else (idx | (8 if v[i, j] < 0 else 0))
            assert cu[i, j] == exp, (v[i, j], cu[i, j], exp)


def test_if3_picks_lower_error_option(orc):
    wl = W.activation(rows=32, cols=512)
    bits = bits_of(wl.tensors()["a"])
    codes, scales, gs, z = _block_views(orc, bits, ROW, IF3M, 0, 3)
    cu = orc.unpack_codes(codes)
    n_int = 0
    for r in range(z.shape[0]):
        for b in range(z.shape[1] // 16):
            S = int(scales[r, b])
            d = f32(f32(orc.e4m3_decode(S & 0x7F)) * f32(gs))
            if d == 0:
                continue
            y = (z[r, 16 * b:16 * b + 16] * f32(f32(1.0) / d)).astype(np.float32)
            fp = np.array([_nearest_even(E2M0, float(t)) for t in y])
            k = np.clip(np.round((y * f32(0.75)).astype(np.float32)), -3, 3)
            it = (k * f32(4.0 / 3.0)).astype(np.float32).astype(np.float64)
            e_fp, e_int = np.sum((y - fp) ** 2), np.sum((y - it) ** 2)
            flag = bool(S & 0x80)
            n_int += flag
            chosen, other = (e_int, e_fp) if flag else (e_fp, e_int)
            assert chosen <= other * (1 + 1e-5) + 1e-12, (r, b)
            if flag:
                c = cu[r, 16 * b:16 * b + 16]
                kk = np.where(c & 8, -(c & 7).astype(int), (c & 7).astype(int))
                assert np.array_equal(kk, k.astype(int))
    assert 0 < n_int < scales.size


def test_mxfp3_shared_exponent(orc):
    rng = np.random.default_rng(31)
    x = rng.standard_normal((4, 256)) * 2.0 ** rng.integers(-20, 20, (4, 8)).repeat(32, 1)
    xb = bf16(x)
    codes, scales, gs = orc.quantize(bits_of(xb), ROW, MX3, 0, 0)
    assert gs == 1.0
    xv = xb.float().numpy()
    cu = orc.unpack_codes(codes)
    for r in range(4):
        for gi in range(8):
            grp = xv[r, 32 * gi:32 * gi + 32].astype(np.float64)
            E = int(np.clip(np.frexp(np.abs(grp).max())[1] - 1 - 2, -127, 127))
            assert scales[r, 2 * gi] == scales[r, 2 * gi + 1] == E + 127
            vals = np.array([E2M0[c & 3] * (-1 if c & 8 else 1) for c in cu[r, 32 * gi:32 * gi + 32]])
            # every code is a nearest E2M0 level of x / 2^E (saturating at 4)
            y = np.minimum(np.abs(grp / 2.0 ** E), 4.0)
            nearest = np.min(np.abs(E2M0[None, :] - y[:, None]), axis=1)
            assert np.allclose(np.abs(np.abs(vals) - y), nearest)


def test_3bit_error_ordering_follows_the_3bit_table(orc):
    """The IF4 page's 3-bit table ranks the formats by perplexity (IF3 10.67 <
    NVFP3 11.12 < NVINT3 12.78 < MXFP3 70.04).  The quantization MSE under
    the readings ranks them the same way on Gaussian and on Laplace
    per-channel data (reported; gated on the order)."""
    rng = np.random.default_rng(16)
    data = {"N(0,1)": bf16(rng.standard_normal((256, 1024))),
            "laplace channels": W.activation(rows=128, cols=1024).tensors()["a"]}
    for name, x in data.items():
        m = [_mse(orc, x, mode, 0, [0]) for mode in (IF3M, NF3, NI3, MX3)]
        print(f"\n{name}: MSE IF3 {m[0]:.4g}  NVFP3 {m[1]:.4g}  NVINT3 {m[2]:.4g}  MXFP3 {m[3]:.4g}", end="")
        assert m[0] < m[1] < m[2] < m[3]


def test_table1_mse_on_gaussian(orc):
    """The MSE column of the IF4 page's Table 1 (tests/golden/if4_table1_mse.txt):
    NVFP4, 4/6, IF4 and MXFP4 on 2^20 standard normal values, each within 2% of
    the printed value (the table prints two digits; measured: 9.03, 7.57,
    6.15, 13.20, and NVINT4 7.43).  This pins the readings behind 4/6 (two candidate scales,
    original-domain error, M = 256) and IF4 (INT4 levels k * 6/7, y-domain
    error, flag) against numbers the pages print."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "if4_table1_mse.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    rng = np.random.default_rng(16)
    x = bf16(rng.standard_normal((1024, 1024)))
    for name, mode, want in rows:
        got = _mse(orc, x, int(mode), 0, [0]) * 1e3
        print(f"\n{name}: MSE {got:.3f}e-3 (Table 1: {want})", end="")
        assert abs(got - float(want)) <= 0.02 * float(want), (name, got, want)


def test_mxfp4_needs_whole_groups(orc):
    x = bf16(np.ones((4, 48)))
    with pytest.raises(Exception):
        orc.quantize(bits_of(x), ROW, MX, 0, 0)


# ------------------------------------------------------------------- structural
@pytest.mark.parametrize("mode,g", [(RTN, 0), (SR, 0), (EDEN, 128), (IF4, 0), (FO6, 0), (SR, 32), (SS, 0),
                                    (SS, 64), (MX, 0), (MX, 128), (NI4, 0), (NI4, 32),
                                    (NF3, 0), (NI3, 16), (IF3M, 0), (IF3M, 128), (MX3, 0)])
def test_transposed_is_rowwise_of_transpose(orc, mode, g):
    rng = np.random.default_rng(6)
    x = bf16(rng.standard_normal((256, 64)))
    a = orc.quantize(bits_of(x), TR, mode, g, 17)
    b = orc.quantize(bits_of(x.t().contiguous()), ROW, mode, g, 17)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


def test_leading_dimension_and_amax_in(orc):
    rng = np.random.default_rng(7)
    full = bf16(rng.standard_normal((64, 160)))
    bits = bits_of(full)
    cols = 128
    dense = bits_of(full[:, :cols].contiguous())
    for layout in (ROW, TR):
        a = orc.quantize(bits, layout, EDEN, 32, 5, cols=cols)
        b = orc.quantize(dense, layout, EDEN, 32, 5)
        assert all(np.array_equal(u, v) for u, v in zip(a[:2], b[:2])) and a[2] == b[2]
        A = orc.amax(dense, layout, 32, 5)
        c = orc.quantize(dense, layout, EDEN, 32, 5, amax_in=A)
        assert all(np.array_equal(u, v) for u, v in zip(b[:2], c[:2])) and b[2] == c[2]


@pytest.mark.parametrize("mode", [RTN, SR, EDEN, IF4, FO6])
def test_zero_tensor_and_zero_block(orc, mode):
    g = 16 if mode == EDEN else 0
    z = np.zeros((4, 64), dtype=np.uint16)
    codes, scales, gs = orc.quantize(z, ROW, mode, g, 1)
    assert gs == 1.0 and not codes.any() and not scales.any()
    x = np.zeros((4, 64), dtype=np.float32)
    x[1, 20] = 3.0
    codes, scales, gs = orc.quantize(bits_of(bf16(x)), ROW, mode, 0 if mode != EDEN else 16, 1)
    assert scales[1, 1] != 0 and scales[0].sum() == 0 and scales[1, [0, 2, 3]].sum() == 0


def test_nibble_order_and_scale_layout(orc):
    x = np.zeros((2, 32), dtype=np.float32)
    x[0, 0] = 6.0   # element 0 -> low nibble of byte 0
    x[0, 3] = -3.0  # element 3 -> high nibble of byte 1
    x[1, 31] = 1.0  # last element -> high nibble of byte 15, scale index 1
    codes, scales, gs = orc.quantize(bits_of(bf16(x)), ROW, RTN, 0, 0)
    assert gs == np.float32(6.0) / np.float32(2688.0)
    assert codes[0, 0] & 15 == 7 and codes[0, 0] >> 4 == 0
    assert codes[0, 1] >> 4 == 8 | 5 and codes[0, 1] & 15 == 0
    assert codes[1, 15] >> 4 == 7 and scales[1, 0] == 0 and scales[1, 1] != 0
    assert scales.shape == (2, 2) and codes.shape == (2, 16)


def test_rtn_error_bound(orc):
    rng = np.random.default_rng(9)
    x = bf16(rng.standard_normal((32, 256)) * np.exp(rng.uniform(-4, 4, size=(32, 1))))
    for g in (0, 64):
        codes, scales, gs = orc.quantize(bits_of(x), ROW, RTN, g, 2)
        q = deq(orc, codes, scales, gs, RTN, g, 2)
        z = orc.rht_view(bits_of(x), ROW, g, 2) if g else x.float().numpy()
        d = np.vectorize(lambda s: np.float32(orc.e4m3_decode(int(s))) * np.float32(gs))(scales)
        dd = np.repeat(d, 16, axis=1).astype(np.float64)
        y = np.abs(z) / dd
        bound = np.where(y > 6, y - 6, 1.0) * dd * (1 + 1e-5)
        assert np.all(np.abs(q - z) <= bound)


def test_gaussian_top_interval_share_reported(orc):
    """Soft reproduction: about 19.3% of Gaussian values land in [4, 6] under absmax-to-6 SR scaling
    (palettes post, interval decomposition); reported, loosely bounded."""
    rng = np.random.default_rng(10)
    x = bf16(rng.standard_normal((256, 1024)))
    codes, scales, gs = orc.quantize(bits_of(x), ROW, SR, 0, 0)
    d = np.vectorize(lambda s: np.float32(orc.e4m3_decode(int(s))) * np.float32(gs))(scales)
    y = np.abs(x.float().numpy()) / np.repeat(d, 16, axis=1)
    share = np.mean(y >= 4.0)
    print(f"\nshare of |y| in [4,6]: {share:.4f}")
    assert 0.15 < share < 0.21


@pytest.mark.parametrize("mode", [RTN, SR, EDEN, IF4, FO6])
def test_quantize_rotated_equals_quantize(orc, mode):
    """Quantizing the oracle's own rotated view gives the oracle's quantization."""
    rng = np.random.default_rng(12)
    x = bf16(rng.standard_normal((128, 256)))
    for layout in (ROW, TR):
        z = orc.rht_view(bits_of(x), layout, 128, 8)
        a = orc.amax(bits_of(x), layout, 128, 8)
        ref = orc.quantize(bits_of(x), layout, mode, 128, 8)
        got = orc.quantize_rotated(z, mode, 8, a)
        assert np.array_equal(ref[0], got[0]) and np.array_equal(ref[1], got[1]) and ref[2] == got[2]
        # a slice of view rows gives those rows of the full result
        part = orc.quantize_rotated(z[37:41], mode, 8, a, row0=37)
        assert np.array_equal(part[0], ref[0][37:41]) and np.array_equal(part[1], ref[1][37:41])

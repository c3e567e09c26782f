"""Which end-to-end differences of a rotated quantization are explained by the
rotation's rounding.

With a rotation the GPU's rotated values z_g differ from the oracle's z_o by a
few fp32 roundings (another summation order).  The GPU's codes and scales are
checked bit for bit against the oracle applied to z_g; against the oracle
applied to x, a code or scale may then differ only where one of the oracle's
decisions lies within the difference |z_g - z_o| of a decision threshold.
This module names those decisions and their thresholds, and propagates the
block's measured |z_g - z_o| to each decision value:

  block scale   s_f = a_b / RN(m s_g)   (a_b = max |z|, m the element maximum)
                thresholds: midpoints between E4M3 values (round to nearest)
                or the E4M3 values (round up, SR); MX formats: the exponent of
                a_b, thresholds at powers of two
  element       y = z / d, d = dec(S) s_g
                thresholds: the element grid's rounding points (E2M1, INT4,
                INT3, E2M0, and the integer options of IF4 / IF3 at y K1);
                SR: l + U (u - l) with the element's uniform U, and the grid
                points
  MS-EDEN scale t = dec(S) sum(y^2) / sum(y v); threshold lo + U (hi - lo)
                between its E4M3 neighbours, U the block's uniform
  selection     IF4 / IF3 option, 4/6 scale, scale-search candidate:
                the two smallest squared errors, compared

A difference is explained when the oracle's decision value is within the
propagated bound (plus a few fp32 ulps of slack for the evaluation order) of
one of its thresholds.  Values are evaluated in float64 from the oracle's
fp32 z; nothing here computes a code or a scale that is compared.
"""
import numpy as np

import oracle

RTN, SR, MS_EDEN, IF4, FOUR_OVER_SIX, SCALE_SEARCH, MXFP4, NVINT4 = 0, 1, 2, 3, 4, 5, 6, 7
NVFP3, NVINT3, IF3, MXFP3 = 8, 9, 10, 11

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_T = (E2M1_GRID[1:] + E2M1_GRID[:-1]) / 2            # 0.25 0.75 1.25 1.75 2.5 3.5 5
E2M0_T = np.array([0.5, 1.5, 3.0])
SLACK_ULPS = 4

_E4M3 = None


def e4m3_values():
    global _E4M3
    if _E4M3 is None:
        _E4M3 = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], dtype=np.float64)
    return _E4M3


def _ulp32(v):
    return np.spacing(np.abs(np.asarray(v, dtype=np.float32))).astype(np.float64)


def _near(v, thresholds, tol):
    """|v| within tol of any threshold (elementwise over v)."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    t = np.asarray(thresholds, dtype=np.float64)
    return np.any(np.abs(v[..., None] - t) <= np.asarray(tol, dtype=np.float64)[..., None], axis=-1)


def element_max(mode):
    return {NVINT4: 7.0, NVFP3: 4.0, IF3: 4.0, NVINT3: 3.0}.get(mode, 6.0)


def element_thresholds(mode):
    """Rounding points of the element grids a mode uses, in the y domain."""
    if mode in (NVINT4,):
        return [np.arange(7) + 0.5]
    if mode in (NVINT3,):
        return [np.arange(3) + 0.5]
    if mode in (NVFP3, MXFP3):
        return [E2M0_T]
    if mode == IF4:
        k1 = float(np.float32(7.0) / np.float32(6.0))
        return [E2M1_T, (np.arange(7) + 0.5) / k1]
    if mode == IF3:
        return [E2M0_T, (np.arange(3) + 0.5) / 0.75]
    return [E2M1_T]


def _rtn_values(y):
    """Nearest E2M1 value of |y| (float64, saturating), signed."""
    a = np.minimum(np.abs(y), 6.0)
    idx = np.argmin(np.abs(a[..., None] - E2M1_GRID), axis=-1)
    return np.sign(y) * E2M1_GRID[idx]


class Block:
    """One scale group (16 elements; 32 for the MX formats): oracle z_o, GPU
    z_g, tensor scale, the view index of its first element and its first
    16-element block."""

    def __init__(self, mode, z_o, z_g, s_g, seed, elem0, block_index):
        self.mode, self.s_g, self.seed = mode, float(s_g), seed
        self.zo = np.asarray(z_o, dtype=np.float64)
        self.n = self.zo.size
        self.dz = np.abs(np.asarray(z_g, dtype=np.float64) - self.zo)
        self.elem0, self.block_index = elem0, block_index
        self.a_b = float(np.abs(self.zo).max())
        self.da = float(self.dz.max())

    # -- block scale ------------------------------------------------------
    def scale_fragile(self, m=None):
        mode = self.mode
        if mode in (MXFP4, MXFP3):
            # the exponent of the group maximum; the group is this block and its pair,
            # whose maximum is at least a_b: a power of two within reach decides it
            return bool(self.a_b > 0 and abs(self.a_b - 2.0 ** np.round(np.log2(self.a_b))) <=
                        self.da + SLACK_ULPS * _ulp32(self.a_b))
        m = element_max(mode) if m is None else m
        q = float(np.float32(np.float32(m) * np.float32(self.s_g)))
        s_f = self.a_b / q
        tol = self.da / q + SLACK_ULPS * _ulp32(s_f)
        v = e4m3_values()
        points = v if mode == SR else (v[1:] + v[:-1]) / 2
        return bool(_near(s_f, points, tol))

    def _d(self, m=None):
        """d = dec(S) s_g of the oracle's round-to-nearest scale for element maximum m."""
        m = element_max(self.mode) if m is None else m
        q = float(np.float32(np.float32(m) * np.float32(self.s_g)))
        s_f = np.float32(self.a_b / q)
        S = oracle.e4m3_ru_sat(s_f) if self.mode == SR else oracle.e4m3_rne_sat(s_f)
        return float(np.float32(oracle.e4m3_decode(S) * np.float32(self.s_g))), S

    # -- elements ---------------------------------------------------------
    def element_fragile(self):
        """Per element: its y lies near a rounding point of the mode's grids."""
        if self.mode in (MXFP4, MXFP3):
            e = np.floor(np.log2(self.a_b)) - 2 if self.a_b > 0 else -127
            d = 2.0 ** max(e, -127)
        else:
            d, _ = self._d()
        if d == 0:
            return np.zeros(self.n, dtype=bool)
        y = self.zo / d
        tol = self.dz / d + SLACK_ULPS * _ulp32(y) + 1e-300
        out = np.zeros(self.n, dtype=bool)
        for t in element_thresholds(self.mode):
            out |= _near(y, t, tol)
        if self.mode == FOUR_OVER_SIX:
            d4, _ = self._d(4.0)
            if d4:
                y4 = self.zo / d4
                out |= _near(y4, E2M1_T, self.dz / d4 + SLACK_ULPS * _ulp32(y4))
        if self.mode == SR:
            a = np.minimum(np.abs(y), 6.0)
            hi_idx = np.clip(np.searchsorted(E2M1_GRID, a, side="right"), 1, 7)
            lo, hi = E2M1_GRID[hi_idx - 1], E2M1_GRID[hi_idx]
            u = np.array([oracle.uniform_element(self.seed, self.elem0 + i) for i in range(self.n)])
            out |= np.abs(a - (lo + u * (hi - lo))) <= tol
            out |= _near(a, E2M1_GRID[1:], tol)
        return out

    # -- selections and the MS-EDEN scale --------------------------------
    def _err_y(self, d, kind):
        """Squared error per element and its derivative bound in the y domain."""
        y = self.zo / d
        if kind == "fp":
            v = _rtn_values(y)
        elif kind == "if4int":
            k1, k2 = float(np.float32(7.0) / np.float32(6.0)), float(np.float32(6.0) / np.float32(7.0))
            v = np.clip(np.round(y * k1), -7, 7) * k2
        elif kind == "e2m0":
            a = np.minimum(np.abs(y), 4.0)
            g = np.array([0.0, 1.0, 2.0, 4.0])
            v = np.sign(y) * g[np.argmin(np.abs(a[..., None] - g), axis=-1)]
        else:  # if3 integer option
            v = np.clip(np.round(y * 0.75), -3, 3) / 0.75
        r = y - v
        return float(np.sum(r * r)), float(np.sum(2 * np.abs(r) * self.dz / d))

    def selection_fragile(self):
        mode = self.mode
        if mode in (IF4, IF3):
            d, _ = self._d()
            if d == 0:
                return False
            ea, da = self._err_y(d, "fp" if mode == IF4 else "e2m0")
            eb, db = self._err_y(d, "if4int" if mode == IF4 else "if3int")
            return abs(ea - eb) <= da + db + SLACK_ULPS * 2.0 ** -23 * (ea + eb) + 1e-300
        if mode in (FOUR_OVER_SIX, SCALE_SEARCH):
            errs, bounds = [], []
            v = e4m3_values()
            if mode == FOUR_OVER_SIX:
                cands = [self._d(6.0)[1], self._d(4.0)[1]]
            else:
                s0 = self._d(6.0)[1]
                cands = sorted({min(max(s0 + dlt, 0), 0x7E) for dlt in range(-9, 10)})
            for S in cands:
                d = float(np.float32(v[S] * np.float32(self.s_g)))
                if d == 0:
                    deq = np.zeros(self.n)
                else:
                    deq = _rtn_values(self.zo / d) * d
                r = self.zo - deq
                errs.append(float(np.sum(r * r)))
                bounds.append(float(np.sum(2 * np.abs(r) * self.dz)))
            order = np.argsort(errs)
            if len(order) < 2:
                return False
            i, j = order[0], order[1]
            return abs(errs[i] - errs[j]) <= bounds[i] + bounds[j] + SLACK_ULPS * 2.0 ** -23 * (errs[i] + errs[j]) + \
                1e-300
        return False

    def eden_scale_fragile(self):
        d, S = self._d()
        if d == 0:
            return False
        y = self.zo / d
        dy = self.dz / d
        v = _rtn_values(y)
        num, den = float(np.sum(y * y)), float(np.sum(y * v))
        if num <= 0 or den <= 0:
            return False
        dec = e4m3_values()[S]
        t = dec * num / den
        dt = dec * float(np.sum(np.abs(2 * y * den - v * num) * dy)) / den ** 2 + SLACK_ULPS * float(_ulp32(t))
        vals = e4m3_values()
        if t >= 448.0:
            return bool(abs(t - 448.0) <= dt)
        lo_i = int(np.searchsorted(vals, t, side="right") - 1)
        lo, hi = vals[lo_i], vals[min(lo_i + 1, 0x7E)]
        u = oracle.uniform_block(self.seed, self.block_index)
        return bool(abs(t - (lo + u * (hi - lo))) <= dt or abs(t - lo) <= dt or abs(t - hi) <= dt)


def explain(mode, z_o, z_g, s_g, seed, elem0, block_index, codes_differ, scale_differs):
    """Whether the differences of one scale group are explained; returns (bool, reason).

    codes_differ: one boolean per element (codes that differ); scale_differs: bool."""
    b = Block(mode, z_o, z_g, s_g, seed, elem0, block_index)
    ef = b.element_fragile()
    if scale_differs:
        if mode not in (MXFP4, MXFP3) and b.scale_fragile():
            return True, "block scale near an E4M3 decision point"
        if mode in (MXFP4, MXFP3) and b.scale_fragile():
            return True, "group maximum near a power of two"
        if mode == FOUR_OVER_SIX and b.scale_fragile(4.0):
            return True, "4/6: the m = 4 scale near an E4M3 decision point"
        if b.selection_fragile():
            return True, "selection errors within the bound"
        if mode == MS_EDEN and (b.eden_scale_fragile() or ef.any()):
            return True, "MS-EDEN corrected scale near its stochastic-rounding threshold"
        return False, "scale differs with no decision near a threshold"
    cd = np.asarray(codes_differ, dtype=bool)
    if np.all(ef[cd]):
        return True, "every differing element near a rounding point"
    if b.selection_fragile():
        return True, "selection errors within the bound"
    return False, f"elements {np.flatnonzero(cd & ~ef).tolist()} differ away from every rounding point"

"""The kernels' code searches, restated on the CPU: a table on a uniform grid gives exactly
the number of thresholds (NF4: midpoints) strictly below a value, for every fp32 value.

A table cuts the value range into cells that hold at most one threshold; for y in cell k
  #{t < y} = #{t < left edge of cell k} + [y > the threshold inside cell k].
How the kernels find the cell:
- Block-GTQ widths 2..7: v = y 2^-p + 1/2 rounded toward -infinity and saturated to [0, 1]
  (NaN to 0), then cell = floor(v 2^q); the grid is [-2^(p-1), 2^(p-1)) in cells of 2^(p-q),
  plus a top cell 2^q for v = 1.
- Block-GTQ width 8: y clamped into [-K/s, (K - 1/2)/s] (NaN to the lowest cell), then
  cell = floor(y s) + K.
- NF4: u in [-1, 1): v = u/2 + 1/2 as above, cell = floor(32 v), top cell 32.
This test checks the grid property on the stored thresholds (the oracle's codebooks and NF4
midpoints) and the identity on random values, on every threshold and cell edge and their
fp32 neighbours, and on zeros, infinities, huge and tiny values and NaN. The rounding toward
-infinity of the kernels' multiply-add is reproduced exactly with rational arithmetic.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import codebooks as cb

SAT_P = {2: 1, 3: 2, 4: 3, 5: 3, 6: 3, 7: 3}            # range 2^(p-1)
SAT_Q = {2: 2, 3: 3, 4: 5, 5: 6, 6: 7, 7: 8}            # 2^q cells
HALF_CELLS_8 = 288
SCALE_8 = 64.0


def _f32_down(x: Fraction) -> np.float32:
    """The largest fp32 value not above x (x finite)."""
    v = np.float32(float(x))
    while Fraction(float(v)) > x:
        v = np.nextafter(v, np.float32(-np.inf))
    return v


def _sat_cell(y: np.float32, p: int, q: int) -> int:
    """floor(2^q * sat(round_down(y 2^-p + 1/2))), NaN -> 0."""
    if np.isnan(y):
        return 0
    if np.isinf(y):
        return (1 << q) if y > 0 else 0
    exact = Fraction(float(y)) / (1 << p) + Fraction(1, 2)
    if exact <= 0:
        return 0
    if exact >= 1:
        return 1 << q
    v = _f32_down(exact)
    return int(np.floor(Fraction(float(v)) * (1 << q)))


def _table(t: np.ndarray, lo0: float, cw: float, cells: int, top_open: bool):
    below, tau = [], []
    for k in range(cells):
        lo = lo0 + k * cw
        hi = np.inf if (top_open and k == cells - 1) else lo + cw
        inside = [x for x in t if lo <= float(x) < hi]
        assert len(inside) <= 1, (k, inside)
        below.append(int(np.sum(t.astype(np.float64) < lo)))
        tau.append(inside[0] if inside else np.float32(np.inf))
    return np.array(below), np.array(tau, dtype=np.float32)


def _values(t: np.ndarray, edges: np.ndarray, seed: int, scale: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    parts = [(rng.standard_normal(4000) * scale).astype(np.float32),
             np.array([0.0, -0.0, np.inf, -np.inf, 1e30, -1e30, 1e-40, -1e-40, 3.4e38, -3.4e38], np.float32)]
    for anchors in (t.astype(np.float32), edges.astype(np.float32)):
        parts += [anchors, np.nextafter(anchors, np.float32(np.inf)), np.nextafter(anchors, np.float32(-np.inf))]
    return np.concatenate(parts).astype(np.float32)


@pytest.mark.parametrize("w", sorted(SAT_P))
def test_saturating_grid_equals_threshold_count(w):
    _, t = cb.stored_codebook(w)
    t = t.astype(np.float32)
    p, q = SAT_P[w], SAT_Q[w]
    R = float(1 << (p - 1))
    assert float(t[0]) >= -R and float(t[-1]) < R
    cw = 2.0 ** (p - q)
    below, tau = _table(t, -R, cw, (1 << q) + 1, top_open=True)
    y = _values(t, np.arange(-R - 3 * cw, R + 3 * cw, cw), w, 3.0)
    got = np.array([below[c] + (yy > tau[c]) for yy, c in ((yy, _sat_cell(yy, p, q)) for yy in y)])
    np.testing.assert_array_equal(got, np.searchsorted(t, y, side="left"))
    assert below[_sat_cell(np.float32(np.nan), p, q)] + 0 == 0


def test_clamped_grid_equals_threshold_count_width8():
    _, t = cb.stored_codebook(8)
    t = t.astype(np.float32)
    K, s = HALF_CELLS_8, SCALE_8
    assert float(t[0]) >= -K / s and float(t[-1]) < K / s
    below, tau = _table(t, -K / s, 1.0 / s, 2 * K, top_open=False)
    y = _values(t, np.arange(-K - 3, K + 3) / s, 8, 3.0)
    lo, hi = np.float32(-K / s), np.float32((K - 0.5) / s)
    yc = np.minimum(np.maximum(np.where(np.isnan(y), lo, y), lo), hi)
    cell = (np.floor(yc.astype(np.float64) * s) + K).astype(np.int64)
    got = below[cell] + (y > tau[cell])
    np.testing.assert_array_equal(got, np.searchsorted(t, y, side="left"))


def test_nf4_grid_equals_midpoint_count():
    m = np.asarray(cb.nf4_midpoints(), dtype=np.float32)
    assert float(m[0]) >= -1.0 and float(m[-1]) < 1.0
    below, tau = _table(m, -1.0, 1.0 / 16.0, 33, top_open=True)
    u = _values(m, np.arange(-1.25, 1.25, 1.0 / 16.0), 5, 0.5)
    got = np.array([below[c] + (uu > tau[c]) for uu, c in ((uu, _sat_cell(uu, 1, 5)) for uu in u)])
    np.testing.assert_array_equal(got, np.searchsorted(m, u, side="left"))

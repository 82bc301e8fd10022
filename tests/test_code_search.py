"""The quantizer's code search, restated on the CPU: a table on a uniform grid gives exactly
the number of thresholds strictly below y, for every fp32 y.

For width w (2..8) the kernel cuts [-R_w, R_w) into cells of 1/s_w with s_w = 2^max(w-2, 1)
and R_w = 1, 2, 2.5, 3, 3.5, 4, 4.5. If no cell holds two thresholds, then for y in cell k
  #{t < y} = #{t < left edge of cell k} + [y > the threshold inside cell k],
with y clamped into the grid first (a NaN clamps to the lowest cell and compares false, so
it gets code 0). This test checks the grid property on the stored thresholds (the oracle's
codebooks) and the identity on random values, on every threshold and cell edge and their
fp32 neighbours, and on zeros, infinities, huge values and NaN.
"""
import numpy as np
import pytest

from oracle import codebooks as cb

HALF_CELLS = {2: 2, 3: 4, 4: 10, 5: 24, 6: 56, 7: 128, 8: 288}


def _scale(w):
    return float(1 << max(w - 2, 1))


def _table(w):
    _, t = cb.stored_codebook(w)
    t = t.astype(np.float32)
    K, s = HALF_CELLS[w], _scale(w)
    below, tau = [], []
    for k in range(2 * K):
        lo, hi = (k - K) / s, (k - K + 1) / s
        inside = [x for x in t if lo <= float(x) < hi]
        assert len(inside) <= 1, (w, k, inside)
        below.append(int(np.sum(t.astype(np.float64) < lo)))
        tau.append(inside[0] if inside else np.float32(np.inf))
    assert float(t[0]) >= -K / s and float(t[-1]) < K / s
    return t, np.array(below), np.array(tau, dtype=np.float32)


def _grid_code(y, w, below, tau):
    K, s = HALF_CELLS[w], _scale(w)
    lo, hi = np.float32(-K / s), np.float32((K - 0.5) / s)
    yc = np.minimum(np.maximum(np.where(np.isnan(y), lo, y), lo), hi)
    cell = (np.floor(yc.astype(np.float64) * s) + K).astype(np.int64)
    assert cell.min() >= 0 and cell.max() < 2 * K
    return below[cell] + (y > tau[cell])


@pytest.mark.parametrize("w", sorted(HALF_CELLS))
def test_grid_search_equals_threshold_count(w):
    t, below, tau = _table(w)
    K, s = HALF_CELLS[w], _scale(w)
    rng = np.random.default_rng(w)
    parts = [rng.standard_normal(50000).astype(np.float32) * 3,
             np.array([0.0, -0.0, np.inf, -np.inf, 1e30, -1e30, 1e-40, -1e-40, 3.4e38, -3.4e38], np.float32)]
    for anchors in (t, (np.arange(-K - 3, K + 3) / s).astype(np.float32)):
        parts += [anchors, np.nextafter(anchors, np.float32(np.inf)), np.nextafter(anchors, np.float32(-np.inf))]
    y = np.concatenate(parts).astype(np.float32)
    got = _grid_code(y, w, below, tau)
    ref = np.searchsorted(t, y, side="left")          # number of thresholds strictly below y
    np.testing.assert_array_equal(got, ref)
    nan_code = _grid_code(np.array([np.nan], np.float32), w, below, tau)
    assert nan_code[0] == 0

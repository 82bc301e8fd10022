"""Pins for the CPU oracle: closed forms, textbook constants, brute force, invariants.

None of these compares the oracle with itself: each value on the right-hand
side comes from mathematics, an independent routine (quadrature, exhaustive
search, dynamic programming, Monte Carlo) or a published constant.
"""
import itertools
import math
import os

import numpy as np
import pytest
from scipy import integrate
from scipy.stats import norm

from oracle import blockgtq as bg
from oracle import codebooks as cb
from oracle import nqkv
from oracle import rope

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return rows


# ----------------------------------------------------------------- pin 1: RoPE blocks

def test_rope_logit_is_sum_of_block_terms():
    """Block-GTQ abstract: under RoPE a key's logit contribution is a position-dependent
    sum over 2-D frequency blocks. Checked at every key position of the tiny workload."""
    rng = np.random.default_rng(0)
    d, base = 128, 1e4
    q = rng.standard_normal(d)
    for n in range(512):
        k = rng.standard_normal(d) * 10.0 ** rng.uniform(-1, 1, d)
        direct = float(np.dot(rope.rotate(q, 512.0, base), rope.rotate(k, float(n), base)))
        terms = rope.block_logit_terms(q, k, 512.0, float(n), base)
        assert abs(math.fsum(terms) - direct) <= 1e-12 * max(1.0, float(np.sum(np.abs(q) * np.abs(k))))


def test_rope_preserves_block_energy():
    rng = np.random.default_rng(1)
    k = rng.standard_normal(128) * 3.0
    e0 = rope.block_energy(k)
    for pos in (1.0, 17.0, 511.0, 131071.0):
        e1 = rope.block_energy(rope.rotate(k, pos, 1e6))
        np.testing.assert_allclose(e1, e0, rtol=1e-13, atol=0)


def test_rope_pairing_is_rotate_half():
    """A planted change of pairing (adjacent dims instead of (i, i + d/2)) breaks the identity."""
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal(8), rng.standard_normal(8)
    perm = np.array([0, 2, 4, 6, 1, 3, 5, 7])           # interleaved pairing
    direct = np.dot(rope.rotate(q, 5.0, 1e4), rope.rotate(k, 2.0, 1e4))
    wrong = np.sum(rope.block_logit_terms(q[perm], k[perm], 5.0, 2.0, 1e4))
    assert abs(direct - wrong) > 1e-6


# ----------------------------------------------------------------- pin 2: Lloyd-Max

def test_lloyd_max_closed_form_one_bit():
    c, t = cb.lloyd_max_f64(1)
    assert abs(c[1] - math.sqrt(2.0 / math.pi)) < 1e-14
    assert abs(c[0] + math.sqrt(2.0 / math.pi)) < 1e-14
    assert t[0] == 0.0
    assert abs(cb.quantizer_mse(c, t) - (1.0 - 2.0 / math.pi)) < 1e-14


def test_lloyd_max_textbook_distortions():
    """Agreement within one unit of the last quoted digit (the table quotes 4 significant
    digits; 0.0345478 is quoted as 0.03454 there)."""
    for bits, mse in _golden_rows("lloyd_max_textbook.txt"):
        c, t = cb.lloyd_max_f64(int(bits))
        got = cb.quantizer_mse(c, t)
        unit = 10.0 ** (math.floor(math.log10(mse)) - 3)
        assert abs(got - mse) <= unit, (bits, got, mse)


@pytest.mark.parametrize("w", [1, 2, 3, 4, 5, 6])
def test_lloyd_max_centroids_are_conditional_means(w):
    """Independent check by adaptive quadrature of x phi(x) and phi(x) over each cell."""
    c, t = cb.lloyd_max_f64(w)
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    for ci, ai, bi in zip(c, a, b):
        num = integrate.quad(lambda x: x * norm.pdf(x), ai, bi, epsabs=1e-14, epsrel=1e-13)[0]
        den = integrate.quad(norm.pdf, ai, bi, epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(num / den - ci) < 1e-11
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=0)


def test_lloyd_max_mse_by_quadrature():
    for w in (2, 3, 4, 8):
        c, t = cb.lloyd_max_f64(w)
        a = np.concatenate([[-np.inf], t])
        b = np.concatenate([t, [np.inf]])
        mse = math.fsum(integrate.quad(lambda x: (x - ci) ** 2 * norm.pdf(x), ai, bi,
                                       epsabs=1e-15, epsrel=1e-13)[0] for ai, bi, ci in zip(a, b, c))
        assert abs(mse - cb.quantizer_mse(c, t)) < 1e-12


def test_stored_codebooks_symmetric_and_sorted():
    for w in range(1, 9):
        c16, t32 = cb.stored_codebook(w)
        assert len(c16) == 2 ** w and len(t32) == 2 ** w - 1
        assert np.all(np.diff(c16.astype(np.float64)) > 0)
        assert np.all(np.diff(t32.astype(np.float64)) > 0)
        np.testing.assert_array_equal(c16, -c16[::-1])
        assert t32[(len(t32) - 1) // 2] == 0.0          # middle threshold is exactly 0
        # each stored centroid is the fp16 value nearest the exact one
        exact, _ = cb.lloyd_max_f64(w)
        assert np.all(np.abs(c16.astype(np.float64) - exact) <= np.spacing(np.abs(c16)).astype(np.float64) / 2)


def test_delta_table_convex_and_close_to_exact():
    delta = cb.delta_table().astype(np.float64)
    assert delta[0] == 1.0
    gains = delta[:-1] - delta[1:]
    assert np.all(gains > 0)
    assert np.all(np.diff(gains) < 0)                   # strictly convex
    for w in range(1, 9):
        # The exact Lloyd-Max quantizer is MSE-optimal, so rounding its centroids to fp16 can
        # only raise the MSE, and by at most the largest squared centroid shift.
        c, t = cb.lloyd_max_f64(w)
        exact = cb.quantizer_mse(c, t)
        shift = np.max(np.abs(cb.stored_codebook(w)[0].astype(np.float64) - c))
        assert exact * (1 - 1e-7) <= delta[w] <= exact * (1 + 1e-7) + shift ** 2


def test_delta_table_is_the_stored_quantizers_mse():
    """delta[w] is the MSE on N(0,1) of the quantizer as stored (fp16 centroids, fp32
    thresholds), by adaptive quadrature of (x - c)^2 phi(x) over its cells, within one fp32
    ulp; for w >= 3 that is several ulps away from the exact Lloyd-Max MSE, so the table
    cannot be the exact quantizer's."""
    delta = cb.delta_table()
    for w in range(1, 9):
        c16, t32 = cb.stored_codebook(w)
        c = c16.astype(np.float64)
        edges = np.concatenate([[-np.inf], t32.astype(np.float64), [np.inf]])
        mse = math.fsum(integrate.quad(lambda x: (x - ci) ** 2 * norm.pdf(x), lo, hi, epsabs=1e-16, epsrel=1e-13)[0]
                        for lo, hi, ci in zip(edges[:-1], edges[1:], c))
        ulp = float(np.spacing(delta[w]))
        assert abs(float(delta[w]) - mse) <= ulp, (w, float(delta[w]), mse)
        if w >= 3:
            ce, te = cb.lloyd_max_f64(w)
            assert abs(float(delta[w]) - cb.quantizer_mse(ce, te)) > 2 * ulp


@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_stored_quantizer_monte_carlo(w):
    """10^7 N(0,1) draws through the fp32 threshold quantizer: MSE within 3 sigma of delta(w)."""
    rng = np.random.default_rng(100 + w)
    x = rng.standard_normal(10_000_000).astype(np.float32)
    c16, t32 = cb.stored_codebook(w)
    codes = np.searchsorted(t32, x, side="left")
    err = (x.astype(np.float64) - c16.astype(np.float64)[codes]) ** 2
    mean, sd = err.mean(), err.std() / math.sqrt(len(err))
    assert abs(mean - float(cb.delta_table()[w])) < 3 * sd


def test_threshold_count_is_nearest_centroid():
    """code = #{t < y} equals the brute-force nearest fp16 centroid (away from exact ties)."""
    rng = np.random.default_rng(3)
    for w in range(1, 9):
        c16, t32 = cb.stored_codebook(w)
        y = (rng.standard_normal(20000) * 1.5).astype(np.float32)
        codes = np.sum(y[:, None] > t32[None, :], axis=1)
        dist = np.abs(y[:, None].astype(np.float64) - c16[None, :].astype(np.float64))
        near = np.argmin(dist, axis=1)
        srt = np.sort(dist, axis=1)
        clear = srt[:, 1] - srt[:, 0] > 1e-6
        np.testing.assert_array_equal(codes[clear], near[clear])


# ----------------------------------------------------------------- pin 3: NF4

def test_nf4_matches_published_table():
    vals = np.array([r[0] for r in _golden_rows("nf4_qlora.txt")])
    got = cb.nf4_values().astype(np.float64)
    assert got.shape == (16,)
    np.testing.assert_allclose(got, vals, rtol=0, atol=5e-7)


def test_nf4_structure_and_quantile_spacing():
    v = cb.nf4_values().astype(np.float64)
    assert np.all(np.diff(v) > 0) and v[0] == -1.0 and v[-1] == 1.0
    assert np.sum(v == 0.0) == 1 and np.sum(v < 0) == 7 and np.sum(v > 0) == 8
    # Undo the normalisation with the quantile of the outermost level; the levels are then
    # standard-normal quantiles at evenly spaced probabilities on each side (scipy's norm.cdf).
    off = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))
    z = norm.ppf(off)
    ppos = norm.cdf(v[v > 0] * z)
    pneg = norm.cdf(-v[v < 0] * z)
    np.testing.assert_allclose(np.diff(ppos), (off - 0.5) / 8, rtol=1e-5)
    np.testing.assert_allclose(np.diff(np.sort(pneg)), (off - 0.5) / 7, rtol=1e-5)


def test_nf4_midpoints_between_levels():
    v = cb.nf4_values()
    m = cb.nf4_midpoints()
    assert np.all(m > v[:-1]) and np.all(m < v[1:])


# ----------------------------------------------------------------- pin 4/5/6: greedy allocation

def _objective(E, w):
    delta = cb.delta_table().astype(np.float64)
    return math.fsum(float(e) * delta[int(x)] for e, x in zip(E, w))


def _brute_min(E, bits, w_max):
    h = len(E)
    delta = cb.delta_table().astype(np.float64)
    grid = np.array(list(itertools.product(range(w_max + 1), repeat=h)), dtype=np.int64)
    grid = grid[grid.sum(axis=1) == bits * h]
    obj = (delta[grid] * np.asarray(E)[None, :]).sum(axis=1)
    best = obj.min()
    return best, grid[np.isclose(obj, best, rtol=1e-13, atol=0)]


def _dp_min(E, bits, w_max):
    delta = cb.delta_table().astype(np.float64)
    budget = bits * len(E)
    dp = np.full(budget + 1, np.inf)
    dp[0] = 0.0
    for e in E:
        nxt = np.full(budget + 1, np.inf)
        for s in range(budget + 1):
            for w in range(min(w_max, s) + 1):
                nxt[s] = min(nxt[s], dp[s - w] + e * delta[w])
        dp = nxt
    return dp[budget]


@pytest.mark.parametrize("d", [4, 8, 12])
def test_greedy_matches_exhaustive_search(d):
    rng = np.random.default_rng(d)
    h = d // 2
    for trial in range(3):
        E = np.exp(rng.standard_normal(h) * 1.5)
        for bits in range(1, 9):
            w = bg.greedy_widths(E, bits, 8)
            assert int(w.sum()) == bits * h
            best, argmins = _brute_min(E, bits, 8)
            assert abs(_objective(E, w) - best) <= 1e-12 * best
            if len(argmins) == 1:
                np.testing.assert_array_equal(w, argmins[0])


def test_greedy_matches_dynamic_programming_d16():
    rng = np.random.default_rng(16)
    for trial in range(3):
        E = np.exp(rng.standard_normal(8) * 2.0)
        for bits in range(1, 9):
            w = bg.greedy_widths(E, bits, 8)
            best = _dp_min(E, bits, 8)
            assert abs(_objective(E, w) - best) <= 1e-12 * best


def test_greedy_budget_and_wmax():
    rng = np.random.default_rng(5)
    E = np.exp(rng.standard_normal(64) * 2.0)
    E[[3, 40]] *= 400.0
    for bits in (2, 3, 4):
        for w_max in (bits, 6, 8):
            w = bg.greedy_widths(E, bits, w_max)
            assert int(2 * w.sum()) == bits * 128            # allocated bits equal the budget
            assert w.max() <= w_max and w.min() >= 0
    assert np.all(bg.greedy_widths(E, 4, 4) == 4)            # budget at w_max forces uniform
    with pytest.raises(ValueError):
        bg.greedy_widths(E, 5, 4)


def test_greedy_tie_breaks_to_lowest_block():
    w = bg.greedy_widths(np.array([1.0, 1.0, 1.0]), 1, 8)
    np.testing.assert_array_equal(w, [1, 1, 1])
    # one step only: three equal candidates, the first wins
    E = np.array([2.0, 2.0])
    delta = cb.delta_table().astype(np.float64)
    w = np.zeros(2, dtype=int)
    gains = [E[b] * (delta[w[b]] - delta[w[b] + 1]) for b in range(2)]
    assert gains[0] == gains[1]
    np.testing.assert_array_equal(bg.greedy_widths(E, 1, 8), [1, 1])
    # a tie that decides the result: E = (1, 1, 4), budget 3. With delta = (1, 0.3634,
    # 0.1175, 0.0345, ..) the gains are: step 1 (0.637, 0.637, 2.55) -> block 2; step 2
    # (0.637, 0.637, 0.984) -> block 2; step 3 (0.637, 0.637, 0.332): blocks 0 and 1 tie
    # exactly (the same product), the lower one wins -> (1, 0, 2), not (0, 1, 2)
    E = np.array([1.0, 1.0, 4.0])
    assert E[2] * (delta[1] - delta[2]) > delta[0] - delta[1] > E[2] * (delta[2] - delta[3])
    np.testing.assert_array_equal(bg.greedy_widths(E, 1, 8), [1, 0, 2])
    assert _objective(E, [1, 0, 2]) == _objective(E, [0, 1, 2])      # both optimal: only the rule decides


def test_equal_energies_give_uniform_tqmse():
    d = 128
    E = np.ones((1, 64))
    for bits in (2, 3, 4):
        a = bg.allocate(E, d, bits)
        assert np.all(a["w"] == bits)
        assert np.all(a["g"] == np.float32(1.0))
        assert np.all(a["f"] == np.float32(1.0 / math.sqrt(d)))
        rng = np.random.default_rng(bits)
        X = rng.standard_normal((2, 1, 40, d)).astype(np.float32)
        u = bg.allocate(E, d, bits, mode=bg.MODE_UNIFORM)
        c1 = bg.quantize(X, X, a, bits)
        c2 = bg.quantize(X, X, u, bits)
        np.testing.assert_array_equal(c1["Kc"], c2["Kc"])
        np.testing.assert_array_equal(c1["Kn"], c2["Kn"])


def test_block_gains_restore_unit_variance():
    """After the global sqrt(d)/||k|| scaling, block b's coordinates have variance
    (E_b/2) d / sum E; g_b^2 times that is 1 for every block (closed form)."""
    rng = np.random.default_rng(9)
    E = np.exp(rng.standard_normal(64))
    g, f = bg.block_gains(E, 128)
    var = (E / 2.0) * 128 / E.sum()
    np.testing.assert_allclose(g.astype(np.float64) ** 2 * var, 1.0, rtol=2e-7)
    np.testing.assert_allclose(f.astype(np.float64) * math.sqrt(128) * g.astype(np.float64), 1.0, rtol=2e-7)


# ----------------------------------------------------------------- calibration energy

def test_energy_matches_exact_mean():
    rng = np.random.default_rng(11)
    K = (rng.standard_normal((3, 2, 200, 16)) * 10.0 ** rng.uniform(-1, 1, 16)).astype(np.float32)
    E, N = bg.calibration_energies(K, n_calib=150)
    assert N == 450
    for hh in range(2):
        X = K[:, hh, :150].reshape(-1, 16).astype(np.float64)
        for b in range(8):
            exact = math.fsum((X[:, b] ** 2 + X[:, b + 8] ** 2).tolist()) / N
            assert abs(E[hh, b] - exact) <= 1e-13 * exact


def crafted_energy_keys():
    """bf16-exact keys [1][1][8192][128] whose fp64 energies depend on the summation order.

    8192 pooled tokens = 128 chunks of 64 = 2 segments of 64 chunks. Block b sums
    x_b^2 + x_{b+64}^2; only blocks 0..3 are non-zero. The large terms are powers of two,
    so a small term is lost exactly when it is below half an ulp of the running sum, or a tie
    against an even mantissa.
    """
    K = np.zeros((1, 1, 8192, 128), dtype=np.float32)
    # block 0: 2^53 (x = y = 2^26) at u = 0, then 1 at the first token of chunks 1..127
    K[0, 0, 0, 0] = K[0, 0, 0, 64] = 2.0 ** 26
    K[0, 0, 64::64, 0] = 1.0
    # block 1: 2^54 (x = 2^27) at u = 0; 1 at u = 1..63 (chunk 0) and u = 64..127 (chunk 1)
    K[0, 0, 0, 1] = 2.0 ** 27
    K[0, 0, 1:128, 1] = 1.0
    # block 2: 2^52 (x = 2^26) at u = 63, the last token of chunk 0; 0.25 (x = 0.5) at u = 0..62
    K[0, 0, 63, 2] = 2.0 ** 26
    K[0, 0, 0:63, 2] = 0.5
    # block 3: 2^53 (x = y = 2^26) at u = 4096, the first token of segment 1; 1 at the
    # first token of every other chunk
    K[0, 0, 4096, 3] = K[0, 0, 4096, 67] = 2.0 ** 26
    K[0, 0, 0::64, 3] = 1.0
    K[0, 0, 4096, 3] = 2.0 ** 26
    return K


def test_energy_summation_order_by_hand():
    """Reading R2 fixes the fp64 order of the energy sum: 64-token chunks, 64-chunk segments,
    then the segments, each level left to right. Worked by hand (N = 8192):
      block 0: chunk 0 = 2^53, chunks 1..127 = 1 each. Segment 0 = 2^53 + 63 ones, each a tie
        that rounds back to 2^53 (ulp 2); segment 1 = 64 (exact). E = (2^53 + 64) / 8192
        = 2^40 + 2^-7. (Summing the chunk sums straight, or the tokens, loses all 127 ones:
        2^40; chunks of 32 or segments of 32 chunks keep 96: 2^40 + 96/8192.)
      block 1: chunk 0 = 2^54 + 63 ones, each below half an ulp (2) -> 2^54; chunk 1 = 64,
        added exactly. E = (2^54 + 64) / 8192 = 2^41 + 2^-7. (Chunks of 128 lose the 64.)
      block 2: inside chunk 0, 63 quarters sum exactly to 15.75 before 2^52 arrives (ulp 1):
        2^52 + 15.75 rounds to 2^52 + 16. E = (2^52 + 16) / 8192 = 2^39 + 2^-9. (Summing
        the chunk right to left loses every quarter: 2^39.)
      block 3: segment 0 = 64 ones = 64; segment 1 = 2^53 + 63 ones lost = 2^53. E =
        (64 + 2^53) / 8192 = 2^40 + 2^-7. (A sum of the chunk sums left to right gives the
        same; starting from the large term loses the first segment's 64: 2^40.)
    """
    K = crafted_energy_keys()
    E, N = bg.calibration_energies(K.astype(np.float32), 0)
    assert N == 8192
    want = [2.0 ** 40 + 2.0 ** -7, 2.0 ** 41 + 2.0 ** -7, 2.0 ** 39 + 2.0 ** -9, 2.0 ** 40 + 2.0 ** -7]
    for b, v in enumerate(want):
        assert E[0, b] == v, (b, E[0, b], v)
    assert np.all(E[0, 4:] == 0.0)


def test_energy_is_rope_invariant():
    rng = np.random.default_rng(12)
    d, T = 32, 300
    k0 = rng.standard_normal((T, d)) * 10.0 ** rng.uniform(-1, 1, d // 2).repeat(2).reshape(2, -1).T.reshape(-1)
    k1 = np.stack([rope.rotate(k0[t], float(t), 1e4) for t in range(T)])
    E0, _ = bg.calibration_energies(k0[None, None], 0)
    E1, _ = bg.calibration_energies(k1[None, None], 0)
    np.testing.assert_allclose(E1, E0, rtol=1e-12)


# ----------------------------------------------------------------- pin 8: quantizer

def test_quantizer_zero_row_and_known_norm():
    X = np.zeros((2, 128), dtype=np.float32)
    X[1] = 1.0
    for w in (1, 3, 8):
        codes, n16 = bg.quantize_rows(X, np.full(128, w), np.ones(128, np.float32))
        assert n16[0] == 0 and np.all(codes[0] == 2 ** (w - 1) - 1)   # y = 0 sits on the middle threshold
        assert float(n16[1]) == 11.3125                                  # fp16(sqrt(128))
    # y = 1 * fp32(sqrt 128) / 11.3125 = 1.000107..., width 1: above 0 -> code 1
    codes, _ = bg.quantize_rows(X[1:], np.full(128, 1), np.ones(128, np.float32))
    assert np.all(codes == 1)


def test_quantizer_tie_goes_to_lower_code():
    """A coordinate landing exactly on a threshold takes the lower code.

    d = 4, row (t, r, 0, 0) with r chosen so the fp16 norm is exactly 2; then
    a = fp32(sqrt 4) / 2 = 1 and y_0 = t, the sixth width-3 threshold.
    """
    c16, t32 = cb.stored_codebook(3)
    x = np.zeros(4, dtype=np.float32)
    x[0] = t32[5]
    x[1] = np.float32(math.sqrt(4.0 - float(x[0]) ** 2))
    codes, n16 = bg.quantize_rows(x[None], np.full(4, 3), np.ones(4, np.float32))
    assert float(n16[0]) == 2.0
    assert codes[0, 0] == 5                      # thresholds 0..4 lie strictly below y_0
    x[0] = np.nextafter(t32[5], np.float32(10))
    codes, _ = bg.quantize_rows(x[None], np.full(4, 3), np.ones(4, np.float32))
    assert codes[0, 0] == 6
    # with the block gain g_0 = 2 the coordinate t/2 lands on the threshold (y_0 = (t/2 * 1) * 2
    # = t exactly: code 5), and the next fp32 value above t/2 lands above it (code 6)
    g = np.ones(4, np.float32)
    g[0] = 2.0
    x[0] = t32[5] / np.float32(2)
    x[1] = np.float32(math.sqrt(4.0 - float(x[0]) ** 2))              # the norm stays exactly 2
    codes, n16 = bg.quantize_rows(x[None], np.full(4, 3), g)
    assert float(n16[0]) == 2.0 and codes[0, 0] == 5
    x[0] = np.nextafter(t32[5] / np.float32(2), np.float32(10))
    codes, n16 = bg.quantize_rows(x[None], np.full(4, 3), g)
    assert float(n16[0]) == 2.0 and codes[0, 0] == 6


def _norm_row(ones_at):
    """fp32 row of 128: 4098 at coordinate 0, 1.0 at the given coordinates, 0 elsewhere."""
    x = np.zeros(128, dtype=np.float32)
    x[0] = 4098.0
    x[list(ones_at)] = 1.0
    return x


def test_row_norm_summation_order_by_hand():
    """Reading R5 fixes the fp32 order of the sum of squares: eight partial sums over
    j = r (mod 8), j ascending, combined ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7)).

    Worked by hand. 4098^2 = 16793604 is exact in fp32 (ulp 2 in [2^24, 2^25)), and its
    square root 4098 is the midpoint of the fp16 neighbours 4096 and 4100, so it rounds to
    4096 (even mantissa); any extra mass that survives gives a root above 4098 and the fp16
    norm 4100. Adding 1 to an even value v in [2^24, 2^25) is a tie and rounds back to v:
    a lone 1 added after the large square is lost, while 1s summed among themselves first
    survive once they reach 2.
      A: 1s at j = 1..127. s0 absorbs the 15 at j = 8, 16, ..; s1..s7 = 16 each; the tree
         adds 112 -> 16793716 -> 4100. (A left-to-right sum loses every 1 -> 4096.)
      B: 1s at j = 4 (mod 8). They all land in s4 = 16 -> 16793620 -> 4100. (Partial sums
         mod 4 put them in s0 with the large square, where each is lost -> 4096.)
      C: 1s at j = 0 (mod 8), j > 0. All fall into s0 after the large square: lost -> 4096.
         (An exact fp64 sum keeps them -> 4100.)
      D: 1s at j = 2, 3, 6, 7. s2 + s3 = 2 and s6 + s7 = 2; (s0 + s1) + (s2 + s3) = 16793606,
         plus (s4 + s5) + (s6 + s7) = 2 gives 16793608, whose root 4098.000488 is above the
         midpoint -> 4100. (Combining s0 .. s7 one after the other loses every 1 -> 4096.)
    Codes at width 3 (g = 1): the 4098 coordinate lands far above every threshold (code
    7), the 1s just above the middle threshold 0 (code 4), the zeros on it (code 3).
    """
    cases = {"A": (range(1, 128), 4100.0), "B": (range(4, 128, 8), 4100.0),
             "C": (range(8, 128, 8), 4096.0), "D": ((2, 3, 6, 7), 4100.0)}
    for name, (ones, want) in cases.items():
        x = _norm_row(ones)
        codes, n16 = bg.quantize_rows(x[None], np.full(128, 3), np.ones(128, np.float32))
        assert float(n16[0]) == want, name
        expect = np.full(128, 3, dtype=np.uint8)
        expect[list(ones)] = 4
        expect[0] = 7
        np.testing.assert_array_equal(codes[0], expect, err_msg=name)


def test_nan_coordinate_takes_code_zero():
    """code = #{t < y}: no threshold compares below a NaN, so a NaN y takes code 0 (the rule
    as stated, not a search that sorts NaN last)."""
    _, t32 = cb.stored_codebook(3)
    got = bg.threshold_count(t32, np.array([np.nan, -np.inf, np.inf, 0.0], dtype=np.float32))
    np.testing.assert_array_equal(got, [0, 0, 7, 3])


def _textbook_levels():
    rows = _golden_rows("lloyd_max_centroids_textbook.txt")
    return {int(r[0]): r[1:] for r in rows}


def test_dequantizer_by_hand():
    """k_hat = norm * c16_w[code] * f_b and v_hat = norm * c16[code] / sqrt(d), value by value.

    d = 8 (blocks b = 0..3 cover dims b and b + 4), widths (2, 3, 0, 1), dequant factors
    (0.5, 0.25, 1, 2), one token with key norm 2 and codes (3, 5, 1, 0 | 0, 7, 2, 1) on dims
    0..7. The fp16 centroids used are c2 = (-1.5107421875, -0.452880859375, +.., +..),
    c3[5] = 0.755859375, c3[7] = 2.15234375, c1 = (-0.7978515625, +0.7978515625): the fp16
    roundings of the textbook Lloyd-Max levels (checked against them below). So
      dim 0: 2 * c2[3] * 0.5  = 1.5107421875     dim 4: 2 * c2[0] * 0.5  = -1.5107421875
      dim 1: 2 * c3[5] * 0.25 = 0.3779296875     dim 5: 2 * c3[7] * 0.25 = 1.076171875
      dim 2, 6: width 0 -> 0                     dim 3: 2 * c1[0] * 2 = -3.19140625
      dim 7: 2 * c1[1] * 2 = 3.19140625
    Values at width 2, norm 4, codes (0, 1, 2, 3, 3, 2, 1, 0) on dims 0..7:
      v_hat = 4 * c2[code] / sqrt(8).
    """
    c1 = [-0.7978515625, 0.7978515625]
    c2 = [-1.5107421875, -0.452880859375, 0.452880859375, 1.5107421875]
    c3_5, c3_7 = 0.755859375, 2.15234375
    tb = _textbook_levels()
    assert abs(c1[1] - tb[1][0]) < 1e-3
    assert abs(c2[2] - tb[2][0]) < 1e-3 and abs(c2[3] - tb[2][1]) < 1e-3
    assert abs(c3_5 - tb[3][1]) < 1e-3 and abs(c3_7 - tb[3][3]) < 1e-3
    alloc = {"w": np.array([[2, 3, 0, 1]]), "f": np.array([[0.5, 0.25, 1.0, 2.0]], dtype=np.float32)}
    Kc = np.array([3, 5, 1, 0, 0, 7, 2, 1], dtype=np.uint8).reshape(1, 1, 1, 8)
    Kn = np.array([2.0], dtype=np.float16).reshape(1, 1, 1)
    khat = bg.dequantize_keys(Kc, Kn, alloc)[0, 0, 0]
    want = [1.5107421875, 0.3779296875, 0.0, -3.19140625, -1.5107421875, 1.076171875, 0.0, 3.19140625]
    np.testing.assert_array_equal(khat, want)
    Vc = np.array([0, 1, 2, 3, 3, 2, 1, 0], dtype=np.uint8).reshape(1, 1, 1, 8)
    Vn = np.array([4.0], dtype=np.float16).reshape(1, 1, 1)
    vhat = bg.dequantize_values(Vc, Vn, 2)[0, 0, 0]
    s8 = math.sqrt(8.0)
    want_v = [4 * c2[0] / s8, 4 * c2[1] / s8, 4 * c2[2] / s8, 4 * c2[3] / s8,
              4 * c2[3] / s8, 4 * c2[2] / s8, 4 * c2[1] / s8, 4 * c2[0] / s8]
    np.testing.assert_allclose(vhat, want_v, rtol=1e-15, atol=0)


def test_append_one_token_at_a_time_equals_batch():
    """Append-only cache (NQKV assumptions): a per-row quantizer gives identical codes."""
    rng = np.random.default_rng(13)
    X = (rng.standard_normal((1, 1, 70, 128)) * 3).astype(np.float32)
    E, _ = bg.calibration_energies(X, 0)
    a = bg.allocate(E, 128, 3)
    full = bg.quantize(X, X, a, 3)
    for t in range(70):
        one = bg.quantize(X[:, :, t:t + 1], X[:, :, t:t + 1], a, 3)
        np.testing.assert_array_equal(one["Kc"][0, 0, 0], full["Kc"][0, 0, t])
        assert one["Kn"][0, 0, 0] == full["Kn"][0, 0, t]


# ----------------------------------------------------------------- pin 7: packed byte count

def test_packed_bytes_per_token():
    assert bg.tile_record_bytes(128, 3, 3) == 32 * 100                 # 48 + 48 + 4 bytes per token
    fp16_bytes = 2 * 2 * 128
    assert fp16_bytes / (bg.tile_record_bytes(128, 3, 3) / 32) == 5.12
    assert bg.tile_record_bytes(128, 2, 2) == 32 * 68
    assert bg.tile_record_bytes(128, 4, 4) == 32 * 132
    # the tile records, plus one 128-byte header (64 bytes of fields, 8 per KV head, rounded up)
    assert bg.packed_bytes(1, 2, 131072, 128, 3, 3) == 26_214_400 + 128
    assert bg.packed_bytes(1, 2, 100, 128, 3, 3) == 2 * 4 * 3200 + 128   # ragged tail rounds up to tiles
    assert bg.header_bytes(8) == 128 and bg.header_bytes(9) == 256
    # keys only (bits_v = 0): K part and K norms, 48 + 2 bytes per token at K3
    assert bg.tile_record_bytes(128, 3, 0) == 32 * 50
    # NF4: 128 bytes of codes + one fp16 scale per 256 values
    assert (128 + 2) * 8 / 256 == 4.0625
    assert round(16 / 4.0625, 2) == 3.94


# ----------------------------------------------------------------- layout

def _alloc_with(w_blocks, d=128):
    h = d // 2
    return {"w": np.array([w_blocks]), "g": np.ones((1, h), np.float32),
            "f": np.full((1, h), 1 / math.sqrt(d), np.float32), "E": np.ones((1, h)),
            "d": d, "bits_k": int(sum(w_blocks)) * 2 // d, "w_max": 8, "mode": 0}


def test_k_stream_order_by_hand():
    """d = 8 (4 blocks), widths [2, 5, 0, 1]: the stream holds block 1 (width 5), block 0
    (width 2), block 3 (width 1); block 2 has no bits. Each block is a pair of codes."""
    w = np.array([2, 5, 0, 1])
    assert bg.k_stream_blocks(w) == [1, 0, 3]
    np.testing.assert_array_equal(bg.k_bit_offsets(w), [10, 0, -1, 14])


def test_pack_bits_by_hand():
    words = bg.pack_bits(np.array([[0b101, 0b11, 0b1]]), [3, 30, 1])
    assert words.shape == (1, 2)
    assert int(words[0, 0]) == 0b101 | (0b11 << 3)
    assert int(words[0, 1]) == 1 << 1
    np.testing.assert_array_equal(bg.unpack_bits(words, [3, 30, 1]), [[0b101, 0b11, 0b1]])


def test_pack_single_code_position_by_hand():
    """Every block 3 bits wide, so the K stream is blocks 0..63 in order, 6 bits per block.

    K: token 9, dim 3 + 64 (second code of block 3) with code 0b101 sits at stream bits
    18 + 3 = 21..23, i.e. word 0 of token 9 -> word-planar index 0 * 32 + 9. Token 5, dim 5
    (first code of block 5) with code 0b111 sits at bits 30..32 and straddles words 0 and 1
    -> indices 5 and 32 + 5.
    V: token 13, dim 70, code 0b011 sits at bits 39..41 of dim 70's stream, i.e. bits 7..9
    of its word 1 -> index 1 * 128 + 70.
    """
    w = [3] * 64
    a = _alloc_with(w)
    Kc = np.zeros((1, 1, 32, 128), np.uint8)
    Kc[0, 0, 9, 3 + 64] = 0b101
    Kc[0, 0, 5, 5] = 0b111
    Vc = np.zeros((1, 1, 32, 128), np.uint8)
    Vc[0, 0, 13, 70] = 0b011
    Kn = np.zeros((1, 1, 32), np.float16)
    Vn = np.zeros((1, 1, 32), np.float16)
    Kn[0, 0, 3] = 1.5
    Vn[0, 0, 7] = -2.0
    codes = {"Kc": Kc, "Kn": Kn, "Vc": Vc, "Vn": Vn}
    packed = bg.pack_cache(codes, a, 3, 32)
    norms = packed[0, 0, 0, 4 * 384:4 * 384 + 128].copy().view("<f2")       # K norms, then V norms
    assert norms[3] == 1.5 and norms[32 + 7] == -2.0 and np.count_nonzero(norms) == 2
    kw = packed[0, 0, 0, :4 * 384].copy().view("<u4")
    vw = packed[0, 0, 0, 4 * 384 + 128:].copy().view("<u4")
    assert vw.shape == (384,)
    nz = {i: int(x) for i, x in enumerate(kw) if x}
    assert nz == {9: 0b101 << 21, 5: 0b11 << 30, 37: 1}
    vnz = {i: int(x) for i, x in enumerate(vw) if x}
    assert vnz == {1 * 128 + 70: 0b011 << 7}


def test_pack_unpack_roundtrip_mixed_widths():
    rng = np.random.default_rng(14)
    d, h = 128, 64
    w = np.full(h, 3)
    w[:8] = [8, 0, 6, 0, 1, 5, 2, 2]
    w[8] = 3 * h - int(w.sum() - w[8])
    assert 0 <= w[8] <= 8
    a = _alloc_with(list(w))
    T = 77
    wd = np.concatenate([w, w])
    Kc = np.zeros((2, 1, T, d), np.uint8)
    for j in range(d):
        Kc[..., j] = rng.integers(0, 2 ** wd[j], size=(2, 1, T)) if wd[j] else 0
    Vc = rng.integers(0, 8, size=(2, 1, T, d)).astype(np.uint8)
    Kn = rng.standard_normal((2, 1, T)).astype(np.float16)
    Vn = rng.standard_normal((2, 1, T)).astype(np.float16)
    packed = bg.pack_cache({"Kc": Kc, "Kn": Kn, "Vc": Vc, "Vn": Vn}, a, 3, 100)
    assert packed.shape == (2, 1, 4, 3200)
    u = bg.unpack_cache(packed, a, 3, T)
    np.testing.assert_array_equal(u["Kc"], Kc)
    np.testing.assert_array_equal(u["Vc"], Vc)
    np.testing.assert_array_equal(u["Kn"], Kn)
    np.testing.assert_array_equal(u["Vn"], Vn)
    tail = bg.unpack_cache(packed, a, 3, 128)
    assert np.all(tail["Kc"][:, :, T:] == 0) and np.all(tail["Kn"][:, :, T:] == 0)


# ----------------------------------------------------------------- pin 9: attention

def test_attention_single_token_returns_its_value():
    rng = np.random.default_rng(15)
    q = rng.standard_normal((1, 4, 16))
    K = rng.standard_normal((1, 2, 1, 16))
    V = rng.standard_normal((1, 2, 1, 16))
    out = bg.decode_attention(q, K, V)
    np.testing.assert_allclose(out[0, :2], np.repeat(V[0, 0], 2, axis=0), rtol=1e-15)
    np.testing.assert_allclose(out[0, 2:], np.repeat(V[0, 1], 2, axis=0), rtol=1e-15)


def test_attention_zero_query_is_mean_of_values():
    rng = np.random.default_rng(16)
    K = rng.standard_normal((1, 1, 50, 8))
    V = rng.standard_normal((1, 1, 50, 8))
    out = bg.decode_attention(np.zeros((1, 1, 8)), K, V)
    np.testing.assert_allclose(out[0, 0], V[0, 0].mean(axis=0), rtol=1e-13)


def test_attention_matches_online_softmax_restatement():
    """Two-pass softmax vs the running-max (online) form over 7 chunks, both fp64."""
    rng = np.random.default_rng(17)
    d = 32
    q = rng.standard_normal((1, 1, d)) * 3
    K = rng.standard_normal((1, 1, 300, d)) * 2
    V = rng.standard_normal((1, 1, 300, d))
    ref = bg.decode_attention(q, K, V)[0, 0]
    m, l, o = -np.inf, 0.0, np.zeros(d)
    for chunk in np.array_split(np.arange(300), 7):
        s = K[0, 0, chunk] @ q[0, 0] / math.sqrt(d)
        mn = max(m, s.max())
        scale = math.exp(m - mn) if np.isfinite(m) else 0.0
        p = np.exp(s - mn)
        l = l * scale + p.sum()
        o = o * scale + p @ V[0, 0, chunk]
        m = mn
    np.testing.assert_allclose(o / l, ref, rtol=1e-14, atol=1e-15)


def test_decode_from_packed_equals_direct_dequant():
    rng = np.random.default_rng(18)
    K = (rng.standard_normal((1, 2, 45, 128)) * np.exp(rng.standard_normal(128))).astype(np.float32)
    V = rng.standard_normal((1, 2, 45, 128)).astype(np.float32)
    q = rng.standard_normal((1, 4, 128)).astype(np.float32)
    a = bg.calibrate(K, 3)
    c = bg.quantize(K, V, a, 2)
    packed = bg.pack_cache(c, a, 2, 64)
    out = bg.decode(q, packed, a, 2, 45)
    Khat = bg.dequantize_keys(c["Kc"], c["Kn"], a)
    Vhat = bg.dequantize_values(c["Vc"], c["Vn"], 2)
    np.testing.assert_array_equal(out, bg.decode_attention(q, Khat, Vhat))
    # the dequantised keys approximate the originals (quantizer sanity, not exactness)
    rel = np.linalg.norm(Khat - K) / np.linalg.norm(K)
    assert rel < 0.25


# ----------------------------------------------------------------- packed header

def test_splitmix64_published_vectors():
    """The digest's mixing function against the first outputs of SplitMix64 seeded with 0, as
    published with the reference generator: mix(gamma), mix(2 gamma), mix(3 gamma)."""
    g = 0x9E3779B97F4A7C15
    assert bg.splitmix64(0) == 0xE220A8397B1DCDAF
    assert bg.splitmix64(g) == 0x6E789E6AA1B965F4
    assert bg.splitmix64((2 * g) % (1 << 64)) == 0x06C45D188009454F


def test_header_fields_by_hand():
    """Header of a 2-sequence, 3-KV-head, 77-token K3V2 cache: magic "KVQ1", layout 1,
    d = 128, widths, the record size 4 * 128 * (3 + 2) + 128 = 2688, one digest per head,
    64 + 3 * 8 = 88 bytes padded to 128."""
    w = np.array([[3] * 64, [2] * 32 + [4] * 32, [3] * 64])
    g = np.ones((3, 64), np.float32)
    g[1, 5] = 1.5
    alloc = {"w": w, "g": g, "w_max": 8, "mode": 0}
    h = bg.packed_header(2, 3, 77, 128, 3, 2, alloc)
    assert h.shape == (128,)
    assert bytes(h[:4]) == b"KVQ1"
    assert list(h[4:12]) == [1, 0, 128, 0, 3, 2, 8, 0]
    assert list(h[12:16]) == [0, 0, 0, 0]
    f = h[16:32].view("<u4")
    assert list(f) == [2, 3, 77, 2688]
    assert not h[32:64].any() and not h[88:].any()
    dig = h[64:88].view("<u8")
    assert dig[0] == dig[2] and dig[0] != dig[1]               # same allocation, same digest
    # digest: sum mod 2^64 over blocks of splitmix64(b << 40 | w << 32 | bits(g)); g = 1.0 is 0x3F800000
    want0 = sum(bg.splitmix64((b << 40) | (3 << 32) | 0x3F800000) for b in range(64)) % (1 << 64)
    assert int(dig[0]) == want0
    g2 = g.copy()
    g2[1, 5] = np.float32(1.5) + np.float32(2 ** -23)         # one ulp of one gain changes it
    assert bg.alloc_digest(w[1], g2[1]) != int(dig[1])


# ----------------------------------------------------------------- keys-only cache and recent tokens

def _small_cache(seed, T=45, bits_k=3, bits_v=2):
    rng = np.random.default_rng(seed)
    K = (rng.standard_normal((1, 2, T, 128)) * np.exp(rng.standard_normal(128))).astype(np.float32)
    V = rng.standard_normal((1, 2, T, 128)).astype(np.float32)
    q = rng.standard_normal((1, 4, 128)).astype(np.float32)
    a = bg.calibrate(K, bits_k)
    c = bg.quantize(K, V, a, bits_v)
    return K, V, q, a, c


def test_recent_buffer_alone_is_plain_attention():
    """With no packed token (seq_len 0) and all T tokens in the recent buffer, the decode is
    exact fp64 attention over the raw keys and values."""
    K, V, q, a, _ = _small_cache(31)
    out = bg.decode(q, None, a, 2, 0, K_recent=K, V_recent=V)
    np.testing.assert_array_equal(out, bg.decode_attention(q, K.astype(np.float64), V.astype(np.float64)))


def test_recent_buffer_duplicating_the_cache_changes_nothing():
    """Appending every cached token again as a recent token (with its dequantized key and
    value) doubles each softmax weight's numerator and denominator alike: the output equals
    the packed-only decode (to rounding)."""
    K, V, q, a, c = _small_cache(32)
    packed = bg.pack_cache(c, a, 2, 64)
    ref = bg.decode(q, packed, a, 2, 45)
    Kh = bg.dequantize_keys(c["Kc"], c["Kn"], a)
    Vh = bg.dequantize_values(c["Vc"], c["Vn"], 2)
    out = bg.decode(q, packed, a, 2, 45, K_recent=Kh, V_recent=Vh)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)
    # a recent token far more aligned with q than any cached one takes the whole softmax
    Kr = np.zeros((1, 2, 1, 128))
    Kr[0, :, 0] = 1e4 * q[0, ::2] / np.linalg.norm(q[0, ::2], axis=-1, keepdims=True)
    Vr = np.full((1, 2, 1, 128), 7.0)
    out2 = bg.decode(q[:, ::2], packed, a, 2, 45, K_recent=Kr, V_recent=Vr)
    np.testing.assert_allclose(out2, 7.0, rtol=1e-12)


def test_keys_only_cache_with_exact_values():
    """A keys-only cache (bits_v = 0) holds the K part and K norms of every record; its decode
    with the values given as the dequantized values of a K3V2 cache equals that cache's decode."""
    K, V, q, a, c2 = _small_cache(33)
    c0 = bg.quantize(K, V, a, 0)
    assert c0["Vc"] is None
    pk0 = bg.pack_cache(c0, a, 0, 64)
    pk2 = bg.pack_cache(c2, a, 2, 64)
    assert pk0.shape[-1] == bg.tile_record_bytes(128, 3, 0)
    np.testing.assert_array_equal(pk0, pk2[..., :pk0.shape[-1]])      # same K half, byte for byte
    Vh = bg.dequantize_values(c2["Vc"], c2["Vn"], 2)
    np.testing.assert_array_equal(bg.decode(q, pk0, a, 0, 45, V=Vh), bg.decode(q, pk2, a, 2, 45))


# ----------------------------------------------------------------- NF4

def test_nf4_quantize_special_cases():
    X = np.zeros((1, 2, 3, 128), np.float16)
    X[0, 0, 1, 5] = 3.0
    X[0, 1, 1, 0] = -1.5
    X[0, :, 2, :] = np.float16(-0.25)
    idx, s = nqkv.quantize(X)
    assert idx.shape == (1, 1, 3, 256) and s.shape == (1, 1, 3)
    assert s[0, 0, 0] == 0 and np.all(idx[0, 0, 0] == 7)            # zero block -> the exact-zero level
    assert s[0, 0, 1] == 3.0 and idx[0, 0, 1, 5] == 15               # +absmax -> +1
    assert idx[0, 0, 1, 128] == int(np.searchsorted(cb.nf4_midpoints(), np.float32(-0.5), "left"))
    assert s[0, 0, 2] == 0.25 and np.all(idx[0, 0, 2] == 0)           # every value equals -absmax -> -1


def test_nf4_midpoint_goes_to_lower_index():
    """idx = #{midpoints < u}: a value exactly on midpoint i takes index i (the lower level),
    the next fp32 value above it index i + 1. One 256-value block with absmax 1 (scale 1, so
    u = x exactly): x_0 = 1, x_{1+i} = m_i, x_{16+i} = nextafter(m_i, +inf), the rest 0."""
    m = np.asarray(cb.nf4_midpoints(), dtype=np.float32)
    X = np.zeros((1, 2, 1, 128), np.float32)
    row = X[0, 0, 0]
    row[0] = 1.0
    row[1:16] = m
    row[16:31] = np.nextafter(m, np.float32(2))
    idx, s = nqkv.quantize(X)
    assert s[0, 0, 0] == 1.0
    assert idx[0, 0, 0, 0] == 15
    np.testing.assert_array_equal(idx[0, 0, 0, 1:16], np.arange(15))
    np.testing.assert_array_equal(idx[0, 0, 0, 16:31], np.arange(1, 16))
    assert np.all(idx[0, 0, 0, 31:] == 7)                                # zeros: the exact-zero level


def test_nf4_pack_roundtrip_and_padding():
    rng = np.random.default_rng(19)
    idx = rng.integers(0, 16, size=(2, 3, 21, 256)).astype(np.uint8)
    sc = rng.standard_normal((2, 3, 21)).astype(np.float16)
    codes, scales = nqkv.pack(idx, sc, 21)
    assert codes.shape == (2, 3, 32, 128) and scales.shape == (2, 3, 32)
    assert codes[0, 0, 0, 0] == (idx[0, 0, 0, 0] | (idx[0, 0, 0, 1] << 4))
    assert np.all(codes[:, :, 21:] == 0) and np.all(scales[:, :, 21:] == 0)
    i2, s2 = nqkv.unpack(codes, scales, 21)
    np.testing.assert_array_equal(i2, idx)
    np.testing.assert_array_equal(s2, sc)


def test_nf4_fig5_worked_shape():
    """NQKV Fig. 5 shape: hidden 24, 1024 tokens, block 6 -> 4 blocks per token."""
    rng = np.random.default_rng(20)
    X = rng.standard_normal((1, 4, 1024, 6)).astype(np.float16)
    idx, s = nqkv.quantize(X, block=6)
    assert idx.shape == (1, 4, 1024, 6)
    xh = nqkv.dequantize(idx, s, 4, 6)
    v = cb.nf4_values().astype(np.float64)
    gap = np.max(np.diff(v)) / 2
    # with block == head_dim, block k of a token is head k, so scales align with X's heads
    err = np.abs(xh - X.astype(np.float64))
    bound = s.astype(np.float64)[..., None] * gap * (1 + 1e-6)
    assert np.all(err <= bound)
    # each block's absmax element is reconstructed exactly (+-1 times the fp16 scale)
    amax = np.argmax(np.abs(X.astype(np.float64)), axis=-1)
    got = np.take_along_axis(xh, amax[..., None], -1)[..., 0]
    want = np.take_along_axis(X.astype(np.float64), amax[..., None], -1)[..., 0]
    np.testing.assert_array_equal(got, want)


def test_nf4_decode_masks_padding():
    rng = np.random.default_rng(21)
    X = rng.standard_normal((1, 2, 19, 128)).astype(np.float16)
    q = rng.standard_normal((1, 2, 128)).astype(np.float16)
    idx, s = nqkv.quantize(X)
    kc, ks = nqkv.pack(idx, s, 19)
    out = nqkv.decode(q, kc, ks, kc, ks, 2, 128, 19)
    kc2, ks2 = kc.copy(), ks.copy()
    kc2[:, :, 19:] = 0x77                                             # garbage codes in the padded rows
    ks2[:, :, 19:] = 1.0                                              # and non-zero scales
    out2 = nqkv.decode(q, kc2, ks2, kc2, ks2, 2, 128, 19)
    np.testing.assert_array_equal(out, out2)
    # attention over exactly the 19 quantized tokens, straight from the quantizer's output
    xh = nqkv.dequantize(idx, s, 2, 128)
    np.testing.assert_allclose(out, bg.decode_attention(q.astype(np.float64), xh, xh), rtol=1e-14)

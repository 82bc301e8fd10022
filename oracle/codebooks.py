"""Oracle codebooks: Lloyd-Max scalar quantizers for N(0,1) and the NF4 table.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Lloyd-Max (reading; the Block-GTQ page names TQ-MSE as the base quantizer but
prints no codebook): for width w the 2^w-level MSE-optimal quantizer of a
standard normal, found by the Lloyd fixed-point iteration
    thresholds = midpoints of adjacent centroids,
    centroid of cell (a, b) = E[X | a < X < b] = (phi(a) - phi(b)) / (Phi(b) - Phi(a)),
run in fp64 to convergence. Stored forms (reading):
  * centroids rounded to fp16 (round-to-nearest-even),
  * thresholds = fp32 rounding of the midpoint of adjacent fp16 centroids,
  * delta(w) = fp32 rounding of the MSE on N(0,1) of that stored quantizer,
    delta(0) = 1 (a zero-width coordinate is reconstructed as 0).

NF4 (NQKV review, "What carries the argument": 16 quantiles of the standard
normal, imported from QLoRA, reference [20]): asymmetric construction with an
exact zero — 8 positive quantiles at probabilities evenly spaced from `off`
down to (but excluding) 1/2, 7 negative ones at probabilities evenly spaced
from `off` down to (excluding) 1/2 and mirrored, plus 0, all divided by the
largest so the table spans [-1, 1]. `off` is the mean of 1 - 1/(2*15) and
1 - 1/(2*16), the outermost probability levels of 15- and 16-point grids.
Values are kept in fp32; midpoints in fp32.
"""
from __future__ import annotations

import math
from functools import lru_cache

import numpy as np
from scipy.special import erfc, ndtri

_INV_SQRT2PI = 1.0 / math.sqrt(2.0 * math.pi)


def pdf(x):
    """Standard normal density; 0 at +-inf."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        out = np.exp(-0.5 * x * x) * _INV_SQRT2PI
    return np.where(np.isfinite(x), out, 0.0)


def cdf(x):
    return 0.5 * erfc(-np.asarray(x, dtype=np.float64) / math.sqrt(2.0))


def sf(x):
    return 0.5 * erfc(np.asarray(x, dtype=np.float64) / math.sqrt(2.0))


def cell_mass(a, b):
    """P(a < X < b) for X ~ N(0,1), computed from the nearer tail for accuracy."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    right = sf(a) - sf(b)          # accurate when a >= 0
    left = cdf(b) - cdf(a)         # accurate when b <= 0
    mid = 1.0 - cdf(a) - sf(b)     # straddles 0
    return np.where(a >= 0, right, np.where(b <= 0, left, mid))


def _first_moment(a, b):
    """Integral of x phi(x) over (a, b)."""
    return pdf(a) - pdf(b)


def _second_moment(a, b):
    """Integral of x^2 phi(x) over (a, b) = P + a phi(a) - b phi(b)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        apa = np.where(np.isfinite(a), a * pdf(a), 0.0)
        bpb = np.where(np.isfinite(b), b * pdf(b), 0.0)
    return cell_mass(a, b) + apa - bpb


def quantizer_mse(centroids, thresholds) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1), Q mapping cell i (t_{i-1}, t_i) to centroids[i]."""
    c = np.asarray(centroids, dtype=np.float64)
    t = np.asarray(thresholds, dtype=np.float64)
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    m0 = cell_mass(a, b)
    m1 = _first_moment(a, b)
    m2 = _second_moment(a, b)
    return float(np.sum(m2 - 2.0 * c * m1 + c * c * m0))


def _conditional_means(c):
    """Lloyd map: conditional mean of each cell bounded by midpoints of c, and the cell masses."""
    t = 0.5 * (c[:-1] + c[1:])
    a = np.concatenate([[-np.inf], t])
    b = np.concatenate([t, [np.inf]])
    p = cell_mass(a, b)
    return _first_moment(a, b) / p, a, b, p


@lru_cache(maxsize=None)
def lloyd_max_f64(w: int):
    """Exact (fp64-converged) Lloyd-Max centroids and thresholds for 2^w levels of N(0,1).

    The solution is the fixed point of the Lloyd conditions (each threshold is
    the midpoint of its neighbouring centroids; each centroid is the conditional
    mean of its cell). It is reached by Lloyd iterations from the compander
    (N(0,3) quantile) start, then Newton's method on the same equations with
    the exact tridiagonal Jacobian of the Lloyd map, until the residual
    max|c - M(c)| is at rounding level.
    Returns (centroids[2^w], thresholds[2^w - 1]) as float64 arrays.
    """
    if not 1 <= w <= 8:
        raise ValueError("width must be in 1..8")
    n = 1 << w
    c = math.sqrt(3.0) * ndtri((np.arange(n) + 0.5) / n)
    for _ in range(200):
        c, _a, _b, _p = _conditional_means(c)
    for _ in range(100):
        m, a, b, p = _conditional_means(c)
        resid = c - m
        if float(np.max(np.abs(resid))) < 1e-15:
            break
        # dM_i/da = phi(a)(M_i - a)/P_i, dM_i/db = phi(b)(b - M_i)/P_i, a = t_{i-1}, b = t_i
        with np.errstate(invalid="ignore"):
            dma = np.where(np.isfinite(a), pdf(a) * (m - a) / p, 0.0)
            dmb = np.where(np.isfinite(b), pdf(b) * (b - m) / p, 0.0)
        jac = np.eye(n)
        for i in range(n):
            if i > 0:
                jac[i, i - 1] -= 0.5 * dma[i]
                jac[i, i] -= 0.5 * dma[i]
            if i < n - 1:
                jac[i, i + 1] -= 0.5 * dmb[i]
                jac[i, i] -= 0.5 * dmb[i]
        c = c - np.linalg.solve(jac, resid)
    t = 0.5 * (c[:-1] + c[1:])
    return c, t


@lru_cache(maxsize=None)
def stored_codebook(w: int):
    """Stored forms used by the quantizer and the decode.

    Returns (centroids_f16[2^w] np.float16, thresholds_f32[2^w-1] np.float32).
    """
    c, _ = lloyd_max_f64(w)
    c16 = c.astype(np.float16)
    c16d = c16.astype(np.float64)
    t32 = (0.5 * (c16d[:-1] + c16d[1:])).astype(np.float32)
    return c16, t32


@lru_cache(maxsize=None)
def delta_table():
    """delta[w] for w = 0..8 as float32: MSE on N(0,1) of the stored width-w quantizer; delta[0] = 1."""
    out = [1.0]
    for w in range(1, 9):
        c16, t32 = stored_codebook(w)
        out.append(quantizer_mse(c16.astype(np.float64), t32.astype(np.float64)))
    return np.array(out, dtype=np.float64).astype(np.float32)


@lru_cache(maxsize=None)
def nf4_values():
    """The 16 NF4 levels as float32, ascending, from -1 to 1 with an exact 0."""
    off = 0.5 * ((1.0 - 1.0 / (2 * 15)) + (1.0 - 1.0 / (2 * 16)))
    pos = ndtri(np.linspace(off, 0.5, 9)[:-1])          # 8 positive quantiles
    neg = -ndtri(np.linspace(off, 0.5, 8)[:-1])         # 7 negative quantiles
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    v = v / np.max(np.abs(v))
    return v.astype(np.float32)


@lru_cache(maxsize=None)
def nf4_midpoints():
    """fp32 decision boundaries between adjacent NF4 levels (15 values)."""
    v = nf4_values().astype(np.float64)
    return (0.5 * (v[:-1] + v[1:])).astype(np.float32)

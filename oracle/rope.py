"""RoPE block decomposition — the premise of Block-GTQ. TEST INFRASTRUCTURE ONLY.

Page "RoPE-aware bit allocation for KV cache quantization", abstract: with
RoPE, the logit a cached key later produces splits into one term per 2-D
frequency block, each depending on the position gap. Reading (rotate-half pairing): block i
holds dims (i, i + h), h = d/2, and rotates by angle p * theta_i with
theta_i = base^(-2i/d).
"""
from __future__ import annotations

import numpy as np


def theta(d: int, base: float) -> np.ndarray:
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def rotate(x: np.ndarray, pos: float, base: float) -> np.ndarray:
    """R_pos x for one vector x[d] (fp64): each block (x_i, x_{i+h}) rotated by pos*theta_i."""
    x = np.asarray(x, dtype=np.float64)
    h = x.shape[-1] // 2
    ang = pos * theta(x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[:h] = x[:h] * c - x[h:] * s
    out[h:] = x[h:] * c + x[:h] * s
    return out


def block_logit_terms(q: np.ndarray, k: np.ndarray, m: float, n: float, base: float) -> np.ndarray:
    """Per-block terms of <R_m q, R_n k> written with the pre-RoPE vectors only.

    term_i = (q_i k_i + q_{i+h} k_{i+h}) cos((m-n) theta_i)
             - (q_{i+h} k_i - q_i k_{i+h}) sin((m-n) theta_i).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    h = q.shape[-1] // 2
    ang = (m - n) * theta(q.shape[-1], base)
    dot = q[:h] * k[:h] + q[h:] * k[h:]
    cross = q[h:] * k[:h] - q[:h] * k[h:]
    return dot * np.cos(ang) - cross * np.sin(ang)


def block_energy(k: np.ndarray) -> np.ndarray:
    """||k_b||^2 per block b for one vector k[d]."""
    k = np.asarray(k, dtype=np.float64)
    h = k.shape[-1] // 2
    return k[:h] * k[:h] + k[h:] * k[h:]

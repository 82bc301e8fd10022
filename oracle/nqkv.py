"""NQKV-style per-block NF4 variant: the oracle. TEST INFRASTRUCTURE ONLY.

Source: pith.science review of "NQKV: A KV Cache Quantization Scheme Based on
Normal Distribution Characteristics" (arXiv 2505.16210):
  * "What carries the argument": the hidden dimension of each key/value is
    cut into blocks (256 values in the experiments), each block gets a scale
    and 4-bit NF4 indices; dequantization is a table lookup; the token
    dimension is padded to a multiple of 16 for GEMM.
  * Referee report, major comment 1 (with Fig. 5): each block is rescaled by
    its maximum absolute value, with no mean subtraction.
  * Assumptions: the cache is append-only, so blocks are encoded per token.
  * Figs. 6-7: padding with zeros is done during computation.

Readings: blocks run along each token's head-major hidden vector (the
review's core-claim paragraph puts the blocks on the token axis; the figure
captions and the mechanism paragraph put them on the hidden axis, which is
what is followed). Scale s = fp16(absmax of the block); u = fp32(x) /
fp32(s) (u = 0 when s = 0); index = #{NF4 midpoints strictly below u}.
Padded tokens hold index 0 and scale 0 and are masked out of the softmax.
Storage per (sequence, block): codes[T_pad][128 bytes] with value 2k in the
low nibble of byte k and value 2k+1 in the high nibble, scales[T_pad] fp16.
"""
from __future__ import annotations

import math

import numpy as np

from . import codebooks

BLOCK = 256
PAD = 16


def padded_len(T: int) -> int:
    return -(-T // PAD) * PAD


def quantize(X: np.ndarray, block: int = BLOCK) -> tuple[np.ndarray, np.ndarray]:
    """X: [B][H][T][d] stored values. Returns (idx uint8 [B][nblk][T][block], scale fp16 [B][nblk][T]).

    Block k of token t holds hidden values k*block .. k*block + block - 1 of the
    head-major hidden vector (head hh, dim j) -> hh*d + j.
    """
    B, H, T, d = X.shape
    hidden = np.transpose(np.asarray(X, dtype=np.float32), (0, 2, 1, 3)).reshape(B, T, H * d)
    nblk = H * d // block
    blocks = hidden.reshape(B, T, nblk, block)
    s16 = np.max(np.abs(blocks), axis=-1).astype(np.float16)
    s32 = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(s32[..., None] == 0, np.float32(0.0),
                     blocks / np.where(s32 == 0, np.float32(1.0), s32)[..., None]).astype(np.float32)
    mids = codebooks.nf4_midpoints()
    idx = np.sum(mids < u[..., None], axis=-1).astype(np.uint8)       # #{midpoints < u}
    return np.transpose(idx, (0, 2, 1, 3)), np.transpose(s16, (0, 2, 1))


def pack(idx: np.ndarray, scale: np.ndarray, capacity: int) -> tuple[np.ndarray, np.ndarray]:
    """Byte codes [B][nblk][T_pad][block/2] and scales [B][nblk][T_pad] (fp16); pad = 0."""
    B, nblk, T, blk = idx.shape
    Tp = padded_len(capacity)
    codes = np.zeros((B, nblk, Tp, blk // 2), dtype=np.uint8)
    codes[:, :, :T] = (idx[..., 0::2] & 0xF) | ((idx[..., 1::2] & 0xF) << 4)
    sc = np.zeros((B, nblk, Tp), dtype=np.float16)
    sc[:, :, :T] = scale
    return codes, sc


def unpack(codes: np.ndarray, scales: np.ndarray, seq_len: int) -> tuple[np.ndarray, np.ndarray]:
    lo = codes & 0xF
    hi = codes >> 4
    idx = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    return idx[:, :, :seq_len], scales[:, :, :seq_len]


def dequantize(idx: np.ndarray, scale: np.ndarray, n_heads: int, d: int) -> np.ndarray:
    """x_hat = scale * NF4[idx] (fp64) back in [B][H][T][d] layout."""
    B, nblk, T, blk = idx.shape
    vals = codebooks.nf4_values().astype(np.float64)[idx] * scale.astype(np.float64)[..., None]
    hidden = np.transpose(vals, (0, 2, 1, 3)).reshape(B, T, n_heads, d)
    return np.transpose(hidden, (0, 2, 1, 3))


def decode(q: np.ndarray, kcodes, kscales, vcodes, vscales, n_heads: int, d: int, seq_len: int) -> np.ndarray:
    """MHA decode attention over the dequantized cache; padded tokens excluded (fp64)."""
    ki, ks = unpack(kcodes, kscales, seq_len)
    vi, vs = unpack(vcodes, vscales, seq_len)
    Khat = dequantize(ki, ks, n_heads, d)
    Vhat = dequantize(vi, vs, n_heads, d)
    B = q.shape[0]
    out = np.zeros((B, n_heads, d), dtype=np.float64)
    for b in range(B):
        for hh in range(n_heads):
            logits = Khat[b, hh] @ np.asarray(q[b, hh], dtype=np.float64) / math.sqrt(float(d))
            m = np.max(logits)
            p = np.exp(logits - m)
            out[b, hh] = (p @ Vhat[b, hh]) / np.sum(p)
    return out

"""Planted mistakes in the oracle, on the CPU: each case replaces one oracle function, for the
length of the case, by a copy with one plausible slip (a dropped term or factor, a flipped
tie rule, another summation order, a transposed index, a swapped nibble) and checks that the
pins in test_oracle_pins.py catch it: at least one of the pins named with the case must fail.
A case whose pins all pass would mean that mistake could enter the oracle unnoticed.
Nothing here touches the CUDA path.
"""
import math

import numpy as np
import pytest
from scipy.special import ndtri

from oracle import blockgtq as bg
from oracle import codebooks as cb
from oracle import nqkv
from oracle import rope
from tests import test_oracle_pins as pins

@pytest.fixture(autouse=True, scope="module")
def _true_tables_cached():
    """Fill the oracle's cached tables before any mutation, so that no cached table is ever
    built from a mutated function and carried into later tests."""
    for w in range(1, 9):
        cb.lloyd_max_f64(w)
        cb.stored_codebook(w)
    cb.delta_table()
    cb.nf4_values()
    cb.nf4_midpoints()


_orig = {
    "calibration_energies": bg.calibration_energies,
    "block_gains": bg.block_gains,
    "quantize_rows": bg.quantize_rows,
    "nqkv_unpack": nqkv.unpack,
}


# ---------------------------------------------------------------- calibration energy

def energy_one_chain(K, n_calib=0):
    """All terms summed left to right in one chain (no 64-token chunks, no segments)."""
    B, H, T, d = K.shape
    h, n = d // 2, (T if n_calib <= 0 else n_calib)
    X = np.transpose(np.asarray(K[:, :, :n], np.float64), (1, 0, 2, 3)).reshape(H, B * n, d)
    terms = X[..., :h] * X[..., :h] + X[..., h:] * X[..., h:]
    acc = np.zeros((H, h))
    for u in range(B * n):
        acc = acc + terms[:, u]
    return acc / float(B * n), B * n


def energy_without_partner(K, n_calib=0):
    """Block b counted from x_b alone (x_{b+h} dropped)."""
    K2 = np.array(K, dtype=np.float64, copy=True)
    K2[..., K2.shape[-1] // 2:] = 0.0
    return _orig["calibration_energies"](K2, n_calib)


def energy_over_sequence_length(K, n_calib=0):
    """Divided by the tokens of one sequence instead of all pooled tokens."""
    E, N = _orig["calibration_energies"](K, n_calib)
    return E * K.shape[0], N


# ---------------------------------------------------------------- greedy allocation

def _greedy(E, bits, w_max, gain_of, better, cap=True):
    D = np.asarray(cb.delta_table(), dtype=np.float64)
    if not (1 <= bits <= w_max <= 8):
        raise ValueError("need 1 <= bits <= w_max <= 8")
    w = np.zeros(len(E), dtype=np.int64)
    for _ in range(bits * len(E)):
        best_b, best = -1, -math.inf
        for b in range(len(E)):
            if (w[b] < w_max if cap else w[b] < 8):
                g = gain_of(float(E[b]), D, int(w[b]))
                if better(g, best):
                    best_b, best = b, g
        w[best_b] += 1
    return w


def greedy_ties_to_highest(E, bits, w_max, delta=None):
    return _greedy(E, bits, w_max, lambda e, D, w: e * (D[w] - D[w + 1]), lambda g, best: g >= best)


def greedy_ignores_wmax(E, bits, w_max, delta=None):
    return _greedy(E, bits, w_max, lambda e, D, w: e * (D[w] - D[w + 1]), lambda g, best: g > best, cap=False)


def greedy_gain_is_distortion(E, bits, w_max, delta=None):
    """Gain taken as the distortion left at the current width, not its decrease."""
    return _greedy(E, bits, w_max, lambda e, D, w: e * D[w + 1], lambda g, best: g > best)


def gains_without_factor_two(E, d):
    """g_b = sqrt(S / (d E_b)): the factor 2 (two coordinates per block) dropped."""
    g, _ = _orig["block_gains"](E, d)
    g = (g.astype(np.float64) / math.sqrt(2.0)).astype(np.float32)
    f = np.array([np.float32(1.0 / (math.sqrt(float(d)) * float(x))) for x in g], dtype=np.float32)
    return g, f


# ---------------------------------------------------------------- quantizer

def norms_in_fp64(X):
    X64 = np.asarray(X, dtype=np.float64)
    return np.sqrt(np.sum(X64 * X64, axis=-1)).astype(np.float32).astype(np.float16)


def norms_one_fp32_chain(X):
    X32 = np.asarray(X, dtype=np.float32)
    s = np.zeros(X32.shape[:-1], np.float32)
    for j in range(X32.shape[-1]):
        s = (s + (X32[..., j] * X32[..., j]).astype(np.float32)).astype(np.float32)
    return np.sqrt(s).astype(np.float32).astype(np.float16)


def count_ties_up(t32, y):
    """A y on a threshold takes the upper code."""
    y = np.asarray(y, dtype=np.float32)
    return np.sum(np.asarray(t32, np.float32) <= y[..., None], axis=-1).astype(np.uint8)


def quantize_without_sqrt_d(X, widths_dim, gains_dim):
    """a = 1 / norm instead of sqrt(d) / norm (restated in full: scaling the row before the
    real quantizer would change its norm as well)."""
    X32 = np.asarray(X, dtype=np.float32)
    n16 = bg.row_norms_f16(X32)
    n32 = n16.astype(np.float32)
    a = np.where(n32 == 0, np.float32(0), np.float32(1) / np.where(n32 == 0, np.float32(1), n32)).astype(np.float32)
    y = ((X32 * a[..., None]).astype(np.float32) * np.asarray(gains_dim, np.float32)).astype(np.float32)
    codes = np.zeros(X32.shape, np.uint8)
    for w in range(1, 9):
        sel = np.asarray(widths_dim) == w
        if np.any(sel):
            codes[..., sel] = bg.threshold_count(cb.stored_codebook(w)[1], y[..., sel])
    return codes, n16


def quantize_without_gains(X, widths_dim, gains_dim):
    return _orig["quantize_rows"](X, widths_dim, np.ones(np.asarray(X).shape[-1], np.float32))


# ---------------------------------------------------------------- dequantizer and attention

def keys_without_factor(Kc, Kn, alloc):
    a = dict(alloc)
    a["f"] = np.ones_like(np.asarray(alloc["f"], dtype=np.float32))
    B, H, T, d = Kc.shape
    out = np.zeros((B, H, T, d))
    for hh in range(H):
        wd = bg.widths_per_dim(a["w"][hh])
        for j in range(d):
            if wd[j]:
                c16, _ = cb.stored_codebook(int(wd[j]))
                out[:, hh, :, j] = Kn[:, hh].astype(np.float64) * c16.astype(np.float64)[Kc[:, hh, :, j]]
    return out


def values_without_sqrt_d(Vc, Vn, bits_v):
    c16, _ = cb.stored_codebook(bits_v)
    return Vn.astype(np.float64)[..., None] * c16.astype(np.float64)[Vc]


def attention(q, Khat, Vhat, scale=True, kv_of=lambda hq, G, Hkv: hq // G):
    B, Hq, d = q.shape
    Hkv = Khat.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d))
    for b in range(B):
        for hq in range(Hq):
            kv = kv_of(hq, G, Hkv)
            s = Khat[b, kv] @ np.asarray(q[b, hq], np.float64)
            if scale:
                s = s / math.sqrt(float(d))
            p = np.exp(s - np.max(s))
            out[b, hq] = (p @ Vhat[b, kv]) / np.sum(p)
    return out


def widths_interleaved(w_blocks):
    """Per-dim widths (w_0, w_0, w_1, w_1, ..) instead of block b on dims b and b + h."""
    return np.repeat(np.asarray(w_blocks), 2)


def nf4_scales_shifted(idx, scale, n_heads, d):
    """Each token dequantized with the next token's block scales."""
    return _nf4_dequantize(idx, np.roll(scale, -1, axis=2), n_heads, d)


def decode_recent_in_own_softmax(q, packed, alloc, bits_v, seq_len, V=None, K_recent=None, V_recent=None):
    """Recent tokens attended in a softmax of their own, averaged with the packed tokens'."""
    if K_recent is None or seq_len == 0:
        return _decode(q, packed, alloc, bits_v, seq_len, V=V, K_recent=K_recent, V_recent=V_recent)
    return 0.5 * (_decode(q, packed, alloc, bits_v, seq_len, V=V) + bg.decode_attention(q, K_recent, V_recent))


def decode_keys_only_values_rounded(q, packed, alloc, bits_v, seq_len, V=None, K_recent=None, V_recent=None):
    """A keys-only cache's values rounded to fp16 instead of taken exactly."""
    if bits_v == 0 and V is not None:
        V = np.asarray(V).astype(np.float16).astype(np.float64)
    return _decode(q, packed, alloc, bits_v, seq_len, V=V, K_recent=K_recent, V_recent=V_recent)


# ---------------------------------------------------------------- layout, header, RoPE, NF4

def pack_msb_first(values, widths):
    v = np.asarray(values, dtype=np.uint64)
    rev = np.zeros_like(v)
    for i, w in enumerate(widths):
        for p in range(w):
            rev[..., i] |= ((v[..., i] >> np.uint64(p)) & np.uint64(1)) << np.uint64(w - 1 - p)
    return _pack_bits(rev, widths)


def stream_widths_ascending(w_blocks):
    w_blocks = [int(x) for x in w_blocks]
    return [b for w in range(1, 9) for b in range(len(w_blocks)) if w_blocks[b] == w]


def splitmix_wrong_shift(z):
    m = (1 << 64) - 1
    z = (z + 0x9E3779B97F4A7C15) & m
    z = ((z ^ (z >> 31)) * 0xBF58476D1CE4E5B9) & m
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
    return z ^ (z >> 31)


def rotate_interleaved(x, pos, base):
    """Pairs (x_2i, x_2i+1) rotated instead of (x_i, x_{i+h})."""
    x = np.asarray(x, dtype=np.float64)
    ang = pos * rope.theta(x.shape[-1], base)
    c, s = np.cos(ang), np.sin(ang)
    out = np.empty_like(x)
    out[0::2] = x[0::2] * c - x[1::2] * s
    out[1::2] = x[1::2] * c + x[0::2] * s
    return out


def rotate_backwards(x, pos, base):
    return _rotate(x, -pos, base)


def nf4_mean_scale(X, block=nqkv.BLOCK):
    """Block scale from the mean absolute value instead of the maximum."""
    B, H, T, d = X.shape
    hidden = np.transpose(np.asarray(X, np.float32), (0, 2, 1, 3)).reshape(B, T, H * d)
    blocks = hidden.reshape(B, T, H * d // block, block)
    s16 = np.mean(np.abs(blocks), axis=-1).astype(np.float16)
    s32 = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        u = np.where(s32[..., None] == 0, np.float32(0), blocks / np.where(s32 == 0, 1, s32)[..., None]).astype(np.float32)
    idx = np.sum(cb.nf4_midpoints() < u[..., None], axis=-1).astype(np.uint8)
    return np.transpose(idx, (0, 2, 1, 3)), np.transpose(s16, (0, 2, 1))


def nf4_ties_up(X, block=nqkv.BLOCK):
    """#{midpoints <= u}: on the fp32 grid the same as comparing with each midpoint moved one
    fp32 step down, which the real quantizer is run with."""
    down = np.nextafter(_nf4_midpoints(), np.float32(-2))
    try:
        cb.nf4_midpoints = lambda: down
        return _nf4_quantize(X, block)
    finally:
        cb.nf4_midpoints = _nf4_midpoints


def nf4_nibbles_swapped(idx, scale, capacity):
    return _nf4_pack(np.concatenate([idx[..., 1::2, None], idx[..., 0::2, None]], axis=-1).reshape(idx.shape),
                     scale, capacity)


def nf4_unpack_padding_too(codes, scales, seq_len):
    return _orig["nqkv_unpack"](codes, scales, codes.shape[2])


# ---------------------------------------------------------------- codebooks

def lloyd_five_iterations(w):
    """Lloyd-Max stopped after five Lloyd iterations from the compander start."""
    n = 1 << w
    c = math.sqrt(3.0) * ndtri((np.arange(n) + 0.5) / n)
    for _ in range(5):
        c = cb._conditional_means(c)[0]
    return c, 0.5 * (c[:-1] + c[1:])


def thresholds_from_exact_centroids(w):
    """Stored thresholds as midpoints of the exact centroids instead of the stored fp16 ones."""
    c, _ = cb.lloyd_max_f64(w)
    return c.astype(np.float16), (0.5 * (c[:-1] + c[1:])).astype(np.float32)


def centroids_rounded_toward_zero(w):
    c, _ = cb.lloyd_max_f64(w)
    c16 = c.astype(np.float16)
    away = np.abs(c16.astype(np.float64)) > np.abs(c)
    c16 = np.where(away, np.nextafter(c16, np.float16(0)), c16).astype(np.float16)
    c16d = c16.astype(np.float64)
    return c16, (0.5 * (c16d[:-1] + c16d[1:])).astype(np.float32)


def delta_of_exact_quantizer():
    """Distortions of the exact Lloyd-Max quantizers instead of the stored ones."""
    return np.array([1.0] + [cb.quantizer_mse(*cb.lloyd_max_f64(w)) for w in range(1, 9)]).astype(np.float32)


def nf4_sides_swapped():
    """Eight negative and seven positive quantiles instead of seven and eight."""
    off = 0.5 * ((1.0 - 1.0 / 30) + (1.0 - 1.0 / 32))
    pos = ndtri(np.linspace(off, 0.5, 8)[:-1])
    neg = -ndtri(np.linspace(off, 0.5, 9)[:-1])
    v = np.sort(np.concatenate([neg, [0.0], pos]))
    return (v / np.max(np.abs(v))).astype(np.float32)


# ---------------------------------------------------------------- tile records and header

def k_words_token_major(codes, alloc, bits_v, capacity):
    """A token's K words stored contiguously (token-major) instead of word-planar."""
    out = _pack_cache(codes, alloc, bits_v, capacity).copy()
    nk = bg.tile_k_words(int(alloc["bits_k"]), int(alloc["d"]))
    kw = out[..., :4 * nk].copy().view("<u4")
    kw = kw.reshape(kw.shape[:-1] + (nk // bg.TILE, bg.TILE)).swapaxes(-1, -2).reshape(kw.shape)
    out[..., :4 * nk] = np.ascontiguousarray(kw).view(np.uint8)
    return out


def norms_k_and_v_swapped(codes, alloc, bits_v, capacity):
    out = _pack_cache(codes, alloc, bits_v, capacity).copy()
    a = 4 * bg.tile_k_words(int(alloc["bits_k"]), int(alloc["d"]))
    kn, vn = out[..., a:a + 64].copy(), out[..., a + 64:a + 128].copy()
    out[..., a:a + 64], out[..., a + 64:a + 128] = vn, kn
    return out


def block_pair_reversed(codes, alloc, bits_v, capacity):
    """Each block's pair streamed as (dim b + h, dim b) instead of (dim b, dim b + h)."""
    c = dict(codes)
    h = codes["Kc"].shape[-1] // 2
    c["Kc"] = np.concatenate([codes["Kc"][..., h:], codes["Kc"][..., :h]], axis=-1)
    return _pack_cache(c, alloc, bits_v, capacity)


def header_record_without_norms(batch, n_kv_heads, capacity, d, bits_k, bits_v, alloc):
    """Record size written without the 32 K and 32 V norms."""
    hdr = _packed_header(batch, n_kv_heads, capacity, d, bits_k, bits_v, alloc).copy()
    fields = hdr[16:32].view("<u4")
    fields[3] = 4 * d * (bits_k + bits_v)
    return hdr


_decode = bg.decode
_nf4_dequantize = nqkv.dequantize
_pack_cache = bg.pack_cache
_packed_header = bg.packed_header
_pack_bits = bg.pack_bits
_rotate = rope.rotate
_nf4_quantize = nqkv.quantize
_nf4_pack = nqkv.pack
_nf4_midpoints = cb.nf4_midpoints

# (name, module, attribute, replacement, pins: callables that must not all pass)
CASES = [
    ("energy: one left-to-right chain", bg, "calibration_energies", energy_one_chain,
     [pins.test_energy_summation_order_by_hand]),
    ("energy: partner coordinate dropped", bg, "calibration_energies", energy_without_partner,
     [pins.test_energy_matches_exact_mean]),
    ("energy: divided by one sequence's tokens", bg, "calibration_energies", energy_over_sequence_length,
     [pins.test_energy_matches_exact_mean]),
    ("greedy: ties to the highest block", bg, "greedy_widths", greedy_ties_to_highest,
     [pins.test_greedy_tie_breaks_to_lowest_block]),
    ("greedy: w_max ignored", bg, "greedy_widths", greedy_ignores_wmax,
     [pins.test_greedy_budget_and_wmax]),
    ("greedy: gain is the distortion left", bg, "greedy_widths", greedy_gain_is_distortion,
     [lambda: pins.test_greedy_matches_exhaustive_search(8), pins.test_greedy_matches_dynamic_programming_d16]),
    ("gains: factor 2 dropped", bg, "block_gains", gains_without_factor_two,
     [pins.test_block_gains_restore_unit_variance]),
    ("row norm: fp64 sum", bg, "row_norms_f16", norms_in_fp64,
     [pins.test_row_norm_summation_order_by_hand]),
    ("row norm: one fp32 chain", bg, "row_norms_f16", norms_one_fp32_chain,
     [pins.test_row_norm_summation_order_by_hand]),
    ("code: ties to the upper code", bg, "threshold_count", count_ties_up,
     [pins.test_quantizer_tie_goes_to_lower_code]),
    ("quantizer: sqrt(d) dropped from the scale", bg, "quantize_rows", quantize_without_sqrt_d,
     [pins.test_quantizer_tie_goes_to_lower_code]),
    ("quantizer: block gains not applied", bg, "quantize_rows", quantize_without_gains,
     [pins.test_quantizer_tie_goes_to_lower_code]),
    ("dequantizer: f_b dropped", bg, "dequantize_keys", keys_without_factor,
     [pins.test_dequantizer_by_hand]),
    ("dequantizer: 1/sqrt(d) dropped from values", bg, "dequantize_values", values_without_sqrt_d,
     [pins.test_dequantizer_by_hand]),
    ("attention: logits not scaled", bg, "decode_attention", lambda q, K, V: attention(q, K, V, scale=False),
     [pins.test_attention_matches_online_softmax_restatement]),
    ("attention: q head j reads KV head j mod Hkv", bg, "decode_attention",
     lambda q, K, V: attention(q, K, V, kv_of=lambda hq, G, Hkv: hq % Hkv),
     [pins.test_attention_single_token_returns_its_value]),
    ("widths: per-dim widths interleaved", bg, "widths_per_dim", widths_interleaved,
     [pins.test_dequantizer_by_hand]),
    ("NF4: each token dequantized with the next token's scales", nqkv, "dequantize", nf4_scales_shifted,
     [pins.test_nf4_fig5_worked_shape]),
    ("decode: recent tokens in a softmax of their own", bg, "decode", decode_recent_in_own_softmax,
     [pins.test_recent_buffer_duplicating_the_cache_changes_nothing]),
    ("decode: keys-only values rounded to fp16", bg, "decode", decode_keys_only_values_rounded,
     [pins.test_keys_only_cache_with_exact_values]),
    ("layout: codes packed most significant bit first", bg, "pack_bits", pack_msb_first,
     [pins.test_pack_bits_by_hand]),
    ("layout: stream by ascending width", bg, "k_stream_blocks", stream_widths_ascending,
     [pins.test_k_stream_order_by_hand]),
    ("header: a SplitMix64 shift changed", bg, "splitmix64", splitmix_wrong_shift,
     [pins.test_splitmix64_published_vectors]),
    ("RoPE: interleaved pairs", rope, "rotate", rotate_interleaved,
     [pins.test_rope_logit_is_sum_of_block_terms, pins.test_energy_is_rope_invariant]),
    ("RoPE: rotation the other way", rope, "rotate", rotate_backwards,
     [pins.test_rope_logit_is_sum_of_block_terms]),
    ("NF4: scale from the mean absolute value", nqkv, "quantize", nf4_mean_scale,
     [pins.test_nf4_quantize_special_cases]),
    ("NF4: a value on a midpoint takes the upper index", nqkv, "quantize", nf4_ties_up,
     [pins.test_nf4_midpoint_goes_to_lower_index]),
    ("NF4: nibbles swapped", nqkv, "pack", nf4_nibbles_swapped,
     [pins.test_nf4_pack_roundtrip_and_padding]),
    ("NF4: padded rows attended", nqkv, "unpack", nf4_unpack_padding_too,
     [pins.test_nf4_decode_masks_padding]),
    ("layout: K words token-major", bg, "pack_cache", k_words_token_major,
     [pins.test_pack_single_code_position_by_hand, pins.test_pack_unpack_roundtrip_mixed_widths]),
    ("layout: K and V norms swapped", bg, "pack_cache", norms_k_and_v_swapped,
     [pins.test_pack_single_code_position_by_hand]),
    ("layout: a block's two codes in reverse order", bg, "pack_cache", block_pair_reversed,
     [pins.test_pack_single_code_position_by_hand]),
    ("header: record size without the norms", bg, "packed_header", header_record_without_norms,
     [pins.test_header_fields_by_hand]),
    ("Lloyd-Max: not run to convergence", cb, "lloyd_max_f64", lloyd_five_iterations,
     [lambda: pins.test_lloyd_max_centroids_are_conditional_means(3), pins.test_lloyd_max_textbook_distortions]),
    ("codebook: thresholds from the exact centroids", cb, "stored_codebook", thresholds_from_exact_centroids,
     [pins.test_threshold_count_is_nearest_centroid]),
    ("codebook: centroids rounded toward zero", cb, "stored_codebook", centroids_rounded_toward_zero,
     [pins.test_stored_codebooks_symmetric_and_sorted]),
    ("greedy table: exact instead of stored distortions", cb, "delta_table", delta_of_exact_quantizer,
     [pins.test_delta_table_is_the_stored_quantizers_mse]),
    ("NF4 levels: the two sides swapped", cb, "nf4_values", nf4_sides_swapped,
     [pins.test_nf4_matches_published_table, pins.test_nf4_structure_and_quantile_spacing]),
]


@pytest.mark.parametrize("name,module,attr,bad,checks", CASES, ids=[c[0] for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, module, attr, bad, checks):
    monkeypatch.setattr(module, attr, bad)
    caught = []
    for check in checks:
        try:
            check()
        except (AssertionError, IndexError, ValueError):
            # a failed assertion, or a pin that can no longer run on the mutated oracle (a code
            # out of its codebook's range, a shape that no longer fits); a NameError or
            # TypeError would be a broken stand-in and is not taken as a catch
            caught.append(check)
    assert caught, f"no pin catches the planted mistake: {name}"


def test_pins_pass_on_the_oracle_as_it_stands():
    """The same pins, unmutated, pass (so a caught mistake is the mistake, not a broken pin)."""
    for _, _, _, _, checks in CASES:
        for check in checks:
            check()

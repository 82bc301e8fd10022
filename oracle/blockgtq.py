"""Block-GTQ on a TQ-MSE-style scalar quantizer: the oracle. TEST INFRASTRUCTURE ONLY.

Source: page "RoPE-aware bit allocation for KV cache quantization" (Liang,
Zhang, Jia; arXiv 2606.24033), abstract. As summarised there: per layer and KV
head an energy score is computed for each RoPE block without labels, and
integer bit widths are then handed out greedily by marginal gain; the
allocator sits on TurboQuant-MSE; K and V get matched budgets (K2V2, K3V3, ...);
the baseline gives every coordinate the same width (uniform TQ-MSE); attention
is served straight from a packed cache.

The page names these steps without defining them. The readings taken here
(each restated in the function that uses it):

  energy     E_b = mean over calibration tokens of ||k_b||^2, block b = dims
             (b, b + d/2); fp64, summed in a fixed order (64-token chunks,
             64-chunk segments, then segments).
  greedy     d/2 * bits_k steps; each adds one bit to the block with the
             largest E_b * (delta(w_b) - delta(w_b + 1)) among blocks below
             w_max; ties go to the lowest block index.
  gain       g_b = sqrt(2 sum(E) / (d E_b)) (unit variance per coordinate of
             block b after the global sqrt(d)/||k|| scaling), 1 if E_b = 0;
             f_b = 1 / (sqrt(d) g_b) is the matching dequant factor.
  quantizer  per token row: fp16 norm of the row (fp32 sum of squares in a fixed order of
             eight interleaved partial sums), a = sqrt(d)/norm in fp32,
             y = (x * a) * g_b in fp32, code = #{thresholds strictly below y}
             of the width-w_b Lloyd-Max codebook. Values use width bits_v, g = 1.
  layout     32-token tiles; per token one K bit stream (codes in width-class
             order), per dim one V bit stream over the tile's tokens, both stored
             word-planar (see pack_cache).
  attention  softmax over cached positions 0..T-1 of q . k_hat / sqrt(d),
             k_hat = norm * c[code] * f_b, v_hat = norm * c[code] / sqrt(d).
"""
from __future__ import annotations

import math

import numpy as np

from . import codebooks

TILE = 32            # tokens per packed tile
CALIB_CHUNK = 64     # tokens per fixed-order partial sum of the energy score
CALIB_SEGMENT = 64   # chunk sums per fixed-order segment sum

MODE_BLOCKGTQ = 0
MODE_UNIFORM = 1


# --------------------------------------------------------------------------- calibration

def calibration_energies(K: np.ndarray, n_calib: int = 0) -> tuple[np.ndarray, int]:
    """Label-free energy score per (KV head, RoPE block).

    K: [B][H][T][d] array whose values are exactly the stored keys (any float type).
    n_calib: number of leading tokens of every sequence to use (0 = all T).
    The calibration tokens of all sequences are pooled in the order
    u = s * n_calib + t. Each term is fl(fl(x_b^2) + fl(x_{b+h}^2)) in fp64. The
    sum has a fixed three-level order, every level left to right: terms within
    chunks of 64 consecutive pooled tokens, chunk sums within segments of 64
    consecutive chunks, then the segment sums; the last chunk and segment may be
    shorter. The total is divided by N = B * n_calib.
    Returns (E [H][d/2] float64, N).
    """
    B, H, T, d = K.shape
    h = d // 2
    n = T if n_calib <= 0 else n_calib
    if n > T:
        raise ValueError("n_calib exceeds the sequence length")
    X = np.asarray(K[:, :, :n, :], dtype=np.float64)
    X = np.transpose(X, (1, 0, 2, 3)).reshape(H, B * n, d)            # pooled token order
    terms = X[:, :, :h] * X[:, :, :h] + X[:, :, h:] * X[:, :, h:]     # [H][N][h]
    N = B * n
    chunk_sums = []
    for c0 in range(0, N, CALIB_CHUNK):
        acc = np.zeros((H, h), dtype=np.float64)
        for u in range(c0, min(N, c0 + CALIB_CHUNK)):
            acc = acc + terms[:, u, :]
        chunk_sums.append(acc)
    total = np.zeros((H, h), dtype=np.float64)
    for s0 in range(0, len(chunk_sums), CALIB_SEGMENT):
        seg = np.zeros((H, h), dtype=np.float64)
        for c in chunk_sums[s0:s0 + CALIB_SEGMENT]:
            seg = seg + c
        total = total + seg
    return total / float(N), N


def greedy_widths(E: np.ndarray, bits: int, w_max: int, delta: np.ndarray | None = None) -> np.ndarray:
    """Greedy integer bit allocation by marginal gain for one KV head.

    E: [h] energies. Runs bits * h steps; at each step the block b with
    w_b < w_max maximising E_b * (delta[w_b] - delta[w_b + 1]) (fp64, delta
    taken from the fp32 table) gets one more bit; ties go to the lowest b.
    """
    if delta is None:
        delta = codebooks.delta_table()
    D = np.asarray(delta, dtype=np.float64)
    h = len(E)
    if not (1 <= bits <= w_max <= 8):
        raise ValueError("need 1 <= bits <= w_max <= 8")
    w = np.zeros(h, dtype=np.int64)
    for _ in range(bits * h):
        best_b, best_gain = -1, -math.inf
        for b in range(h):
            if w[b] < w_max:
                gain = float(E[b]) * (D[w[b]] - D[w[b] + 1])
                if gain > best_gain:
                    best_b, best_gain = b, gain
        w[best_b] += 1
    return w


def block_gains(E: np.ndarray, d: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-block gain g_b (fp32) and dequant factor f_b (fp32) for one KV head.

    S = sum_b E_b left to right (fp64); g_b = fp32(sqrt((2 S) / (d E_b))) if E_b > 0
    else 1; f_b = fp32(1 / (sqrt(d) * g_b)) with g_b taken as its fp32 value.
    """
    E = np.asarray(E, dtype=np.float64)
    S = 0.0
    for e in E:
        S = S + float(e)
    g = np.ones(len(E), dtype=np.float32)
    for b, e in enumerate(E):
        if e > 0.0 and S > 0.0:
            g[b] = np.float32(math.sqrt((2.0 * S) / (float(d) * float(e))))
    f = np.array([np.float32(1.0 / (math.sqrt(float(d)) * float(gb))) for gb in g], dtype=np.float32)
    return g, f


def allocate(E: np.ndarray, d: int, bits_k: int, w_max: int = 8, mode: int = MODE_BLOCKGTQ) -> dict:
    """Allocation for every KV head: widths w [H][h], gains g, dequant factors f, energies E."""
    H, h = E.shape
    assert h == d // 2
    w = np.zeros((H, h), dtype=np.int64)
    g = np.ones((H, h), dtype=np.float32)
    f = np.zeros((H, h), dtype=np.float32)
    for hh in range(H):
        if mode == MODE_BLOCKGTQ:
            w[hh] = greedy_widths(E[hh], bits_k, w_max)
            g[hh], f[hh] = block_gains(E[hh], d)
        elif mode == MODE_UNIFORM:
            w[hh] = bits_k
            g[hh] = 1.0
            f[hh] = np.float32(1.0 / math.sqrt(float(d)))
        else:
            raise ValueError("mode")
    return {"E": E.copy(), "w": w, "g": g, "f": f, "d": d, "bits_k": bits_k, "w_max": w_max, "mode": mode}


def calibrate(K: np.ndarray, bits_k: int, n_calib: int = 0, w_max: int = 8, mode: int = MODE_BLOCKGTQ) -> dict:
    E, _ = calibration_energies(K, n_calib)
    return allocate(E, K.shape[-1], bits_k, w_max, mode)


# --------------------------------------------------------------------------- quantizer

def row_norms_f16(X: np.ndarray) -> np.ndarray:
    """fp16 norm of every row: fp16(fp32 sqrt(s2)), round to nearest even.

    s2 is an fp32 sum of the squares in a fixed order (reading R5; the page fixes neither the
    precision nor the order of this sum). Eight partial sums s_r, r = 0..7, each run over the
    coordinates j = r, r + 8, r + 16, ... in ascending j, one step being
    s_r = fl32(s_r + fl32(x_j * x_j)); they are then combined as
        s2 = fl32( fl32(fl32(s_0 + s_1) + fl32(s_2 + s_3))
                 + fl32(fl32(s_4 + s_5) + fl32(s_6 + s_7)) ).
    (The square is exact for 16-bit inputs.) The eight short chains keep the summation's
    dependency depth at 16 instead of d.
    """
    X32 = np.asarray(X, dtype=np.float32)
    d = X32.shape[-1]
    sq = (X32 * X32).astype(np.float32)
    s = [np.zeros(X32.shape[:-1], dtype=np.float32) for _ in range(8)]
    for j in range(d):
        r = j % 8
        s[r] = (s[r] + sq[..., j]).astype(np.float32)
    f32 = np.float32
    lo = ((s[0] + s[1]).astype(f32) + (s[2] + s[3]).astype(f32)).astype(f32)
    hi = ((s[4] + s[5]).astype(f32) + (s[6] + s[7]).astype(f32)).astype(f32)
    s2 = (lo + hi).astype(f32)
    return np.sqrt(s2).astype(np.float32).astype(np.float16)


def threshold_count(t32: np.ndarray, y: np.ndarray) -> np.ndarray:
    """code = #{thresholds t with t < y}, counted by comparison: a y on a threshold takes the
    lower code, and a NaN y (no threshold compares below it) takes code 0."""
    y = np.asarray(y, dtype=np.float32)
    t = np.asarray(t32, dtype=np.float32)
    return np.sum(t < y[..., None], axis=-1).astype(np.uint8)


def quantize_rows(X: np.ndarray, widths_dim: np.ndarray, gains_dim: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """TQ-MSE-style scalar quantizer for rows X[..., d].

    X holds exactly the stored values (converted to fp32 exactly).
    norm = row_norms_f16; a = fp32(sqrt(d)) / fp32(norm) (a = 0 when norm = 0);
    y_j = fp32(fp32(x_j * a) * g_j); code_j = #{thresholds of width w_j strictly
    below y_j} (0 where w_j = 0). Returns (codes uint8 [..., d], norms fp16 [...]).
    """
    X32 = np.asarray(X, dtype=np.float32)
    d = X32.shape[-1]
    n16 = row_norms_f16(X32)
    sqd = np.float32(math.sqrt(float(d)))
    n32 = n16.astype(np.float32)
    with np.errstate(divide="ignore"):
        a = np.where(n32 == 0, np.float32(0.0), sqd / np.where(n32 == 0, np.float32(1.0), n32)).astype(np.float32)
    y = (X32 * a[..., None]).astype(np.float32)
    y = (y * np.asarray(gains_dim, dtype=np.float32)).astype(np.float32)
    codes = np.zeros(X32.shape, dtype=np.uint8)
    for w in range(1, 9):
        sel = np.asarray(widths_dim) == w
        if not np.any(sel):
            continue
        _, t32 = codebooks.stored_codebook(w)
        codes[..., sel] = threshold_count(t32, y[..., sel])
    return codes, n16


def widths_per_dim(w_blocks: np.ndarray) -> np.ndarray:
    return np.concatenate([w_blocks, w_blocks])


def quantize(K: np.ndarray, V: np.ndarray, alloc: dict, bits_v: int) -> dict:
    """Codes and fp16 norms for K (Block-GTQ widths and gains) and V (uniform bits_v, g = 1;
    bits_v = 0: keys only, V is not quantized)."""
    B, H, T, d = K.shape
    Kc = np.zeros((B, H, T, d), dtype=np.uint8)
    Kn = np.zeros((B, H, T), dtype=np.float16)
    for hh in range(H):
        wd = widths_per_dim(alloc["w"][hh])
        gd = np.concatenate([alloc["g"][hh], alloc["g"][hh]])
        Kc[:, hh], Kn[:, hh] = quantize_rows(K[:, hh], wd, gd)
    if bits_v == 0:                     # keys only: values stay unquantized outside the cache
        return {"Kc": Kc, "Kn": Kn, "Vc": None, "Vn": None}
    Vc, Vn = quantize_rows(V, np.full(d, bits_v), np.ones(d, dtype=np.float32))
    return {"Kc": Kc, "Kn": Kn, "Vc": Vc, "Vn": Vn}


# --------------------------------------------------------------------------- packed layout

def tile_k_words(bits_k: int, d: int) -> int:
    return bits_k * d


def tile_v_words(bits_v: int, d: int) -> int:
    return bits_v * d


def tile_record_bytes(d: int, bits_k: int, bits_v: int) -> int:
    """Bytes of one 32-token tile record: K words, 32 K norms, 32 V norms (fp16), V words;
    a keys-only record (bits_v = 0) ends after the K norms."""
    if bits_v == 0:
        return 4 * tile_k_words(bits_k, d) + 2 * TILE
    return 4 * tile_k_words(bits_k, d) + 4 * tile_v_words(bits_v, d) + 2 * TILE * 2


def packed_bytes(batch: int, n_kv_heads: int, capacity: int, d: int, bits_k: int, bits_v: int) -> int:
    """Header plus tile records (bits_v = 0: keys only)."""
    n_tiles = -(-capacity // TILE)
    return header_bytes(n_kv_heads) + batch * n_kv_heads * n_tiles * tile_record_bytes(d, bits_k, bits_v)


def k_stream_blocks(w_blocks: np.ndarray) -> list[int]:
    """Blocks in the order their codes appear in a token's K bit stream: widths descending
    (8 down to 1), blocks ascending within one width; blocks of width 0 are left out."""
    w_blocks = [int(x) for x in w_blocks]
    return [b for w in range(8, 0, -1) for b in range(len(w_blocks)) if w_blocks[b] == w]


def k_bit_offsets(w_blocks: np.ndarray) -> np.ndarray:
    """Bit offset of block b's code pair in a token's K stream (-1 for width 0): the code of
    dim b sits at that offset and the code of dim b + d/2 right after it."""
    off = np.full(len(w_blocks), -1, dtype=np.int64)
    acc = 0
    for b in k_stream_blocks(w_blocks):
        off[b] = acc
        acc += 2 * int(w_blocks[b])
    return off


def pack_bits(values: np.ndarray, widths: list[int]) -> np.ndarray:
    """Concatenate values[..., i] (widths[i] bits each, least significant bit first) into one
    bit stream and return it as little-endian 32-bit words [..., ceil(sum/32)]."""
    values = np.asarray(values, dtype=np.uint64)
    total = int(sum(widths))
    n_words = -(-total // 32)
    bits = np.zeros(values.shape[:-1] + (32 * n_words,), dtype=np.uint8)
    pos = 0
    for i, w in enumerate(widths):
        for p in range(w):
            bits[..., pos] = ((values[..., i] >> np.uint64(p)) & np.uint64(1)).astype(np.uint8)
            pos += 1
    weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
    return np.sum(bits.reshape(values.shape[:-1] + (n_words, 32)).astype(np.uint64) * weights, axis=-1)


def unpack_bits(words: np.ndarray, widths: list[int]) -> np.ndarray:
    """Inverse of pack_bits: values [..., len(widths)] from words [..., n_words]."""
    words = np.asarray(words, dtype=np.uint64)
    n_words = words.shape[-1]
    bits = ((words[..., :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).reshape(
        words.shape[:-1] + (32 * n_words,))
    out = np.zeros(words.shape[:-1] + (len(widths),), dtype=np.uint64)
    pos = 0
    for i, w in enumerate(widths):
        for p in range(w):
            out[..., i] |= bits[..., pos] << np.uint64(p)
            pos += 1
    return out


# --------------------------------------------------------------------------- packed header
#
# Reading (the pages define no interface): every packed cache starts with a header that
# names its layout and the allocation its K codes were written with, so that a decode given
# another layer's allocation, or a descriptor with other widths, can refuse instead of
# returning wrong attention. Little-endian, header_bytes(n_kv_heads) long:
#   0 u32 magic "KVQ1"     4 u16 layout version    6 u16 head_dim
#   8 u8 bits_k            9 u8 bits_v (0: keys only)   10 u8 w_max   11 u8 mode
#  12 u32 status (0; an append that found a mismatch records its kvq_status here)
#  16 i32 batch           20 i32 n_kv_heads       24 i32 capacity    28 u32 record bytes
#  32..63 zero            64 u64 digest of each KV head's allocation, head order
# then zero padding to a multiple of 128 bytes; the tile records follow.

HEADER_MAGIC = 0x3151564B        # bytes "KVQ1"
LAYOUT_VERSION = 1
_M64 = (1 << 64) - 1


def splitmix64(z: int) -> int:
    """The SplitMix64 output function (Steele, Lea and Flood, "Fast splittable pseudorandom
    number generators", OOPSLA 2014; constants as published by Vigna): one 64-bit mix."""
    z = (z + 0x9E3779B97F4A7C15) & _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def alloc_digest(w_blocks, g_blocks) -> int:
    """64-bit digest of one KV head's allocation: the sum mod 2^64, over blocks b, of
    splitmix64(b << 40 | w_b << 32 | fp32 bits of g_b). Any change of a width or a gain
    changes it (up to 64-bit collisions); the sum does not depend on the order it is taken in."""
    g32 = np.asarray(g_blocks, dtype=np.float32).view(np.uint32)
    acc = 0
    for b in range(len(w_blocks)):
        acc = (acc + splitmix64((b << 40) | (int(w_blocks[b]) << 32) | int(g32[b]))) & _M64
    return acc


def header_bytes(n_kv_heads: int) -> int:
    return -(-(64 + 8 * n_kv_heads) // 128) * 128


def packed_header(batch: int, n_kv_heads: int, capacity: int, d: int, bits_k: int, bits_v: int,
                  alloc: dict) -> np.ndarray:
    """Header bytes of a packed cache written with allocation `alloc` (see the layout above)."""
    out = np.zeros(header_bytes(n_kv_heads), dtype=np.uint8)
    fields = np.zeros(8, dtype="<u4")
    fields[0] = HEADER_MAGIC
    fields[1] = LAYOUT_VERSION | (d << 16)
    fields[2] = bits_k | (bits_v << 8) | (int(alloc["w_max"]) << 16) | (int(alloc["mode"]) << 24)
    fields[3] = 0
    fields[4] = batch
    fields[5] = n_kv_heads
    fields[6] = capacity
    fields[7] = tile_record_bytes(d, bits_k, bits_v)
    out[:32] = fields.view(np.uint8)
    dig = np.array([alloc_digest(alloc["w"][h], alloc["g"][h]) for h in range(n_kv_heads)], dtype="<u8")
    out[64:64 + 8 * n_kv_heads] = dig.view(np.uint8)
    return out


def pack_cache_bytes(codes: dict, alloc: dict, bits_v: int, capacity: int) -> np.ndarray:
    """The whole packed buffer: header, then the tile records of pack_cache, flat."""
    rec = pack_cache(codes, alloc, bits_v, capacity)
    B, H = rec.shape[:2]
    hdr = packed_header(B, H, capacity, int(alloc["d"]), int(alloc["bits_k"]), bits_v, alloc)
    return np.concatenate([hdr, rec.reshape(-1)])


def pack_cache(codes: dict, alloc: dict, bits_v: int, capacity: int) -> np.ndarray:
    """Packed cache bytes [B][Hkv][n_tiles][record] for capacity tokens per sequence.

    Tile record (little-endian 32-bit words, then fp16 norms):
      K part, bits_k * d words, stored word-planar: word 32 i + t is word i of token t's
        K stream (i < 4 bits_k). A token's K stream is its K codes concatenated, least
        significant bit first, in the order of k_stream_blocks; each block gives the code
        of dim b (w_b bits) and then the code of dim b + d/2 (w_b bits). The stream is
        exactly bits_k * d bits long.
      32 fp16 K norms, then 32 fp16 V norms, in token order.
      V part, bits_v * d words, stored word-planar: word d i + j is word i of dim j's V
        stream (i < bits_v), which is the codes of tokens 0..31 of the tile at dim j,
        concatenated, bits_v bits each, least significant bit first.
    Keys and their norms come first and values with theirs last, so that a reader can fetch
    either half of a record in one contiguous piece. A keys-only record (bits_v = 0) holds the
    K part and the K norms only.
    Tokens at or beyond the sequence length T are stored with code 0 and norm 0.
    """
    Kc, Kn, Vc, Vn = codes["Kc"], codes["Kn"], codes["Vc"], codes["Vn"]
    B, H, T, d = Kc.shape
    h = d // 2
    bits_k = int(alloc["bits_k"])
    n_tiles = -(-capacity // TILE)
    if T > capacity:
        raise ValueError("more tokens than capacity")
    cap = n_tiles * TILE

    def padded(a, fill=0):
        out = np.full(a.shape[:2] + (cap,) + a.shape[3:], fill, dtype=a.dtype)
        out[:, :, :T] = a
        return out

    keys_only = bits_v == 0
    Kc, Kn = padded(Kc), padded(Kn)
    Kc = Kc.reshape(B, H, n_tiles, TILE, d)
    if not keys_only:
        Vc, Vn = padded(Vc), padded(Vn)
        Vc = Vc.reshape(B, H, n_tiles, TILE, d)
    rec = tile_record_bytes(d, bits_k, bits_v)
    out = np.zeros((B, H, n_tiles, rec), dtype=np.uint8)
    for hh in range(H):
        w_blocks = alloc["w"][hh]
        order = k_stream_blocks(w_blocks)
        dims = [j for b in order for j in (b, b + h)]
        widths = [int(w_blocks[b]) for b in order for _ in (0, 1)]
        kstream = pack_bits(Kc[:, hh][..., dims], widths)                     # [B][n_tiles][32][kw]
        if kstream.shape[-1] != tile_k_words(bits_k, d) // TILE:
            raise ValueError("widths do not fill the K budget")
        kwords = np.transpose(kstream, (0, 1, 3, 2)).reshape(B, n_tiles, -1)   # word-planar
        parts = [kwords.astype("<u4").view(np.uint8).reshape(B, n_tiles, -1),
                 Kn[:, hh].reshape(B, n_tiles, TILE).astype("<f2").view(np.uint8).reshape(B, n_tiles, -1)]
        if not keys_only:
            vstream = pack_bits(np.transpose(Vc[:, hh], (0, 1, 3, 2)), [bits_v] * TILE)   # [B][n_tiles][d][bv]
            vwords = np.transpose(vstream, (0, 1, 3, 2)).reshape(B, n_tiles, -1)
            parts += [Vn[:, hh].reshape(B, n_tiles, TILE).astype("<f2").view(np.uint8).reshape(B, n_tiles, -1),
                      vwords.astype("<u4").view(np.uint8).reshape(B, n_tiles, -1)]
        out[:, hh] = np.concatenate(parts, axis=-1)
    return out


def unpack_cache(packed: np.ndarray, alloc: dict, bits_v: int, seq_len: int) -> dict:
    """Inverse of pack_cache for the first seq_len tokens: codes and norms per token."""
    B, H, n_tiles, rec = packed.shape
    d = int(alloc["d"])
    h = d // 2
    bits_k = int(alloc["bits_k"])
    nk, nv = tile_k_words(bits_k, d), tile_v_words(bits_v, d)
    cap = n_tiles * TILE
    Kc = np.zeros((B, H, n_tiles, TILE, d), dtype=np.uint8)
    Vc = np.zeros((B, H, n_tiles, TILE, d), dtype=np.uint8)
    keys_only = bits_v == 0
    kw = packed[..., :4 * nk].copy().view("<u4")
    norms = packed[..., 4 * nk:4 * nk + (2 if keys_only else 4) * TILE].copy().view("<f2")
    vw = None if keys_only else packed[..., 4 * nk + 4 * TILE:].copy().view("<u4")
    Kn = norms[..., :TILE].reshape(B, H, cap)
    Vn = None if keys_only else norms[..., TILE:].reshape(B, H, cap)
    for hh in range(H):
        w_blocks = alloc["w"][hh]
        order = k_stream_blocks(w_blocks)
        dims = [j for b in order for j in (b, b + h)]
        widths = [int(w_blocks[b]) for b in order for _ in (0, 1)]
        kstream = np.transpose(kw[:, hh].reshape(B, n_tiles, nk // TILE, TILE), (0, 1, 3, 2))
        Kc[:, hh][..., dims] = unpack_bits(kstream, widths).astype(np.uint8)
        if not keys_only:
            vstream = np.transpose(vw[:, hh].reshape(B, n_tiles, bits_v, d), (0, 1, 3, 2))   # [B][n][d][bv]
            Vc[:, hh] = np.transpose(unpack_bits(vstream, [bits_v] * TILE), (0, 1, 3, 2)).astype(np.uint8)
    Kc = Kc.reshape(B, H, cap, d)[:, :, :seq_len]
    if keys_only:
        return {"Kc": Kc, "Kn": Kn[:, :, :seq_len].astype(np.float16), "Vc": None, "Vn": None}
    Vc = Vc.reshape(B, H, cap, d)[:, :, :seq_len]
    return {"Kc": Kc, "Kn": Kn[:, :, :seq_len].astype(np.float16),
            "Vc": Vc, "Vn": Vn[:, :, :seq_len].astype(np.float16)}


# --------------------------------------------------------------------------- dequant + attention

def dequantize_keys(Kc: np.ndarray, Kn: np.ndarray, alloc: dict) -> np.ndarray:
    """k_hat[b,h,t,j] = norm * c_{w}[code] * f_b in fp64 (0 where w_b = 0)."""
    B, H, T, d = Kc.shape
    out = np.zeros((B, H, T, d), dtype=np.float64)
    for hh in range(H):
        wd = widths_per_dim(alloc["w"][hh])
        fd = np.concatenate([alloc["f"][hh], alloc["f"][hh]]).astype(np.float64)
        for j in range(d):
            if wd[j] == 0:
                continue
            c16, _ = codebooks.stored_codebook(int(wd[j]))
            cval = c16.astype(np.float64)[Kc[:, hh, :, j]]
            out[:, hh, :, j] = Kn[:, hh].astype(np.float64) * cval * fd[j]
    return out


def dequantize_values(Vc: np.ndarray, Vn: np.ndarray, bits_v: int) -> np.ndarray:
    """v_hat = norm * c_{bits_v}[code] / sqrt(d) in fp64."""
    d = Vc.shape[-1]
    c16, _ = codebooks.stored_codebook(bits_v)
    return Vn.astype(np.float64)[..., None] * c16.astype(np.float64)[Vc] / math.sqrt(float(d))


def decode_attention(q: np.ndarray, Khat: np.ndarray, Vhat: np.ndarray) -> np.ndarray:
    """out[b, hq] = sum_t softmax_t(q . k_hat_t / sqrt(d)) v_hat_t over all given tokens (fp64).

    q: [B][Hq][d]; Khat, Vhat: [B][Hkv][T][d]; q-head hq reads KV head hq // (Hq / Hkv).
    """
    B, Hq, d = q.shape
    Hkv = Khat.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        for hq in range(Hq):
            kv = hq // G
            logits = Khat[b, kv] @ np.asarray(q[b, hq], dtype=np.float64) / math.sqrt(float(d))
            m = np.max(logits)
            p = np.exp(logits - m)
            out[b, hq] = (p @ Vhat[b, kv]) / np.sum(p)
    return out


def decode(q: np.ndarray, packed: np.ndarray, alloc: dict, bits_v: int, seq_len: int, V=None, K_recent=None,
           V_recent=None) -> np.ndarray:
    """Fused-path reference: unpack the stored bits, dequantize, attend (fp64).

    Keys-only cache (bits_v = 0; the Block-GTQ page reports key errors with only the keys
    quantized): the values of positions 0..seq_len-1 are the stored values V
    [B][Hkv][>= seq_len][d], taken exactly. Recent-token buffer (reading: the Block-GTQ page
    reports its results with no buffer of fp16 recent keys, which names the variant; here the
    R most recent tokens keep their keys and values unquantized): K_recent, V_recent [B][Hkv][R][d] hold positions
    seq_len .. seq_len + R - 1, attended in the same softmax with their exact values.
    seq_len may be 0 when R > 0.
    """
    parts_k, parts_v = [], []
    if seq_len > 0:
        u = unpack_cache(packed, alloc, bits_v, seq_len)
        parts_k.append(dequantize_keys(u["Kc"], u["Kn"], alloc))
        if bits_v == 0:
            parts_v.append(np.asarray(V, dtype=np.float64)[:, :, :seq_len])
        else:
            parts_v.append(dequantize_values(u["Vc"], u["Vn"], bits_v))
    if K_recent is not None and K_recent.shape[2] > 0:
        parts_k.append(np.asarray(K_recent, dtype=np.float64))
        parts_v.append(np.asarray(V_recent, dtype=np.float64))
    Khat = np.concatenate(parts_k, axis=2)
    Vhat = np.concatenate(parts_v, axis=2)
    return decode_attention(q, Khat, Vhat)

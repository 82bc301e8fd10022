"""Shared helpers for the GPU parity tests: run the oracle on the same inputs and compare."""
import math

import numpy as np

from oracle import blockgtq as bg

TOL = 2e-3   # max_j |o_j - o*_j| / max_j |o*_j| per (sequence, q-head)


def host_f32(t):
    """Exact fp32 host copy of a device tensor in any float dtype."""
    return t.detach().float().cpu().numpy()


def rel_err(out, ref):
    """Max over (b, h) of max_j |o - ref| / max_j |ref|."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.max(np.abs(out - ref), axis=-1)
    den = np.max(np.abs(ref), axis=-1)
    return float(np.max(num / den))


def compare_alloc(gpu_heads, ref):
    """Bit-exact comparison of the library allocation with the oracle's."""
    H = ref["w"].shape[0]
    assert len(gpu_heads) == H
    for h in range(H):
        g = gpu_heads[h]
        np.testing.assert_array_equal(g["E"].view(np.uint64), ref["E"][h].astype(np.float64).view(np.uint64))
        np.testing.assert_array_equal(g["w"], ref["w"][h])
        np.testing.assert_array_equal(g["g"].view(np.uint32), ref["g"][h].view(np.uint32))
        np.testing.assert_array_equal(g["f"].view(np.uint32), ref["f"][h].view(np.uint32))
        np.testing.assert_array_equal(g["bit_off"], bg.k_bit_offsets(ref["w"][h]))
        assert g["k_words"] == int(2 * ref["w"][h].sum())
        check_classes(g, ref["w"][h])
        check_plan(g, ref["w"][h])
        assert g["digest"] == bg.alloc_digest(ref["w"][h], ref["g"][h])


def check_classes(g, w):
    """The class table lists the stream order: widths descending, blocks ascending inside a
    class, bit offsets consistent with 2 * w bits per block."""
    order = bg.k_stream_blocks(w)
    n = len(order)
    assert g["n_blocks"] == n
    assert list(g["stream_block"][:n]) == order and all(x == 255 for x in g["stream_block"][n:])
    widths = sorted({int(x) for x in w if x > 0}, reverse=True)
    assert g["n_classes"] == len(widths)
    bit = 0
    for c, cw in enumerate(widths):
        blocks = [b for b in range(len(w)) if w[b] == cw]
        assert g["class_width"][c] == cw and g["class_blocks"][c] == len(blocks)
        assert order[g["class_first"][c]:g["class_first"][c] + len(blocks)] == blocks
        assert g["class_bit"][c] == bit
        bit += 2 * cw * len(blocks)
    assert all(x == 0 for x in g["class_width"][len(widths):])


def check_plan(g, w):
    """Decode plan: width classes in stream order cut into slots of 4 consecutive block pairs;
    slot s covers columns 4s..4s+3, starts at the bit offset of its first block, and every
    block with w > 0 owns exactly one column."""
    order = bg.k_stream_blocks(w)
    off = bg.k_bit_offsets(w)
    cb = g["plan_col_block"]
    n_slots = int(g["plan_n_slots"])
    assert g["plan_k_cols"] == -(-4 * n_slots // 8) * 8
    widths = sorted({int(x) for x in w if x > 0}, reverse=True)
    expect_slots = sum(-(-sum(1 for x in w if x == cw) // 4) for cw in widths)
    assert n_slots == expect_slots
    blocks = [int(x) for x in cb if x >= 0]
    assert sorted(blocks) == [b for b in range(len(w)) if w[b] > 0]
    for s in range(24):
        e = int(g["plan_slot"][s])
        if s >= n_slots:
            assert e == 0 and all(int(x) == -1 for x in cb[4 * s:4 * s + 4])
            continue
        width, bit = e & 0xff, e >> 8
        b0 = int(cb[4 * s])
        assert b0 >= 0 and w[b0] == width and off[b0] == bit
        for k in range(4):
            bk = int(cb[4 * s + k])
            if bk >= 0:
                assert w[bk] == width and off[bk] == bit + 2 * width * k
    # columns follow the stream order, padding aside
    assert blocks == order


def oracle_pipeline(K, V, q, bits_k, bits_v, n_calib=0, w_max=8, mode=0, capacity=None):
    """Oracle calibrate -> quantize -> pack -> decode on host fp32 copies."""
    Kh, Vh = host_f32(K), host_f32(V)
    alloc = bg.calibrate(Kh, bits_k, n_calib=n_calib, w_max=w_max, mode=mode)
    T = Kh.shape[2]
    cap = T if capacity is None else capacity
    codes = bg.quantize(Kh, Vh, alloc, bits_v)
    packed = bg.pack_cache(codes, alloc, bits_v, cap)
    out = None
    if q is not None:
        out = bg.decode(host_f32(q), packed, alloc, bits_v, T)
    return alloc, packed, out


def tiles_written(T):
    return -(-T // bg.TILE)


def split_packed(packed_np, B, H, cap, bits_k, bits_v):
    """(header bytes, records [B][H][n_tiles][record]) of a host copy of a packed cache."""
    hb = bg.header_bytes(H)
    rec = bg.tile_record_bytes(128, bits_k, bits_v)
    n = B * H * tiles_written(cap) * rec
    return packed_np[:hb], packed_np[hb:hb + n].reshape(B, H, tiles_written(cap), rec)


def check_packed(packed_np, ref_alloc, ref_records, B, H, cap, bits_k, bits_v, n_tiles=None):
    """Header and (the first n_tiles of) the records byte for byte against the oracle."""
    hdr, recs = split_packed(packed_np, B, H, cap, bits_k, bits_v)
    np.testing.assert_array_equal(hdr, bg.packed_header(B, H, cap, 128, bits_k, bits_v, ref_alloc))
    if n_tiles is None:
        np.testing.assert_array_equal(recs, ref_records)
    else:
        np.testing.assert_array_equal(recs[:, :, :n_tiles], ref_records[:, :, :n_tiles])

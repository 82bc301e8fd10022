"""GPU parity through the C ABI: libkvq against the CPU oracle on the same seeded inputs.

Bit-exact: energies, widths, gains, dequant factors, packed codes and norms (NF4 codes
and scales). Attention: max_j |o - o*| / max_j |o*| <= 2e-3 per (sequence, q-head).
"""
import math

import numpy as np
import pytest

from oracle import blockgtq as bg
from oracle import nqkv
from packed_cache_attention_b200 import kvq
from packed_cache_attention_b200 import workloads as wl
from tests.parity_util import (TOL, check_packed, compare_alloc, host_f32, oracle_pipeline, rel_err, split_packed,
                               tiles_written)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    kvq.lib()
    kvq._check("kvq_init", kvq.lib().kvq_init())
    return torch.device("cuda:0")


def run_gpu(K, V, q, bits_k, bits_v, n_calib=0, w_max=8, mode=0, capacity=None, seq_len=None):
    import torch
    B, H, T, _ = K.shape
    cap = T if capacity is None else capacity
    alloc = kvq.kvq_calibrate(K, bits_k, w_max=w_max, n_calib=n_calib, mode=mode)
    cache = kvq.cache_desc(B, H, cap, bits_k, bits_v)
    packed = kvq.kvq_quantize(K, V, alloc, cache)
    out = None
    if q is not None:
        ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, q.shape[1]), dtype=torch.uint8, device=K.device)
        out = kvq.kvq_decode_attn(q, packed, alloc, cache, T if seq_len is None else seq_len, ws=ws)
        assert kvq.kvq_workspace_status(ws) == 0
    torch.cuda.synchronize()
    heads = kvq.parse_alloc(alloc.cpu().numpy())
    return heads, packed.cpu().numpy(), (out.cpu().numpy() if out is not None else None), cache


def packed_view(packed_np, B, H, cap, bits_k, bits_v):
    """The tile records of a host copy of a packed cache (the header skipped)."""
    return split_packed(packed_np, B, H, cap, bits_k, bits_v)[1]


CASES = [
    # (B, Hq, Hkv, T, dtype, bits_k, bits_v, profile, n_calib, mode, w_max)
    (1, 1, 1, 512, "f32", 3, 3, "loguniform", 0, 0, 8),
    (1, 4, 1, 1, "bf16", 3, 3, "lognormal_outliers", 0, 0, 8),
    (2, 8, 2, 33, "bf16", 2, 2, "lognormal_outliers", 0, 0, 8),
    (1, 8, 1, 100, "f16", 4, 4, "lognormal_outliers", 0, 0, 8),
    (2, 6, 2, 257, "bf16", 3, 2, "loguniform", 100, 0, 8),
    (1, 2, 2, 64, "bf16", 3, 3, "lognormal_outliers", 0, 1, 8),
    (1, 4, 2, 95, "f32", 2, 4, "lognormal_outliers", 0, 0, 4),
    (1, 16, 2, 1000, "bf16", 1, 1, "lognormal_outliers", 0, 0, 8),
    (1, 8, 1, 700, "bf16", 8, 8, "loguniform", 0, 0, 8),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}Hq{c[1]}Hkv{c[2]}T{c[3]}{c[4]}K{c[5]}V{c[6]}m{c[9]}")
def test_small_cases_match_oracle(dev, case):
    B, Hq, Hkv, T, dtype, bk, bv, prof, n_calib, mode, w_max = case
    x = wl.make_blockgtq_inputs(B, Hq, Hkv, 128, T, dtype, 1e4, prof, seed=T + bk, device=dev)
    heads, packed, out, _ = run_gpu(x["K"], x["V"], x["q"], bk, bv, n_calib, w_max, mode)
    ref_alloc, ref_packed, ref_out = oracle_pipeline(x["K"], x["V"], x["q"], bk, bv, n_calib, w_max, mode)
    compare_alloc(heads, ref_alloc)
    check_packed(packed, ref_alloc, ref_packed, B, Hkv, T, bk, bv)
    assert rel_err(out, ref_out) <= TOL


def test_tiny_workload_seed0(dev):
    """The tiny single-head workload exactly as stated: fp32, T 512, K3V3, seed 0."""
    W = wl.WORKLOADS["tiny"]
    x = wl.make_blockgtq_inputs(W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim, W.seq_len, W.dtype, W.rope_base,
                                W.key_profile, seed=0, device=dev)
    heads, packed, out, _ = run_gpu(x["K"], x["V"], x["q"], W.bits_k, W.bits_v)
    ref_alloc, ref_packed, ref_out = oracle_pipeline(x["K"], x["V"], x["q"], W.bits_k, W.bits_v)
    compare_alloc(heads, ref_alloc)
    np.testing.assert_array_equal(packed_view(packed, 1, 1, W.seq_len, W.bits_k, W.bits_v), ref_packed)
    assert rel_err(out, ref_out) <= TOL


def test_crafted_energy_order_and_norm_overflow(dev):
    """Keys whose fp64 energies depend on the fixed summation order (64-token chunks, 64-chunk
    segments, then segments): the kernel's energies equal the oracle's bit for bit. Their
    rows of 2^26 and 2^27 have norms beyond the fp16 range, so they store norm +inf with every
    code taken at y = 0; the packed cache equals the oracle's byte for byte."""
    import torch
    from tests.test_oracle_pins import crafted_energy_keys
    Kh = crafted_energy_keys()
    K = torch.from_numpy(Kh).to(dev).to(torch.bfloat16)
    assert torch.equal(K.float().cpu(), torch.from_numpy(Kh))       # bf16-exact by construction
    gen = torch.Generator(device=dev).manual_seed(3)
    V = torch.randn(K.shape, generator=gen, device=dev).to(torch.bfloat16)
    for mode in (0, 1):
        heads, packed, _, _ = run_gpu(K, V, None, 3, 3, mode=mode)
        ref_alloc, ref_packed, _ = oracle_pipeline(K, V, None, 3, 3, mode=mode)
        compare_alloc(heads, ref_alloc)
        np.testing.assert_array_equal(packed_view(packed, 1, 1, 8192, 3, 3), ref_packed)
    u = bg.unpack_cache(ref_packed, ref_alloc, 3, 8192)
    assert np.isinf(float(u["Kn"][0, 0, 0])) and np.isinf(float(u["Kn"][0, 0, 4096]))


def _tie_rows(rng, T, widths, gains, n_ties=24):
    """fp32 rows [T][128] in which n_ties coordinates of every row land exactly on a threshold:
    fl32(fl32(x a) g) = t with a = fp32(sqrt 128) / fp16 norm of the row (the oracle's R5)."""
    X = (rng.standard_normal((T, 128)) * 2.0).astype(np.float32)
    sqd = np.float32(math.sqrt(128.0))
    hit = np.zeros((T, 128), dtype=bool)
    for t in range(T):
        cols = rng.choice(128, size=n_ties, replace=False)
        for _ in range(4):                       # the fp16 norm settles after a pass or two
            n16 = bg.row_norms_f16(X[t][None])[0]
            a = np.float32(sqd / np.float32(n16))
            for j in cols:
                w = int(widths[j])
                if w == 0:
                    continue
                _, t32 = bg.codebooks.stored_codebook(w)
                tau = t32[rng.integers(len(t32))]
                g = np.float32(gains[j])
                v0 = np.float32(tau / (a * g))
                for k in range(-6, 7):
                    v = np.float32(v0 + np.float32(k) * np.spacing(v0))
                    if np.float32(np.float32(v * a) * g) == tau:
                        X[t, j] = v
                        break
        n16 = bg.row_norms_f16(X[t][None])[0]
        a = np.float32(sqd / np.float32(n16))
        for j in cols:
            w = int(widths[j])
            if w:
                y = np.float32(np.float32(X[t, j] * a) * np.float32(gains[j]))
                hit[t, j] = bool(np.any(bg.codebooks.stored_codebook(w)[1] == y))
    return X, hit


@pytest.mark.parametrize("mode", [1, 0])
def test_threshold_ties_at_full_head_dim(dev, mode):
    """Coordinates exactly on a threshold at d = 128 take the lower code on the GPU as in the
    oracle: fp32 keys and values built so that fl32(x a) (times g_b in Block-GTQ mode) equals
    a stored threshold; the packed cache is compared byte for byte."""
    import torch
    rng = np.random.default_rng(77 + mode)
    T = 64
    x = wl.make_blockgtq_inputs(1, 2, 1, 128, T, "f32", 1e4, "loguniform", seed=8, device=dev)
    Kh = host_f32(x["K"])
    ref_alloc = bg.calibrate(Kh, 3, mode=mode)
    wk = bg.widths_per_dim(ref_alloc["w"][0])
    gk = np.concatenate([ref_alloc["g"][0], ref_alloc["g"][0]])
    # keep the calibration input, change the rows that are quantized: calibrate on K, then
    # quantize rows built against that allocation (the allocation only depends on K's energies)
    Kt, hit_k = _tie_rows(rng, T, wk, gk)
    Vt, hit_v = _tie_rows(rng, T, np.full(128, 4), np.ones(128, np.float32))
    assert hit_k.sum() > T and hit_v.sum() > T
    alloc = kvq.kvq_calibrate(x["K"], 3, mode=mode)
    cache = kvq.cache_desc(1, 1, T, 3, 4)
    Kd = torch.from_numpy(Kt).reshape(1, 1, T, 128).to(dev)
    Vd = torch.from_numpy(Vt).reshape(1, 1, T, 128).to(dev)
    packed = kvq.kvq_quantize(Kd, Vd, alloc, cache).cpu().numpy()
    codes = bg.quantize(Kt.reshape(1, 1, T, 128), Vt.reshape(1, 1, T, 128), ref_alloc, 4)
    ref_packed = bg.pack_cache(codes, ref_alloc, 4, T)
    np.testing.assert_array_equal(packed_view(packed, 1, 1, T, 3, 4), ref_packed)
    # the oracle took the lower code at every tie: the threshold itself is not below y
    for X, hit, C, wd in ((Kt, hit_k, codes["Kc"][0, 0], wk), (Vt, hit_v, codes["Vc"][0, 0], np.full(128, 4))):
        t_idx, j_idx = np.nonzero(hit)
        for t, j in zip(t_idx[:50], j_idx[:50]):
            _, t32 = bg.codebooks.stored_codebook(int(wd[j]))
            n16 = bg.row_norms_f16(X[t][None])[0]
            a = np.float32(np.float32(math.sqrt(128.0)) / np.float32(n16))
            y = np.float32(X[t, j] * a) if X is Vt else np.float32(np.float32(X[t, j] * a) * np.float32(gk[j]))
            assert C[t, j] == int(np.sum(t32 < y)) and np.any(t32 == y)


def test_capacity_larger_than_tokens_and_prefix_decode(dev):
    import torch
    x = wl.make_blockgtq_inputs(1, 8, 2, 128, 150, "bf16", 5e5, "lognormal_outliers", seed=7, device=dev)
    heads, packed, _, cache = run_gpu(x["K"], x["V"], None, 3, 3, capacity=1000)
    ref_alloc, ref_packed, _ = oracle_pipeline(x["K"], x["V"], None, 3, 3, capacity=1000)
    got = packed_view(packed, 1, 2, 1000, 3, 3)[:, :, :tiles_written(150)]
    np.testing.assert_array_equal(got, ref_packed[:, :, :tiles_written(150)])
    # decode over a prefix of the quantized tokens
    alloc_t = kvq.kvq_calibrate(x["K"], 3)
    packed_t = kvq.kvq_quantize(x["K"], x["V"], alloc_t, cache)
    for sl in (1, 31, 32, 97, 150):
        out = kvq.kvq_decode_attn(x["q"], packed_t, alloc_t, cache, sl).cpu().numpy()
        ref = bg.decode(host_f32(x["q"]), ref_packed, ref_alloc, 3, sl)
        assert rel_err(out, ref) <= TOL, sl


def test_zero_rows_and_single_token(dev):
    import torch
    x = wl.make_blockgtq_inputs(1, 4, 1, 128, 40, "bf16", 1e4, "loguniform", seed=3, device=dev)
    K, V = x["K"].clone(), x["V"].clone()
    K[0, 0, 5] = 0
    V[0, 0, 6] = 0
    heads, packed, out, _ = run_gpu(K, V, x["q"], 3, 3)
    ref_alloc, ref_packed, ref_out = oracle_pipeline(K, V, x["q"], 3, 3)
    np.testing.assert_array_equal(packed_view(packed, 1, 1, 40, 3, 3), ref_packed)
    assert rel_err(out, ref_out) <= TOL


def test_repeated_decode_reuses_workspace(dev):
    """The split tickets are reset by the last CTA, so one zeroed workspace serves many calls."""
    import torch
    x = wl.make_blockgtq_inputs(1, 16, 2, 128, 4096, "bf16", 1e6, "lognormal_outliers", seed=11, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], 3)
    cache = kvq.cache_desc(1, 2, 4096, 3, 3)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, 16), dtype=torch.uint8, device=dev)
    outs = [kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 4096, ws=ws).clone() for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o, outs[0])
    assert kvq.kvq_workspace_status(ws) == 0


def test_workspace_serves_every_length_of_a_cache(dev):
    """One workspace sized for a cache serves decodes of any length in any order, including a
    long length (two-level split merge) right after short ones (one split, one-level merge):
    each output equals the decode with a freshly zeroed workspace, bit for bit."""
    import torch
    T = 131072
    x = wl.make_blockgtq_inputs(1, 16, 2, 128, T, "bf16", 1e6, "lognormal_outliers", seed=17, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], 3)
    cache = kvq.cache_desc(1, 2, T, 3, 3)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    nbytes = kvq.kvq_decode_workspace_bytes(cache, 16)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    for n in (300, 5000, T, 700, 40000, T, 1):
        got = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, n, ws=ws).clone()
        fresh = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        want = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, n, ws=fresh)
        assert torch.equal(got, want), n
        assert kvq.kvq_workspace_status(ws) == 0


APPEND_CASES = [("bf16", 3, 3), ("f16", 5, 7), ("f32", 2, 4)]


@pytest.mark.parametrize("case", APPEND_CASES, ids=lambda c: f"{c[0]}K{c[1]}V{c[2]}")
def test_append_in_pieces_equals_one_quantize(dev, case):
    """The cache only grows ([NQKV] assumptions), so appending a sequence piece by piece
    (single tokens on both sides of tile boundaries, ragged chunks) must store the same bytes
    as one quantize call, whatever the buffer held before; decode over the grown cache then
    matches the oracle at every prefix length reached."""
    import torch
    dtype, bk, bv = case
    T = 200
    x = wl.make_blockgtq_inputs(2, 8, 2, 128, T, dtype, 1e6, "lognormal_outliers", seed=5 + bk, device=dev)
    K, V, q = x["K"], x["V"], x["q"]
    alloc = kvq.kvq_calibrate(K, bk)
    cache = kvq.cache_desc(2, 2, 256, bk, bv)
    one = kvq.kvq_quantize(K, V, alloc, cache)
    grown = torch.full_like(one, 0xAB)
    cuts = [0, 1, 2, 31, 32, 33, 64, 100, 101, 150, 199, 200]
    ref_alloc = bg.calibrate(host_f32(K), bk)
    for a, b in zip(cuts[:-1], cuts[1:]):
        kvq.kvq_append(K[:, :, a:b], V[:, :, a:b], alloc, cache, a, grown)
        if b in (33, 101, 200):
            out = kvq.kvq_decode_attn(q, grown, alloc, cache, b).cpu().numpy()
            ref_packed = bg.pack_cache(bg.quantize(host_f32(K[:, :, :b]), host_f32(V[:, :, :b]), ref_alloc, bv),
                                       ref_alloc, bv, b)
            ref = bg.decode(host_f32(q), ref_packed, ref_alloc, bv, b)
            assert rel_err(out, ref) <= TOL, b
    torch.cuda.synchronize()
    nt = tiles_written(T)
    g = packed_view(grown.cpu().numpy(), 2, 2, 256, bk, bv)[:, :, :nt]
    o = packed_view(one.cpu().numpy(), 2, 2, 256, bk, bv)[:, :, :nt]
    np.testing.assert_array_equal(g, o)


def test_append_edges_match_oracle(dev):
    """Appends at the cache's edges: the first token into a buffer of garbage, a run that ends
    exactly at the capacity, and a one-token append into a tile whose other 31 tokens are
    stored; each stored tile equals the oracle's, and decode over 1 and over all tokens
    matches the oracle."""
    import torch
    T = 96
    x = wl.make_blockgtq_inputs(1, 8, 2, 128, T, "bf16", 1e6, "lognormal_outliers", seed=21, device=dev)
    K, V, q = x["K"], x["V"], x["q"]
    alloc = kvq.kvq_calibrate(K, 3)
    cache = kvq.cache_desc(1, 2, T, 3, 3)
    grown = torch.full((kvq.kvq_packed_bytes(cache),), 0xC3, dtype=torch.uint8, device=dev)
    ref_alloc = bg.calibrate(host_f32(K), 3)
    kvq.kvq_append(K[:, :, :1], V[:, :, :1], alloc, cache, 0, grown)
    out1 = kvq.kvq_decode_attn(q, grown, alloc, cache, 1).cpu().numpy()
    ref1 = bg.pack_cache(bg.quantize(host_f32(K[:, :, :1]), host_f32(V[:, :, :1]), ref_alloc, 3), ref_alloc, 3, 1)
    assert rel_err(out1, bg.decode(host_f32(q), ref1, ref_alloc, 3, 1)) <= TOL
    kvq.kvq_append(K[:, :, 1:63], V[:, :, 1:63], alloc, cache, 1, grown)
    kvq.kvq_append(K[:, :, 64:], V[:, :, 64:], alloc, cache, 64, grown)     # ends at the capacity
    kvq.kvq_append(K[:, :, 63:64], V[:, :, 63:64], alloc, cache, 63, grown)  # last hole of tile 1
    ref = bg.pack_cache(bg.quantize(host_f32(K), host_f32(V), ref_alloc, 3), ref_alloc, 3, T)
    np.testing.assert_array_equal(packed_view(grown.cpu().numpy(), 1, 2, T, 3, 3), ref)
    out = kvq.kvq_decode_attn(q, grown, alloc, cache, T).cpu().numpy()
    assert rel_err(out, bg.decode(host_f32(q), ref, ref_alloc, 3, T)) <= TOL


def test_append_full_size_matches_one_quantize(dev):
    """At the 128K Qwen2.5-3B shape, in the calls the benchmark times (a 4096-token chunk and
    a single token appended at the end of a cache that already holds the rest), the grown
    cache is byte-identical to one quantize call over the whole sequence."""
    import torch
    W = wl.WORKLOADS["qwen3b"]
    x = wl.make_blockgtq_inputs(W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim, W.seq_len, W.dtype, W.rope_base,
                                W.key_profile, seed=3, device=dev, with_q=False)
    K, V, T = x["K"], x["V"], W.seq_len
    alloc = kvq.kvq_calibrate(K, W.bits_k)
    cache = kvq.cache_desc(W.batch, W.n_kv_heads, T, W.bits_k, W.bits_v)
    one = kvq.kvq_quantize(K, V, alloc, cache)
    grown = torch.full_like(one, 0x5A)
    a = T - 4096 - 1
    kvq.kvq_append(K[:, :, :a], V[:, :, :a], alloc, cache, 0, grown)
    kvq.kvq_append(K[:, :, a:T - 1], V[:, :, a:T - 1], alloc, cache, a, grown)
    kvq.kvq_append(K[:, :, T - 1:], V[:, :, T - 1:], alloc, cache, T - 1, grown)
    torch.cuda.synchronize()
    assert torch.equal(grown, one)


# ----------------------------------------------------------------------------- header, keys only, timeouts

def _layer(dev, seed, T=300, Hq=8, Hkv=2, bk=3, bv=3, cap=None):
    x = wl.make_blockgtq_inputs(1, Hq, Hkv, 128, T, "bf16", 1e6, "lognormal_outliers", seed=seed, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], bk)
    cache = kvq.cache_desc(1, Hkv, T if cap is None else cap, bk, bv)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    return x, alloc, cache, packed


def test_decode_refuses_another_layers_allocation(dev):
    """The packed header names the allocation its codes were written with (per-head digest):
    a decode given another layer's allocation, or a descriptor with other widths, records
    KVQ_ERR_MISMATCH and leaves the output untouched."""
    import torch
    x, alloc, cache, packed = _layer(dev, 61)
    _, alloc_b, _, _ = _layer(dev, 62)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, 8), dtype=torch.uint8, device=dev)
    out = torch.full((1, 8, 128), 12345.0, device=dev)
    kvq.kvq_decode_attn(x["q"], packed, alloc_b, cache, 300, out=out, ws=ws)
    assert kvq.kvq_workspace_status(ws) == kvq.KVQ_ERR_MISMATCH
    assert torch.all(out == 12345.0)
    kvq.kvq_workspace_init(ws)
    other = kvq.cache_desc(1, 2, 300, 3, 2)                     # V width the cache was not written with
    ws2 = torch.zeros(kvq.kvq_decode_workspace_bytes(other, 8), dtype=torch.uint8, device=dev)
    kvq.kvq_decode_attn(x["q"], packed, alloc, other, 300, out=out, ws=ws2)
    assert kvq.kvq_workspace_status(ws2) == kvq.KVQ_ERR_MISMATCH
    assert torch.all(out == 12345.0)
    # the right allocation still decodes, matching the oracle
    got = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 300, ws=ws).cpu().numpy()
    assert kvq.kvq_workspace_status(ws) == 0
    _, _, ref = oracle_pipeline(x["K"], x["V"], x["q"], 3, 3)
    assert rel_err(got, ref) <= TOL


def test_decode_refuses_a_slot_plan_past_the_key_stream(dev):
    """An allocation whose decode plan points a slot of KV head 0 past the key stream (its
    digest still matching the cache) is refused before any lookup: KVQ_ERR_MISMATCH, the
    query rows of head 0 untouched, head 1 decoded as with the intact allocation."""
    import torch
    x, alloc, cache, packed = _layer(dev, 65)
    bad = alloc.clone()
    off = kvq.HeadAlloc.plan_slot.offset                         # head 0, slot 0
    word = 3 | ((128 * 3 + 5) << 8)                              # width 3, first code past 384 bits
    bad[off:off + 4] = torch.tensor(list(int(word).to_bytes(4, "little")), dtype=torch.uint8, device=dev)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, 8), dtype=torch.uint8, device=dev)
    out = torch.full((1, 8, 128), 3.0, device=dev)
    kvq.kvq_decode_attn(x["q"], packed, bad, cache, 300, out=out, ws=ws)
    assert kvq.kvq_workspace_status(ws) == kvq.KVQ_ERR_MISMATCH
    assert torch.all(out[:, :4] == 3.0)
    good = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 300)
    assert torch.equal(out[:, 4:], good[:, 4:])


def test_append_refuses_another_allocation(dev):
    """An append (t_begin > 0) extends only a cache whose header names its allocation: with
    another layer's allocation it writes nothing and leaves KVQ_ERR_MISMATCH in the header,
    which the decode then reports; quantizing from token 0 writes a fresh header."""
    import torch
    x, alloc, cache, packed = _layer(dev, 63, T=200, cap=256)
    _, alloc_b, _, _ = _layer(dev, 64, T=200)
    before = packed.clone()
    kvq.kvq_append(x["K"][:, :, 100:150], x["V"][:, :, 100:150], alloc_b, cache, 100, packed)
    assert kvq.kvq_packed_status(packed) == kvq.KVQ_ERR_MISMATCH
    hb = kvq.kvq_packed_header_bytes(2)
    assert torch.equal(packed[hb:], before[hb:])
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, 8), dtype=torch.uint8, device=dev)
    out = torch.full((1, 8, 128), 7.0, device=dev)
    kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 200, out=out, ws=ws)
    assert kvq.kvq_workspace_status(ws) == kvq.KVQ_ERR_MISMATCH and torch.all(out == 7.0)
    kvq.kvq_quantize(x["K"], x["V"], alloc, cache, packed=packed)
    assert kvq.kvq_packed_status(packed) == 0
    assert torch.equal(packed, before)


def test_decode_wait_timeout_is_reported(dev):
    """Bounded waits (SURVEY failure detection, on the device): with the test hook that makes
    the decode issue no copy at all, every warpgroup's first wait runs out with nothing in
    flight; the call records KVQ_ERR_TIMEOUT, writes nothing, and the context stays usable."""
    import torch
    x, alloc, cache, packed = _layer(dev, 65, T=5000)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, 8), dtype=torch.uint8, device=dev)
    out = torch.full((1, 8, 128), -3.0, device=dev)
    try:
        kvq.kvq_debug_decode(wait_limit=3, no_loads=True)
        kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 5000, out=out, ws=ws)
        torch.cuda.synchronize()
    finally:
        kvq.kvq_debug_decode(wait_limit=2000, no_loads=False)
    assert kvq.kvq_workspace_status(ws) == kvq.KVQ_ERR_TIMEOUT
    assert torch.all(out == -3.0)
    kvq.kvq_workspace_init(ws)
    got = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 5000, ws=ws).cpu().numpy()
    assert kvq.kvq_workspace_status(ws) == 0
    _, _, ref = oracle_pipeline(x["K"], x["V"], x["q"], 3, 3)
    assert rel_err(got, ref) <= TOL


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_keys_only_quantize_matches_oracle(dev, dtype):
    """A keys-only cache (bits_v = 0) holds each record's K words and K norms only, byte for
    byte as the oracle packs them; appends in pieces store the same bytes."""
    import torch
    T = 150
    x = wl.make_blockgtq_inputs(2, 8, 2, 128, T, dtype, 1e6, "lognormal_outliers", seed=66, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], 3)
    cache = kvq.cache_desc(2, 2, 160, 3, 0)
    packed = kvq.kvq_quantize(x["K"], None, alloc, cache)
    Kh = host_f32(x["K"])
    ra = bg.calibrate(Kh, 3)
    ref = bg.pack_cache_bytes(bg.quantize(Kh, None, ra, 0), ra, 0, 160)
    got = packed.cpu().numpy()
    nt = tiles_written(T)
    rec = bg.tile_record_bytes(128, 3, 0)
    hb = bg.header_bytes(2)
    n = 2 * 2 * tiles_written(160) * rec
    np.testing.assert_array_equal(got[:hb], ref[:hb])
    np.testing.assert_array_equal(got[hb:hb + n].reshape(2, 2, -1, rec)[:, :, :nt],
                                  ref[hb:hb + n].reshape(2, 2, -1, rec)[:, :, :nt])
    grown = torch.full_like(packed, 0x11)
    for a, b in [(0, 1), (1, 40), (40, 64), (64, 150)]:
        kvq.kvq_append(x["K"][:, :, a:b], None, alloc, cache, a, grown)
    g2 = grown.cpu().numpy()
    np.testing.assert_array_equal(g2[:hb], ref[:hb])
    np.testing.assert_array_equal(g2[hb:hb + n].reshape(2, 2, -1, rec)[:, :, :nt],
                                  ref[hb:hb + n].reshape(2, 2, -1, rec)[:, :, :nt])


@pytest.mark.parametrize("case", [("bf16", 2, 4000), ("f16", 3, 777), ("bf16", 4, 33)], ids=lambda c: f"{c[0]}K{c[1]}T{c[2]}")
def test_keys_only_decode_matches_oracle(dev, case):
    """Keys-only cache: packed keys, values read from the caller's unquantized
    tensor; attention within tolerance of the oracle's fp64 attention over k-hat and the exact
    values, at every prefix length checked."""
    dtype, bk, T = case
    x = wl.make_blockgtq_inputs(1, 8, 2, 128, T, dtype, 1e6, "lognormal_outliers", seed=80 + bk, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], bk)
    cache = kvq.cache_desc(1, 2, T + 7, bk, 0)
    packed = kvq.kvq_quantize(x["K"], None, alloc, cache)
    Kh, Vh, qh = host_f32(x["K"]), host_f32(x["V"]), host_f32(x["q"])
    ra = bg.calibrate(Kh, bk)
    rp = bg.pack_cache(bg.quantize(Kh, None, ra, 0), ra, 0, T + 7)
    for sl in sorted({1, T // 2, T}):
        out = kvq.kvq_decode_attn_ex(x["q"], packed, alloc, cache, sl, V=x["V"]).cpu().numpy()
        ref = bg.decode(qh, rp, ra, 0, sl, V=Vh)
        assert rel_err(out, ref) <= TOL, sl


@pytest.mark.parametrize("case", [(3000, 64, "bf16"), (300, 1000, "f32"), (0, 37, "bf16"), (5000, 1, "f16")],
                         ids=lambda c: f"T{c[0]}R{c[1]}{c[2]}")
def test_recent_tokens_join_the_softmax(dev, case):
    """Recent tokens kept unquantized (the buffer of fp16 recent keys the Block-GTQ page reports
    its results without): R tokens after the packed ones, in the caller's dtype, attended in
    the same softmax; within tolerance of the oracle's fp64 attention over the packed
    tokens' k-hat, v-hat and the recent tokens' exact keys and values. T = 0 attends over the
    recent tokens alone."""
    T, R, rdtype = case
    xs = wl.make_blockgtq_inputs(1, 16, 2, 128, T + R, "bf16", 1e6, "lognormal_outliers", seed=90 + R, device=dev)
    K, V, q = xs["K"], xs["V"], xs["q"]
    Tc = max(T, 1)
    Kc = K[:, :, :Tc].contiguous()
    alloc = kvq.kvq_calibrate(Kc, 3)
    cache = kvq.cache_desc(1, 2, Tc, 3, 3)
    packed = kvq.kvq_quantize(Kc, V[:, :, :Tc].contiguous(), alloc, cache)
    tdt = wl.torch_dtype(rdtype)
    Kr = K[:, :, T:T + R].to(tdt).contiguous()
    Vr = V[:, :, T:T + R].to(tdt).contiguous()
    out = kvq.kvq_decode_attn_ex(q, packed, alloc, cache, T, K_recent=Kr, V_recent=Vr).cpu().numpy()
    Kh = host_f32(Kc)
    ra = bg.calibrate(Kh, 3)
    rp = bg.pack_cache(bg.quantize(Kh, host_f32(V[:, :, :Tc]), ra, 3), ra, 3, Tc)
    ref = bg.decode(host_f32(q), rp, ra, 3, T, K_recent=host_f32(Kr), V_recent=host_f32(Vr))
    assert rel_err(out, ref) <= TOL


# ----------------------------------------------------------------------------- full-size workloads

def _sample_tiles(n_tiles, k=6, seed=0):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n_tiles, size=min(k, n_tiles), replace=False).tolist())
    pick |= {0, n_tiles - 1}
    return sorted(pick)


@pytest.mark.parametrize("name", ["llama8b", "qwen3b", "qwen3b_256k", "batched"])
def test_full_size_workloads(dev, name):
    """Full sizes, in the launch configuration the benchmark times: allocation bit-exact over
    the whole calibration set; packed records bit-exact on sampled tiles of every head;
    attention within tolerance on all heads (sampled sequences for the batched case)."""
    import torch
    W = wl.WORKLOADS[name]
    x = wl.make_blockgtq_inputs(W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim, W.seq_len, W.dtype, W.rope_base,
                                W.key_profile, seed=0, device=dev)
    K, V, q = x["K"], x["V"], x["q"]
    alloc = kvq.kvq_calibrate(K, W.bits_k, n_calib=W.n_calib)
    cache = kvq.cache_desc(W.batch, W.n_kv_heads, W.seq_len, W.bits_k, W.bits_v)
    packed = kvq.kvq_quantize(K, V, alloc, cache)
    out = kvq.kvq_decode_attn(q, packed, alloc, cache, W.seq_len).cpu().numpy()
    heads = kvq.parse_alloc(alloc.cpu().numpy())

    n_cal = W.n_calib if W.n_calib else W.seq_len
    Kcal = host_f32(K[:, :, :n_cal])
    ref_alloc = bg.calibrate(Kcal, W.bits_k, n_calib=0)
    compare_alloc(heads, ref_alloc)

    hdr, got = split_packed(packed.cpu().numpy(), W.batch, W.n_kv_heads, W.seq_len, W.bits_k, W.bits_v)
    np.testing.assert_array_equal(hdr, bg.packed_header(W.batch, W.n_kv_heads, W.seq_len, 128, W.bits_k, W.bits_v,
                                                        ref_alloc))
    for b in sorted({0, W.batch - 1, W.batch // 2}):
        # the oracle quantizes and packs the whole sequence itself, then decodes its own cache
        codes = bg.quantize(host_f32(K[b:b + 1]), host_f32(V[b:b + 1]), ref_alloc, W.bits_v)
        ref_packed = bg.pack_cache(codes, ref_alloc, W.bits_v, W.seq_len)
        np.testing.assert_array_equal(got[b:b + 1], ref_packed)
        ref = bg.decode(host_f32(q[b:b + 1]), ref_packed, ref_alloc, W.bits_v, W.seq_len)
        assert rel_err(out[b:b + 1], ref) <= TOL, b


# ----------------------------------------------------------------------------- NF4

NF4_CASES = [(1, 2, 1, "f16"), (2, 4, 15, "f16"), (1, 6, 16, "bf16"), (2, 2, 33, "f32"), (1, 56, 200, "f16")]


@pytest.mark.parametrize("case", NF4_CASES, ids=lambda c: f"B{c[0]}H{c[1]}T{c[2]}{c[3]}")
def test_nf4_small_cases_match_oracle(dev, case):
    B, H, T, dtype = case
    x = wl.make_nf4_inputs(B, H, 128, T, dtype, seed=T, device=dev)
    cap = T + 5
    packed = kvq.kvq_nf4_quantize(x["K"], x["V"], capacity=cap)
    out = kvq.kvq_nf4_decode_attn(x["q"], packed, cap, T).cpu().numpy()
    kc, vc, ks, vs = kvq.nf4_sections(packed.cpu().numpy(), B, H, cap)
    ki, ksc = nqkv.quantize(host_f32(x["K"]))
    vi, vsc = nqkv.quantize(host_f32(x["V"]))
    rkc, rks = nqkv.pack(ki, ksc, cap)
    rvc, rvs = nqkv.pack(vi, vsc, cap)
    np.testing.assert_array_equal(kc, rkc)
    np.testing.assert_array_equal(vc, rvc)
    np.testing.assert_array_equal(ks.view(np.uint16), rks.view(np.uint16))
    np.testing.assert_array_equal(vs.view(np.uint16), rvs.view(np.uint16))
    ref = nqkv.decode(host_f32(x["q"]), rkc, rks, rvc, rvs, H, 128, T)
    assert rel_err(out, ref) <= TOL


def test_nf4_edge_blocks(dev):
    """NF4 special blocks, byte for byte against the oracle: an all-zero block (scale 0, every
    index at the exact-zero level), values exactly on every midpoint of the table with the
    block's absmax 1 (u = x, each takes the lower index), and a block whose absmax exceeds
    the fp16 range (scale +inf, every u = 0)."""
    import torch
    B, H, T = 1, 4, 20
    mids = bg.codebooks.nf4_midpoints()
    X = np.random.default_rng(5).standard_normal((B, H, T, 128)).astype(np.float32)
    X[0, 0:2, 3] = 0.0                                  # block 0 of token 3: all zero
    X[0, 2:4, 4] = 0.0                                  # block 1 of token 4: midpoints, absmax 1
    X[0, 2, 4, :15] = mids
    X[0, 2, 4, 15] = 1.0
    X[0, 3, 4, :15] = -mids[::-1]
    X[0, 0, 5, 7] = 1.0e5                               # block 0 of token 5: absmax beyond fp16
    K = torch.from_numpy(X).to(dev)
    V = torch.from_numpy(X[:, ::-1].copy()).to(dev)
    packed = kvq.kvq_nf4_quantize(K, V, capacity=T)
    kc, vc, ks, vs = kvq.nf4_sections(packed.cpu().numpy(), B, H, T)
    for got_c, got_s, Xs in ((kc, ks, X), (vc, vs, X[:, ::-1].copy())):
        ri, rs = nqkv.quantize(Xs)
        rc, rsc = nqkv.pack(ri, rs, T)
        np.testing.assert_array_equal(got_c, rc)
        np.testing.assert_array_equal(got_s.view(np.uint16), rsc.view(np.uint16))
    ri, rs = nqkv.quantize(X)
    assert float(rs[0, 0, 3]) == 0.0 and np.all(ri[0, 0, 3] == 7)
    assert float(rs[0, 1, 4]) == 1.0 and list(ri[0, 1, 4, :15]) == list(range(15))
    assert np.isinf(float(rs[0, 0, 5])) and np.all(ri[0, 0, 5] == 7)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_nf4_append_in_pieces_equals_one_quantize(dev, dtype):
    """NF4 append ([NQKV] assumptions: append-only cache; Fig. 6 decoding phase): pieces of one
    token and ragged runs store the rows below the last padding boundary exactly as one
    quantize call, whatever the buffer held; decode over the grown cache matches the oracle."""
    import torch
    B, H, T, cap = 2, 4, 45, 64
    x = wl.make_nf4_inputs(B, H, 128, T, dtype, seed=9, device=dev)
    K, V, q = x["K"], x["V"], x["q"]
    one = kvq.kvq_nf4_quantize(K, V, capacity=cap)
    grown = torch.full_like(one, 0x3C)
    for a, b in zip([0, 1, 2, 15, 16, 17, 33, 44], [1, 2, 15, 16, 17, 33, 44, 45]):
        kvq.kvq_nf4_append(K[:, :, a:b], V[:, :, a:b], cap, a, grown)
    torch.cuda.synchronize()
    kc, vc, ks, vs = kvq.nf4_sections(grown.cpu().numpy(), B, H, cap)
    ok, ov, oks, ovs = kvq.nf4_sections(one.cpu().numpy(), B, H, cap)
    rows = -(-T // 16) * 16
    np.testing.assert_array_equal(kc[:, :, :rows], ok[:, :, :rows])
    np.testing.assert_array_equal(vc[:, :, :rows], ov[:, :, :rows])
    np.testing.assert_array_equal(ks[:, :, :rows].view(np.uint16), oks[:, :, :rows].view(np.uint16))
    np.testing.assert_array_equal(vs[:, :, :rows].view(np.uint16), ovs[:, :, :rows].view(np.uint16))
    out = kvq.kvq_nf4_decode_attn(q, grown, cap, T).cpu().numpy()
    ki, ksc = nqkv.quantize(host_f32(K))
    vi, vsc = nqkv.quantize(host_f32(V))
    rkc, rks = nqkv.pack(ki, ksc, cap)
    rvc, rvs = nqkv.pack(vi, vsc, cap)
    ref = nqkv.decode(host_f32(q), rkc, rks, rvc, rvs, H, 128, T)
    assert rel_err(out, ref) <= TOL


def test_nf4_full_size(dev):
    """OPT-30B shape at full size: whole (sequence, block) rows bit-exact on sampled blocks,
    attention of their heads against the oracle's own quantized cache."""
    W = wl.WORKLOADS["nqkv_opt30b"]
    x = wl.make_nf4_inputs(W.batch, W.n_q_heads, W.head_dim, W.seq_len, W.dtype, seed=0, device=dev)
    packed = kvq.kvq_nf4_quantize(x["K"], x["V"])
    out = kvq.kvq_nf4_decode_attn(x["q"], packed, W.seq_len, W.seq_len).cpu().numpy()
    kc, vc, ks, vs = kvq.nf4_sections(packed.cpu().numpy(), W.batch, W.n_q_heads, W.seq_len)
    for b in (0, W.batch - 1):
        for blk in (0, 9, W.n_q_heads // 2 - 1):
            hs = slice(2 * blk, 2 * blk + 2)
            ki, ksc = nqkv.quantize(host_f32(x["K"][b:b + 1, hs]))
            vi, vsc = nqkv.quantize(host_f32(x["V"][b:b + 1, hs]))
            rkc, rks = nqkv.pack(ki, ksc, W.seq_len)
            rvc, rvs = nqkv.pack(vi, vsc, W.seq_len)
            np.testing.assert_array_equal(kc[b, blk], rkc[0, 0])
            np.testing.assert_array_equal(vc[b, blk], rvc[0, 0])
            np.testing.assert_array_equal(ks[b, blk].view(np.uint16), rks[0, 0].view(np.uint16))
            np.testing.assert_array_equal(vs[b, blk].view(np.uint16), rvs[0, 0].view(np.uint16))
            ref = nqkv.decode(host_f32(x["q"][b:b + 1, hs]), rkc, rks, rvc, rvs, 2, 128, W.seq_len)
            assert rel_err(out[b:b + 1, hs], ref) <= TOL

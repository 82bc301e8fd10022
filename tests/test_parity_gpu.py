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
from tests.parity_util import TOL, compare_alloc, host_f32, oracle_pipeline, rel_err, tiles_written

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
    rec = bg.tile_record_bytes(128, bits_k, bits_v)
    return packed_np[:B * H * tiles_written(cap) * rec].reshape(B, H, tiles_written(cap), rec)


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
    got = packed_view(packed, B, Hkv, T, bk, bv)
    np.testing.assert_array_equal(got, ref_packed)
    assert rel_err(out, ref_out) <= TOL


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


# ----------------------------------------------------------------------------- full-size workloads

def _sample_tiles(n_tiles, k=6, seed=0):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n_tiles, size=min(k, n_tiles), replace=False).tolist())
    pick |= {0, n_tiles - 1}
    return sorted(pick)


@pytest.mark.parametrize("name", ["llama8b", "qwen3b", "batched"])
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

    rec = bg.tile_record_bytes(128, W.bits_k, W.bits_v)
    nt = tiles_written(W.seq_len)
    got = packed.cpu().numpy().reshape(W.batch, W.n_kv_heads, nt, rec)
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

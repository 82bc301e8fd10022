"""The C ABI without a GPU: library loads, every declared symbol is exported, host-side
tables agree bit-for-bit with the oracle, size queries follow the layout, and bad
arguments are rejected before anything is launched."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import blockgtq as bg
from oracle import codebooks as cb
from packed_cache_attention_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvq.h")


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(kvq.LIB_PATH):
        from packed_cache_attention_b200 import build
        build.build()
    return kvq.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*[\w][\w\s\*]*?\b(kvq_\w+)\s*\(", text, flags=re.M)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 18
    raw = ctypes.CDLL(kvq.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) <= set(kvq._SIGNATURES), set(names) - set(kvq._SIGNATURES)


def test_struct_sizes_match_header(L):
    assert ctypes.sizeof(kvq.HeadAlloc) == 2048
    assert kvq.HeadAlloc.digest.offset == 1608
    assert ctypes.sizeof(kvq.PackedHeader) == 64
    assert ctypes.sizeof(kvq.Tensor4) == 48
    assert kvq.kvq_alloc_bytes(3) == 3 * 2048
    assert kvq.kvq_abi_version() == 4
    for h in (1, 2, 8, 9, 56):
        assert kvq.kvq_packed_header_bytes(h) == bg.header_bytes(h)


@pytest.mark.parametrize("w", range(1, 9))
def test_library_codebooks_equal_oracle(L, w):
    c16, t32, delta = kvq.kvq_codebook(w)
    oc, ot = cb.stored_codebook(w)
    np.testing.assert_array_equal(c16.view(np.uint16), oc.view(np.uint16))
    np.testing.assert_array_equal(t32.view(np.uint32), ot.view(np.uint32))
    assert np.float32(delta) == cb.delta_table()[w]


def test_library_nf4_equal_oracle(L):
    lv, mid = kvq.kvq_nf4_table()
    np.testing.assert_array_equal(lv.view(np.uint32), cb.nf4_values().view(np.uint32))
    np.testing.assert_array_equal(mid.view(np.uint32), cb.nf4_midpoints().view(np.uint32))


def test_size_queries_follow_layout(L):
    for (B, H, cap, bk, bv) in [(1, 2, 131072, 3, 3), (1, 8, 32768, 2, 2), (16, 8, 16384, 4, 4), (2, 1, 77, 3, 2),
                                (1, 8, 32768, 2, 0), (3, 5, 100, 3, 0)]:
        c = kvq.cache_desc(B, H, cap, bk, bv)
        assert kvq.kvq_packed_bytes(c) == bg.packed_bytes(B, H, cap, 128, bk, bv)
        assert kvq.kvq_decode_workspace_bytes(c, 8 * H) > 0
    assert kvq.kvq_packed_bytes(kvq.cache_desc(1, 2, 131072, 3, 3)) == 26_214_400 + 128
    assert kvq.kvq_packed_bytes(kvq.cache_desc(1, 1, 10, 9, 3)) == 0
    assert kvq.kvq_packed_bytes(kvq.cache_desc(1, 1, 10, 3, 9)) == 0
    # NF4 at the OPT-30B shape: 130 bytes per 256 values, K and V
    assert kvq.kvq_nf4_packed_bytes(8, 56, 8192) == 2 * 8 * 28 * 8192 * 130
    assert kvq.kvq_nf4_packed_bytes(1, 3, 16) == 0            # odd head count
    # counters + energies + segment sums + chunk sums
    assert kvq.kvq_calibrate_workspace_bytes(16, 8, 2048) >= 8 * (16 * 2048 // 64) * 64 * 8 + 8 * 64 * 8


def test_status_strings(L):
    for s in range(11):
        assert kvq.kvq_status_string(s) and kvq.kvq_status_string(s) != "unknown status"
    assert kvq.kvq_status_string(0) == "ok"


_KEEP = []


def buf(nbytes=4 << 20):
    """Address of a real zeroed buffer of `nbytes` (on the GPU when there is one, else host
    memory), kept alive for the session. Every call below is rejected by host validation
    before any launch; the buffers are real and large enough for the shapes passed, so that
    even a launch that slipped through validation would stay inside them."""
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.zeros(int(nbytes), dtype=torch.uint8, device=dev)
    _KEEP.append(t)
    return t.data_ptr()


WS_BYTES = 4 << 20


def _t4(B=1, H=2, T=64, d=128, dtype=kvq.KVQ_BF16, sb=None, sh=None, st=128):
    sh = T * st if sh is None else sh
    sb = H * sh if sb is None else sb
    return kvq.Tensor4(B, H, T, d, sb, sh, st, dtype, 0)


def _calib(L, K, kd, p, alloc=None, ws=None, ws_bytes=WS_BYTES):
    alloc = buf(64 << 10) if alloc is None else alloc
    ws = buf(WS_BYTES) if ws is None else ws
    return L.kvq_calibrate(K, ctypes.byref(kd) if kd else None, ctypes.byref(p) if p else None, alloc, ws, ws_bytes,
                           None)


def test_calibrate_rejects_bad_arguments(L):
    p = kvq.CalibParams(3, 8, 0, 0)
    mem = buf()
    assert _calib(L, None, _t4(), p) == 1                                  # null K
    assert _calib(L, mem, _t4(d=64), p) == 2                              # head_dim != 128
    assert _calib(L, mem, _t4(dtype=7), p) == 3                           # unknown dtype
    assert _calib(L, mem + 2, _t4(), p) == 1                              # misaligned row start
    assert _calib(L, mem, _t4(st=129), p) == 1                            # stride not 16-byte multiple
    assert _calib(L, mem, _t4(), kvq.CalibParams(9, 8, 0, 0)) == 4        # budget above 8
    assert _calib(L, mem, _t4(), kvq.CalibParams(5, 4, 0, 0)) == 4        # budget above w_max
    assert _calib(L, mem, _t4(), kvq.CalibParams(0, 8, 0, 0)) == 4
    assert _calib(L, mem, _t4(), kvq.CalibParams(3, 8, 65, 0)) == 5       # n_calib > seq_len
    assert _calib(L, mem, _t4(), kvq.CalibParams(3, 8, 0, 2)) == 1        # unknown mode
    assert _calib(L, mem, _t4(), p, ws_bytes=64) == 6                     # workspace too small
    assert _calib(L, mem, _t4(), p, ws=0) == 6


def test_quantize_and_decode_reject_bad_arguments(L):
    mem = buf()
    kd = _t4(T=100)
    c = kvq.cache_desc(1, 2, 64, 3, 3)
    q = lambda kd_, c_: L.kvq_quantize(mem, ctypes.byref(kd_), mem, ctypes.byref(kd_), mem, ctypes.byref(c_),
                                       mem, None)
    assert q(kd, c) == 5                                                   # seq_len beyond capacity
    assert q(_t4(H=3), kvq.cache_desc(1, 2, 128, 3, 3)) == 2               # head count mismatch
    assert q(_t4(), kvq.cache_desc(1, 2, 128, 0, 3)) == 1                  # bad cache descriptor
    qd = kvq.Tensor4(1, 32, 1, 128, 32 * 128, 128, 128, kvq.KVQ_BF16, 0)
    dec = lambda qd_, c_, sl, wsb=WS_BYTES: L.kvq_decode_attn(mem, ctypes.byref(qd_), mem, mem, ctypes.byref(c_),
                                                              sl, mem, buf(WS_BYTES), wsb, None)
    assert dec(qd, kvq.cache_desc(1, 2, 128, 3, 3), 64) == 9               # 16 q-heads per KV head
    assert dec(qd, kvq.cache_desc(1, 8, 128, 3, 3), 129) == 5              # seq_len > capacity
    assert dec(qd, kvq.cache_desc(1, 8, 128, 3, 3), 0) == 5
    assert dec(qd, kvq.cache_desc(1, 8, 128, 3, 3), 64, wsb=16) == 6
    qd2 = kvq.Tensor4(1, 32, 2, 128, 64 * 128, 256, 128, kvq.KVQ_BF16, 0)
    assert dec(qd2, kvq.cache_desc(1, 8, 128, 3, 3), 64) == 2              # more than one query token
    assert L.kvq_nf4_quantize(mem, ctypes.byref(_t4(H=3)), mem, ctypes.byref(_t4(H=3)), 64, mem, None) == 2
    assert L.kvq_workspace_init(None, 0, None) == 6


def test_empty_inputs_are_refused(L):
    """Zero tokens, zero sequences or zero heads are refused on the host, before any launch."""
    mem = buf()
    p = kvq.CalibParams(3, 8, 0, 0)
    c = kvq.cache_desc(1, 2, 64, 3, 3)
    assert _calib(L, mem, _t4(T=0), p) == 2
    assert _calib(L, mem, _t4(B=0), p) == 2
    assert _calib(L, mem, _t4(H=0), p) == 2
    assert L.kvq_quantize(mem, ctypes.byref(_t4(T=0)), mem, ctypes.byref(_t4(T=0)), mem, ctypes.byref(c), mem,
                          None) == 2
    assert L.kvq_append(mem, ctypes.byref(_t4(T=0)), mem, ctypes.byref(_t4(T=0)), mem, ctypes.byref(c), 0, mem,
                        None) == 2
    assert L.kvq_nf4_quantize(mem, ctypes.byref(_t4(T=0)), mem, ctypes.byref(_t4(T=0)), 64, mem, None) == 2
    qd = kvq.Tensor4(1, 2, 1, 128, 2 * 128, 128, 128, kvq.KVQ_BF16, 0)
    assert L.kvq_nf4_decode_attn(mem, ctypes.byref(qd), mem, 64, 0, mem, buf(WS_BYTES), WS_BYTES, None) == 5
    assert kvq.kvq_packed_bytes(kvq.cache_desc(1, 2, 0, 3, 3)) == 0
    assert kvq.kvq_packed_bytes(kvq.cache_desc(0, 2, 64, 3, 3)) == 0
    assert kvq.kvq_nf4_packed_bytes(1, 2, 0) == 0


def test_nf4_append_rejects_ranges_outside_the_cache(L):
    mem = buf()
    app = lambda kd_, cap, t0: L.kvq_nf4_append(mem, ctypes.byref(kd_), mem, ctypes.byref(kd_), cap, t0, mem, None)
    assert app(_t4(T=1), 64, -1) == 5                                     # negative first token
    assert app(_t4(T=8), 64, 60) == 5                                     # range runs past capacity
    assert app(_t4(T=1, H=3), 64, 0) == 2                                 # odd head count


def test_append_rejects_ranges_outside_the_cache(L):
    """Append checks its token range against the capacity before anything is launched."""
    mem = buf()
    app = lambda kd_, c_, t0: L.kvq_append(mem, ctypes.byref(kd_), mem, ctypes.byref(kd_), mem, ctypes.byref(c_),
                                           t0, mem, None)
    c = kvq.cache_desc(1, 2, 64, 3, 3)
    assert app(_t4(T=1), c, -1) == 5                                      # negative first token
    assert app(_t4(T=1), c, 64) == 5                                      # first token at capacity
    assert app(_t4(T=10), c, 60) == 5                                     # range runs past capacity
    assert app(_t4(T=1, H=3), c, 0) == 2                                  # head count mismatch
    assert app(_t4(T=1), kvq.cache_desc(1, 2, 64, 0, 3), 0) == 1          # bad cache descriptor


def test_binding_raises_on_missing_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kvq, "_lib", None)
    monkeypatch.setattr(kvq, "LIB_PATH", str(tmp_path / "libkvq.so"))
    with pytest.raises(RuntimeError, match="missing"):
        kvq.lib()

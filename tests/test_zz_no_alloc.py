"""Allocation-free decode entry point (collected last on purpose).

kvq_decode_attn_noalloc serves callers that cannot allocate device memory (a plain-C host
with no CUDA allocator of its own, an engine plugin that may not allocate on its hot path):
it uses the library's fixed device scratch array as its workspace instead of one the caller
provides. It must give the same attention output as kvq_decode_attn (and as the oracle) on
the same packed cache, call after call, including when the number of splits changes between
calls and when its first call runs on a non-blocking stream; it must leave a clear status
word behind, and refuse shapes whose workspace would not fit in the array.
"""
import ctypes

import numpy as np
import pytest

from oracle import blockgtq as bg
from packed_cache_attention_b200 import kvq
from packed_cache_attention_b200 import workloads as wl
from tests.parity_util import TOL, host_f32, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _setup(dev, Hq, Hkv, T, seed):
    x = wl.make_blockgtq_inputs(1, Hq, Hkv, 128, T, "bf16", 1e6, "lognormal_outliers", seed=seed, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], 3)
    cache = kvq.cache_desc(1, Hkv, T, 3, 3)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    return x, alloc, cache, packed


def test_noalloc_decode_matches_workspace_decode_twice(dev):
    import torch
    x, alloc, cache, packed = _setup(dev, 16, 2, 5000, 5)
    ref = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 5000).cpu().numpy()
    # second call with a different query and length, so stale scratch contents would show
    q2 = torch.flip(x["q"], dims=[1]).contiguous()
    ref2 = kvq.kvq_decode_attn(q2, packed, alloc, cache, 4321).cpu().numpy()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()              # created non-blocking: not ordered after stream 0
    with torch.cuda.stream(side):
        out1 = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 5000, stream=side)
        out2 = kvq.kvq_decode_attn_noalloc(q2, packed, alloc, cache, 4321, stream=side)
    side.synchronize()
    out3 = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 5000).cpu().numpy()
    out1, out2 = out1.cpu().numpy(), out2.cpu().numpy()
    assert rel_err(out1, ref) <= TOL
    assert rel_err(out2, ref2) <= TOL
    assert rel_err(out3, ref) <= TOL
    assert kvq.kvq_decode_noalloc_status() == 0


def test_noalloc_split_count_changes_between_calls(dev):
    """300 and 5000 tokens over 2 and then 1 KV heads use different split and merge-group
    counts, which move the ticket layout inside the shared array; each output matches the
    oracle's fp64 attention over its own packed cache."""
    for Hq, Hkv, T in [(16, 2, 300), (16, 2, 5000), (8, 1, 300), (8, 1, 5000), (16, 2, 300)]:
        x, alloc, cache, packed = _setup(dev, Hq, Hkv, T, 40 + T + Hkv)
        out = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, T).cpu().numpy()
        K, V, q = host_f32(x["K"]), host_f32(x["V"]), host_f32(x["q"])
        ra = bg.calibrate(K, 3)
        rp = bg.pack_cache(bg.quantize(K, V, ra, 3), ra, 3, T)
        assert rel_err(out, bg.decode(q, rp, ra, 3, T)) <= TOL, (Hkv, T)
    assert kvq.kvq_decode_noalloc_status() == 0


def test_noalloc_status_reports_and_clears_a_timeout(dev):
    """A wait that gives up inside an allocation-free call is recorded in the scratch array's
    status word: kvq_decode_noalloc_status reports it once and clears it, and the next call
    decodes normally."""
    import torch
    x, alloc, cache, packed = _setup(dev, 16, 2, 3000, 71)
    out = torch.full((1, 16, 128), 5.0, device=dev)
    try:
        kvq.kvq_debug_decode(wait_limit=3, no_loads=True)
        kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 3000, out=out)
        torch.cuda.synchronize()
    finally:
        kvq.kvq_debug_decode(wait_limit=2000, no_loads=False)
    assert kvq.kvq_decode_noalloc_status() == kvq.KVQ_ERR_TIMEOUT
    assert kvq.kvq_decode_noalloc_status() == 0
    assert torch.all(out == 5.0)
    got = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 3000).cpu().numpy()
    assert kvq.kvq_decode_noalloc_status() == 0
    ref = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 3000).cpu().numpy()
    assert rel_err(got, ref) <= TOL


def test_noalloc_rejects_shapes_beyond_scratch(dev):
    """64 sequences x 8 KV heads need more than 2 MiB of split partials: refused before any
    launch. Every buffer passed is real and sized for the shape."""
    import torch
    L = kvq.lib()
    limit = kvq.kvq_decode_noalloc_scratch_bytes()
    assert limit == 2 << 20
    big = kvq.cache_desc(64, 8, 32, 3, 3)
    assert kvq.kvq_decode_workspace_bytes(big, 64) > limit
    q = torch.zeros((64, 64, 128), dtype=torch.bfloat16, device=dev)
    packed = torch.zeros(kvq.kvq_packed_bytes(big), dtype=torch.uint8, device=dev)
    alloc = torch.zeros(kvq.kvq_alloc_bytes(8), dtype=torch.uint8, device=dev)
    out = torch.zeros((64, 64, 128), dtype=torch.float32, device=dev)
    qd = kvq.tensor4(q)
    st = L.kvq_decode_attn_noalloc(q.data_ptr(), ctypes.byref(qd), packed.data_ptr(), alloc.data_ptr(),
                                   ctypes.byref(big), 32, out.data_ptr(), None)
    assert st == 6    # KVQ_ERR_WORKSPACE

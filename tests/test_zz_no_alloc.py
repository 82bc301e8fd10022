"""Allocation-free decode entry point (collected last on purpose).

kvq_decode_attn_noalloc serves callers that cannot allocate device memory: it uses the
library's fixed device scratch array as its workspace instead of one the caller provides.
It must give the same attention output as kvq_decode_attn on the same packed cache, call
after call, and refuse shapes whose workspace would not fit in the array.
"""
import ctypes

import numpy as np
import pytest

from packed_cache_attention_b200 import kvq
from packed_cache_attention_b200 import workloads as wl
from tests.parity_util import TOL, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def test_noalloc_decode_matches_workspace_decode_twice(dev):
    import torch
    x = wl.make_blockgtq_inputs(1, 16, 2, 128, 5000, "bf16", 1e6, "lognormal_outliers", seed=5, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], 3)
    cache = kvq.cache_desc(1, 2, 5000, 3, 3)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    ref = kvq.kvq_decode_attn(x["q"], packed, alloc, cache, 5000).cpu().numpy()
    # second call with a different query and length, so stale scratch contents would show
    q2 = torch.flip(x["q"], dims=[1]).contiguous()
    ref2 = kvq.kvq_decode_attn(q2, packed, alloc, cache, 4321).cpu().numpy()
    out1 = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 5000).cpu().numpy()
    out2 = kvq.kvq_decode_attn_noalloc(q2, packed, alloc, cache, 4321).cpu().numpy()
    out3 = kvq.kvq_decode_attn_noalloc(x["q"], packed, alloc, cache, 5000).cpu().numpy()
    assert rel_err(out1, ref) <= TOL
    assert rel_err(out2, ref2) <= TOL
    assert rel_err(out3, ref) <= TOL


def test_noalloc_rejects_shapes_beyond_scratch(dev):
    L = kvq.lib()
    limit = kvq.kvq_decode_noalloc_scratch_bytes()
    assert limit == 2 << 20
    big = kvq.cache_desc(64, 8, 131072, 3, 3)
    assert kvq.kvq_decode_workspace_bytes(big, 64) > limit
    qd = kvq.Tensor4(64, 64, 1, 128, 64 * 128, 128, 128, kvq.KVQ_BF16, 0)
    fake = 0x100000   # rejected on the host before any launch, never dereferenced
    st = L.kvq_decode_attn_noalloc(fake, ctypes.byref(qd), fake, fake, ctypes.byref(big), 1000, fake, None)
    assert st == 6    # KVQ_ERR_WORKSPACE

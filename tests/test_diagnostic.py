"""Key-side diagnostic of the allocation: Block-GTQ against uniform TQ-MSE at equal K budgets.

The page "RoPE-aware bit allocation for KV cache quantization" (abstract) reports that
allocating integer widths per RoPE block by marginal gain beats giving every coordinate the
same width at the same bits per dimension, measured on logits (mean absolute error) and on
attention distributions (KL divergence). Those measurements need trained models; here they
are restated on synthetic keys from the Llama-3.1-8B-shaped generator (log-normal block
scales, two outlier blocks x20, RoPE base 5e5) with random queries, through the oracle. The
pages' own numbers are not reproduced: only the direction of the comparison and its growth
with the budget are checked.

For a query independent of the keys, the expected squared logit error is the keys' total
squared quantization error, which is exactly what the greedy allocation minimises under the
N(0,1) distortion model, so the allocation must win on this diagnostic.
"""
import math

import numpy as np
import pytest

from oracle import blockgtq as bg
from packed_cache_attention_b200 import workloads as wl


def _inputs(seed=0, T=1024, n_q=4):
    x = wl.make_blockgtq_inputs(1, n_q, 1, 128, T, "f32", 5e5, "lognormal_outliers", seed=seed)
    K = x["K"].double().numpy()
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_q, 128))
    return K, q


def _diagnostic(K, q, bits, mode):
    alloc = bg.calibrate(K, bits, mode=mode)
    codes = bg.quantize(K, K, alloc, 2)
    Khat = bg.dequantize_keys(codes["Kc"], codes["Kn"], alloc)[0, 0]
    k = K[0, 0]
    exact = q @ k.T / math.sqrt(128.0)
    approx = q @ Khat.T / math.sqrt(128.0)
    mae = float(np.mean(np.abs(exact - approx)))

    def log_softmax(z):
        z = z - z.max(axis=1, keepdims=True)
        return z - np.log(np.exp(z).sum(axis=1, keepdims=True))

    lp, lq = log_softmax(exact), log_softmax(approx)
    kl = float(np.mean(np.sum(np.exp(lp) * (lp - lq), axis=1)))
    return mae, kl


@pytest.fixture(scope="module")
def results():
    K, q = _inputs()
    return {(b, m): _diagnostic(K, q, b, m) for b in (2, 3, 4) for m in (bg.MODE_BLOCKGTQ, bg.MODE_UNIFORM)}


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_block_gtq_beats_uniform_at_equal_budget(results, bits):
    mae_g, kl_g = results[(bits, bg.MODE_BLOCKGTQ)]
    mae_u, kl_u = results[(bits, bg.MODE_UNIFORM)]
    assert mae_g < mae_u, (bits, mae_g, mae_u)
    assert kl_g < kl_u, (bits, kl_g, kl_u)


def test_errors_shrink_with_the_budget(results):
    for mode in (bg.MODE_BLOCKGTQ, bg.MODE_UNIFORM):
        maes = [results[(b, mode)][0] for b in (2, 3, 4)]
        assert maes[0] > maes[1] > maes[2], (mode, maes)

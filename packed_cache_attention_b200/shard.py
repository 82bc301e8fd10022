"""Sharding of the packed-cache path over ranks (one process per GPU).

The path's units are (sequence, KV head) pairs: a KV head's allocation is calibrated over
its own keys only, and its packed cache, quantization and decode never read another head's
data. So ranks split the KV heads into contiguous ranges; each rank calibrates, quantizes and
decodes its heads for every sequence, and nothing crosses ranks until the outputs, which are
gathered in rank order (a fixed order, so the assembled output is the same bytes whatever the
number of ranks). A rank that owns no head contributes an empty slice.

The gather goes through torch.distributed (NCCL between GPUs, gloo on CPU); everything else
is the single-GPU library call on the rank's own slice.
"""
from __future__ import annotations

import torch


def kv_head_ranges(n_kv_heads: int, world: int) -> list[range]:
    """Contiguous KV-head ranges, one per rank, sizes differing by at most one."""
    if world < 1:
        raise ValueError("world must be >= 1")
    return [range(r * n_kv_heads // world, (r + 1) * n_kv_heads // world) for r in range(world)]


def query_heads(kv: range, group: int) -> range:
    """Query heads that read the KV heads of `kv` (head hq reads KV head hq // group)."""
    return range(kv.start * group, kv.stop * group)


def gather_outputs(local: torch.Tensor, kv: range, n_kv_heads: int, group: int, world: int) -> torch.Tensor:
    """Assemble out [B][Hq][d] from every rank's slice local [B][len(kv) * group][d].

    All ranks call it with their own slice; the result on every rank is the full output,
    rank r's query heads at their place. Uses all_gather on padded slices so ranks with
    fewer heads take part in the same collective.
    """
    import torch.distributed as dist

    ranges = kv_head_ranges(n_kv_heads, world)
    width = max(len(r) for r in ranges) * group
    B, _, d = local.shape
    pad = torch.zeros((B, width, d), dtype=local.dtype, device=local.device)
    pad[:, :local.shape[1]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad)
    out = torch.empty((B, n_kv_heads * group, d), dtype=local.dtype, device=local.device)
    for r, kvr in enumerate(ranges):
        qh = query_heads(kvr, group)
        out[:, qh.start:qh.stop] = parts[r][:, :len(qh)]
    return out


def decode_step_sharded(K, V, q, bits_k: int, bits_v: int, world: int, rank: int, n_calib: int = 0, kvq=None):
    """One calibrate -> quantize -> decode pass of this rank's KV heads through libkvq, then
    the gathered output. K, V: [B][Hkv][T][128] and q: [B][Hq][128] (the full tensors or
    views of them; only this rank's heads are read)."""
    if kvq is None:
        from . import kvq as kvq_mod
        kvq = kvq_mod
    B, Hkv, T, d = K.shape
    G = q.shape[1] // Hkv
    kv = kv_head_ranges(Hkv, world)[rank]
    if len(kv) == 0:
        local = torch.zeros((B, 0, d), dtype=torch.float32, device=q.device)
    else:
        Kl, Vl = K[:, kv.start:kv.stop], V[:, kv.start:kv.stop]
        qh = query_heads(kv, G)
        ql = q[:, qh.start:qh.stop].contiguous()
        alloc = kvq.kvq_calibrate(Kl, bits_k, n_calib=n_calib)
        cache = kvq.cache_desc(B, len(kv), T, bits_k, bits_v)
        packed = kvq.kvq_quantize(Kl, Vl, alloc, cache)
        local = kvq.kvq_decode_attn(ql, packed, alloc, cache, T)
    return gather_outputs(local, kv, Hkv, G, world)

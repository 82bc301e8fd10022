"""Seeded synthetic inputs for the packed-cache path.

This module only draws random tensors with the shapes and value distributions
of the workloads the pages measure on; it holds none of the method's
arithmetic (no energy, allocation, quantizer, packing or attention). Both the
CUDA path and the CPU oracle consume exactly the tensors built here.

RoPE is applied here because the cache stores post-RoPE keys: the decode
query and the cached keys come out of the model already rotated (page
"RoPE-aware bit allocation for KV cache quantization", abstract: under RoPE a
key's share of a later logit splits over 2-D frequency blocks). The pairing is
rotate-half: block i = dims (i, i + d/2), angle p * base^(-2i/d).

Workloads (all seeded; synthetic stand-ins for the pages' models):
  tiny        1 KV head, 1 q head, d 128, T 512, fp32. sigma_b = 10^U(-1,1)
              per RoPE block, RoPE base 1e4.                       K3V3
  llama8b     B1, Hq 32, Hkv 8, d 128, T 32768, bf16. sigma_{h,b} =
              exp(N(0,1)) plus 2 outlier blocks x20, RoPE base 5e5. K2V2
  qwen3b      B1, Hq 16, Hkv 2, d 128, T 131072, bf16, base 1e6.    K3V3
  batched     B16, Hq 32, Hkv 8, d 128, T 16384, bf16, base 5e5,
              calibration on the first 2048 tokens of each sequence. K4V4
  nqkv_opt30b B8, H 56 (MHA), d 128, T 8192, fp16, no RoPE, entries
              N(0, s^2) with s log-uniform in [0.2, 5] per 256-value block.
"""
from __future__ import annotations

import dataclasses
import math

import torch

__all__ = ["Workload", "WORKLOADS", "make_blockgtq_inputs", "make_nf4_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "blockgtq" or "nf4"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int
    dtype: str           # "f32", "f16", "bf16"
    rope_base: float     # 0 = no RoPE
    key_profile: str     # "loguniform", "lognormal_outliers", "nf4_blocks"
    bits_k: int = 0
    bits_v: int = 0
    n_calib: int = 0     # calibration tokens per sequence (0 = all)


WORKLOADS = {
    "tiny": Workload("tiny", "blockgtq", 1, 1, 1, 128, 512, "f32", 1e4, "loguniform", 3, 3, 0),
    "llama8b": Workload("llama8b", "blockgtq", 1, 32, 8, 128, 32768, "bf16", 5e5,
                        "lognormal_outliers", 2, 2, 0),
    "qwen3b": Workload("qwen3b", "blockgtq", 1, 16, 2, 128, 131072, "bf16", 1e6,
                       "lognormal_outliers", 3, 3, 0),
    "qwen3b_256k": Workload("qwen3b_256k", "blockgtq", 1, 16, 2, 128, 262144, "bf16", 1e6,
                            "lognormal_outliers", 3, 3, 0),
    "batched": Workload("batched", "blockgtq", 16, 32, 8, 128, 16384, "bf16", 5e5,
                        "lognormal_outliers", 4, 4, 2048),
    "nqkv_opt30b": Workload("nqkv_opt30b", "nf4", 8, 56, 56, 128, 8192, "f16", 0.0, "nf4_blocks"),
}

_TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TORCH_DTYPE[name]


def _rope_rotate_(x: torch.Tensor, positions: torch.Tensor, base: float) -> torch.Tensor:
    """Rotate-half RoPE on the last dim of a float64 tensor, in place on a copy.

    x: [..., T, d] float64, positions: [T] float64.
    """
    d = x.shape[-1]
    h = d // 2
    i = torch.arange(h, dtype=torch.float64, device=x.device)
    theta = torch.pow(torch.tensor(base, dtype=torch.float64, device=x.device), -2.0 * i / d)
    ang = positions[:, None].to(torch.float64) * theta[None, :]          # [T, h]
    c, s = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    r1 = x1 * c - x2 * s
    r2 = x2 * c + x1 * s
    return torch.cat([r1, r2], dim=-1)


def _key_sigmas(profile: str, n_kv_heads: int, h: int, gen: torch.Generator) -> torch.Tensor:
    """Per (KV head, RoPE block) standard deviations, float64 [Hkv, h]."""
    if profile == "loguniform":
        u = torch.rand((n_kv_heads, h), generator=gen, dtype=torch.float64)
        return torch.pow(torch.tensor(10.0, dtype=torch.float64), 2.0 * u - 1.0)
    if profile == "lognormal_outliers":
        sig = torch.exp(torch.randn((n_kv_heads, h), generator=gen, dtype=torch.float64))
        outl = torch.randperm(h, generator=gen)[:2]            # same two blocks for every head
        sig[:, outl] *= 20.0
        return sig
    raise ValueError(profile)


def make_blockgtq_inputs(batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int, seq_len: int,
                         dtype: str = "bf16", rope_base: float = 1e6,
                         key_profile: str = "lognormal_outliers", seed: int = 0,
                         device: str | torch.device = "cpu", with_q: bool = True):
    """Keys, values and one decode query per q-head, all contiguous.

    Returns dict with K, V: [B][Hkv][T][d] in `dtype`, q: [B][Hq][d] in `dtype`
    (fp32 for dtype f32), sigma: [Hkv][d/2] float64 (the generator's block scales).
    Small parameters come from a CPU generator seeded with `seed`; the bulk
    normals come from a generator on `device` seeded with `seed + 1` (so the
    same seed gives different bulk values on CPU and CUDA; each test uses one).
    """
    assert head_dim % 2 == 0
    h = head_dim // 2
    cpu_gen = torch.Generator(device="cpu").manual_seed(seed)
    sigma = _key_sigmas(key_profile, n_kv_heads, h, cpu_gen)
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    tdt = _TORCH_DTYPE[dtype]
    K = torch.empty((batch, n_kv_heads, seq_len, head_dim), dtype=tdt, device=dev)
    V = torch.empty_like(K)
    sig_full = torch.cat([sigma, sigma], dim=1).to(dev)                # dims i and i+h share block i
    pos = torch.arange(seq_len, dtype=torch.float64, device=dev)
    chunk = max(1, (1 << 24) // max(1, head_dim))                      # tokens per generation chunk
    for b in range(batch):
        for hh in range(n_kv_heads):
            for t0 in range(0, seq_len, chunk):
                t1 = min(seq_len, t0 + chunk)
                z = torch.randn((t1 - t0, head_dim), generator=gen, dtype=torch.float64, device=dev)
                k = z * sig_full[hh][None, :]
                if rope_base > 0:
                    k = _rope_rotate_(k, pos[t0:t1], rope_base)
                K[b, hh, t0:t1] = k.to(tdt)
                v = torch.randn((t1 - t0, head_dim), generator=gen, dtype=torch.float64, device=dev)
                V[b, hh, t0:t1] = v.to(tdt)
    out = {"K": K, "V": V, "sigma": sigma}
    if with_q:
        q = torch.randn((batch, n_q_heads, 1, head_dim), generator=gen, dtype=torch.float64, device=dev)
        if rope_base > 0:
            q = _rope_rotate_(q, torch.tensor([float(seq_len)], dtype=torch.float64, device=dev), rope_base)
        out["q"] = q[:, :, 0, :].to(tdt).contiguous()
    return out


def make_nf4_inputs(batch: int, n_heads: int, head_dim: int, seq_len: int, dtype: str = "f16",
                    block: int = 256, s_lo: float = 0.2, s_hi: float = 5.0, seed: int = 0,
                    device: str | torch.device = "cpu", with_q: bool = True):
    """NQKV-style K, V with one scale per 256-value block of each token's hidden vector.

    Entries are N(0, s^2), s = 10^U(log10 s_lo, log10 s_hi) drawn per (token, block),
    independently for K and V. Layout [B][H][T][d]; q [B][H][d] ~ N(0, 1).
    """
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed + 1)
    tdt = _TORCH_DTYPE[dtype]
    hidden = n_heads * head_dim
    assert hidden % block == 0 and block % head_dim == 0
    nblk = hidden // block
    lo, hi = math.log10(s_lo), math.log10(s_hi)
    K = torch.empty((batch, n_heads, seq_len, head_dim), dtype=tdt, device=dev)
    V = torch.empty_like(K)
    chunk = max(1, (1 << 24) // hidden)
    for dst in (K, V):
        for b in range(batch):
            for t0 in range(0, seq_len, chunk):
                t1 = min(seq_len, t0 + chunk)
                n = t1 - t0
                u = torch.rand((n, nblk, 1), generator=gen, dtype=torch.float32, device=dev)
                s = torch.pow(10.0, lo + (hi - lo) * u)
                z = torch.randn((n, nblk, block), generator=gen, dtype=torch.float32, device=dev) * s
                z = z.reshape(n, n_heads, head_dim).permute(1, 0, 2)          # [H][n][d]
                dst[b, :, t0:t1] = z.to(tdt)
    out = {"K": K, "V": V}
    if with_q:
        out["q"] = torch.randn((batch, n_heads, head_dim), generator=gen, dtype=torch.float32,
                               device=dev).to(tdt)
    return out

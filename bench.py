"""Benchmark of the packed-cache hot path (libkvq) on B200.

One step = one pass of the whole path over a stack of L = 36 layers shaped like the
Qwen2.5-3B 128K decode workload (16 q-heads, 2 KV heads, head_dim 128, batch 1,
131072 tokens, bf16, K3V3): for every layer calibrate (energy reduction + greedy
allocation) and quantize/pack its K and V (the prefill write of the cache), then one
decode step of attention through all layers reading the packed caches. Qwen2.5-3B has
36 layers; with 36 x 160 MB touched per step, every layer's inputs and cache have left
L2 by the time they are read again.

Prints one JSON line (rank 0). `--impl reference` times the CPU oracle instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed-KV decode attn: KV-tokens/s & % HBM peak; quantize/pack tokens/s"
UNIT = "layer-tokens/s"
LAYERS = 36
WORKLOAD = "qwen3b"


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (ms) over all ranks of the default process
    group (the slowest rank sets the job's time); the values unchanged on a single rank."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world, layers, batch, seq_len, ms_per_step):
    """Whole-job layer-tokens/s: every rank processes its own replica of the workload (the
    (sequence, KV head) units are independent), so the units of all ranks count, over the
    slowest rank's time."""
    return world * layers * batch * seq_len / (ms_per_step * 1e-3)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="libkvq", choices=["libkvq", "reference"])
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=0, help="override the context length (profiling only)")
    ap.add_argument("--no-nf4", action="store_true", help="skip the NF4-variant measurement")
    ap.add_argument("--nf4-batch", type=int, default=0, help="override the NF4 batch (profiling only)")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload decode/quantize lines")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash(name: str) -> str:
    with open(os.path.join(ROOT, "packed_cache_attention_b200", "csrc", name), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def recorded_traffic(kernel: str, src: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash(src)
    with open(path) as fh:
        for line in fh:
            f = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
            if f.get("kernel") == kernel and f.get("src_sha") == want and f.get("workload") == WORKLOAD:
                return int(f["bytes_per_launch"])
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 20 ms during the timed region (about
    0.1 s at the default 20 steps)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------ GPU arm

def run_gpu(args, rank, world, local_rank):
    import torch
    from packed_cache_attention_b200 import kvq
    from packed_cache_attention_b200 import workloads as wl

    dist = world > 1
    if dist:
        import torch.distributed as tdist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    W = wl.WORKLOADS[WORKLOAD]
    T = args.seq_len or W.seq_len
    B, Hq, Hkv, d = W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim
    bk, bv = W.bits_k, W.bits_v
    L = args.layers
    kvq.lib()
    kvq._check("kvq_init", kvq.lib().kvq_init())

    # Inputs for all layers, resident in HBM; one seed per (rank, layer).
    Ks, Vs, qs = [], [], []
    for layer in range(L):
        x = wl.make_blockgtq_inputs(B, Hq, Hkv, d, T, W.dtype, W.rope_base, W.key_profile,
                                    seed=1000 * rank + layer, device=dev)
        Ks.append(x["K"]); Vs.append(x["V"]); qs.append(x["q"])
    cache = kvq.cache_desc(B, Hkv, T, bk, bv)
    allocs = [torch.empty(kvq.kvq_alloc_bytes(Hkv), dtype=torch.uint8, device=dev) for _ in range(L)]
    packs = [torch.empty(kvq.kvq_packed_bytes(cache), dtype=torch.uint8, device=dev) for _ in range(L)]
    outs = [torch.empty((B, Hq, d), dtype=torch.float32, device=dev) for _ in range(L)]
    cws = torch.zeros(kvq.kvq_calibrate_workspace_bytes(B, Hkv, T), dtype=torch.uint8, device=dev)
    dws = [torch.zeros(kvq.kvq_decode_workspace_bytes(cache, Hq), dtype=torch.uint8, device=dev) for _ in range(L)]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev: ev[0].record(stream)
        for layer in range(L):
            kvq.kvq_calibrate(Ks[layer], bk, n_calib=W.n_calib, alloc=allocs[layer], ws=cws, stream=stream)
        if ev: ev[1].record(stream)
        for layer in range(L):
            kvq.kvq_quantize(Ks[layer], Vs[layer], allocs[layer], cache, packed=packs[layer], stream=stream)
        if ev: ev[2].record(stream)
        for layer in range(L):
            kvq.kvq_decode_attn(qs[layer], packs[layer], allocs[layer], cache, T, out=outs[layer], ws=dws[layer],
                                stream=stream)
        if ev: ev[3].record(stream)

    def barrier():
        if dist:
            tdist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(3, args.warmup)):
        step()
    barrier()
    for w in dws:
        assert kvq.kvq_workspace_status(w) == 0

    sampler = ClockSampler(local_rank)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    cal_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    qnt_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in evs)
    total_ms, cal_ms, qnt_ms, dec_ms = max_over_ranks([total_ms, cal_ms, qnt_ms, dec_ms], dev)

    # ---------------------------------------------------------------- end to end through the C ABI
    e2e = None
    if args.e2e_steps > 0:
        hK = [k.cpu().pin_memory() for k in Ks]
        hV = [v.cpu().pin_memory() for v in Vs]
        hq = [q.cpu().pin_memory() for q in qs]
        hout = [torch.empty((B, Hq, d), dtype=torch.float32).pin_memory() for _ in range(L)]
        h2d = sum(x.numel() * x.element_size() for x in hK + hV + hq)
        d2h = sum(x.numel() * x.element_size() for x in hout)

        def e2e_step():
            for layer in range(L):
                Ks[layer].copy_(hK[layer], non_blocking=True)
                Vs[layer].copy_(hV[layer], non_blocking=True)
                qs[layer].copy_(hq[layer], non_blocking=True)
            step()
            for layer in range(L):
                hout[layer].copy_(outs[layer], non_blocking=True)

        e2e_step()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        z.record(stream)
        barrier()
        e2e_ms = a.elapsed_time(z) / args.e2e_steps
        e2e_ms = max_over_ranks([e2e_ms], dev)[0]
        e2e = {"value": job_throughput(world, L, B, T, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    nf4 = (measure_nf4(kvq, wl, dev, stream, hbm_peak=peaks()[0], batch=args.nf4_batch)
           if (rank == 0 and not args.no_nf4) else None)
    append = measure_append(kvq, Ks[0], Vs[0], allocs[0], cache, packs[0], stream, T) if rank == 0 else None
    configs = None
    if rank == 0 and not args.no_configs:
        del Ks, Vs
        torch.cuda.empty_cache()
        configs = measure_configs(kvq, wl, dev, stream, hbm_peak=peaks()[0])

    steps = args.steps
    ms_step = total_ms / steps
    tokens = world * L * B * T
    hbm, peak_kind = peaks()
    q_bytes = B * Hkv * T * d * 2 * 2 + kvq.kvq_packed_bytes(cache)
    d_bytes = kvq.kvq_packed_bytes(cache)
    c_bytes = B * Hkv * T * d * 2
    q_launch_ms = qnt_ms / (steps * L)
    d_launch_ms = dec_ms / (steps * L)
    c_launch_ms = cal_ms / (steps * L)
    q_gbs = q_bytes / (q_launch_ms * 1e-3) / 1e9
    d_gbs = d_bytes / (d_launch_ms * 1e-3) / 1e9
    c_gbs = c_bytes / (c_launch_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": job_throughput(world, L, B, T, ms_step),
        "unit": UNIT,
        "n_gpus": world,
        "steps": steps,
        "warmup": max(3, args.warmup),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 in; f64 norms/energies, f32 scaling, u32 bit planes; f16 mma + f32 accumulate",
        "data": "synthetic (seeded Qwen2.5-3B-shaped K/V/q, lognormal block scales + 2 outlier blocks, RoPE 1e6)",
        "config": {"workload": f"{WORKLOAD}: {L} layers x (Hq {Hq}, Hkv {Hkv}, d {d}, B {B}, T {T}, bf16), K{bk}V{bv}",
                   "layers": L, "global_batch": B * world, "seq_len": T, "parallelism": f"replicas{world}",
                   "l2": "inputs larger than L2: each step touches 36 x 160 MB; no explicit flush"},
        "roofline": {"bound": "hbm", "achieved": q_gbs, "peak": hbm, "unit": "GB/s", "frac": q_gbs / hbm,
                     "traffic": recorded_traffic("kvq_quant_pack", "quantize.cuh"),
                     "kernel": "kvq_quant_pack", "bytes_per_launch": q_bytes, "launch_ms": q_launch_ms,
                     "peak_kind": peak_kind},
        "breakdown": {
            "decode": {"kv_tokens_per_s": tokens / (dec_ms / steps * 1e-3), "launch_ms": d_launch_ms,
                       "bytes_per_launch": d_bytes, "gb_s": d_gbs, "hbm_frac": d_gbs / hbm,
                       "traffic": recorded_traffic("kvq_decode_gtq", "decode.cuh")},
            "quantize": {"tokens_per_s": tokens / (qnt_ms / steps * 1e-3), "launch_ms": q_launch_ms,
                         "bytes_per_launch": q_bytes, "gb_s": q_gbs, "hbm_frac": q_gbs / hbm},
            "calibrate": {"tokens_per_s": tokens / (cal_ms / steps * 1e-3), "launch_ms": c_launch_ms,
                          "bytes_per_launch": c_bytes, "gb_s": c_gbs, "hbm_frac": c_gbs / hbm},
            "bytes_per_token_per_kv_head": d_bytes // (B * Hkv * T),
            "compression_vs_bf16": (2 * 2 * d) / (d_bytes / (B * Hkv * T)),
        },
        "nf4": nf4,
        "append": append,
        "workloads": configs,
        "e2e": e2e,
        "gpu_launches": steps * L * 4,
        "clocks": clocks,
    }
    return result


def measure_append(kvq, K, V, alloc, cache, packed, stream, T, iters=50, chunk=4096):
    """Decode-step growth of the packed cache: one token appended at position T - 1 (a partly
    filled tile, so the value words are merged), and a 4096-token chunk (chunked prefill).
    The same tokens are re-appended, so the cache content is unchanged."""
    import torch

    def timed(fn, n):
        fn()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        z.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(z) / n

    def graphed(fn, n):
        """Device time per call: n calls captured in one CUDA graph (no host gaps)."""
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn(side)
            side.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                for _ in range(n):
                    fn(side)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        z.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(z) / n

    k1, v1 = K[:, :, T - 1:T], V[:, :, T - 1:T]
    kc, vc = K[:, :, T - chunk:T], V[:, :, T - chunk:T]
    one = lambda st: kvq.kvq_append(k1, v1, alloc, cache, T - 1, packed, stream=st)
    big = lambda st: kvq.kvq_append(kc, vc, alloc, cache, T - chunk, packed, stream=st)
    try:
        one_ms, chunk_ms, how = graphed(one, iters), graphed(big, iters), "cuda graph of 50 calls"
    except Exception as e:  # noqa: BLE001 - capture unavailable: host-issued calls instead
        one_ms, chunk_ms = timed(lambda: one(stream), iters), timed(lambda: big(stream), iters)
        how = f"host-issued calls ({type(e).__name__})"
    B, H = K.shape[0], K.shape[1]
    per_tok = 2 * 2 * K.shape[3] + kvq.kvq_packed_bytes(cache) // (B * H * T)
    return {"one_token_launch_ms": one_ms, "chunk_tokens": chunk, "chunk_launch_ms": chunk_ms,
            "chunk_tokens_per_s": B * H * chunk / (chunk_ms * 1e-3),
            "chunk_gb_s": B * H * chunk * per_tok / (chunk_ms * 1e-3) / 1e9, "timing": how}


def timed_launches(fn, stream, iters, flush):
    """Mean device time (ms) of fn() over `iters` launches, each preceded by a write of a
    buffer larger than L2 (outside the timed interval) so every launch starts cold."""
    import torch
    for _ in range(3):
        fn()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    for a, z in evs:
        flush.add_(1)
        a.record(stream)
        fn()
        z.record(stream)
    torch.cuda.synchronize()
    return sum(a.elapsed_time(z) for a, z in evs) / iters


def measure_configs(kvq, wl, dev, stream, hbm_peak, iters=10):
    """Decode and quantize/pack of the other Block-GTQ workloads, one layer each, every launch
    after an L2 flush: Llama-3.1-8B-shaped 32K (K2V2), batched 16 x 16K (K4V4), the 128K
    Qwen2.5-3B shape at 262144 tokens (K3V3), a keys-only K2 cache at the Llama shape (bf16
    values), and the Qwen 128K layer with 128 recent tokens kept unquantized."""
    import torch
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)     # 256 MB > L2
    res = {}
    for name in ("llama8b", "batched", "qwen3b_256k"):
        W = wl.WORKLOADS[name]
        x = wl.make_blockgtq_inputs(W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim, W.seq_len, W.dtype,
                                    W.rope_base, W.key_profile, seed=5, device=dev)
        alloc = kvq.kvq_calibrate(x["K"], W.bits_k, n_calib=W.n_calib)
        cache = kvq.cache_desc(W.batch, W.n_kv_heads, W.seq_len, W.bits_k, W.bits_v)
        packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
        out = torch.empty((W.batch, W.n_q_heads, W.head_dim), dtype=torch.float32, device=dev)
        ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, W.n_q_heads), dtype=torch.uint8, device=dev)
        d_ms = timed_launches(lambda: kvq.kvq_decode_attn(x["q"], packed, alloc, cache, W.seq_len, out=out, ws=ws,
                                                          stream=stream), stream, iters, flush)
        q_ms = timed_launches(lambda: kvq.kvq_quantize(x["K"], x["V"], alloc, cache, packed=packed, stream=stream),
                              stream, iters, flush)
        assert kvq.kvq_workspace_status(ws) == 0
        tok = W.batch * W.seq_len
        rec = (kvq.kvq_packed_bytes(cache) - kvq.kvq_packed_header_bytes(W.n_kv_heads))
        qb = W.batch * W.n_kv_heads * W.seq_len * W.head_dim * 2 * 2 + rec
        res[name] = {"workload": f"{name}: B{W.batch} Hq{W.n_q_heads} Hkv{W.n_kv_heads} T{W.seq_len} K{W.bits_k}V{W.bits_v}",
                     "decode": {"launch_ms": d_ms, "bytes_per_launch": rec, "gb_s": rec / (d_ms * 1e-3) / 1e9,
                                "kv_tokens_per_s": tok / (d_ms * 1e-3)},
                     "quantize": {"launch_ms": q_ms, "bytes_per_launch": qb, "gb_s": qb / (q_ms * 1e-3) / 1e9,
                                  "tokens_per_s": tok / (q_ms * 1e-3)}}
        for k in ("decode", "quantize"):
            res[name][k]["hbm_frac"] = res[name][k]["gb_s"] / hbm_peak
        if name == "llama8b":
            # keys only: K2 codes packed, values read as bf16
            ck = kvq.cache_desc(W.batch, W.n_kv_heads, W.seq_len, W.bits_k, 0)
            pk = kvq.kvq_quantize(x["K"], None, alloc, ck)
            wk = torch.zeros(kvq.kvq_decode_workspace_bytes(ck, W.n_q_heads), dtype=torch.uint8, device=dev)
            k_ms = timed_launches(lambda: kvq.kvq_decode_attn_ex(x["q"], pk, alloc, ck, W.seq_len, V=x["V"], out=out,
                                                                 ws=wk, stream=stream), stream, iters, flush)
            assert kvq.kvq_workspace_status(wk) == 0
            kb = (kvq.kvq_packed_bytes(ck) - kvq.kvq_packed_header_bytes(W.n_kv_heads)) + x["V"].numel() * 2
            res["keys_only_llama8b"] = {"workload": f"llama8b keys only: K{W.bits_k}, bf16 values",
                                        "decode": {"launch_ms": k_ms, "bytes_per_launch": kb,
                                                   "gb_s": kb / (k_ms * 1e-3) / 1e9,
                                                   "hbm_frac": kb / (k_ms * 1e-3) / 1e9 / hbm_peak}}
        del x, packed, out, ws, alloc
        torch.cuda.empty_cache()
    # recent tokens kept unquantized: the 128K layer plus 128 bf16 tokens
    W = wl.WORKLOADS["qwen3b"]
    R = 128
    x = wl.make_blockgtq_inputs(W.batch, W.n_q_heads, W.n_kv_heads, W.head_dim, W.seq_len, W.dtype, W.rope_base,
                                W.key_profile, seed=6, device=dev)
    alloc = kvq.kvq_calibrate(x["K"], W.bits_k)
    cache = kvq.cache_desc(W.batch, W.n_kv_heads, W.seq_len, W.bits_k, W.bits_v)
    packed = kvq.kvq_quantize(x["K"], x["V"], alloc, cache)
    Kr = x["K"][:, :, -R:].contiguous()
    Vr = x["V"][:, :, -R:].contiguous()
    out = torch.empty((W.batch, W.n_q_heads, W.head_dim), dtype=torch.float32, device=dev)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cache, W.n_q_heads), dtype=torch.uint8, device=dev)
    r_ms = timed_launches(lambda: kvq.kvq_decode_attn_ex(x["q"], packed, alloc, cache, W.seq_len, K_recent=Kr,
                                                         V_recent=Vr, out=out, ws=ws, stream=stream),
                          stream, iters, flush)
    assert kvq.kvq_workspace_status(ws) == 0
    rb = (kvq.kvq_packed_bytes(cache) - kvq.kvq_packed_header_bytes(W.n_kv_heads)) + 2 * Kr.numel() * 2
    res["recent_qwen3b"] = {"workload": f"qwen3b 128K + {R} recent bf16 tokens",
                            "decode": {"launch_ms": r_ms, "bytes_per_launch": rb, "gb_s": rb / (r_ms * 1e-3) / 1e9,
                                       "hbm_frac": rb / (r_ms * 1e-3) / 1e9 / hbm_peak}}
    del x, packed, out, ws, flush
    torch.cuda.empty_cache()
    return res


def measure_nf4(kvq, wl, dev, stream, hbm_peak, iters=10, batch=0):
    """NQKV-style NF4 variant at the OPT-30B shape (one layer: B8 x 56 heads x 8192 tokens,
    fp16), timed outside the step: quantize/pack and MHA decode, CUDA events per launch."""
    import torch
    W = wl.WORKLOADS["nqkv_opt30b"]
    B, H, T, d = (batch or W.batch), W.n_q_heads, W.seq_len, W.head_dim
    x = wl.make_nf4_inputs(B, H, d, T, W.dtype, seed=7, device=dev)
    packed = torch.empty(kvq.kvq_nf4_packed_bytes(B, H, T, d), dtype=torch.uint8, device=dev)
    out = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    ws = torch.zeros(kvq.kvq_nf4_decode_workspace_bytes(B, H, T, d), dtype=torch.uint8, device=dev)

    def timed(fn):
        for _ in range(3):
            fn()
        a = torch.cuda.Event(enable_timing=True)
        z = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(iters):
            fn()
        z.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(z) / iters

    q_ms = timed(lambda: kvq.kvq_nf4_quantize(x["K"], x["V"], capacity=T, packed=packed, stream=stream))
    d_ms = timed(lambda: kvq.kvq_nf4_decode_attn(x["q"], packed, T, T, out=out, ws=ws, stream=stream))
    in_bytes = 2 * B * H * T * d * 2
    pk_bytes = packed.numel()
    res = {"workload": f"nqkv_opt30b: B{B} x H{H} x T{T} x d{d}, fp16, NF4 block 256",
           "quantize": {"tokens_per_s": B * T / (q_ms * 1e-3), "launch_ms": q_ms, "bytes_per_launch": in_bytes + pk_bytes,
                        "gb_s": (in_bytes + pk_bytes) / (q_ms * 1e-3) / 1e9},
           "decode": {"kv_tokens_per_s": B * T / (d_ms * 1e-3), "launch_ms": d_ms, "bytes_per_launch": pk_bytes,
                      "gb_s": pk_bytes / (d_ms * 1e-3) / 1e9},
           "bytes_per_token_per_256_values": 130}
    for k in ("quantize", "decode"):
        res[k]["hbm_frac"] = res[k]["gb_s"] / hbm_peak
    del x, packed
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------------------------------ CPU oracle

def oracle_sample(n_tokens: int, seed: int = 0, workload: str = WORKLOAD, batch: int = 0):
    """Time the oracle's calibrate + quantize/pack + decode on the first n_tokens of one layer
    of a workload (all KV heads and q-heads; `batch` sequences, default the workload's).
    Returns (seconds, layer-tokens)."""
    import numpy as np
    import torch
    from oracle import blockgtq as bg
    from packed_cache_attention_b200 import workloads as wl
    W = wl.WORKLOADS[workload]
    B = batch or W.batch
    x = wl.make_blockgtq_inputs(B, W.n_q_heads, W.n_kv_heads, W.head_dim, n_tokens, W.dtype, W.rope_base,
                                W.key_profile, seed=seed, device="cpu")
    K = x["K"].float().numpy()
    V = x["V"].float().numpy()
    q = x["q"].float().numpy()
    t0 = time.perf_counter()
    alloc = bg.calibrate(K, W.bits_k, n_calib=min(W.n_calib, n_tokens) if W.n_calib else 0)
    codes = bg.quantize(K, V, alloc, W.bits_v)
    packed = bg.pack_cache(codes, alloc, W.bits_v, n_tokens)
    bg.decode(q, packed, alloc, W.bits_v, n_tokens)
    return time.perf_counter() - t0, B * n_tokens


def oracle_nf4_sample(n_tokens: int, batch: int = 1, seed: int = 0):
    """Time the oracle's NF4 quantize/pack of K and V and its MHA decode on the first n_tokens
    of `batch` sequences of the OPT-30B-shaped workload (56 heads). Returns (seconds, layer-tokens)."""
    from oracle import nqkv
    from packed_cache_attention_b200 import workloads as wl
    W = wl.WORKLOADS["nqkv_opt30b"]
    y = wl.make_nf4_inputs(batch, W.n_q_heads, W.head_dim, n_tokens, W.dtype, seed=seed, device="cpu")
    K, V, q = (t.float().numpy() for t in (y["K"], y["V"], y["q"]))
    t0 = time.perf_counter()
    ki, ks = nqkv.quantize(K)
    vi, vs = nqkv.quantize(V)
    kc, kss = nqkv.pack(ki, ks, n_tokens)
    vc, vss = nqkv.pack(vi, vs, n_tokens)
    nqkv.decode(q, kc, kss, vc, vss, W.n_q_heads, W.head_dim, n_tokens)
    return time.perf_counter() - t0, batch * n_tokens


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(n_tokens: int = 131072):
    """The oracle on the host cores: the 128K layer on one core, then bounded samples of every
    workload on one core and with numpy's default thread count (all cores)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        secs, toks = oracle_sample(n_tokens)
    ncpu = os.cpu_count() or 1
    per = {}
    samples = {"tiny": (512, 0), "llama8b": (4096, 0), "qwen3b": (8192, 0), "batched": (2048, 2)}
    for name, (n, bsz) in samples.items():
        row = {}
        for label, lim in (("one_core", 1), ("all_cores", None)):
            with threadpool_limits(limits=lim):
                sec, tk = oracle_sample(n, workload=name, batch=bsz)
            row[label] = tk / sec
        row["sample"] = f"first {n} tokens" + (f" of {bsz} sequences" if bsz else "")
        per[name] = row
    row = {}
    for label, lim in (("one_core", 1), ("all_cores", None)):
        with threadpool_limits(limits=lim):
            sec, tk = oracle_nf4_sample(1024)
        row[label] = tk / sec
    row["sample"] = "first 1024 tokens of 1 sequence, 56 heads"
    per["nqkv_opt30b"] = row
    return {"value": toks / secs, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"one layer of {WORKLOAD}, first {n_tokens} tokens of both KV heads: calibrate + quantize/pack "
                      f"+ decode for 16 q-heads ({secs:.1f} s)",
            "host": {"nproc": ncpu, "cpu_model": cpu_model()},
            "per_workload_layer_tokens_per_s": per}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from threadpoolctl import threadpool_limits
    n_tokens = 2048
    with threadpool_limits(limits=1):
        for i in range(args.warmup):
            oracle_sample(n_tokens, seed=i)
        t0 = time.perf_counter()
        toks = 0
        for i in range(args.steps):
            s, t = oracle_sample(n_tokens, seed=100 + i)
            toks += t
        total = time.perf_counter() - t0
    value = toks / total
    return {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64/f32 (numpy oracle)", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": f"{WORKLOAD}: one layer, first {n_tokens} tokens per step (bounded sample)",
                       "layers": 1, "global_batch": 1, "seq_len": n_tokens, "parallelism": "cpu"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"{n_tokens} tokens of one layer per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline()       # before any CUDA work in this process
    res = run_gpu(args, rank, world, local_rank)
    if rank == 0:
        res["cpu_baseline"] = base
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as tdist
        tdist.barrier()
        tdist.destroy_process_group()


if __name__ == "__main__":
    main()

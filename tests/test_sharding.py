"""Sharding of the path over ranks, on CPU: two gloo ranks split the KV heads of one
workload, each runs its share (here through the CPU oracle, since there is no GPU), and the
outputs gathered in rank order equal the single-rank result byte for byte. The (sequence, KV
head) units never exchange data: calibration, quantization and decode of a head read that
head alone."""
import os
import socket
import time
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import blockgtq as bg
from packed_cache_attention_b200 import shard
from packed_cache_attention_b200 import workloads as wl

B, HQ, HKV, T, BK, BV = 2, 6, 3, 200, 3, 3


def _inputs():
    x = wl.make_blockgtq_inputs(B, HQ, HKV, 128, T, "bf16", 5e5, "lognormal_outliers", seed=12, device="cpu")
    return x["K"].float().numpy(), x["V"].float().numpy(), x["q"].float().numpy()


def _oracle_heads(K, V, q, kv: range):
    """The oracle's calibrate -> quantize -> pack -> decode on the KV heads of `kv` alone."""
    G = HQ // HKV
    Kl, Vl = K[:, kv.start:kv.stop], V[:, kv.start:kv.stop]
    qh = shard.query_heads(kv, G)
    a = bg.calibrate(Kl, BK)
    p = bg.pack_cache(bg.quantize(Kl, Vl, a, BV), a, BV, T)
    return bg.decode(q[:, qh.start:qh.stop], p, a, BV, T)


class OracleLib:
    """Stands in for the ctypes binding on the CPU: the calls decode_step_sharded makes, with
    the same arguments and result types (fp32 output), computed by the oracle."""

    @staticmethod
    def kvq_calibrate(K, bits_k, n_calib=0):
        return bg.calibrate(K.numpy(), bits_k, n_calib)

    @staticmethod
    def cache_desc(batch, n_kv_heads, capacity, bits_k, bits_v):
        return {"batch": batch, "n_kv_heads": n_kv_heads, "capacity": capacity, "bits_k": bits_k, "bits_v": bits_v}

    @staticmethod
    def kvq_quantize(K, V, alloc, cache):
        assert K.shape[1] == cache["n_kv_heads"] == len(alloc["w"])
        codes = bg.quantize(K.numpy(), V.numpy(), alloc, cache["bits_v"])
        return bg.pack_cache(codes, alloc, cache["bits_v"], cache["capacity"])

    @staticmethod
    def kvq_decode_attn(q, packed, alloc, cache, seq_len):
        return torch.from_numpy(bg.decode(q.numpy(), packed, alloc, cache["bits_v"], seq_len)).float()


def _step_rank(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        K, V, q = (torch.from_numpy(a) for a in _inputs())
        full = shard.decode_step_sharded(K, V, q, BK, BV, world, rank, kvq=OracleLib)
        np.save(os.path.join(out_dir, f"step{rank}.npy"), full.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        K, V, q = _inputs()
        kv = shard.kv_head_ranges(HKV, world)[rank]
        local = torch.from_numpy(_oracle_heads(K, V, q, kv)) if len(kv) else torch.zeros((B, 0, 128),
                                                                                          dtype=torch.float64)
        full = shard.gather_outputs(local, kv, HKV, HQ // HKV, world)
        np.save(os.path.join(out_dir, f"out{rank}.npy"), full.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_kv_head_ranges_cover_every_head_once():
    for n, w in [(8, 2), (3, 2), (2, 3), (16, 8), (1, 4)]:
        rs = shard.kv_head_ranges(n, w)
        assert len(rs) == w and [h for r in rs for h in r] == list(range(n))
        assert max(len(r) for r in rs) - min(len(r) for r in rs) <= 1
    assert list(shard.query_heads(range(1, 3), 4)) == list(range(4, 12))


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 4])
def test_sharded_heads_equal_single_rank(tmp_path, world):
    """3 KV heads over 2 ranks (1 + 2 heads) and over 4 ranks (one rank with none): the
    gathered output equals the single-rank oracle result exactly."""
    mp.start_processes(_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    K, V, q = _inputs()
    ref = _oracle_heads(K, V, q, range(HKV))
    for r in range(world):
        got = np.load(tmp_path / f"out{r}.npy")
        np.testing.assert_array_equal(got, ref)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 4])
def test_decode_step_sharded_equals_single_rank(tmp_path, world):
    """The library's own sharded step (head ranges, query-head slices, padded all-gather), run
    over gloo ranks with the oracle standing in for the kernels: every rank ends with the
    single-rank output, fp32 bits equal."""
    mp.start_processes(_step_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    K, V, q = _inputs()
    ref = _oracle_heads(K, V, q, range(HKV)).astype(np.float32)
    for r in range(world):
        got = np.load(tmp_path / f"step{r}.npy")
        assert got.dtype == np.float32
        np.testing.assert_array_equal(got, ref)


def _rank_that_leaves(rank, world, port, out_dir):
    """Rank 1 leaves the job before the gather (it exits between steps, with nothing in
    flight); rank 0 goes on to the gather and records what happened."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    if rank == 1:
        dist.destroy_process_group()
        return
    t0 = time.monotonic()
    try:
        shard.gather_outputs(torch.zeros((1, 2, 128)), range(0, 1), 2, 2, world)
        outcome = "returned"
    except Exception as e:                                   # the collective reports the missing rank
        outcome = "error " + type(e).__name__
    with open(os.path.join(out_dir, "rank0.txt"), "w") as fh:
        fh.write(f"{outcome} {time.monotonic() - t0:.1f}")


@pytest.mark.timeout(120)
def test_gather_reports_a_rank_that_left(tmp_path):
    """A rank that left is seen by the others at their next collective: the gather raises
    within the process group's timeout instead of waiting for good."""
    mp.start_processes(_rank_that_leaves, args=(2, _free_port(), str(tmp_path)), nprocs=2, start_method="spawn")
    outcome, seconds = (tmp_path / "rank0.txt").read_text().rsplit(" ", 1)
    assert outcome.startswith("error"), outcome
    assert float(seconds) < 60

"""Host logic of bench.py (CPU only): work counts, multi-rank aggregation.

The multi-GPU path of the benchmark shards whole batches across ranks with no
data-path collective; the only cross-rank step is taking the slowest rank's
time.  That logic is checked here with two gloo ranks on the CPU.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from differential_attention_07_b200 import inputs


def test_algorithmic_work_counts():
    # 768 FLOP per causal (query, key <= query) pair per head
    assert bench.prefill_flops(inputs.WORKLOADS["motif4k"]) == 768 * 4 * 16 * 4096 * 4097 // 2
    assert abs(bench.prefill_flops(inputs.WORKLOADS["lc16k"]) / 1e12 - 1.6494) < 1e-4
    # grouped: 24 signal + 8 noise score maps, 24 + 8 P.V products (one V per group)
    g = inputs.WORKLOADS["grouped"]
    pairs = 4096 * 4097 // 2
    assert bench.prefill_flops(g) == (32 * 128 + 32 * 256) * pairs * 2
    # decode: K1 + K2 + V read once
    assert bench.decode_bytes(inputs.WORKLOADS["decode"]) == 64 * 16 * 8192 * 256 * 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        dev = torch.device("cpu")
        bench.barrier(dev)
        elapsed = [0.5, 2.0][rank]                      # rank 1 is the slow one
        value, t = bench.aggregate_throughput(100.0, elapsed, dev, world)
        m = bench.max_over_ranks(float(rank + 10), dev)
        q.put((rank, value, t, m))
        bench.barrier(dev)
    finally:
        dist.destroy_process_group()


def test_two_rank_aggregation_uses_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, t, m in res:
        assert t == 2.0                     # max over ranks
        assert value == 100.0 * world / 2.0  # all ranks' units over the slowest time
        assert m == 11.0


def test_single_process_aggregation_is_identity():
    value, t = bench.aggregate_throughput(7.0, 0.5, torch.device("cpu"), 1)
    assert (value, t) == (14.0, 0.5)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""


def test_traffic_figure_is_dropped_when_the_kernel_source_changes(monkeypatch):
    t = bench.prefill_traffic()
    assert t is None or t > 0
    monkeypatch.setitem(bench.PREFILL_TRAFFIC, "source_sha256_16", "0" * 16)
    assert bench.prefill_traffic() is None


def test_window_pair_count():
    # W(W+1)/2 pairs for the first W queries, then W per query
    assert bench.causal_pairs(16384, 128) == 128 * 129 // 2 + (16384 - 128) * 128
    assert bench.causal_pairs(100, 0) == bench.causal_pairs(100, 100) == 5050
    w = inputs.WORKLOADS["swa16k"]
    assert bench.prefill_flops(w) == 768 * 16 * bench.causal_pairs(16384, 128)
    assert bench.prefill_bytes(w) == 16384 * 16 * 1024

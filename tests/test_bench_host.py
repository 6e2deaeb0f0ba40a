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


# ------------------------------------------------------------------ one problem split over ranks
SHARD_SHAPES = [  # (B, N, H, H_N, H_V)
    (3, 5, 4, 4, 4),      # plain heads
    (1, 6, 16, 16, 16),   # one sequence (the long-context case): heads are the only split
    (2, 4, 6, 2, 2),      # groups of 3 signal heads sharing a noise and a V head
    (2, 4, 6, 2, 6),      # grouped noise heads, one V per signal head
    (2, 3, 3, 1, 1),      # a single group: the heads split leaves one rank idle
]


def _standin(x, H, H_N, H_V):
    """A stand-in for the kernel that is pure data movement: output channels
    0..63 copy Q1 of the row's signal head, 64..127 copy the first 64
    channels of its V head, with K2 of its noise head added to 64..127 (so
    every index map of the shard views is exercised)."""
    B, N = x["q1"].shape[:2]
    out = torch.zeros(B, N, H, 128)
    for h in range(H):
        n, hv = h // (H // H_N), h // (H // H_V)
        out[:, :, h, :64] = x["q1"][:, :, h].float()
        out[:, :, h, 64:] = x["v"][:, :, hv, :64].float() + x["k2"][:, :, n].float()
    return out


def _shard_worker(rank, world, port, q):
    import dataclasses
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        dev = torch.device("cpu")
        res = []
        for (B, N, H, H_N, H_V) in SHARD_SHAPES:
            w = dataclasses.replace(inputs.WORKLOADS["tiny"], B=B, N=N, H=H, H_N=H_N, H_V=H_V)
            x = inputs.workload_inputs(w)                      # the same global inputs on every rank
            for mode in ("batch", "heads"):
                plan = bench.shard_plan(w, world, rank, mode)
                xs = bench.shard_inputs(x, plan)
                out_full = torch.zeros(B, N, H, 128)
                if plan["b1"] > plan["b0"] and plan["h1"] > plan["h0"]:
                    sw = bench.shard_work(w, plan)
                    out_full[plan["b0"]:plan["b1"], :, plan["h0"]:plan["h1"]] = _standin(
                        xs, sw.H, sw.H_N, sw.H_V)
                cover = torch.zeros(B, H)
                cover[plan["b0"]:plan["b1"], plan["h0"]:plan["h1"]] = 1
                dist.all_reduce(cover)
                bench.gather_output(out_full, dev)
                res.append((mode, (B, N, H, H_N, H_V), cover.numpy(), out_full.numpy()))
        q.put((rank, res))
        bench.barrier(dev)
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_cover_one_problem_and_gather_to_its_layout():
    """Batch and head splits of one global problem over two gloo ranks:
    every (b, signal head) is computed by exactly one rank, and the gathered
    output equals the unsharded output layout [B, N, H, 128]."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    import dataclasses
    for i, (mode, shape, cover, out) in enumerate(got[0]):
        B, N, H, H_N, H_V = shape
        assert (cover == 1).all(), (mode, shape)                   # exactly once each
        w = dataclasses.replace(inputs.WORKLOADS["tiny"], B=B, N=N, H=H, H_N=H_N, H_V=H_V)
        ref = _standin(inputs.workload_inputs(w), H, H_N, H_V).numpy()
        assert (out == ref).all(), (mode, shape)
        assert (got[1][i][3] == ref).all()                         # every rank holds it


def test_shard_plan_keeps_groups_whole():
    import dataclasses
    g = inputs.WORKLOADS["grouped"]                      # 24 signal heads in 8 groups of 3
    plans = [bench.shard_plan(g, 8, r, "heads") for r in range(8)]
    assert [(p["h0"], p["h1"], p["n0"], p["n1"], p["v0"], p["v1"]) for p in plans] == [
        (3 * r, 3 * r + 3, r, r + 1, r, r + 1) for r in range(8)]
    lc = inputs.WORKLOADS["lc16k"]                       # B = 1: heads are the only split
    plans = [bench.shard_plan(lc, 4, r, "heads") for r in range(4)]
    assert [(p["h0"], p["h1"]) for p in plans] == [(0, 4), (4, 8), (8, 12), (12, 16)]
    assert sum(bench.prefill_flops(bench.shard_work(lc, p)) for p in plans) == bench.prefill_flops(lc)
    m = inputs.WORKLOADS["motif4k"]
    plans = [bench.shard_plan(m, 3, r, "batch") for r in range(3)]
    assert [(p["b0"], p["b1"]) for p in plans] == [(0, 1), (1, 2), (2, 4)]
    assert bench.shard_plan(m, 1, 0, "heads") == bench.shard_plan(m, 1, 0, "replica")
    w = dataclasses.replace(m, H=6, H_N=2, H_V=3)        # groups: lcm(3, 2) = 6 heads, one unit
    assert [bench.shard_plan(w, 2, r, "heads")["h1"] for r in range(2)] == [0, 6]

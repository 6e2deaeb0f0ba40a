"""Benchmark of differential attention on B200 (headline: the forward pass).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one causal prefill of the Motif-2.6B-shaped workload (batch 4,
sequence 4096, 16 heads, Q/K head dim 64, V head dim 128, bf16) through the C
ABI: the fp16 V staging kernel plus the warp-specialised tcgen05 prefill
kernel.  Rank 0 prints one JSON line:

* value        prefill TFLOP/s over all ranks (768 FLOP per causal
               query/key pair per head), inputs resident in HBM;
* e2e          the same metric with pinned-host inputs copied in and the output
               copied out inside the timed region;
* roofline     the prefill kernel alone, timed with CUDA events recorded
               around its launch, against the measured dense-bf16 peak;
* cpu_baseline the float64 oracle on a bounded sample of the same workload
               (rank 0, one GPU only);
* extra        the other workloads at one pass each: long context (1 x 16384),
               grouped (24 signal / 8 noise heads), gated (the grouped shape
               with token-dependent lambda and output gate, no norm: Motif 3
               summary, section 2.2), sliding window (1 x 16384, W = 128),
               RoPE (the 4K shape, theta = 500,000), the backward pass of the
               4K shape and of the gated grouped shape (1280 FLOP per pair per
               signal head; also the saving forward and a training step of
               both), decode (batch 64, 8192 cached keys; GB/s against the
               measured HBM copy bandwidth).

With more than one GPU (torchrun) every rank runs its own batch of the same
shape by default (weak scaling; the path has no exchange step); `--shard
batch|heads` instead splits one global problem by batch entries or by
(whole groups of) heads through strided views, and `--gather` assembles the
output afterwards.  The time is the max over ranks.  `--impl reference`
times the oracle itself on the host cores.
"""
import argparse
import json
import os
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from differential_attention_07_b200 import inputs  # noqa: E402

FLOP_PER_PAIR = 768  # 2*64 + 2*64 (two QK^T) + 2*128 + 2*128 (two P.V)
# Backward, the products it cannot do without: the two score maps again
# (2*64 each), dP = dD V^T (2*128, shared by both maps), dV = (P_1 - lambda
# P_2)^T dD (2*128, shared), dK_1, dK_2, dQ_1, dQ_2 (2*64 each).  The kernels
# execute 1792: the query-tile kernel recomputes both score maps and dP.
BWD_FLOP_PER_PAIR = 1280
# Timed steps of each secondary workload: at least 20 steps and about 25 ms
# of device time (the grouped prefill takes about 0.25 ms a step, the 16K
# prefill 1.6 ms).
EXTRA_STEPS = 20
EXTRA_SECONDS = 0.025


def extra_steps(call, device, minimum=EXTRA_STEPS):
    """Steps for a secondary workload: one untimed call sizes the loop to
    about EXTRA_SECONDS of device time, at least `minimum` steps."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    call()
    e0.record()
    call()
    e1.record()
    torch.cuda.synchronize(device)
    t = max(e0.elapsed_time(e1) / 1e3, 1e-6)
    return max(minimum, int(EXTRA_SECONDS / t + 0.999))


def causal_pairs(N, window=0):
    """Visible (query, key) pairs of one head: key j <= query i, and under a
    sliding window of W keys also j > i - W."""
    if window <= 0 or window >= N:
        return N * (N + 1) // 2
    return window * (window + 1) // 2 + (N - window) * window


def prefill_bytes(w):
    """Algorithmic HBM bytes of one prefill call: Q1, Q2, K1, K2, V read once
    and the output written once (bf16)."""
    per_token = (w.H + w.H_N) * w.d * 2 * 2 + w.H_V * w.dv * 2 + w.H * w.dv * 2
    return w.B * w.N * per_token


def prefill_flops(w):
    """Algorithmic FLOP of one prefill call (causal pairs only).

    Per pair: 2*64 for each score map, 2*128 for each P.V product.  In the
    grouped form a noise map is computed once per noise head; its P.V product
    is shared by the group when the group shares one V head (H_V == H_N),
    otherwise each signal head multiplies it by its own V."""
    pairs = causal_pairs(w.N, w.window) if w.causal else w.N * w.N
    qk_maps = w.H + w.H_N
    pv_maps = w.H + (w.H_N if w.H_V == w.H_N else w.H)
    return (qk_maps * 2 * 64 + pv_maps * 2 * 128) * pairs * w.B


def decode_bytes(w):
    """Algorithmic HBM bytes of one decode call: K1 + K2 + V read once."""
    return w.B * w.H * w.N * (64 + 64 + 128) * 2


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one
# prefill_kernel launch on the 4 x 4096 x 16-head workload, from one ncu
# capture, keyed by a hash of the kernel sources it was taken on.  A kernel
# whose sources no longer hash to this value reports null traffic.
PREFILL_TRAFFIC = {"source_sha256_16": "e4427aace67f1a28", "bytes": 268_173_312 + 47_439_872}


def prefill_traffic():
    import hashlib
    h = hashlib.sha256()
    for f in ("prefill_sm100.cu", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "differential_attention_07_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if h.hexdigest()[:16] != PREFILL_TRAFFIC["source_sha256_16"]:
        return None
    return PREFILL_TRAFFIC["bytes"]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained"),
                    source="measured (MEASURED_PEAKS.json)")
    # The pool's earlier measurement, used when the per-pod file is absent.
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback (MEASURED_PEAKS.json absent)")


# ------------------------------------------------------------------ distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x, device):
    """Max of a float over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_throughput(units_per_rank, elapsed_s_local, device, world):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    t = max_over_ranks(elapsed_s_local, device)
    return units_per_rank * world / t, t


def sum_over_ranks(x, device):
    """Sum of a float over ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ partition
SHARD_MODES = ("replica", "batch", "heads")


def shard_plan(w, world, rank, mode):
    """The part of a workload that `rank` of `world` computes.

    * replica: the whole workload, on inputs of the rank's own seed (every
      rank one independent problem: weak scaling);
    * batch: batch entries [b0, b1) of one global problem;
    * heads: heads of one global problem, whole groups at a time: noise heads
      [n0, n1), their signal heads [h0, h1) and V heads [v0, v1).  A group
      is the least run of signal heads that owns whole noise and V heads
      (lcm of H / H_N and H / H_V signal heads).

    Every (b, signal head) of the global problem falls to exactly one rank
    in the batch and heads modes; the work (b, h) units need no exchange.
    Returns a dict of the index ranges (empty ranges when a rank gets no
    work)."""
    import math
    g_n, g_v = w.H // w.H_N, w.H // w.H_V
    full = dict(b0=0, b1=w.B, h0=0, h1=w.H, n0=0, n1=w.H_N, v0=0, v1=w.H_V)
    if mode == "replica" or world == 1:
        return full
    if mode == "batch":
        return {**full, "b0": rank * w.B // world, "b1": (rank + 1) * w.B // world}
    if mode != "heads":
        raise ValueError(mode)
    unit = g_n * g_v // math.gcd(g_n, g_v)
    units = w.H // unit
    u0, u1 = rank * units // world, (rank + 1) * units // world
    h0, h1 = u0 * unit, u1 * unit
    return {**full, "h0": h0, "h1": h1, "n0": h0 // g_n, "n1": h1 // g_n,
            "v0": h0 // g_v, "v1": h1 // g_v}


def shard_inputs(x, plan):
    """Views of a workload's [B, N, heads, dim] tensors (and the per-head
    lambda / gain, per-token logits and gate) restricted to a shard plan.
    The views keep the global tensors' strides."""
    b = slice(plan["b0"], plan["b1"])
    sig, noise, vh = (slice(plan["h0"], plan["h1"]), slice(plan["n0"], plan["n1"]),
                      slice(plan["v0"], plan["v1"]))
    heads = {"q1": sig, "k1": sig, "q2": noise, "k2": noise, "v": vh, "lam_logits": sig, "gate": sig}
    out = {}
    for k, t in x.items():
        if t is None:
            out[k] = None
        elif k in ("lam", "gain"):
            out[k] = t[sig]
        else:
            out[k] = t[b, :, heads[k]]
    return out


def shard_work(w, plan):
    """The workload restricted to a shard (for its FLOP count)."""
    import dataclasses
    return dataclasses.replace(w, B=plan["b1"] - plan["b0"], H=plan["h1"] - plan["h0"],
                               H_N=max(1, plan["n1"] - plan["n0"]), H_V=max(1, plan["v1"] - plan["v0"]))


def gather_output(out_full, device):
    """Assemble the ranks' output slices: each rank holds the global output
    layout with only its own slice written and zeros elsewhere, so a sum over
    ranks is the unsharded output exactly.  Runs outside the timed region."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(out_full, op=dist.ReduceOp.SUM)
    return out_full


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled (NVML, every ~2 ms, from a
    background thread) while the timed region runs."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device):
        self.device = device
        self.samples = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self._handle = None

    def _open(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            pr = torch.cuda.get_device_properties(self.device)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            self._handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            self._handle = pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)
        self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        return pynvml

    def __enter__(self):
        import threading
        try:
            nv = self._open()
        except Exception:
            return self
        self._stop = threading.Event()

        def run():
            while not self._stop.is_set():
                try:
                    mhz = nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM)
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
                self._stop.wait(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        mhz = sorted(m for m, _ in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b)
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ timing helpers
def time_loop(fn, steps, warmup, device, stream=None, clocks=None, kernel_ops=None):
    """Device time (s) of `steps` calls of fn after `warmup` calls; barrier and
    synchronize on both sides; events on the launching stream.  `clocks` (a
    ClockSampler) samples the SM clock during the timed region only.

    With `kernel_ops` (the ops module) the library also records a pair of
    events around each call's main kernel(s) (diffattn_set_profile_events),
    and the mean of those durations is returned too: the step time and the
    kernel time then come from the same timed calls."""
    import contextlib
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize(device)
    barrier(device)
    s = stream or torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ks = []
    if kernel_ops is not None:
        ks = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for a, b in ks:  # torch creates the CUDA events on first record
            a.record(s)
            b.record(s)
        torch.cuda.synchronize(device)
    with (clocks if clocks is not None else contextlib.nullcontext()):
        e0.record(s)
        for i in range(steps):
            if ks:
                kernel_ops.set_profile_events(*ks[i])
            fn()
        e1.record(s)
        torch.cuda.synchronize(device)
    if ks:
        kernel_ops.set_profile_events(None, None)
    barrier(device)
    t = e0.elapsed_time(e1) / 1e3
    if not ks:
        return t
    return t, sum(a.elapsed_time(b) for a, b in ks) / steps / 1e3


# ------------------------------------------------------------------ CPU baseline
def cpu_baseline(w, budget_s=12.0, seed_rows=0):
    """The float64 oracle on a bounded, row-sampled piece of workload `w`:
    returns (throughput in the workload's unit, description, threads)."""
    import oracle
    x = inputs.workload_inputs(w)
    if w.kind == "decode":
        nseq = 1
        t0 = time.perf_counter()
        while True:
            sub = {k: (v[:nseq] if k not in ("lam", "gain") else v) for k, v in x.items()}
            t0 = time.perf_counter()
            oracle.decode(sub["q1"], sub["q2"], sub["k1"], sub["k2"], sub["v"], sub["lam"],
                          sub["gain"], scale=w.scale, eps=w.eps)
            dt = time.perf_counter() - t0
            if dt > budget_s / 4 or nseq >= w.B:
                break
            nseq = min(w.B, nseq * 4)
        byts = nseq * w.H * w.N * 256 * 2
        return byts / dt / 1e9, f"{nseq} of {w.B} sequences x {w.H} heads x {w.N} keys", oracle.threads()
    # prefill: sample rows uniformly over (b, i, h); work of a row = (i+1) pairs
    nrows = 64
    while True:
        rows = inputs.sample_rows(w.B, w.N, w.H, nrows, seed=w.seed + 7 + seed_rows)
        t0 = time.perf_counter()
        oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=w.scale, eps=w.eps, causal=w.causal, rows=rows)
        dt = time.perf_counter() - t0
        if dt > budget_s / 4 or nrows >= 1 << 16:
            break
        nrows *= 4
    pairs = int((rows[:, 1] + 1).sum()) if w.causal else nrows * w.N
    flops = pairs * FLOP_PER_PAIR
    return flops / dt / 1e12, f"{nrows} sampled query rows of {w.name} ({pairs} causal pairs)", oracle.threads()


# ------------------------------------------------------------------ GPU arm
def to_dev(x, device):
    return {k: v.to(device, non_blocking=True) for k, v in x.items()}


def run_prefill_workload(w, steps, warmup, device, ops, rank=0, clocks=None, plan=None,
                         shard="replica", separate_kernel_loop=False):
    """Time the prefill of workload w.  With a shard plan (batch or heads
    mode) every rank draws the same global inputs and computes its slice of
    them through strided views, writing its slice of a global output.

    The kernel time comes from events the library records around the prefill
    launch in the same timed calls, or, with separate_kernel_loop, from a
    second loop of as many calls (the headline keeps its timed calls free of
    the extra event records)."""
    seed = w.seed + 1000 * rank if shard == "replica" else w.seed
    x = inputs.workload_inputs(inputs.Workload(**{**w.__dict__, "seed": seed}))
    d_full = to_dev(x, device)
    plan = plan or shard_plan(w, 1, 0, "replica")
    d = shard_inputs(d_full, plan)
    sw = shard_work(w, plan)
    empty = plan["b1"] <= plan["b0"] or plan["h1"] <= plan["h0"]
    grouped = w.kind == "grouped"
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    out_full = torch.zeros(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=device)
    out = out_full[plan["b0"]:plan["b1"], :, plan["h0"]:plan["h1"]]
    ws = torch.empty(max(1, ops.fwd_workspace_size(sw.B, sw.N, sw.H, sw.H_V, sw.H_N, sw.rope_theta, sw.window)
                         if not empty else 1), dtype=torch.uint8, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)

    def call():
        if empty:
            return
        f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], scale=w.scale, eps=w.eps,
          causal=w.causal, apply_norm=w.apply_norm, out=out, workspace=ws, dev_status=status,
          window=w.window, rope_theta=w.rope_theta,
          lam_logits=d.get("lam_logits"), gate=d.get("gate"))

    call()
    launches = ops.last_launch_count() if not empty else 0
    if steps is None:
        steps = extra_steps(call, device)
    if separate_kernel_loop:
        t = time_loop(call, steps, warmup, device, clocks=clocks)
        _, tk = time_loop(call, steps, 0, device, kernel_ops=ops)
    else:
        t, tk = time_loop(call, steps, warmup, device, clocks=clocks, kernel_ops=ops)
    torch.cuda.synchronize(device)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} in {w.name}")
    return dict(step_s=t / steps, kernel_s=tk, launches=launches, steps=steps, x=shard_inputs(x, plan), d=d,
                call=call, out=out, out_full=out_full, ws=ws, f=f, work=sw, empty=empty,
                flops=0 if empty else prefill_flops(sw))


def run_decode_workload(w, steps, warmup, device, ops, clocks=None):
    x = inputs.workload_inputs(w)
    d = to_dev(x, device)
    out = torch.empty(w.B, w.H, w.dv, dtype=torch.bfloat16, device=device)
    ws = torch.empty(ops.decode_workspace_size(w.B, w.H, w.N), dtype=torch.uint8, device=device)

    def call():
        ops.diffattn_decode(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                            scale=w.scale, eps=w.eps, out=out, workspace=ws)

    call()
    launches = ops.last_launch_count()
    if steps is None:
        steps = extra_steps(call, device)
    t, tk = time_loop(call, steps, warmup, device, clocks=clocks, kernel_ops=ops)
    return dict(step_s=t / steps, kernel_s=tk, launches=launches, steps=steps)


def e2e_prefill(w, steps, warmup, device, ops, x):
    """Same metric through the public call with pinned-host inputs: H2D copies
    of every input, the call, D2H copy of the output, all inside the timing.

    A step is pipelined over the batch entries on three streams, the way a
    serving loop would use the call: entry b's inputs are copied in while
    entry b-1 is computed and entry b-2's output is copied out.  Copies and
    calls of one step never overlap the next step's."""
    host = {k: v.contiguous().pin_memory() for k, v in x.items() if v is not None}
    dev = {k: torch.empty_like(v, device=device) for k, v in host.items()}
    out = torch.empty(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=device)
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    ws = torch.empty(ops.fwd_workspace_size(w.B, w.N, w.H, w.H_V, w.H_N, w.rope_theta, w.window), dtype=torch.uint8, device=device)
    f = ops.diffattn_grouped_fwd if w.kind == "grouped" else ops.diffattn_fwd
    s_in, s_c, s_out = (torch.cuda.Stream(device) for _ in range(3))
    per_batch = [k for k in dev if dev[k].dim() == 4]          # [B, N, heads, dim] tensors
    shared = [k for k in dev if k not in per_batch]            # lambda, gain

    def step():
        main = torch.cuda.current_stream(device)
        start = torch.cuda.Event()
        start.record(main)
        s_in.wait_event(start)
        with torch.cuda.stream(s_in):
            for k in shared:
                dev[k].copy_(host[k], non_blocking=True)
        for b in range(w.B):
            with torch.cuda.stream(s_in):
                for k in per_batch:
                    dev[k][b].copy_(host[k][b], non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            s_c.wait_event(ready)
            sl = {k: (dev[k][b:b + 1] if k in per_batch else dev[k]) for k in dev}
            f(sl["q1"], sl["q2"], sl["k1"], sl["k2"], sl["v"], sl["lam"], sl["gain"], scale=w.scale,
              eps=w.eps, causal=w.causal, out=out[b:b + 1], workspace=ws, stream=s_c)
            done = torch.cuda.Event()
            done.record(s_c)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                out_host[b].copy_(out[b], non_blocking=True)
        end = torch.cuda.Event()
        end.record(s_out)
        main.wait_event(end)

    t = time_loop(step, steps, warmup, device)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()
    return t / steps, h2d, d2h


def run_backward_workload(w, steps, warmup, device, ops, clocks=None):
    """Time diffattn_bwd (and the forward that saves its state) on workload w
    (any of its options: grouped heads, token lambda, gate, window, RoPE)."""
    x = inputs.workload_inputs(w)
    d = to_dev(x, device)
    dy = inputs.grad_output(w.B, w.N, w.H, w.dv, seed=w.seed).to(device)
    save = torch.empty(ops.fwd_save_size(w.B, w.N, w.H), dtype=torch.uint8, device=device)
    out = torch.empty(w.B, w.N, w.H, w.dv, dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    f = ops.diffattn_grouped_fwd if w.kind == "grouped" else ops.diffattn_fwd
    opts = dict(lam_logits=d.get("lam_logits"), gate=d.get("gate"), window=w.window,
                rope_theta=w.rope_theta)
    fws = torch.empty(1, dtype=torch.uint8, device=device)

    def fwd():
        f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], scale=w.scale, eps=w.eps,
          causal=w.causal, apply_norm=w.apply_norm, out=out, workspace=fws, save=save,
          dev_status=status, **opts)

    # the saving forward's workspace (a grouped call that saves needs no noise outputs)
    a = ops._fwd_args(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], out,
                      scale=w.scale, eps=w.eps, causal=w.causal, apply_norm=w.apply_norm,
                      timeout_ms=0, dev_status=None, save=save, **opts)
    fws = torch.empty(max(1, ops.lib().diffattn_fwd_workspace_size(ops.ctypes.byref(a))),
                      dtype=torch.uint8, device=device)
    fwd()
    grads = ops.diffattn_bwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], dy,
                             save, scale=w.scale, eps=w.eps, causal=w.causal,
                             apply_norm=w.apply_norm, dev_status=status, **opts)
    bws = torch.empty(ops.bwd_workspace_size(w.B, w.N, w.H, w.H_N, w.H_V, w.rope_theta),
                      dtype=torch.uint8, device=device)

    def bwd():
        ops.diffattn_bwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], dy, save,
                         scale=w.scale, eps=w.eps, causal=w.causal, apply_norm=w.apply_norm,
                         grads=grads, workspace=bws, dev_status=status, **opts)

    bwd()
    launches = ops.last_launch_count()
    if steps is None:
        steps = extra_steps(bwd, device)
    tb, tk = time_loop(bwd, steps, warmup, device, clocks=clocks, kernel_ops=ops)
    tb /= steps
    tf = time_loop(fwd, steps, warmup, device) / steps
    torch.cuda.synchronize(device)
    if status.item() != 0:
        raise RuntimeError(f"device status {status.item()} in the backward of {w.name}")
    return dict(bwd_s=tb, kernel_s=tk, fwd_save_s=tf, launches=launches, steps=steps)


def backward_line(w, rb, peaks):
    """The bench's record of one backward workload: 1280 FLOP per visible
    (query, key) pair per signal head (every product the gradient needs:
    both score maps again, dP, dV, dK_1, dK_2, dQ_1, dQ_2)."""
    pairs = (causal_pairs(w.N, w.window) if w.causal else w.N * w.N) * w.B * w.H
    fl = pairs * BWD_FLOP_PER_PAIR
    return {"tflops": round(fl / rb["bwd_s"] / 1e12, 2),
            "kernel_tflops": round(fl / rb["kernel_s"] / 1e12, 2),
            "frac_of_peak": round(fl / rb["kernel_s"] / 1e12 / peaks["bf16_tflops"], 4),
            "ms": round(rb["bwd_s"] * 1e3, 4), "fwd_save_ms": round(rb["fwd_save_s"] * 1e3, 4),
            "train_step_tflops": round(pairs * (FLOP_PER_PAIR + BWD_FLOP_PER_PAIR)
                                       / (rb["bwd_s"] + rb["fwd_save_s"]) / 1e12, 2),
            "flop_per_pair": BWD_FLOP_PER_PAIR, "launches": rb["launches"], "steps": rb["steps"],
            "kernels_timed": "bwd_key_kernel + bwd_query_kernel"}


def gpu_arm(args):
    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    from differential_attention_07_b200 import build, ops
    if rank == 0:
        build.build()
    barrier(device)
    peaks = measured_peaks()
    w = inputs.WORKLOADS[args.workload]
    plan = shard_plan(w, world, rank, args.shard)

    clk = ClockSampler(device)
    r = run_prefill_workload(w, args.steps, args.warmup, device, ops, rank, clocks=clk, plan=plan,
                             shard=args.shard, separate_kernel_loop=True)
    units = r["flops"]                        # this rank's algorithmic FLOP per step
    total_units = sum_over_ranks(units, device)
    t_max = max_over_ranks(r["step_s"] * args.steps, device)
    value = total_units * args.steps / t_max / 1e12
    gathered = None
    if args.gather and args.shard != "replica":  # outside the timed region
        gather_output(r["out_full"], device)
        gathered = bool(torch.isfinite(r["out_full"].float()).all().item())
    e2e_s, h2d, d2h = (e2e_prefill(r["work"], max(3, args.steps // 4), 2, device, ops, r["x"])
                       if not r["empty"] else (0.0, 0, 0))
    e2e_value = total_units / max_over_ranks(e2e_s, device)

    achieved = units / r["kernel_s"] / 1e12 if not r["empty"] else 0.0
    result = {
        "metric": "diff-attn fwd TFLOP/s (bf16 causal)",
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_max / args.steps * 1e3, 4),
        "higher_is_better": True,
        "scaling": "weak" if args.shard == "replica" else "strong",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B{w.B} N{w.N} H{w.H} d64 dv128 causal prefill",
                   "global_batch": w.B * world if args.shard == "replica" else w.B,
                   "seq_len": w.N, "heads": w.H,
                   "parallelism": {"replica": f"dp{world} (independent batches)",
                                   "batch": f"batch split over {world} ranks (one global problem)",
                                   "heads": f"heads split over {world} ranks (one global problem)"}[args.shard],
                   "l2": "inputs 201 MB per rank, larger than the 126 MB L2; no flush"},
        "e2e": {"value": round(e2e_value / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1),
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4),
                     "peak_source": "bf16 burst, " + peaks["source"],
                     "kernel": "prefill_kernel", "traffic": prefill_traffic(),
                     "traffic_unit": "bytes per launch (ncu)"},
        "gpu_launches": r["launches"] * args.steps,
        "clocks": clk.summary(),
    }
    if gathered is not None:
        result["gathered"] = gathered
    if world == 1 and not args.no_extra:
        extra = {}
        for name in ("lc16k", "grouped", "gated", "swa16k", "rope4k"):
            wx = inputs.WORKLOADS[name]
            cx = ClockSampler(device)
            rx = run_prefill_workload(wx, None, 3, device, ops, clocks=cx)
            fx = prefill_flops(wx)
            extra[name] = {"tflops": round(fx / rx["step_s"] / 1e12, 2),
                           "kernel_tflops": round(fx / rx["kernel_s"] / 1e12, 2),
                           "frac_of_peak": round(fx / rx["kernel_s"] / 1e12 / peaks["bf16_tflops"], 4),
                           "ms": round(rx["step_s"] * 1e3, 4), "steps": rx["steps"],
                           "sm_mhz": cx.summary()["sm_mhz"]}
            if wx.window:  # few keys per query: the HBM bytes bound it, not the tensor cores
                gb = prefill_bytes(wx) / rx["step_s"] / 1e9
                extra[name]["gbs"] = round(gb, 1)
                extra[name]["hbm_frac"] = round(gb / peaks["hbm_gbs"], 4)
            del rx
        for key, name in (("bwd4k", "motif4k"), ("bwd_gated", "gated")):
            # the gated workload is Motif 3's attention: grouped, token lambda, gate
            wb = inputs.WORKLOADS[name]
            cb = ClockSampler(device)
            rb = run_backward_workload(wb, None, 3, device, ops, clocks=cb)
            extra[key] = backward_line(wb, rb, peaks)
            extra[key]["sm_mhz"] = cb.summary()["sm_mhz"]
            del rb
        wd = inputs.WORKLOADS["decode"]
        cd = ClockSampler(device)
        rd = run_decode_workload(wd, None, 3, device, ops, clocks=cd)
        bd = decode_bytes(wd)
        extra["decode"] = {"gbs": round(bd / rd["step_s"] / 1e9, 1),
                           "split_kernel_gbs": round(bd / rd["kernel_s"] / 1e9, 1),
                           "roofline": {"bound": "hbm", "achieved": round(bd / rd["step_s"] / 1e9, 1),
                                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                        "peak_source": "HBM copy, " + peaks["source"],
                                        "frac": round(bd / rd["step_s"] / 1e9 / peaks["hbm_gbs"], 4)},
                           "us": round(rd["step_s"] * 1e6, 2), "launches": rd["launches"],
                           "steps": rd["steps"], "sm_mhz": cd.summary()["sm_mhz"]}
        result["extra"] = extra
    if world == 1 and rank == 0 and not args.no_cpu:
        v, sample, cores = cpu_baseline(w, budget_s=args.cpu_budget)
        result["cpu_baseline"] = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores,
                                  "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(result), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def reference_arm(args):
    """The oracle as it stands, timed on the host cores (rank 0 only)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    w = inputs.WORKLOADS[args.workload]
    import oracle
    x = inputs.workload_inputs(w)
    per_step = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = None
    nrows = 16
    while True:  # size one step's row sample to about per_step seconds
        rows = inputs.sample_rows(w.B, w.N, w.H, nrows, seed=w.seed + 99)
        t0 = time.perf_counter()
        oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=w.scale, eps=w.eps, causal=w.causal, rows=rows)
        if time.perf_counter() - t0 > per_step / 4 or nrows >= 1 << 16:
            break
        nrows *= 2
    nrows = int(nrows * min(4.0, per_step / max(1e-3, time.perf_counter() - t0)))
    total_flops, total_t = 0, 0.0
    for s in range(args.warmup + args.steps):
        rows = inputs.sample_rows(w.B, w.N, w.H, nrows, seed=w.seed + 100 + s)
        t0 = time.perf_counter()
        oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=w.scale, eps=w.eps, causal=w.causal, rows=rows)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            total_t += dt
            total_flops += int((rows[:, 1] + 1).sum()) * FLOP_PER_PAIR
    value = total_flops / total_t / 1e12
    sample = f"{nrows} sampled query rows per step of {w.name}"
    print(json.dumps({
        "impl": "reference", "metric": "diff-attn fwd TFLOP/s (bf16 causal)",
        "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B{w.B} N{w.N} H{w.H} d64 dv128 causal prefill",
                   "global_batch": w.B, "seq_len": w.N, "heads": w.H},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="motif4k", choices=["motif4k", "lc16k", "grouped"])
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-baseline leg")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--shard", choices=SHARD_MODES, default="replica",
                    help="multi-GPU split: independent problems per rank (replica), or one global "
                         "problem split by batch entries or by heads")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard batch|heads, assemble the output on every rank afterwards")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        reference_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()

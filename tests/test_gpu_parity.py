"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Tolerance (fixed by the workload definition): on the normalised bf16 output,
max abs error <= 2e-2 and mean abs error <= 2e-3 against the unrounded float64
oracle.  Small shapes span several 128-row tiles plus a ragged tail; the
full-size workloads run in the launch configuration the benchmark times.
Every case is compared element by element.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _dev(x):
    return {k: v.cuda() for k, v in x.items()}


def _errs(y_gpu, ref):
    y = y_gpu.detach().float().cpu().double().numpy()
    assert np.all(np.isfinite(y)), "non-finite output"
    e = np.abs(y - ref)
    return float(e.max()), float(e.mean())


def _assert_parity(y_gpu, ref, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    mx, mn = _errs(y_gpu, ref)
    assert mx <= max_abs and mn <= mean_abs, f"max abs {mx:.3e}, mean abs {mn:.3e}"
    return mx, mn


def _run_prefill(x, *, grouped=False, causal=True, apply_norm=True, scale=0.125, eps=1e-5,
                 status=None):
    d = _dev(x)
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    y = f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], scale=scale, eps=eps,
          causal=causal, apply_norm=apply_norm, dev_status=status)
    torch.cuda.synchronize()
    return y


def _oracle_prefill(x, rows=None, causal=True, apply_norm=True, scale=0.125, eps=1e-5):
    return oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                          scale=scale, eps=eps, causal=causal, apply_norm=apply_norm, rows=rows)


def test_tiny_workload(cuda_ok):
    w = inputs.WORKLOADS["tiny"]
    x = inputs.workload_inputs(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_prefill(x, status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_prefill(x))


@pytest.mark.parametrize("N", [1, 2, 64, 127, 128, 129, 255, 300, 513])
def test_prefill_ragged_lengths(cuda_ok, N):
    x = inputs.prefill_inputs(2, N, 3, seed=N, lam=(0.0, 0.9), gain_std=0.1)
    y = _run_prefill(x)
    _assert_parity(y, _oracle_prefill(x))


def test_prefill_multi_tile_many_heads(cuda_ok):
    x = inputs.prefill_inputs(3, 700, 5, seed=17, lam=(0.2, 0.8), gain_std=0.1)
    y = _run_prefill(x)
    _assert_parity(y, _oracle_prefill(x))


@pytest.mark.parametrize("N", [200, 640])
def test_prefill_growing_scores_force_rescales(cuda_ok, N):
    """Key magnitudes that grow along the sequence (and a late spike) make the
    running maximum jump by more than 2^8 repeatedly, so the kernel's stale
    maximum must be corrected (O rescaled, the step's exponentials redone)."""
    x = inputs.prefill_inputs(2, N, 3, seed=N + 1, lam=(0.2, 0.8), gain_std=0.1)
    grow = (1.0 + 5.0 * torch.arange(N, dtype=torch.float32) / N)[None, :, None, None]
    x["k1"] = (x["k1"].float() * grow).to(torch.bfloat16)
    x["k2"] = (x["k2"].float() * grow.flip(1)).to(torch.bfloat16)
    spike = N - N // 5
    x["k1"][:, spike] = (x["q1"][:, -1].float() * 4.0).to(torch.bfloat16)
    y = _run_prefill(x)
    _assert_parity(y, _oracle_prefill(x))


@pytest.mark.parametrize("B,N,H", [(40, 100, 8), (64, 64, 6), (8, 700, 8)])
def test_prefill_many_tiles_per_cta(cuda_ok, B, N, H):
    """More query tiles than SMs, many of them one or two key steps long, so
    each persistent CTA runs several tiles back to back and the work-item
    ring wraps around."""
    x = inputs.prefill_inputs(B, N, H, seed=B + N + H, lam=(0.0, 0.9), gain_std=0.1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_prefill(x, status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_prefill(x))


@pytest.mark.parametrize("N", [100, 384, 450])
def test_prefill_non_causal(cuda_ok, N):
    x = inputs.prefill_inputs(2, N, 2, seed=5 + N, lam=(0.2, 0.8), gain_std=0.1)
    y = _run_prefill(x, causal=False)
    _assert_parity(y, _oracle_prefill(x, causal=False))


def test_prefill_without_norm(cuda_ok):
    """apply_norm off returns D itself, whose scale varies by row (early rows
    average few keys).  Both sides are divided by the oracle's RMS of the row,
    which puts the error in the units of the normalised output, where the
    2e-2 / 2e-3 bar applies."""
    x = inputs.prefill_inputs(2, 333, 2, seed=23, lam=(0.2, 0.8))
    y = _run_prefill(x, apply_norm=False).float().cpu().double().numpy()
    ref = _oracle_prefill(x, apply_norm=False)
    rms = np.sqrt((ref ** 2).mean(-1, keepdims=True))
    e = np.abs(y / rms - ref / rms)
    assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (e.max(), e.mean())


def test_prefill_lambda_zero_and_one(cuda_ok):
    x = inputs.prefill_inputs(1, 260, 4, seed=29, gain_std=0.1)
    x["lam"] = torch.tensor([0.0, 1.0, 0.5, 0.999], dtype=torch.float32)
    _assert_parity(_run_prefill(x), _oracle_prefill(x))


def test_prefill_identical_maps_lambda_one_is_zero(cuda_ok):
    """Q2=Q1, K2=K1, lambda=1: D is exactly zero in every precision, so Y = 0."""
    x = inputs.prefill_inputs(1, 200, 2, seed=31)
    x["q2"], x["k2"] = x["q1"].clone(), x["k1"].clone()
    x["lam"] = torch.ones(2, dtype=torch.float32)
    y = _run_prefill(x)
    assert torch.count_nonzero(y).item() == 0


def test_prefill_strided_views(cuda_ok):
    """Q1/Q2/K1/K2/V as column slices of one fused [B, N, H, 448] projection."""
    B, N, H = 2, 300, 3
    x = inputs.prefill_inputs(B, N, H, seed=37, gain_std=0.1)
    fused = torch.cat([x["q1"], x["q2"], x["k1"], x["k2"], x["v"]], dim=3).cuda()
    q1, q2, k1, k2, v = torch.split(fused, [64, 64, 64, 64, 128], dim=3)
    out = torch.full((B, N, H, 256), float("nan"), dtype=torch.bfloat16, device="cuda")[..., :128]
    y = ops.diffattn_fwd(q1, q2, k1, k2, v, x["lam"].cuda(), x["gain"].cuda(), out=out)
    torch.cuda.synchronize()
    _assert_parity(y, _oracle_prefill(x))


def test_prefill_writes_every_row_and_is_deterministic(cuda_ok):
    x = inputs.prefill_inputs(2, 390, 3, seed=41, gain_std=0.1)
    d = _dev(x)
    outs = []
    for _ in range(2):
        out = torch.full((2, 390, 3, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], out=out)
        outs.append(out)
    torch.cuda.synchronize()
    assert not torch.isnan(outs[0]).any()
    assert torch.equal(outs[0], outs[1])


def test_row0_closed_form_on_gpu(cuda_ok):
    """Row 0 sees only key 0: Y = V[0] / sqrt(mean V[0]^2 + eps/(1-lambda)^2) * gain."""
    x = inputs.prefill_inputs(2, 200, 4, seed=43, gain_std=0.1)
    y = _run_prefill(x)[:, 0].float().cpu().double().numpy()
    v0 = x["v"][:, 0].double().numpy()
    lam = x["lam"].double().numpy()[None, :, None]
    d0 = (1 - lam) * v0
    ref = d0 / np.sqrt((d0 ** 2).mean(-1, keepdims=True) + 1e-5) * x["gain"].double().numpy()[None]
    assert np.abs(y - ref).max() <= MAX_ABS


@pytest.mark.parametrize("H,H_N,H_V,N", [(6, 2, 2, 333), (6, 2, 6, 333), (4, 1, 2, 333),
                                         (3, 3, 1, 333), (10, 2, 2, 333), (15, 5, 5, 200),
                                         (9, 3, 3, 700), (12, 2, 2, 260)])
def test_grouped_small(cuda_ok, H, H_N, H_V, N):
    """Groups of g = 3 or 5 signal heads sharing one V head run as (signal,
    noise) export items and (signal, signal) pair items in one launch; other
    layouts (V per signal head, even g, g = 1) one signal head per item."""
    x = inputs.prefill_inputs(2, N, H, H_N, H_V, seed=47 + H + H_N + H_V, gain_std=0.1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_prefill(x, grouped=True, status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_prefill(x))


@pytest.mark.parametrize("B,N,H,H_N", [(40, 100, 9, 3), (16, 1000, 14, 2), (3, 2000, 21, 3)])
def test_grouped_pairs_many_items(cuda_ok, B, N, H, H_N):
    """Grouped pairs with several items per CTA (more tiles than SMs; g = 3,
    7, 7): pair items wait for export items that other CTAs run, across the
    whole work order."""
    x = inputs.prefill_inputs(B, N, H, H_N, H_N, seed=B + N + H, lam=(0.2, 0.8), gain_std=0.1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_prefill(x, grouped=True, status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_prefill(x))


def test_grouped_g1_equals_ungrouped_bitwise(cuda_ok):
    x = inputs.prefill_inputs(2, 270, 3, seed=53, gain_std=0.1)
    assert torch.equal(_run_prefill(x), _run_prefill(x, grouped=True))


# ------------------------------------------------------------------ decode
def _run_decode(x, **kw):
    d = _dev(x)
    kv = kw.pop("kv_len", None)
    y = ops.diffattn_decode(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                            kv_len=kv.cuda() if kv is not None else None, **kw)
    torch.cuda.synchronize()
    return y


def _oracle_decode(x, kv_len=None, apply_norm=True):
    return oracle.decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         kv_len=kv_len, scale=0.125, eps=1e-5, apply_norm=apply_norm)


@pytest.mark.parametrize("L", [1, 7, 64, 200, 2049, 5000])
def test_decode_lengths(cuda_ok, L):
    x = inputs.decode_inputs(3, L, 4, seed=L, gain_std=0.1)
    _assert_parity(_run_decode(x), _oracle_decode(x))


def test_decode_kv_len_and_splits(cuda_ok):
    B, L, H = 5, 3000, 2
    x = inputs.decode_inputs(B, L, H, seed=61, gain_std=0.1)
    kv = torch.tensor([3000, 1, 64, 65, 2500], dtype=torch.int32)
    ref = _oracle_decode(x, kv_len=kv.numpy())
    ys = []
    for splits in (0, 1, 2, 3, 7, 47):
        y = _run_decode(x, kv_len=kv, num_splits=splits)
        _assert_parity(y, ref)
        ys.append(y.float())
    for y in ys[1:]:
        assert (y - ys[0]).abs().max().item() <= MAX_ABS


def test_decode_equals_last_prefill_row(cuda_ok):
    B, N, H = 2, 333, 3
    x = inputs.prefill_inputs(B, N, H, seed=67, gain_std=0.1)
    yp = _run_prefill(x)
    hm = lambda t: t.permute(0, 2, 1, 3).contiguous()
    xd = dict(q1=x["q1"][:, -1].contiguous(), q2=x["q2"][:, -1].contiguous(), k1=hm(x["k1"]),
              k2=hm(x["k2"]), v=hm(x["v"]), lam=x["lam"], gain=x["gain"])
    yd = _run_decode(xd)
    assert (yd.float() - yp[:, -1].float()).abs().max().item() <= MAX_ABS


def test_decode_bad_kv_len_reports_status(cuda_ok):
    x = inputs.decode_inputs(2, 100, 2, seed=71)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    _run_decode(x, kv_len=torch.tensor([100, 0], dtype=torch.int32), dev_status=st)
    assert st.item() == 1


# ------------------------------------------------------------------ full-size workloads
def _full_parity(name):
    """Every element of a full-size workload, in the benchmark's launch
    configuration, against the whole float64 oracle output (tens of seconds
    of host time on the machine's cores)."""
    w = inputs.WORKLOADS[name]
    x = inputs.workload_inputs(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_prefill(x, grouped=(w.kind == "grouped"), status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_prefill(x))
    # a property that holds at any size: the per-row RMS of Y / gain is
    # sqrt(ms / (ms + eps)) <= 1 (ms = mean D^2); the two maps' common mode
    # cancels, so ms can come within an order of magnitude of eps
    g = x["gain"].cuda()
    r = (y.float() / g[None, None]).pow(2).mean(-1).sqrt()
    assert r.max().item() <= 1.01 and r.min().item() >= 0.5


def test_motif4k_full(cuda_ok):
    _full_parity("motif4k")


def test_lc16k_full(cuda_ok):
    _full_parity("lc16k")


def test_grouped_workload_full(cuda_ok):
    _full_parity("grouped")


def test_decode_workload_full(cuda_ok):
    w = inputs.WORKLOADS["decode"]
    x = inputs.workload_inputs(w)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = _run_decode(x, dev_status=st)
    assert st.item() == 0
    _assert_parity(y, _oracle_decode(x))

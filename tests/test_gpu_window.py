"""Parity of the causal sliding window (CUDA path vs oracle).

Motif 3 summary, section 2.1 (sliding-window layers) and "Practical
Implications" (128-token windows), read as: query i sees keys i-W < j <= i.
Same tolerance as every parity test: max abs <= 2e-2, mean abs <= 2e-3 on the
normalised output.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _check(y, ref):
    y = y.float().cpu().double().numpy() if torch.is_tensor(y) else y
    e = np.abs(y - ref)
    assert np.all(np.isfinite(y))
    assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (e.max(), e.mean())


def _run(x, window, grouped=False, **kw):
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    y = f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], window=window,
          dev_status=st, lam_logits=d.get("lam_logits"), gate=d.get("gate"), **kw)
    torch.cuda.synchronize()
    assert st.item() == 0
    return y


def _oracle(x, window, rows=None):
    return oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                          scale=0.125, eps=1e-5, window=window, rows=rows,
                          lam_logits=x.get("lam_logits"), gate=x.get("gate"))


@pytest.mark.parametrize("W", [1, 7, 63, 64, 65, 100, 128, 129, 300])
def test_window_prefill(cuda_ok, W):
    """Windows below, at and above the 64-key step and the 128-row tile, over
    several tiles and a ragged tail."""
    x = inputs.prefill_inputs(2, 700, 3, seed=W, lam=(0.2, 0.8), gain_std=0.1)
    _check(_run(x, W), _oracle(x, W))


def test_window_covering_everything_equals_no_window(cuda_ok):
    x = inputs.prefill_inputs(2, 333, 2, seed=5, lam=(0.2, 0.8), gain_std=0.1)
    y0 = _run(x, 0)
    for W in (333, 334, 5000):
        assert torch.equal(_run(x, W), y0)


def test_window_grouped_and_gated(cuda_ok):
    """Window with the grouped pair modes, token lambda and the output gate."""
    B, N, H = 2, 500, 6
    x = inputs.prefill_inputs(B, N, H, 2, 2, seed=9, lam=(0.2, 0.8), gain_std=0.1)
    x.update(inputs.gate_inputs(B, N, H, seed=9))
    _check(_run(x, 128, grouped=True), _oracle(x, 128))


def test_window_requires_causal(cuda_ok):
    x = inputs.prefill_inputs(1, 64, 1, seed=1)
    with pytest.raises(ops.DiffAttnError):
        _run(x, 16, causal=False)


def test_window_workload_full(cuda_ok):
    """The sliding-window workload (1 x 16384, 16 heads, W = 128) in the
    benchmark's launch configuration, every element against the oracle."""
    w = inputs.WORKLOADS["swa16k"]
    x = inputs.workload_inputs(w)
    y = _run(x, w.window)
    _check(y, _oracle(x, w.window))


@pytest.mark.parametrize("W", [1, 100, 2048, 3000, 10000])
def test_window_decode(cuda_ok, W):
    B, L, H = 4, 5000, 2
    x = inputs.decode_inputs(B, L, H, seed=W, gain_std=0.1)
    kv = torch.tensor([5000, 1, 777, 4097], dtype=torch.int32)
    d = {k: v.cuda() for k, v in x.items()}
    ref = oracle.decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                        kv_len=kv.numpy(), scale=0.125, eps=1e-5, window=W)
    for splits in (0, 1, 3):
        y = ops.diffattn_decode(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                                kv_len=kv.cuda(), num_splits=splits, window=W)
        torch.cuda.synchronize()
        _check(y, ref)

"""Parity of the rotary position embedding (CUDA path vs oracle).

Motif 2.6B explainer, "The block": RoPE with theta = 500,000, read as each
64-wide map vector (Q1, K1, Q2, K2) rotated by its token position in
interleaved pairs.  The library rotates copies of Q and K in its staging
pass; the caller's tensors stay unchanged.  Same tolerance as every parity
test: max abs <= 2e-2, mean abs <= 2e-3 on the normalised output.
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


def _run(x, theta, grouped=False, window=0):
    d = {k: v.cuda() for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    y = f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], rope_theta=theta,
          window=window, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for k in ("q1", "q2", "k1", "k2"):          # the caller's tensors are untouched
        assert torch.equal(d[k].cpu(), x[k])
    return y


@pytest.mark.parametrize("N", [1, 77, 333, 1000])
def test_rope_prefill(cuda_ok, N):
    x = inputs.prefill_inputs(2, N, 3, seed=N, lam=(0.2, 0.8), gain_std=0.1)
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5, rope_theta=500000.0)
    _check(_run(x, 500000.0), ref)


def test_rope_grouped_windowed_and_strided(cuda_ok):
    """Grouped pairs, a sliding window and Q/K given as slices of a wider
    projection output."""
    B, N, H = 2, 500, 6
    x = inputs.prefill_inputs(B, N, H, 2, 2, seed=17, lam=(0.2, 0.8), gain_std=0.1)
    wide = torch.zeros(B, N, H, 192, dtype=torch.bfloat16)
    wide[..., 64:128] = x["q1"]
    d = {k: v.cuda() for k, v in x.items()}
    q1 = wide.cuda()[..., 64:128]
    y = ops.diffattn_grouped_fwd(q1, d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                                 rope_theta=10000.0, window=200)
    torch.cuda.synchronize()
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5, rope_theta=10000.0, window=200)
    _check(y, ref)


def test_rope_workload_full(cuda_ok):
    """The 4 x 4096 x 16-head workload with theta = 500,000, in the benchmark's
    launch configuration, every element against the oracle (positions up to
    4095)."""
    w = inputs.WORKLOADS["rope4k"]
    x = inputs.workload_inputs(w)
    y = _run(x, w.rope_theta)
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5, rope_theta=w.rope_theta)
    _check(y, ref)

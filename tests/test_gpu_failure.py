"""Failure path of the prefill kernel: bounded waits that run out.

Every mbarrier wait in the prefill kernel is bounded.  With the library's
test hook the producer withholds one K/V load, so the MMA warps' waits run
out after timeout_ms; the kernel must then drain what it issued, free its
TMEM, report DIFFATTN_ERR_TIMEOUT in the device status word and return.  The
device must stay usable: a normal call afterwards still matches the oracle.
Nothing here faults, traps or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def test_withheld_load_reports_timeout_and_device_stays_usable(cuda_ok):
    x = inputs.prefill_inputs(2, 300, 3, seed=11, gain_std=0.1)
    d = {k: v.cuda() for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, 300, 3, 128, dtype=torch.bfloat16, device="cuda")
    ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], out=out,
                     dev_status=st, timeout_ms=50, test_withhold_load=True)
    torch.cuda.synchronize()
    assert st.item() == 6  # DIFFATTN_ERR_TIMEOUT
    assert torch.count_nonzero(out).item() == 0  # nothing was stored

    st.zero_()
    y = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                         dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5)
    err = np.abs(y.float().cpu().double().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_grouped_pairs_time_out_together_and_device_stays_usable(cuda_ok):
    """Grouped pairs in one launch: pair items wait (bounded) for their
    tile's export item.  With every CTA's first load withheld, export items
    never publish, so the pair items' waits run out too; the call reports
    DIFFATTN_ERR_TIMEOUT, stores nothing, and the next call is correct."""
    x = inputs.prefill_inputs(2, 300, 6, 2, 2, seed=12, gain_std=0.1)
    d = {k: v.cuda() for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, 300, 6, 128, dtype=torch.bfloat16, device="cuda")
    ops.diffattn_grouped_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                             out=out, dev_status=st, timeout_ms=50, test_withhold_load=True)
    torch.cuda.synchronize()
    assert st.item() == 6  # DIFFATTN_ERR_TIMEOUT
    assert torch.count_nonzero(out).item() == 0

    st.zero_()
    y = ops.diffattn_grouped_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                                 dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5)
    err = np.abs(y.float().cpu().double().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3

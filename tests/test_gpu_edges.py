"""Edge cases of the CUDA path: empty inputs, extreme sizes, out-of-range
values.  Same tolerance as every parity test (max abs <= 2e-2, mean abs <=
2e-3 on the normalised output)."""
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


@pytest.mark.parametrize("B,N", [(0, 128), (2, 0), (0, 0)])
def test_empty_prefill_launches_nothing(cuda_ok, B, N):
    x = {k: v.cuda() for k, v in inputs.prefill_inputs(B, N, 2, seed=1).items()}
    y = ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    torch.cuda.synchronize()
    assert tuple(y.shape) == (B, N, 2, 128)
    assert ops.last_launch_count() == 0


def test_empty_decode_launches_nothing(cuda_ok):
    x = {k: v.cuda() for k, v in inputs.decode_inputs(0, 64, 2, seed=1).items()}
    y = ops.diffattn_decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    torch.cuda.synchronize()
    assert tuple(y.shape) == (0, 2, 128)
    assert ops.last_launch_count() == 0


def test_long_sequence_sampled(cuda_ok):
    """One head over 65536 tokens (512 query tiles, the longest rows 1024 key
    steps), checked on sampled rows that include the last ones."""
    B, N, H = 1, 65536, 1
    x = inputs.prefill_inputs(B, N, H, seed=3, lam=(0.2, 0.8), gain_std=0.1)
    d = {k: v.cuda() for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                         dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rows = inputs.sample_rows(B, N, H, 24, seed=3)
    rows = torch.cat([rows, torch.tensor([[0, N - 1, 0], [0, N - 129, 0]])])
    b, i, h = rows[:, 0], rows[:, 1], rows[:, 2]
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5, rows=rows)[b.numpy(), i.numpy(), h.numpy()]
    _check(y[b.cuda(), i.cuda(), h.cuda()], ref)


def test_many_one_token_sequences(cuda_ok):
    """256 sequences of one token: every work item is a single-row tile."""
    x = inputs.prefill_inputs(256, 1, 2, seed=4, lam=(0.2, 0.8), gain_std=0.1)
    d = {k: v.cuda() for k, v in x.items()}
    y = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"])
    torch.cuda.synchronize()
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5)
    _check(y, ref)


@pytest.mark.parametrize("window", [0, 64])
def test_v_beyond_fp16_range_is_reported(cuda_ok, window):
    """bf16 can hold values the fp16 P.V product cannot: the staging kernel
    (or, under a sliding window, the kernel's own V conversion) reports
    DIFFATTN_ERR_UNSUPPORTED (2) in the status word; nothing faults and the
    next call is fine."""
    x = {k: v.cuda() for k, v in inputs.prefill_inputs(1, 300, 1, seed=5).items()}
    x["v"][0, 207, 0, 3] = 70000.0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dev_status=st,
                     window=window)
    torch.cuda.synchronize()
    assert st.item() == 2
    x["v"][0, 207, 0, 3] = 1.0
    st.zero_()
    ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dev_status=st,
                     window=window)
    torch.cuda.synchronize()
    assert st.item() == 0

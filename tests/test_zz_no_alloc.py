"""The no-allocation decode entry point (runs last on purpose).

Some callers cannot give the library device memory: an inference server whose
allocator already owns the whole GPU for its KV-cache pool, a latency-critical
path that must not call cudaMalloc (it can synchronise the device), a plugin
with no allocator handle to take a workspace from.  diffattn_decode_noalloc
serves them by keeping the decode's per-split partial states in a fixed
static device array inside the library.  This test calls it through the C ABI
twice in a row, with different inputs and split counts, and checks each
result against diffattn_decode (which uses a caller-owned workspace) and
against the float64 oracle, within the parity tolerance of the other GPU
tests.  It lives in its own file that
sorts last, so a run stopping at the first failure has run everything else.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu


def _dev(x):
    return {k: v.cuda() for k, v in x.items()}


def _both(x, num_splits, kv_len=None):
    d = _dev(x)
    kv = kv_len.cuda() if kv_len is not None else None
    ref = ops.diffattn_decode(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                              kv_len=kv, num_splits=num_splits)
    out = torch.full_like(ref, float("nan"))
    got = ops.diffattn_decode_noalloc(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"],
                                      d["gain"], out=out, kv_len=kv, num_splits=num_splits)
    torch.cuda.synchronize()
    return got.float(), ref.float()


def test_noalloc_decode_matches_workspace_decode_twice(cuda_ok):
    x1 = inputs.decode_inputs(8, 3000, 4, seed=123, gain_std=0.1)
    got1, ref1 = _both(x1, 0)
    x2 = inputs.decode_inputs(3, 777, 2, seed=456, gain_std=0.1)
    got2, ref2 = _both(x2, 5, kv_len=torch.tensor([777, 1, 400], dtype=torch.int32))
    kv2 = torch.tensor([777, 1, 400], dtype=torch.int32)
    exact1 = oracle.decode(x1["q1"], x1["q2"], x1["k1"], x1["k2"], x1["v"], x1["lam"], x1["gain"],
                           scale=0.125, eps=1e-5)
    exact2 = oracle.decode(x2["q1"], x2["q2"], x2["k1"], x2["k2"], x2["v"], x2["lam"], x2["gain"],
                           kv_len=kv2, scale=0.125, eps=1e-5)
    for got, ref, exact in ((got1, ref1, exact1), (got2, ref2, exact2)):
        assert torch.isfinite(got).all()
        err = (got - ref).abs()
        assert err.max().item() <= 2e-2 and err.mean().item() <= 2e-3
        e64 = np.abs(got.cpu().double().numpy() - exact)
        assert e64.max() <= 2e-2 and e64.mean() <= 2e-3, (e64.max(), e64.mean())


def test_noalloc_decode_rejects_sizes_beyond_its_scratch(cuda_ok):
    """Sizes whose partial states do not fit the static array are refused
    before anything is launched (the pointers below are valid and aligned but
    never read)."""
    import ctypes
    buf = torch.zeros(1 << 16, dtype=torch.bfloat16, device="cuda")
    B, H, L = 64, 16, 1 << 16
    assert ops.decode_workspace_size(B, H, L) > 8 << 20
    a = ops.DecodeArgs()
    a.B, a.H, a.L, a.d, a.dv = B, H, L, 64, 128
    a.scale, a.eps, a.flags = 0.125, 1e-5, ops.DIFFATTN_FLAG_APPLY_NORM
    for n in ("q1", "q2", "out"):
        setattr(a, n, buf.data_ptr())
        setattr(a, n + "_stride", ops._S2(H * 128, 128))
    for n in ("k1", "k2", "v"):
        setattr(a, n, buf.data_ptr())
        setattr(a, n + "_stride", ops._S3(H * L * 128, L * 128, 128))
    a.lambda_ = buf.data_ptr()
    st = ops.lib().diffattn_decode_noalloc(ctypes.byref(a), None)
    assert st == 4  # DIFFATTN_ERR_WORKSPACE
    assert b"no-allocation scratch" in ops.lib().diffattn_last_error()

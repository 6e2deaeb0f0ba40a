"""The backward tolerance, derived from the arithmetic (CPU only).

The GPU backward rounds at fixed points: dD and V are fp16 tensor-core
operands, P_1 - lambda P_2 is an fp16 operand, dS_1 and dS_2 are bf16
operands, and every gradient tensor is written in bf16; the rest accumulates
in fp32.  This test applies exactly those roundings to a float64 evaluation of
the gradient and checks that the resulting error against the backward oracle
stays well inside the tolerance the GPU parity tests use (max abs error
<= 2e-2 * max |ref|, mean abs error <= 1e-2 * mean |ref| per gradient): the
tolerance leaves room for fp32 accumulation order and the forward's own
rounding of the saved map outputs, and no more.  It models the arithmetic,
not the CUDA code, and shares nothing with it.
"""
import numpy as np
import torch

import oracle
from differential_attention_07_b200 import inputs


def _f16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)


def _bf16(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


def _rounded_backward(x, dy, scale=0.125, eps=1e-5):
    """The gradient with the kernels' rounding points (one batch entry, one head)."""
    q1, q2, k1, k2, v = (x[k][0, :, 0].double().numpy() for k in ("q1", "q2", "k1", "k2", "v"))
    lam, gain = float(x["lam"][0]), x["gain"][0].double().numpy()
    dy = dy[0, :, 0].double().numpy()
    N = q1.shape[0]
    vis = np.tril(np.ones((N, N), bool))
    P, A = [], []
    for q, k in ((q1, k1), (q2, k2)):
        z = np.where(vis, scale * (q @ k.T), -np.inf)
        w = np.exp(z - z.max(1, keepdims=True))
        P.append(w / w.sum(1, keepdims=True))
        A.append(P[-1] @ v)
    D = A[0] - lam * A[1]
    r = 1 / np.sqrt((D * D).mean(1, keepdims=True) + eps)
    dd = r * gain * dy - r ** 3 / 128 * D * (gain * dy * D).sum(1, keepdims=True)
    delta1, delta2 = (dd * A[0]).sum(1, keepdims=True), -lam * (dd * A[1]).sum(1, keepdims=True)
    dd16, v16 = _f16(dd), _f16(v)
    dP = dd16 @ v16.T
    ds1 = _bf16(P[0] * (dP - delta1))
    ds2 = _bf16(P[1] * (-lam * dP - delta2))
    pc = _f16(P[0] - lam * P[1])
    return {"dq1": _bf16(scale * ds1 @ k1), "dq2": _bf16(scale * ds2 @ k2),
            "dk1": _bf16(scale * ds1.T @ q1), "dk2": _bf16(scale * ds2.T @ q2),
            "dv": _bf16(pc.T @ dd16)}


def test_kernel_roundings_fit_well_inside_the_backward_tolerance():
    for N in (130, 300):
        x = inputs.prefill_inputs(1, N, 1, seed=31, lam=(0.2, 0.8), gain_std=0.1)
        dy = inputs.grad_output(1, N, 1, seed=31)
        g = _rounded_backward(x, dy)
        ref = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                      x["gain"], dy, scale=0.125, eps=1e-5)
        for n, gv in g.items():
            rv = ref[n][0, :, 0]
            e = np.abs(gv - rv)
            assert e.max() <= 0.5 * 2e-2 * np.abs(rv).max(), (N, n, e.max() / np.abs(rv).max())
            assert e.mean() <= 0.5 * 1e-2 * np.abs(rv).mean(), (N, n, e.mean() / np.abs(rv).mean())

"""Parity of the backward pass (diffattn_bwd through the C ABI) with the
float64 backward oracle.

Tolerance, derived from the arithmetic: the gradients are written in bf16
(relative rounding 2^-9), the tensor-core operands dS (bf16), P_1 - lambda
P_2 and dD (fp16) are rounded once per element, and the forward's saved map
outputs carry its own fp16 P.V rounding (about 1e-3 relative).  Each
gradient tensor must be within max abs error <= 2e-2 * max |ref| and mean abs
error <= 1e-2 * mean |ref| of the unrounded float64 oracle; dlambda and dgain
(fp32 sums) within 1e-2 relative.  Small shapes are compared element by
element (several 128-row tiles and a ragged tail), and so is the 4 x 4096 x
16 shape of the benchmark.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu

REL_MAX, REL_MEAN, REL_SUM = 2e-2, 1e-2, 1e-2
NAMES = ("dq1", "dq2", "dk1", "dk2", "dv")


def _dev(x):
    return {k: v.cuda() for k, v in x.items()}


def _opts(x):
    return dict(lam_logits=x.get("lam_logits"), gate=x.get("gate"), window=x.get("window", 0),
                rope_theta=x.get("rope_theta", 0.0))


def _run(x, dy, *, causal=True, apply_norm=True, scale=0.125, eps=1e-5, gain=True):
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    g = d["gain"] if gain else None
    B, N, H, _ = x["q1"].shape
    grouped = x["q2"].shape[2] != H or x["v"].shape[2] != H
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    save = torch.empty(max(ops.fwd_save_size(B, N, H), 16), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], g, scale=scale, eps=eps,
          causal=causal, apply_norm=apply_norm, save=save, dev_status=st, **_opts(d))
    grads = ops.diffattn_bwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], g, dy.cuda(),
                             save, scale=scale, eps=eps, causal=causal, apply_norm=apply_norm,
                             dev_status=st, **_opts(d))
    torch.cuda.synchronize()
    assert st.item() == 0
    return y, {k: v.float().cpu().double().numpy() for k, v in grads.items()}


def _ref(x, dy, *, causal=True, apply_norm=True, scale=0.125, eps=1e-5, gain=True):
    return oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                   x["gain"] if gain else None, dy, scale=scale, eps=eps,
                                   causal=causal, apply_norm=apply_norm, **_opts(x))


def _check(g, ref, names=NAMES, sums=("dlam", "dgain")):
    for n in names:
        assert np.all(np.isfinite(g[n])), n
        e = np.abs(g[n] - ref[n])
        mx, mn = float(e.max()), float(e.mean())
        assert mx <= REL_MAX * np.abs(ref[n]).max(), (n, mx, np.abs(ref[n]).max())
        assert mn <= REL_MEAN * np.abs(ref[n]).mean(), (n, mn, np.abs(ref[n]).mean())
    for n in sums:
        e = np.abs(g[n] - ref[n]).max()
        assert e <= REL_SUM * max(np.abs(ref[n]).max(), 1e-6), (n, e)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("apply_norm", [True, False])
def test_small_element_by_element(cuda_ok, causal, apply_norm):
    """B2 N300 H3: three 128-row tiles (the last ragged), five 64-row blocks."""
    x = inputs.prefill_inputs(2, 300, 3, seed=21, lam=(0.2, 0.8), gain_std=0.1)
    dy = inputs.grad_output(2, 300, 3, seed=21)
    _, g = _run(x, dy, causal=causal, apply_norm=apply_norm)
    ref = _ref(x, dy, causal=causal, apply_norm=apply_norm)
    _check(g, ref, sums=("dlam", "dgain") if apply_norm else ("dlam",))
    if not apply_norm:
        assert np.all(g["dgain"] == 0)


@pytest.mark.parametrize("N", [1, 63, 64, 65, 129])
def test_sizes_around_the_blocks(cuda_ok, N):
    x = inputs.prefill_inputs(1, N, 2, seed=22 + N, lam=(0.2, 0.8), gain_std=0.1)
    dy = inputs.grad_output(1, N, 2, seed=22 + N)
    _, g = _run(x, dy)
    ref = _ref(x, dy)
    if N > 1:
        _check(g, ref)
        return
    # One token: each softmax is constant, so dQ and dK are exactly zero; the
    # GPU's are rounding residue of dP - Delta (dD staged in fp16), far below
    # the scale of dV.  And D = (1 - lambda) V_0, so the norm leaves only eps
    # to depend on lambda: dlambda = -sum_c dD_c V_0c is a near-cancellation
    # of 128 fp32 products of order one, checked to 1e-4 absolute.
    _check(g, ref, names=("dv",), sums=("dgain",))
    assert np.abs(g["dlam"] - ref["dlam"]).max() <= 1e-4
    for n in ("dq1", "dq2", "dk1", "dk2"):
        assert np.abs(g[n]).max() <= 1e-3 * np.abs(ref["dv"]).max(), n


def test_lambda_zero_head_and_no_gain(cuda_ok):
    """lambda = 0 on head 0 (map 2 then gets no gradient there) and gain NULL
    (gradient with respect to a gain of ones)."""
    x = inputs.prefill_inputs(1, 200, 2, seed=23, lam=(0.2, 0.8), lam_head0=0.0)
    dy = inputs.grad_output(1, 200, 2, seed=23)
    _, g = _run(x, dy, gain=False)
    ref = _ref(x, dy, gain=False)
    _check(g, ref)
    assert np.abs(g["dq2"][:, :, 0]).max() == 0 and np.abs(g["dk2"][:, :, 0]).max() == 0


def test_saving_forward_matches_plain_forward(cuda_ok):
    x = inputs.prefill_inputs(2, 300, 3, seed=24, lam=(0.2, 0.8), gain_std=0.1)
    d = _dev(x)
    y0 = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"])
    y1, _ = _run(x, inputs.grad_output(2, 300, 3, seed=24))
    torch.cuda.synchronize()
    assert (y0.float() - y1.float()).abs().max().item() <= 2e-2


def test_autograd_function_matches_oracle(cuda_ok):
    x = inputs.prefill_inputs(1, 160, 2, seed=25, lam=(0.2, 0.8), gain_std=0.1)
    dy = inputs.grad_output(1, 160, 2, seed=25)
    t = {k: v.cuda().requires_grad_(True) for k, v in x.items()}
    y = ops.diff_attention(t["q1"], t["q2"], t["k1"], t["k2"], t["v"], t["lam"], t["gain"])
    y.backward(dy.cuda())
    g = {"d" + k: t[k].grad.float().cpu().double().numpy() for k in ("q1", "q2", "k1", "k2", "v")}
    g["dlam"] = t["lam"].grad.cpu().double().numpy()
    g["dgain"] = t["gain"].grad.cpu().double().numpy()
    _check(g, _ref(x, dy))


def test_benchmark_shape_all_heads(cuda_ok):
    """B4 N4096 H16 (the benchmark's backward workload) in the benchmark's
    launch configuration; every gradient element against the oracle (about
    a second of host time per head)."""
    B, N, H = 4, 4096, 16
    x = inputs.prefill_inputs(B, N, H, seed=1, lam=(0.2, 0.8), gain_std=0.1)
    dy = inputs.grad_output(B, N, H, seed=1)
    _, g = _run(x, dy)
    _check(g, _ref(x, dy))


def test_empty_problem_zeroes_the_sums(cuda_ok):
    x = _dev(inputs.prefill_inputs(0, 128, 2, seed=1))
    save = torch.empty(16, dtype=torch.uint8, device="cuda")
    grads = {k: torch.empty(0, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
             for k in ("dq1", "dq2", "dk1", "dk2")}
    grads["dv"] = torch.empty(0, 128, 2, 128, dtype=torch.bfloat16, device="cuda")
    grads["dlam"] = torch.full((2,), 7.0, device="cuda")
    grads["dgain"] = torch.full((2, 128), 7.0, device="cuda")
    dy = torch.empty(0, 128, 2, 128, dtype=torch.bfloat16, device="cuda")
    ops.diffattn_bwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dy, save,
                     grads=grads)
    torch.cuda.synchronize()
    assert grads["dlam"].abs().max().item() == 0 and grads["dgain"].abs().max().item() == 0


def test_argument_error_enqueues_nothing(cuda_ok):
    """A workspace that is too small is refused before anything is enqueued:
    the caller's dlambda and dgain keep their contents."""
    x = _dev(inputs.prefill_inputs(1, 200, 2, seed=26, lam=(0.2, 0.8), gain_std=0.1))
    save = torch.empty(ops.fwd_save_size(1, 200, 2), dtype=torch.uint8, device="cuda")
    ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], save=save)
    grads = {k: torch.empty(1, 200, 2, 64, dtype=torch.bfloat16, device="cuda")
             for k in ("dq1", "dq2", "dk1", "dk2")}
    grads["dv"] = torch.empty(1, 200, 2, 128, dtype=torch.bfloat16, device="cuda")
    grads["dlam"] = torch.full((2,), 7.0, device="cuda")
    grads["dgain"] = torch.full((2, 128), 7.0, device="cuda")
    dy = inputs.grad_output(1, 200, 2, seed=26).cuda()
    small = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ops.DiffAttnError) as e:
        ops.diffattn_bwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dy, save,
                         grads=grads, workspace=small)
    assert e.value.status == 4  # DIFFATTN_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (grads["dlam"] == 7.0).all() and (grads["dgain"] == 7.0).all()


def test_dD_beyond_fp16_reports_unsupported(cuda_ok):
    """An upstream gradient so large that dD leaves the fp16 range: the call
    returns OK (the condition is only visible on the device) and dev_status
    reads DIFFATTN_ERR_UNSUPPORTED, the caller's sign that these gradients
    are undefined."""
    x = _dev(inputs.prefill_inputs(1, 130, 2, seed=27, lam=(0.2, 0.8), gain_std=0.1))
    dy = inputs.grad_output(1, 130, 2, seed=27, std=1e6).cuda()
    save = torch.empty(ops.fwd_save_size(1, 130, 2), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.diffattn_fwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], save=save,
                     dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ops.diffattn_bwd(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"], dy, save,
                     dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 2  # DIFFATTN_ERR_UNSUPPORTED


# ------------------------------------------------------------------ grouped heads, token lambda, gate, window, RoPE
# Motif 3 summary, section 2.2 (grouped differential output, lambda_t =
# sigma(x_t W^lambda), output gating) and 2.1 (sliding-window layers); Motif
# 2.6B explainer, "The block" (RoPE).  The per-token and per-element
# gradients (dlam_logits, dgate) use the same relative bounds as the others.
def _ext(B, N, H, H_N, H_V, seed, *, logits=False, gate=False, window=0, theta=0.0, gain_std=0.1):
    x = inputs.prefill_inputs(B, N, H, H_N, H_V, seed=seed, lam=(0.2, 0.8), gain_std=gain_std)
    if logits or gate:
        gi = inputs.gate_inputs(B, N, H, seed=seed)
        if logits:
            x["lam_logits"] = gi["lam_logits"]
        if gate:
            x["gate"] = gi["gate"]
    x["window"], x["rope_theta"] = window, theta
    return x, inputs.grad_output(B, N, H, seed=seed)


def _names(x):
    n = list(NAMES)
    if x.get("lam_logits") is not None:
        n.append("dlam_logits")
    if x.get("gate") is not None:
        n.append("dgate")
    return tuple(n)


@pytest.mark.parametrize("H,H_N,H_V", [(6, 2, 2), (6, 2, 6), (4, 1, 2), (6, 3, 2), (9, 3, 3)])
def test_grouped_heads(cuda_ok, H, H_N, H_V):
    """Noise and V heads shared by several signal heads: their gradients are
    summed over the signal heads (fp32 sums, then bf16)."""
    x, dy = _ext(2, 300, H, H_N, H_V, seed=31 + H + H_N + H_V)
    _, g = _run(x, dy)
    _check(g, _ref(x, dy))


@pytest.mark.parametrize("apply_norm", [True, False])
def test_token_lambda_and_gate(cuda_ok, apply_norm):
    x, dy = _ext(2, 333, 3, 3, 3, seed=41 + apply_norm, logits=True, gate=True)
    _, g = _run(x, dy, apply_norm=apply_norm)
    ref = _ref(x, dy, apply_norm=apply_norm)
    _check(g, ref, names=_names(x), sums=("dgain",) if apply_norm else ())
    assert np.all(g["dlam"] == 0)          # the per-head lambda is unused


@pytest.mark.parametrize("W", [1, 50, 128, 200, 1000])
def test_window(cuda_ok, W):
    x, dy = _ext(2, 600, 2, 2, 2, seed=51 + W, window=W)
    _, g = _run(x, dy)
    ref = _ref(x, dy)
    if W > 1:
        _check(g, ref)
        return
    # W = 1: every query sees only itself, so each softmax is constant and
    # dQ, dK are exactly zero; the GPU's are fp32 rounding residue of
    # dP - Delta (both from the same fp16 dD), far below the scale of dV.
    # And D = (1 - lambda) V_i, so the norm leaves only eps to depend on
    # lambda: dlambda sums, over B N rows, near-cancellations of 128 fp32
    # products of order one (about 1e-5 each), checked to 1e-4 sqrt(B N)
    # absolute, as a random walk of those residues.
    _check(g, ref, names=("dv",), sums=("dgain",))
    assert np.abs(g["dlam"] - ref["dlam"]).max() <= 1e-4 * np.sqrt(2 * 600)
    for n in ("dq1", "dq2", "dk1", "dk2"):
        assert np.abs(g[n]).max() <= 1e-3 * np.abs(ref["dv"]).max(), n


@pytest.mark.parametrize("N", [1, 77, 300])
def test_rope(cuda_ok, N):
    x, dy = _ext(1, N, 2, 2, 2, seed=61 + N, theta=10000.0)
    _, g = _run(x, dy)
    ref = _ref(x, dy)
    if N > 1:
        _check(g, ref)
    else:  # one token: dQ and dK are exactly zero (see test_sizes_around_the_blocks)
        _check(g, ref, names=("dv",), sums=("dgain",))


def test_everything_together(cuda_ok):
    """Grouped heads, token lambda, gate, window and RoPE in one call, causal
    and without the norm (Motif 3's formula)."""
    x, dy = _ext(2, 500, 6, 2, 2, seed=71, logits=True, gate=True, window=100, theta=500000.0)
    _, g = _run(x, dy, apply_norm=False)
    _check(g, _ref(x, dy, apply_norm=False), names=_names(x), sums=())


def test_autograd_function_grouped_gated(cuda_ok):
    x, dy = _ext(1, 200, 6, 2, 2, seed=81, logits=True, gate=True, window=64, theta=10000.0)
    t = {k: (v.cuda().requires_grad_(True) if torch.is_tensor(v) else v) for k, v in x.items()}
    y = ops.diff_attention(t["q1"], t["q2"], t["k1"], t["k2"], t["v"], t["lam"], t["gain"],
                           lam_logits=t["lam_logits"], gate=t["gate"], window=64,
                           rope_theta=10000.0)
    y.backward(dy.cuda())
    g = {"d" + k: t[k].grad.float().cpu().double().numpy()
         for k in ("q1", "q2", "k1", "k2", "v", "gain", "lam_logits", "gate")}
    _check(g, _ref(x, dy), names=_names(x) , sums=("dgain",))


def test_grouped_workload_full(cuda_ok):
    """The grouped workload (B2 N4096, 24 signal / 8 noise / 8 V heads), every
    gradient element against the oracle."""
    w = inputs.WORKLOADS["grouped"]
    x = inputs.workload_inputs(w)
    dy = inputs.grad_output(w.B, w.N, w.H, seed=w.seed)
    _, g = _run(x, dy)
    _check(g, _ref(x, dy))


def test_gated_workload_full(cuda_ok):
    """The Motif-3-style workload (grouped, token lambda, gate, no norm),
    every gradient element against the oracle."""
    w = inputs.WORKLOADS["gated"]
    x = inputs.workload_inputs(w)
    dy = inputs.grad_output(w.B, w.N, w.H, seed=w.seed)
    _, g = _run(x, dy, apply_norm=False)
    _check(g, _ref(x, dy, apply_norm=False), names=_names(x), sums=())


def test_saving_forward_with_every_option_matches_plain_forward(cuda_ok):
    """A grouped call that saves runs one signal head per item (the plain
    call shares each noise map over its group); with token lambda, gate,
    window and RoPE both outputs must agree with the oracle."""
    x, dy = _ext(2, 300, 9, 3, 3, seed=91, logits=True, gate=True, window=77, theta=10000.0)
    y1, _ = _run(x, dy)
    d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in x.items()}
    y0 = ops.diffattn_grouped_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                                  **_opts(d))
    torch.cuda.synchronize()
    ref = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                         scale=0.125, eps=1e-5, **_opts(x))
    for y in (y0, y1):
        e = np.abs(y.float().cpu().double().numpy() - ref)
        assert e.max() <= 2e-2 and e.mean() <= 2e-3, (e.max(), e.mean())

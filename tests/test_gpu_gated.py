"""Parity of the token-dependent lambda and the output gate (CUDA path vs oracle).

Motif 3 summary, section 2.2: lambda_t = sigma(x_t W^lambda) per signal head
and token, and GDLA(x_t) = vec(sigma(G_t) (.) D_t) W^O.  The kernels take the
projection outputs (lambda logits, gate logits) and apply sigma; the gate is
the last step of the epilogue.  Same tolerance as every parity test: max abs
<= 2e-2, mean abs <= 2e-3 on the normalised output.  Outputs without the norm
are compared in units of the oracle's per-row RMS of D, so the bar means the
same thing there.
"""
import numpy as np
import pytest
import torch

import oracle
from differential_attention_07_b200 import inputs, ops

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def _gated(B, N, H, H_N=None, H_V=None, seed=0, gain_std=0.1, lam_logits=True, gate=True):
    x = inputs.prefill_inputs(B, N, H, H_N, H_V, seed=seed, lam=(0.2, 0.8), gain_std=gain_std)
    g = inputs.gate_inputs(B, N, H, seed=seed)
    x["lam_logits"] = g["lam_logits"] if lam_logits else None
    x["gate"] = g["gate"] if gate else None
    return x


def _run(x, grouped, apply_norm=True, causal=True):
    d = {k: (v.cuda() if v is not None else None) for k, v in x.items()}
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    f = ops.diffattn_grouped_fwd if grouped else ops.diffattn_fwd
    y = f(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"], scale=0.125, eps=1e-5,
          causal=causal, apply_norm=apply_norm, dev_status=st, lam_logits=d["lam_logits"],
          gate=d["gate"])
    torch.cuda.synchronize()
    assert st.item() == 0
    return y.float().cpu().double().numpy()


def _oracle(x, apply_norm=True, causal=True, rows=None, gate=True):
    return oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                          scale=0.125, eps=1e-5, causal=causal, apply_norm=apply_norm, rows=rows,
                          lam_logits=x["lam_logits"], gate=x["gate"] if gate else None)


def _check(e):
    assert np.all(np.isfinite(e))
    assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (e.max(), e.mean())


# (H, H_N, H_V, N): ungrouped; grouped pairs (export and pair items); grouped one head per item
SHAPES = [(4, 4, 4, 333), (6, 2, 2, 333), (4, 1, 2, 200), (9, 3, 3, 260)]


@pytest.mark.parametrize("H,H_N,H_V,N", SHAPES)
def test_gated_prefill_with_norm(cuda_ok, H, H_N, H_V, N):
    x = _gated(2, N, H, H_N, H_V, seed=H * 31 + N)
    grouped = (H_N, H_V) != (H, H)
    e = np.abs(_run(x, grouped) - _oracle(x))
    _check(e)


@pytest.mark.parametrize("H,H_N,H_V,N", SHAPES)
@pytest.mark.parametrize("causal", [True, False])
def test_gated_prefill_without_norm(cuda_ok, H, H_N, H_V, N, causal):
    """Motif 3's literal output, sigma(G) (.) D with token lambda and no norm.
    The gain is given but must be ignored without the norm."""
    x = _gated(2, N, H, H_N, H_V, seed=H * 17 + N + causal)
    grouped = (H_N, H_V) != (H, H)
    y = _run(x, grouped, apply_norm=False, causal=causal)
    ref = _oracle(x, apply_norm=False, causal=causal)
    dref = _oracle(x, apply_norm=False, causal=causal, gate=False)
    rms = np.sqrt((dref ** 2).mean(-1, keepdims=True))
    _check(np.abs(y - ref) / rms)


def test_token_lambda_only_and_gate_only(cuda_ok):
    for lam_logits, gate in ((True, False), (False, True)):
        x = _gated(2, 333, 4, seed=5 + 2 * lam_logits, lam_logits=lam_logits, gate=gate)
        _check(np.abs(_run(x, False) - _oracle(x)))


def test_gain_is_ignored_without_norm(cuda_ok):
    """The gain belongs to the norm: with the norm off the output is D even
    when a gain is passed (plain inputs, no gate)."""
    x = inputs.prefill_inputs(2, 300, 3, seed=77, lam=(0.2, 0.8), gain_std=0.3)
    x["lam_logits"], x["gate"] = None, None
    y = _run(x, False, apply_norm=False)
    ref = _oracle(x, apply_norm=False)
    rms = np.sqrt((ref ** 2).mean(-1, keepdims=True))
    _check(np.abs(y - ref) / rms)


def test_saturated_logits_match_the_plain_call(cuda_ok):
    """Gate logits of +40 (sigma = 1) and lambda logits equal to logit(lambda_h)
    give the plain per-head call's output within the rounding of sigma."""
    B, N, H = 2, 300, 4
    x = inputs.prefill_inputs(B, N, H, seed=88, lam=(0.2, 0.8), gain_std=0.1)
    d = {k: v.cuda() for k, v in x.items()}
    plain = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"])
    logit = torch.log(d["lam"] / (1 - d["lam"]))
    ll = logit[None, None, :].expand(B, N, H).contiguous()
    gate = torch.full((B, N, H, 128), 40.0, dtype=torch.bfloat16, device="cuda")
    y = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], None, d["gain"],
                         lam_logits=ll, gate=gate)
    torch.cuda.synchronize()
    assert (y.float() - plain.float()).abs().max().item() <= MAX_ABS


def test_strided_logits_and_gate(cuda_ok):
    """Logits and gate as slices of wider tensors (non-contiguous strides)."""
    B, N, H = 2, 200, 4
    x = _gated(B, N, H, seed=99)
    wide_ll = torch.zeros(B, N, H + 3)
    wide_ll[:, :, 1:H + 1] = x["lam_logits"]
    wide_g = torch.zeros(B, N, H, 256, dtype=torch.bfloat16)
    wide_g[..., 128:] = x["gate"]
    d = {k: v.cuda() for k, v in x.items() if v is not None}
    wll, wg = wide_ll.cuda(), wide_g.cuda()
    y = ops.diffattn_fwd(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], d["lam"], d["gain"],
                         lam_logits=wll[:, :, 1:H + 1], gate=wg[..., 128:])
    torch.cuda.synchronize()
    _check(np.abs(y.float().cpu().double().numpy() - _oracle(x)))


def test_gated_workload_full(cuda_ok):
    """The Motif-3-style workload (B2 N4096, 24 signal / 8 noise / 8 V heads,
    token lambda, gate, no norm) in the benchmark's launch configuration,
    every element against the oracle, in units of the oracle's per-row RMS of
    D."""
    w = inputs.WORKLOADS["gated"]
    x = inputs.workload_inputs(w)
    y = _run(x, True, apply_norm=False)
    ref = _oracle(x, apply_norm=False)
    dref = _oracle(x, apply_norm=False, gate=False)
    rms = np.sqrt((dref ** 2).mean(-1, keepdims=True))
    _check(np.abs(y - ref) / rms)


# ------------------------------------------------------------------ decode
def _decode_case(B, L, H, seed):
    x = inputs.decode_inputs(B, L, H, seed=seed, gain_std=0.1)
    x.update(inputs.gate_inputs(B, None, H, seed=seed))
    return x


@pytest.mark.parametrize("apply_norm", [True, False])
def test_gated_decode(cuda_ok, apply_norm):
    B, L, H = 4, 3000, 3
    x = _decode_case(B, L, H, seed=13 + apply_norm)
    kv = torch.tensor([3000, 1, 777, 2048], dtype=torch.int32)
    d = {k: v.cuda() for k, v in x.items()}
    y = ops.diffattn_decode(d["q1"], d["q2"], d["k1"], d["k2"], d["v"], None, d["gain"],
                            kv_len=kv.cuda(), apply_norm=apply_norm, lam_logits=d["lam_logits"],
                            gate=d["gate"])
    torch.cuda.synchronize()
    ref = oracle.decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, x["gain"],
                        kv_len=kv.numpy(), scale=0.125, eps=1e-5, apply_norm=apply_norm,
                        lam_logits=x["lam_logits"], gate=x["gate"])
    unit = 1.0
    if not apply_norm:
        dref = oracle.decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, None,
                             kv_len=kv.numpy(), scale=0.125, eps=1e-5, apply_norm=False,
                             lam_logits=x["lam_logits"])
        unit = np.sqrt((dref ** 2).mean(-1, keepdims=True))
    _check(np.abs(y.float().cpu().double().numpy() - ref) / unit)

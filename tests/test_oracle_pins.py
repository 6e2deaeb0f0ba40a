"""Pins of the float64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not share code with: a
hand-derived worked example, torch's scaled-dot-product attention and rms_norm
(library routines) in the special cases that reduce to them, SciPy's softmax in
a full-matrix brute force, closed forms and invariants of the formula
attn = [softmax(Q1 K1^T) - lambda softmax(Q2 K2^T)] V with the norm after the
subtraction (Motif 2.6B explainer, section "Differential attention" and
figure 1) and of its grouped form D = H_S - lambda Repeat_g(H_N) (Motif 3
summary, section 2.2).  Chosen so that a dropped term, a wrong sign or index,
a transposed operand, an off-by-one causal mask or a misplaced eps fails one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from differential_attention_07_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.double()


def _sdpa(q, k, v, scale, causal):
    """torch SDPA in float64 on token-major [B,N,H,d] tensors -> [B,N,H,dv]."""
    qh, kh, vh = (x.permute(0, 2, 1, 3) for x in (q, k, v))
    o = F.scaled_dot_product_attention(qh, kh, vh, is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3)


def _small(B=2, N=37, H=3, H_N=None, H_V=None, d=64, dv=128, seed=7, lam=(0.2, 0.8),
           gain_std=0.1):
    x = inputs.prefill_inputs(B, N, H, H_N, H_V, d, dv, seed=seed, lam=lam, gain_std=gain_std)
    return {k: _f64(v) for k, v in x.items()}


# ---------------------------------------------------------------------------
# hand-derived worked example
# ---------------------------------------------------------------------------
def test_golden_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "closed_form_n2.json")))
    x = {k: np.array(v, dtype=np.float64) for k, v in g["inputs"].items()
         if k in ("q1", "q2", "k1", "k2", "v", "lambda")}
    s, eps, tol = g["inputs"]["scale"], g["inputs"]["eps"], g["tolerance_abs"]
    e = g["expected"]
    args = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lambda"])
    pre = oracle.prefill(*args, scale=s, eps=eps, causal=True, apply_norm=False)
    np.testing.assert_allclose(pre[0, :, 0, :], e["causal_prenorm"], atol=tol, rtol=0)
    y = oracle.prefill(*args, scale=s, eps=eps, causal=True)
    np.testing.assert_allclose(y[0, :, 0, :], e["causal_norm"], atol=tol, rtol=0)
    ync = oracle.prefill(*args, scale=s, eps=eps, causal=False)
    np.testing.assert_allclose(ync[0, 0, 0, :], e["noncausal_norm_row0"], atol=tol, rtol=0)
    yg = oracle.prefill(*args, np.array([[2.0, 3.0]]), scale=s, eps=eps, causal=True)
    np.testing.assert_allclose(yg[0, 1, 0, :], e["causal_norm_gain23_row1"], atol=tol, rtol=0)
    # decode: query of row 1 against the two cached keys, head-major layout
    hm = lambda a: a.transpose(0, 2, 1, 3)
    yd = oracle.decode(x["q1"][:, 1], x["q2"][:, 1], hm(x["k1"]), hm(x["k2"]), hm(x["v"]),
                       x["lambda"], scale=s, eps=eps)
    np.testing.assert_allclose(yd[0, 0], e["decode_norm"], atol=tol, rtol=0)


# ---------------------------------------------------------------------------
# special cases that reduce to library routines
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("causal", [True, False])
def test_lambda_zero_is_sdpa_then_rms_norm(causal):
    """lambda = 0 is ordinary attention (explainer: 'At lambda = 0 it's just
    ordinary attention'), then the per-head RMS norm with gain."""
    x = _small()
    lam = torch.zeros(3, dtype=torch.float64)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], lam, x["gain"],
                       scale=0.125, eps=1e-5, causal=causal)
    a = _sdpa(x["q1"], x["k1"], x["v"], 0.125, causal)
    ref = torch.stack([F.rms_norm(a[:, :, h], (128,), weight=x["gain"][h], eps=1e-5)
                       for h in range(3)], dim=2)
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12, rtol=0)


def test_map2_is_sdpa():
    """D is affine in lambda: D(0) - D(1) = softmax(s Q2 K2^T) V, checked
    against torch SDPA (pins map 2's operands and indices)."""
    x = _small(seed=11)
    args = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"])
    d0 = oracle.prefill(*args, torch.zeros(3, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False)
    d1 = oracle.prefill(*args, torch.ones(3, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False)
    a2 = _sdpa(x["q2"], x["k2"], x["v"], 0.125, True)
    np.testing.assert_allclose(d0 - d1, a2.numpy(), atol=1e-12, rtol=0)


def test_identical_maps_give_one_minus_lambda():
    """Q2=Q1, K2=K1 gives (1 - lambda) softmax(s Q K^T) V before the norm."""
    x = _small(seed=3)
    lam = x["lam"]
    d = oracle.prefill(x["q1"], x["q1"], x["k1"], x["k1"], x["v"], lam, scale=0.125, eps=1e-5,
                       apply_norm=False)
    a = _sdpa(x["q1"], x["k1"], x["v"], 0.125, True)
    ref = a * (1.0 - lam)[None, None, :, None]
    np.testing.assert_allclose(d, ref.numpy(), atol=1e-12, rtol=0)
    # lambda = 1 with identical maps cancels exactly to zero; the norm keeps it 0
    y = oracle.prefill(x["q1"], x["q1"], x["k1"], x["k1"], x["v"],
                       torch.ones(3, dtype=torch.float64), scale=0.125, eps=1e-5)
    assert np.all(y == 0.0)


def test_brute_force_scipy_softmax_small():
    """Full-matrix brute force with SciPy's softmax for N <= 8."""
    for N in range(1, 9):
        x = _small(B=1, N=N, H=2, d=8, dv=6, seed=100 + N)
        y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                           scale=0.35, eps=1e-5, causal=True)
        for h in range(2):
            mask = np.triu(np.ones((N, N), dtype=bool), 1)
            maps = []
            for q, k in ((x["q1"], x["k1"]), (x["q2"], x["k2"])):
                z = 0.35 * (q[0, :, h].numpy() @ k[0, :, h].numpy().T)
                z[mask] = -np.inf
                maps.append(scipy.special.softmax(z, axis=1) @ x["v"][0, :, h].numpy())
            dd = maps[0] - x["lam"][h].item() * maps[1]
            ref = dd / np.sqrt((dd ** 2).mean(axis=1, keepdims=True) + 1e-5) * x["gain"][h].numpy()
            np.testing.assert_allclose(y[0, :, h], ref, atol=1e-12, rtol=0)


def test_grouped_matches_repeat_interleave():
    """Grouped: signal head h uses noise head h // g and V head h // g
    (Repeat_g interleaves); equal to the ungrouped oracle on repeat_interleave'd
    Q2, K2 and V."""
    x = _small(B=2, N=29, H=6, H_N=2, H_V=2, seed=5)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=1e-5)
    rep = lambda t: t.repeat_interleave(3, dim=2)
    ref = oracle.prefill(x["q1"], rep(x["q2"]), x["k1"], rep(x["k2"]), rep(x["v"]), x["lam"],
                         x["gain"], scale=0.125, eps=1e-5)
    np.testing.assert_array_equal(y, ref)
    # and map 2 of each signal head is SDPA over its noise head
    d0 = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"],
                        torch.zeros(6, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False)
    d1 = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"],
                        torch.ones(6, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False)
    a2 = _sdpa(x["q2"], x["k2"], x["v"], 0.125, True)
    np.testing.assert_allclose(d0 - d1, rep(a2).numpy(), atol=1e-12, rtol=0)


# ---------------------------------------------------------------------------
# invariants and closed forms
# ---------------------------------------------------------------------------
def test_softmax_rows_sum_to_one():
    g = torch.Generator().manual_seed(1)
    for n in (1, 2, 17, 300):
        q = torch.randn(64, generator=g, dtype=torch.float64) * 3
        k = torch.randn(n, 64, generator=g, dtype=torch.float64)
        w = oracle.softmax_row(q, k, 0.125)
        assert np.all(w >= 0)
        assert abs(w.sum() - 1.0) < 1e-12
        ref = scipy.special.softmax(0.125 * (k.numpy() @ q.numpy()))
        np.testing.assert_allclose(w, ref, atol=1e-14, rtol=0)


def test_causal_independence_of_future_keys():
    x = _small(B=1, N=40, H=2, seed=9)
    args = lambda k1, k2, v: (x["q1"], x["q2"], k1, k2, v, x["lam"], x["gain"])
    y = oracle.prefill(*args(x["k1"], x["k2"], x["v"]), scale=0.125, eps=1e-5)
    i = 17
    k1, k2, v = x["k1"].clone(), x["k2"].clone(), x["v"].clone()
    k1[:, i + 1:] += 5.0
    k2[:, i + 1:] -= 3.0
    v[:, i + 1:] *= -2.0
    y2 = oracle.prefill(*args(k1, k2, v), scale=0.125, eps=1e-5)
    np.testing.assert_array_equal(y[:, :i + 1], y2[:, :i + 1])
    assert np.abs(y[:, i + 1:] - y2[:, i + 1:]).max() > 1e-3


def test_row0_closed_form():
    """Row 0 sees only key 0: D = (1 - lambda) V[0], Y = V[0]/rms(V[0]) * gain
    (eps = 0; lambda < 1 so the (1 - lambda) factor cancels in the norm)."""
    x = _small(B=2, N=5, H=3, seed=21)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=0.0)
    v0 = x["v"][:, 0].numpy()                                # [B, H, dv]
    ref = v0 / np.sqrt((v0 ** 2).mean(-1, keepdims=True)) * x["gain"].numpy()[None]
    np.testing.assert_allclose(y[:, 0], ref, atol=1e-12, rtol=0)
    pre = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], scale=0.125,
                         eps=0.0, apply_norm=False)
    np.testing.assert_allclose(pre[:, 0], v0 * (1 - x["lam"].numpy())[None, :, None],
                               atol=1e-14, rtol=0)


def test_v_scale_invariance_exact():
    """With eps = 0, V -> 2V doubles D exactly and the norm undoes it bit for bit."""
    x = _small(seed=31)
    a = (x["q1"], x["q2"], x["k1"], x["k2"])
    y1 = oracle.prefill(*a, x["v"], x["lam"], x["gain"], scale=0.125, eps=0.0)
    y2 = oracle.prefill(*a, 2 * x["v"], x["lam"], x["gain"], scale=0.125, eps=0.0)
    np.testing.assert_array_equal(y1, y2)


def test_gain_is_channelwise():
    x = _small(seed=41)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"])
    y1 = oracle.prefill(*a, None, scale=0.125, eps=1e-5)
    yg = oracle.prefill(*a, x["gain"], scale=0.125, eps=1e-5)
    np.testing.assert_allclose(yg, y1 * x["gain"].numpy()[None, None], atol=1e-13, rtol=0)


def test_eps_inside_sqrt():
    """eps enters as sqrt(mean(D^2) + eps): with D = (1-lambda) V[0] at row 0
    and a large eps the closed form tells the placements apart."""
    x = _small(B=1, N=3, H=1, seed=51, gain_std=0.0)
    eps = 0.5
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], scale=0.125,
                       eps=eps)
    d0 = (1 - x["lam"][0].item()) * x["v"][0, 0, 0].numpy()
    ref = d0 / math.sqrt((d0 ** 2).mean() + eps)
    np.testing.assert_allclose(y[0, 0, 0], ref, atol=1e-13, rtol=0)


def test_decode_equals_last_prefill_row_and_respects_kv_len():
    B, L, H = 3, 50, 2
    x = _small(B=B, N=L, H=H, seed=61)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=1e-5)
    hm = lambda t: t.permute(0, 2, 1, 3).contiguous()
    kv_len = np.array([L, 1, 23])
    q1 = torch.stack([x["q1"][b, kv_len[b] - 1] for b in range(B)])
    q2 = torch.stack([x["q2"][b, kv_len[b] - 1] for b in range(B)])
    yd = oracle.decode(q1, q2, hm(x["k1"]), hm(x["k2"]), hm(x["v"]), x["lam"], x["gain"],
                       kv_len=kv_len, scale=0.125, eps=1e-5)
    for b in range(B):
        np.testing.assert_allclose(yd[b], y[b, kv_len[b] - 1], atol=1e-13, rtol=0)


def test_decode_lambda_zero_is_sdpa():
    x = inputs.decode_inputs(2, 33, 2, seed=71, gain_std=0.1)
    x = {k: _f64(v) for k, v in x.items()}
    lam = torch.zeros(2, dtype=torch.float64)
    y = oracle.decode(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], lam, x["gain"], scale=0.125,
                      eps=1e-5)
    a = F.scaled_dot_product_attention(x["q1"][:, :, None], x["k1"], x["v"], scale=0.125)[:, :, 0]
    ref = torch.stack([F.rms_norm(a[:, h], (128,), weight=x["gain"][h], eps=1e-5)
                       for h in range(2)], dim=1)
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12, rtol=0)


def test_sampled_rows_match_full():
    x = _small(B=2, N=33, H=3, seed=81)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    full = oracle.prefill(*a, scale=0.125, eps=1e-5)
    rows = inputs.sample_rows(2, 33, 3, count=20, seed=1)
    part = oracle.prefill(*a, scale=0.125, eps=1e-5, rows=rows)
    for b, i, h in rows.tolist():
        np.testing.assert_array_equal(part[b, i, h], full[b, i, h])


def test_oracle_rejects_bad_arguments():
    x = _small(B=1, N=4, H=3)
    with pytest.raises(ValueError):
        oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], scale=1, eps=0,
                       rows=[[0, 4, 0]])
    with pytest.raises(ValueError):
        hm = lambda t: t.permute(0, 2, 1, 3).contiguous()
        oracle.decode(x["q1"][:, 0], x["q2"][:, 0], hm(x["k1"]), hm(x["k2"]), hm(x["v"]),
                      x["lam"], kv_len=[0], scale=1, eps=0)


# ---------------------------------------------------------------------------
# token-dependent lambda and output gate (Motif 3 summary, section 2.2:
# lambda_t = sigma(x_t W^lambda); GDLA(x_t) = vec(sigma(G_t) (.) D_t) W^O)
# ---------------------------------------------------------------------------
def _gated_small(B=2, N=37, H=4, H_N=2, H_V=2, seed=91):
    x = _small(B=B, N=N, H=H, H_N=H_N, H_V=H_V, seed=seed)
    x.update({k: _f64(v) for k, v in inputs.gate_inputs(B, N, H, seed=seed).items()})
    return x


@pytest.mark.parametrize("causal", [True, False])
def test_saturated_logits_give_ordinary_attention(causal):
    """lambda logits -40 (sigma = 4e-18) and gate logits +40 (sigma = 1 - 4e-18):
    ordinary attention (torch SDPA) followed by the RMS norm with gain."""
    x = _gated_small()
    B, N, H = x["lam_logits"].shape
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, x["gain"],
                       scale=0.125, eps=1e-5, causal=causal,
                       lam_logits=torch.full((B, N, H), -40.0, dtype=torch.float64),
                       gate=torch.full((B, N, H, 128), 40.0, dtype=torch.float64))
    a = _sdpa(x["q1"], x["k1"], x["v"].repeat_interleave(2, dim=2), 0.125, causal)
    ref = torch.stack([F.rms_norm(a[:, :, h], (128,), weight=x["gain"][h], eps=1e-5)
                       for h in range(H)], dim=2)
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12, rtol=0)


def test_zero_logits_are_one_half():
    """sigma(0) = 1/2: zero lambda logits equal a per-head lambda of 1/2, and
    zero gate logits halve every output element."""
    x = _gated_small(seed=92)
    B, N, H = x["lam_logits"].shape
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"])
    half = oracle.prefill(*a, torch.full((H,), 0.5, dtype=torch.float64), x["gain"],
                          scale=0.125, eps=1e-5)
    y = oracle.prefill(*a, None, x["gain"], scale=0.125, eps=1e-5,
                       lam_logits=torch.zeros(B, N, H, dtype=torch.float64),
                       gate=torch.zeros(B, N, H, 128, dtype=torch.float64))
    np.testing.assert_allclose(y, 0.5 * half, atol=1e-15, rtol=0)


@pytest.mark.parametrize("causal", [True, False])
def test_token_lambda_against_sdpa(causal):
    """Before the norm, D[b, i, h] = A1 - sigma(z[b, i, h]) A2 with A1, A2 from
    torch SDPA (grouped: map 2 and V from head h // 2) and sigma = 1/(1+e^-z)
    from torch.sigmoid: pins the [B, N, H] indexing of the logits."""
    x = _gated_small(seed=93)
    H = x["lam_logits"].shape[2]
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, scale=0.125,
                       eps=1e-5, causal=causal, apply_norm=False, lam_logits=x["lam_logits"])
    rep = lambda t: t.repeat_interleave(H // t.shape[2], dim=2)
    a1 = _sdpa(x["q1"], x["k1"], rep(x["v"]), 0.125, causal)
    a2 = _sdpa(rep(x["q2"]), rep(x["k2"]), rep(x["v"]), 0.125, causal)
    ref = a1 - torch.sigmoid(x["lam_logits"])[..., None] * a2
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12, rtol=0)


def test_gate_is_elementwise_after_the_norm():
    """With the norm on, gated / ungated = sigma(G) element by element: the gate
    is the last step before W^O (a gate before the norm would be partly
    normalised away) and is indexed [b, i, h, c]."""
    x = _gated_small(seed=94)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    y0 = oracle.prefill(*a, scale=0.125, eps=1e-5)
    y = oracle.prefill(*a, scale=0.125, eps=1e-5, gate=x["gate"])
    np.testing.assert_allclose(y, torch.sigmoid(x["gate"]).numpy() * y0, atol=1e-13, rtol=0)


def test_decode_gated_equals_last_prefill_row():
    """Decode with lambda logits [B, H] and gate logits [B, H, dv] equals the
    last prefill row with the same logits at that row."""
    B, L, H = 2, 41, 3
    x = _small(B=B, N=L, H=H, seed=95)
    gl = {k: _f64(v) for k, v in inputs.gate_inputs(B, L, H, seed=95).items()}
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, x["gain"],
                       scale=0.125, eps=1e-5, lam_logits=gl["lam_logits"], gate=gl["gate"])
    hm = lambda t: t.permute(0, 2, 1, 3).contiguous()
    yd = oracle.decode(x["q1"][:, L - 1], x["q2"][:, L - 1], hm(x["k1"]), hm(x["k2"]),
                       hm(x["v"]), None, x["gain"], scale=0.125, eps=1e-5,
                       lam_logits=gl["lam_logits"][:, L - 1], gate=gl["gate"][:, L - 1])
    np.testing.assert_allclose(yd, y[:, L - 1], atol=1e-13, rtol=0)


# ---------------------------------------------------------------------------
# sliding window (Motif 3 summary: sliding-window layers, 128-token windows);
# read as: query i sees the W most recent keys, i - W < j <= i
# ---------------------------------------------------------------------------
def _window_mask(N, W):
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    return (j <= i) & (j > i - W)


def test_window_covering_everything_is_plain_causal():
    x = _small(B=2, N=30, H=2, seed=101)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    ref = oracle.prefill(*a, scale=0.125, eps=1e-5)
    for W in (30, 31, 1000):
        np.testing.assert_array_equal(oracle.prefill(*a, scale=0.125, eps=1e-5, window=W), ref)


def test_window_of_one_is_the_row_itself():
    """W = 1: every map attends to its own key only, D = (1 - lambda) V[i] and
    Y = V[i] / rms(V[i]) * gain (eps = 0)."""
    x = _small(B=2, N=9, H=3, seed=102)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=0.0, window=1)
    v = x["v"].numpy()
    ref = v / np.sqrt((v ** 2).mean(-1, keepdims=True)) * x["gain"].numpy()[None, None]
    np.testing.assert_allclose(y, ref, atol=1e-12, rtol=0)


@pytest.mark.parametrize("W", [2, 5, 17])
def test_window_against_masked_sdpa(W):
    """lambda = 0 against torch SDPA with the explicit window mask, then the
    norm; map 2 through D(0) - D(1) against the same masked SDPA."""
    B, N, H = 2, 40, 2
    x = _small(B=B, N=N, H=H, seed=103 + W)
    mask = _window_mask(N, W)
    sdpa = lambda q, k: F.scaled_dot_product_attention(
        q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3), x["v"].permute(0, 2, 1, 3), attn_mask=mask,
        scale=0.125).permute(0, 2, 1, 3)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"])
    y = oracle.prefill(*a, torch.zeros(H, dtype=torch.float64), x["gain"], scale=0.125, eps=1e-5,
                       window=W)
    a1 = sdpa(x["q1"], x["k1"])
    ref = torch.stack([F.rms_norm(a1[:, :, h], (128,), weight=x["gain"][h], eps=1e-5)
                       for h in range(H)], dim=2)
    np.testing.assert_allclose(y, ref.numpy(), atol=1e-12, rtol=0)
    d0 = oracle.prefill(*a, torch.zeros(H, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False, window=W)
    d1 = oracle.prefill(*a, torch.ones(H, dtype=torch.float64), scale=0.125, eps=1e-5,
                        apply_norm=False, window=W)
    np.testing.assert_allclose(d0 - d1, sdpa(x["q2"], x["k2"]).numpy(), atol=1e-12, rtol=0)


def test_window_edges():
    """Row i under window W ignores keys up to i - W and depends on key i - W + 1."""
    N, W, i = 40, 7, 25
    x = _small(B=1, N=N, H=1, seed=107)
    a = lambda k1, v: (x["q1"], x["q2"], k1, x["k2"], v, x["lam"], x["gain"])
    y = oracle.prefill(*a(x["k1"], x["v"]), scale=0.125, eps=1e-5, window=W)
    k1, v = x["k1"].clone(), x["v"].clone()
    k1[:, : i - W + 1] += 4.0
    v[:, : i - W + 1] *= -3.0
    y2 = oracle.prefill(*a(k1, v), scale=0.125, eps=1e-5, window=W)
    np.testing.assert_array_equal(y[0, i], y2[0, i])
    v3 = x["v"].clone()
    v3[:, i - W + 1] *= -3.0
    y3 = oracle.prefill(*a(x["k1"], v3), scale=0.125, eps=1e-5, window=W)
    assert np.abs(y[0, i] - y3[0, i]).max() > 1e-3


def test_decode_window_equals_last_prefill_row():
    B, L, H, W = 3, 50, 2, 11
    x = _small(B=B, N=L, H=H, seed=109)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=1e-5, window=W)
    hm = lambda t: t.permute(0, 2, 1, 3).contiguous()
    kv_len = np.array([L, 5, 23])
    q1 = torch.stack([x["q1"][b, kv_len[b] - 1] for b in range(B)])
    q2 = torch.stack([x["q2"][b, kv_len[b] - 1] for b in range(B)])
    yd = oracle.decode(q1, q2, hm(x["k1"]), hm(x["k2"]), hm(x["v"]), x["lam"], x["gain"],
                       kv_len=kv_len, scale=0.125, eps=1e-5, window=W)
    for b in range(B):
        np.testing.assert_allclose(yd[b], y[b, kv_len[b] - 1], atol=1e-13, rtol=0)


# ---------------------------------------------------------------------------
# rotary position embedding (Motif 2.6B explainer, "The block": RoPE with
# theta = 500,000); read as interleaved pairs within each 64-wide map vector
# ---------------------------------------------------------------------------
def _rope_complex(x, theta):
    """Rotation written as complex multiplication: pair (x[2c], x[2c+1]) is the
    number x[2c] + i x[2c+1], times exp(i n theta^(-2c/d)) at token n.
    x: [B, N, heads, d] float64."""
    B, N, Hh, d = x.shape
    z = torch.view_as_complex(x.reshape(B, N, Hh, d // 2, 2).contiguous())
    n = torch.arange(N, dtype=torch.float64)[:, None]
    freq = theta ** (-2.0 * torch.arange(d // 2, dtype=torch.float64) / d)
    rot = torch.polar(torch.ones(N, d // 2, dtype=torch.float64), n * freq)
    return torch.view_as_real(z * rot[None, :, None, :]).reshape(B, N, Hh, d)


@pytest.mark.parametrize("theta", [500000.0, 10000.0])
def test_rope_equals_complex_rotation_then_plain(theta):
    """The oracle with RoPE equals the plain oracle on Q/K rotated by the
    complex-number form (grouped shape, so both maps and heads are covered)."""
    x = _small(B=2, N=45, H=4, H_N=2, H_V=2, seed=111)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.125, eps=1e-5, rope_theta=theta)
    r = lambda t: _rope_complex(t, theta)
    ref = oracle.prefill(r(x["q1"]), r(x["q2"]), r(x["k1"]), r(x["k2"]), x["v"], x["lam"],
                         x["gain"], scale=0.125, eps=1e-5)
    np.testing.assert_allclose(y, ref, atol=1e-12, rtol=0)


def test_rope_leaves_row_zero_and_depends_on_relative_position():
    """Token 0 is not rotated, so row 0 is unchanged.  And with the same q at
    every position and the same k at every position, the score of (i, j)
    depends only on i - j: with V one-hot over the keys the output row is the
    weight vector, whose log-weights by distance differ between rows only by
    a constant (the row's normaliser)."""
    x = _small(B=1, N=12, H=1, seed=112)
    a = (x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"])
    y0 = oracle.prefill(*a, scale=0.125, eps=1e-5)
    yr = oracle.prefill(*a, scale=0.125, eps=1e-5, rope_theta=500000.0)
    np.testing.assert_allclose(yr[:, 0], y0[:, 0], atol=1e-14, rtol=0)
    assert np.abs(yr[:, 5:] - y0[:, 5:]).max() > 1e-4
    # relative position: constant q and k, V = one-hot of the key index, no
    # norm, lambda = 0: the output of row i is the weight vector over keys,
    # and weight(i, j) depends only on i - j
    N = 12
    q = x["q1"][:, :1].repeat(1, N, 1, 1)
    k = x["k1"][:, :1].repeat(1, N, 1, 1)
    v = torch.zeros(1, N, 1, 128, dtype=torch.float64)
    v[0, torch.arange(N), 0, torch.arange(N)] = 1.0
    w = oracle.prefill(q, q, k, k, v, torch.zeros(1, dtype=torch.float64), scale=0.125, eps=1e-5,
                       apply_norm=False, rope_theta=500000.0)[0, :, 0, :N]
    s = np.log(w + 1e-300)   # log-weights: s(i, j) - logsumexp_i
    for i in range(2, N):
        d = s[i, :i + 1][::-1]          # by distance i - j = 0, 1, ...
        d_prev = s[i - 1, :i][::-1]
        # differences between distances are the same in both rows
        np.testing.assert_allclose(d[1:i] - d[0], d_prev[1:i] - d_prev[0], atol=1e-9, rtol=0)

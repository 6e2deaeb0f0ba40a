"""Pins of the float64 backward oracle to facts outside itself (CPU only).

The backward pass is the gradient of the forward pass of the Motif 2.6B
explainer (section "Differential attention", figure 1) and of its grouped form
(Motif 3 summary, section 2.2); the pages print no backward formulas.  So the
oracle's gradients are checked against:

* central finite differences of the C forward oracle (itself pinned in
  test_oracle_pins.py) on tiny inputs, for every input, grouped head maps,
  token-dependent lambda logits, output-gate logits, the sliding window and
  the rotary embedding included;
* torch autograd through scaled-dot-product attention (with an explicit
  window mask), rms_norm, sigmoid and complex rotation (library routines) at
  the benchmark's head sizes (d = 64, dv = 128);
* exact invariants of the forward: a shift of every key leaves each softmax
  unchanged (sum_j dK_t[j] = 0); scaling Q_t by c and K_t by 1/c leaves the
  scores unchanged (sum Q_t.dQ_t = sum K_t.dK_t); Y is linear in the gain
  (sum_c gain_c dgain_c = sum dY.Y); with eps = 0 the norm makes Y invariant
  to a scaling of V (sum V.dV = 0); a window covering every key, a saturated
  gate and token logits constant per head reduce to the plain call.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

HEAD_MAPS = [(4, 4), (2, 2), (2, 4)]  # (H_N, H_V) with H = 4


def _rand(shape, rng, std=1.0):
    return rng.standard_normal(shape) * std


def _tiny(H_N, H_V, seed=0, B=2, N=4, H=4, d=3, dv=5):
    rng = np.random.default_rng(seed)
    return {
        "q1": _rand((B, N, H, d), rng), "k1": _rand((B, N, H, d), rng),
        "q2": _rand((B, N, H_N, d), rng), "k2": _rand((B, N, H_N, d), rng),
        "v": _rand((B, N, H_V, dv), rng),
        "lam": rng.uniform(0.2, 0.8, H), "gain": 1.0 + _rand((H, dv), rng, 0.3),
        "dy": _rand((B, N, H, dv), rng),
    }


def _loss(x, scale, eps, causal, apply_norm):
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=scale, eps=eps, causal=causal, apply_norm=apply_norm)
    return float(np.sum(x["dy"] * y))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("apply_norm", [True, False])
@pytest.mark.parametrize("H_N,H_V", HEAD_MAPS)
def test_gradients_match_central_differences(causal, apply_norm, H_N, H_V):
    x = _tiny(H_N, H_V, seed=H_N * 10 + H_V)
    scale, eps, h = 0.7, 1e-3, 1e-5
    g = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                x["gain"], x["dy"], scale=scale, eps=eps, causal=causal,
                                apply_norm=apply_norm)
    names = {"q1": "dq1", "q2": "dq2", "k1": "dk1", "k2": "dk2", "v": "dv", "lam": "dlam",
             "gain": "dgain"}
    for key, gname in names.items():
        num = np.zeros_like(x[key])
        flat = x[key].reshape(-1)
        for e in range(flat.size):
            keep = flat[e]
            flat[e] = keep + h
            up = _loss(x, scale, eps, causal, apply_norm)
            flat[e] = keep - h
            down = _loss(x, scale, eps, causal, apply_norm)
            flat[e] = keep
            num.reshape(-1)[e] = (up - down) / (2 * h)
        ref = max(np.max(np.abs(num)), 1e-3)
        err = np.max(np.abs(g[gname] - num))
        assert err <= 1e-6 * ref, (gname, err, ref)


def _torch_forward(t, scale, eps, causal, apply_norm, g_n, g_v):
    """Y through library routines: SDPA per map, repeat_interleave for the
    grouped head maps, rms_norm with the gain as its weight."""
    def sdpa(q, k, v):
        o = F.scaled_dot_product_attention(q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3),
                                           v.permute(0, 2, 1, 3), is_causal=causal, scale=scale)
        return o.permute(0, 2, 1, 3)
    v1 = t["v"].repeat_interleave(g_v, dim=2)
    q2 = t["q2"].repeat_interleave(g_n, dim=2)
    k2 = t["k2"].repeat_interleave(g_n, dim=2)
    d = sdpa(t["q1"], t["k1"], v1) - t["lam"][None, None, :, None] * sdpa(q2, k2, v1)
    if not apply_norm:
        return d
    return F.rms_norm(d, (d.shape[-1],), eps=eps) * t["gain"]


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("apply_norm", [True, False])
def test_gradients_match_torch_autograd(causal, apply_norm):
    rng = np.random.default_rng(3)
    B, N, H, H_N, H_V, d, dv = 1, 40, 4, 2, 2, 64, 128
    x = {
        "q1": _rand((B, N, H, d), rng), "k1": _rand((B, N, H, d), rng),
        "q2": _rand((B, N, H_N, d), rng), "k2": _rand((B, N, H_N, d), rng),
        "v": _rand((B, N, H_V, dv), rng), "lam": rng.uniform(0.2, 0.8, H),
        "gain": 1.0 + _rand((H, dv), rng, 0.1), "dy": _rand((B, N, H, dv), rng),
    }
    scale, eps = 0.125, 1e-5
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=(k != "dy")) for k, v in x.items()}
    y = _torch_forward(t, scale, eps, causal, apply_norm, H // H_N, H // H_V)
    (y * t["dy"]).sum().backward()
    g = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                x["gain"], x["dy"], scale=scale, eps=eps, causal=causal,
                                apply_norm=apply_norm)
    for key in ("q1", "q2", "k1", "k2", "v", "lam", "gain"):
        ref = t[key].grad.numpy() if t[key].grad is not None else np.zeros_like(x[key])
        err = np.max(np.abs(g["d" + key] - ref))
        assert err <= 1e-9 * max(np.max(np.abs(ref)), 1.0), (key, err)


def _medium(seed, causal=True, apply_norm=True, eps=1e-5):
    rng = np.random.default_rng(seed)
    B, N, H, H_N, H_V, d, dv = 2, 23, 4, 2, 4, 16, 8
    x = {
        "q1": _rand((B, N, H, d), rng), "k1": _rand((B, N, H, d), rng),
        "q2": _rand((B, N, H_N, d), rng), "k2": _rand((B, N, H_N, d), rng),
        "v": _rand((B, N, H_V, dv), rng), "lam": rng.uniform(0.2, 0.8, H),
        "gain": 1.0 + _rand((H, dv), rng, 0.2), "dy": _rand((B, N, H, dv), rng),
    }
    g = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                x["gain"], x["dy"], scale=0.3, eps=eps, causal=causal,
                                apply_norm=apply_norm)
    return x, g


@pytest.mark.parametrize("causal", [True, False])
def test_key_shift_invariance(causal):
    _, g = _medium(1, causal)
    for key in ("dk1", "dk2"):
        s = np.sum(g[key], axis=1)  # over keys, per (b, head, c)
        assert np.max(np.abs(s)) <= 1e-10 * max(np.max(np.abs(g[key])), 1.0), key


@pytest.mark.parametrize("causal", [True, False])
def test_query_key_scaling_symmetry(causal):
    x, g = _medium(2, causal)
    for qn, kn in (("q1", "k1"), ("q2", "k2")):
        lhs = np.sum(x[qn] * g["d" + qn], axis=(1, 3))  # per (b, head)
        rhs = np.sum(x[kn] * g["d" + kn], axis=(1, 3))
        assert np.max(np.abs(lhs - rhs)) <= 1e-10 * max(np.max(np.abs(lhs)), 1.0), qn


def test_gain_identity():
    x, g = _medium(3)
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.3, eps=1e-5)
    lhs = np.sum(x["gain"] * g["dgain"], axis=1)          # per head
    rhs = np.sum(x["dy"] * y, axis=(0, 1, 3))
    assert np.max(np.abs(lhs - rhs)) <= 1e-10 * np.max(np.abs(rhs))


def test_v_scaling_invariance_without_eps():
    x, g = _medium(4, eps=0.0)
    s = np.sum(x["v"] * g["dv"])
    assert abs(s) <= 1e-10 * np.sum(np.abs(x["v"] * g["dv"]))


def test_no_norm_means_no_gain_gradient_and_linear_in_dy():
    x, g = _medium(5, apply_norm=False)
    assert np.all(g["dgain"] == 0)
    # without the norm Y is linear in V, so sum V.dV = sum dY.Y
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=0.3, eps=1e-5, apply_norm=False)
    assert abs(np.sum(x["v"] * g["dv"]) - np.sum(x["dy"] * y)) <= 1e-10 * np.sum(np.abs(x["dy"] * y))


# ------------------------------------------------------------------ token lambda, gate, window, RoPE
# Motif 3 summary, section 2.2 (lambda_t = sigma(x_t W^lambda), output gate
# sigma(G_t)), section 2.1 (sliding-window layers); Motif 2.6B explainer,
# "The block" (rotary embedding).  The gradients of these inputs and of the
# rest under them are checked the same ways as above.
EXT_CASES = [  # (lam_logits, gate, window, rope_theta, H_N, H_V, apply_norm)
    (True, True, 0, 0.0, 2, 2, True),
    (False, False, 2, 10.0, 2, 2, True),
    (True, True, 3, 10.0, 1, 2, True),
    (True, True, 2, 10.0, 2, 4, False),
]


def _tiny_ext(lam_logits, gate, H_N, H_V, seed, B=1, N=5, H=4, d=4, dv=3):
    rng = np.random.default_rng(seed)
    x = {
        "q1": _rand((B, N, H, d), rng), "k1": _rand((B, N, H, d), rng),
        "q2": _rand((B, N, H_N, d), rng), "k2": _rand((B, N, H_N, d), rng),
        "v": _rand((B, N, H_V, dv), rng),
        "lam": rng.uniform(0.2, 0.8, H), "gain": 1.0 + _rand((H, dv), rng, 0.3),
        "dy": _rand((B, N, H, dv), rng),
    }
    if lam_logits:
        x["lam_logits"] = _rand((B, N, H), rng, 1.5)
    if gate:
        x["gate"] = _rand((B, N, H, dv), rng, 2.0)
    return x


def _loss_ext(x, scale, eps, apply_norm, window, theta):
    y = oracle.prefill(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                       scale=scale, eps=eps, causal=True, apply_norm=apply_norm,
                       lam_logits=x.get("lam_logits"), gate=x.get("gate"), window=window,
                       rope_theta=theta)
    return float(np.sum(x["dy"] * y))


def _bwd_ext(x, scale, eps, apply_norm, window, theta):
    return oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"],
                                   x["gain"], x["dy"], scale=scale, eps=eps, causal=True,
                                   apply_norm=apply_norm, lam_logits=x.get("lam_logits"),
                                   gate=x.get("gate"), window=window, rope_theta=theta)


@pytest.mark.parametrize("case", EXT_CASES)
def test_extended_gradients_match_central_differences(case):
    lam_logits, gate, window, theta, H_N, H_V, apply_norm = case
    x = _tiny_ext(lam_logits, gate, H_N, H_V, seed=window * 7 + H_N + H_V)
    scale, eps, h = 0.7, 1e-3, 1e-5
    g = _bwd_ext(x, scale, eps, apply_norm, window, theta)
    names = {"q1": "dq1", "q2": "dq2", "k1": "dk1", "k2": "dk2", "v": "dv", "gain": "dgain",
             "lam_logits": "dlam_logits", "gate": "dgate"}
    if not lam_logits:
        names["lam"] = "dlam"
    for key, gname in names.items():
        if key not in x:
            assert np.all(g[gname] == 0), gname
            continue
        num = np.zeros_like(x[key])
        flat = x[key].reshape(-1)
        for e in range(flat.size):
            keep = flat[e]
            flat[e] = keep + h
            up = _loss_ext(x, scale, eps, apply_norm, window, theta)
            flat[e] = keep - h
            down = _loss_ext(x, scale, eps, apply_norm, window, theta)
            flat[e] = keep
            num.reshape(-1)[e] = (up - down) / (2 * h)
        ref = max(np.max(np.abs(num)), 1e-3)
        err = np.max(np.abs(g[gname] - num))
        assert err <= 1e-6 * ref, (gname, err, ref)
    if lam_logits:
        assert np.all(g["dlam"] == 0)   # the per-head lambda is unused


def _torch_forward_ext(t, scale, eps, apply_norm, g_n, g_v, window, theta):
    """Y through library routines: complex multiplication for the rotary
    embedding, SDPA with an explicit boolean mask per map, repeat_interleave
    for the grouped head maps, sigmoid for lambda and the gate, rms_norm."""
    N = t["q1"].shape[1]

    def rope(x):
        if theta <= 0:
            return x
        d = x.shape[-1]
        ang = torch.arange(N, dtype=torch.float64)[:, None] * theta ** (
            -2.0 * torch.arange(d // 2, dtype=torch.float64)[None, :] / d)
        rotor = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
        xc = torch.view_as_complex(x.reshape(*x.shape[:-1], d // 2, 2).contiguous())
        return torch.view_as_real(xc * rotor).reshape(x.shape)

    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    mask = (j <= i) & ((j > i - window) if window > 0 else torch.ones(N, N, dtype=torch.bool))

    def sdpa(q, k, v):
        o = F.scaled_dot_product_attention(q.permute(0, 2, 1, 3), k.permute(0, 2, 1, 3),
                                           v.permute(0, 2, 1, 3), attn_mask=mask, scale=scale)
        return o.permute(0, 2, 1, 3)
    v1 = t["v"].repeat_interleave(g_v, dim=2)
    q2 = rope(t["q2"]).repeat_interleave(g_n, dim=2)
    k2 = rope(t["k2"]).repeat_interleave(g_n, dim=2)
    lam = torch.sigmoid(t["lam_logits"])[..., None]
    d = sdpa(rope(t["q1"]), rope(t["k1"]), v1) - lam * sdpa(q2, k2, v1)
    y = F.rms_norm(d, (d.shape[-1],), eps=eps) * t["gain"] if apply_norm else d
    return torch.sigmoid(t["gate"]) * y


@pytest.mark.parametrize("apply_norm", [True, False])
def test_extended_gradients_match_torch_autograd(apply_norm):
    rng = np.random.default_rng(11)
    B, N, H, H_N, H_V, d, dv, window, theta = 1, 40, 4, 2, 2, 64, 128, 7, 10000.0
    x = {
        "q1": _rand((B, N, H, d), rng), "k1": _rand((B, N, H, d), rng),
        "q2": _rand((B, N, H_N, d), rng), "k2": _rand((B, N, H_N, d), rng),
        "v": _rand((B, N, H_V, dv), rng), "lam": rng.uniform(0.2, 0.8, H),
        "gain": 1.0 + _rand((H, dv), rng, 0.1), "dy": _rand((B, N, H, dv), rng),
        "lam_logits": _rand((B, N, H), rng, 1.5), "gate": _rand((B, N, H, dv), rng, 2.0),
    }
    scale, eps = 0.125, 1e-5
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=(k not in ("dy", "lam")))
         for k, v in x.items()}
    y = _torch_forward_ext(t, scale, eps, apply_norm, H // H_N, H // H_V, window, theta)
    (y * t["dy"]).sum().backward()
    g = _bwd_ext(x, scale, eps, apply_norm, window, theta)
    for key in ("q1", "q2", "k1", "k2", "v", "gain", "lam_logits", "gate"):
        ref = t[key].grad.numpy() if t[key].grad is not None else np.zeros_like(x[key])
        err = np.max(np.abs(g["d" + key] - ref))
        assert err <= 1e-9 * max(np.max(np.abs(ref)), 1.0), (key, err)


def test_window_covering_everything_changes_nothing():
    x, _ = _medium(6)
    a = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                x["dy"], scale=0.3, eps=1e-5)
    b = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                x["dy"], scale=0.3, eps=1e-5, window=x["q1"].shape[1])
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_saturated_gate_is_no_gate():
    """Gate logits of +40: sigma = 1 to double precision, so every gradient is
    the ungated one and the gate's own gradient vanishes."""
    x, g0 = _medium(7)
    gate = np.full(x["dy"].shape, 40.0)
    g = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                x["dy"], scale=0.3, eps=1e-5, gate=gate)
    for k in ("dq1", "dq2", "dk1", "dk2", "dv", "dlam", "dgain"):
        assert np.max(np.abs(g[k] - g0[k])) <= 1e-12 * max(np.max(np.abs(g0[k])), 1.0), k
    assert np.max(np.abs(g["dgate"])) <= 1e-15


def test_constant_token_logits_are_the_per_head_lambda():
    """Logits l_h constant over tokens make lambda_h = sigma(l_h): the other
    gradients equal the per-head call's, and the logits' gradients of head h
    sum to sigma'(l_h) dlambda_h."""
    x, _ = _medium(8)
    B, N, H = x["dy"].shape[:3]
    logit = np.log(x["lam"] / (1.0 - x["lam"]))           # sigma(logit) = lam
    ll = np.broadcast_to(logit, (B, N, H)).copy()
    g0 = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], x["lam"], x["gain"],
                                 x["dy"], scale=0.3, eps=1e-5)
    g = oracle.prefill_backward(x["q1"], x["q2"], x["k1"], x["k2"], x["v"], None, x["gain"],
                                x["dy"], scale=0.3, eps=1e-5, lam_logits=ll)
    for k in ("dq1", "dq2", "dk1", "dk2", "dv", "dgain"):
        assert np.max(np.abs(g[k] - g0[k])) <= 1e-10 * max(np.max(np.abs(g0[k])), 1.0), k
    lhs = g["dlam_logits"].sum(axis=(0, 1))
    rhs = x["lam"] * (1.0 - x["lam"]) * g0["dlam"]
    assert np.max(np.abs(lhs - rhs)) <= 1e-10 * max(np.max(np.abs(rhs)), 1.0)

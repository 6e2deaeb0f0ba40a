"""Pins of the float64 backward oracle to facts outside itself (CPU only).

The backward pass is the gradient of the forward pass of the Motif 2.6B
explainer (section "Differential attention", figure 1) and of its grouped form
(Motif 3 summary, section 2.2); the pages print no backward formulas.  So the
oracle's gradients are checked against:

* central finite differences of the C forward oracle (itself pinned in
  test_oracle_pins.py) on tiny inputs, for every input, grouped head maps
  included;
* torch autograd through scaled-dot-product attention and rms_norm (library
  routines) at the benchmark's head sizes (d = 64, dv = 128);
* exact invariants of the forward: a shift of every key leaves each softmax
  unchanged (sum_j dK_t[j] = 0); scaling Q_t by c and K_t by 1/c leaves the
  scores unchanged (sum Q_t.dQ_t = sum K_t.dK_t); Y is linear in the gain
  (sum_c gain_c dgain_c = sum dY.Y); with eps = 0 the norm makes Y invariant
  to a scaling of V (sum V.dV = 0).
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

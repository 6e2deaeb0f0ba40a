"""Float64 CPU oracle for the gradient of the differential-attention prefill.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the
package's smoke check and the benchmark's CPU-baseline leg may import it.  It
shares no code with the CUDA path.

The pages give the forward pass only (Motif 2.6B explainer, section
"Differential attention" and figure 1; Motif 3 summary, section 2.2, for the
grouped head map, the token-dependent lambda and the output gate, section 2.1
for sliding-window layers; Motif 2.6B explainer, "The block", for the rotary
embedding); the model is trained with it (Motif 2.6B explainer, section "A
schedule for the data"), so the backward pass is the gradient of that forward
pass, nothing more.  This module writes the chain rule out step by step, per
batch entry and signal head, on whole N x N matrices (NumPy matmuls are the
only library steps):

    Q~_t = R Q_t, K~_t = R K_t        (rotary embedding by token position;
                                       R = identity without it)
    Z_t = s Q~_t K~_t^T               (masked entries: -inf; causal: j <= i,
                                       window W: also j > i - W)
    P_t = softmax_rows(Z_t)            A_t = P_t V
    lambda_i = sigma(l_i)              (token logits; else the head's lambda)
    D   = A_1 - lambda_i A_2           (row-wise lambda)
    Yn  = D r gain,  r = (mean_c D^2 + eps)^(-1/2)     (APPLY_NORM; else Yn = D)
    Y   = sigma(G) Yn                  (output gate; else Y = Yn)

Given dY (the gradient of a scalar loss with respect to Y):

    dG        = dY Yn sigma'(G),  dYn = dY sigma(G)       (gate; else dYn = dY)
    dgain_c   = sum_i dYn_ic D_ic r_i
    dD        = r (dYn gain) - (r^3 / dv) D sum_c (dYn gain D)_c   (norm; else dYn)
    dA_1 = dD,  dA_2 = -lambda_i dD,  dlambda_i = -sum_c dD_ic A_2ic
    dl_i = dlambda_i sigma'(l_i)       (token logits; else dlambda[h] = sum_i dlambda_i)
    per map:  dP_t = dA_t V^T,  Delta_t = rowsum(dA_t A_t),
              dZ_t = P_t (dP_t - Delta_t),
              dQ~_t = s dZ_t K~_t,  dK~_t = s dZ_t^T Q~_t,  dV += P_t^T dA_t
    dQ_t = R^T dQ~_t,  dK_t = R^T dK~_t   (the inverse rotation)

Grouped head maps accumulate: noise head n(h) = h // (H / H_N) collects the
dQ_2 / dK_2 of all its signal heads, V head h // (H / H_V) the dV.

Pins (tests/test_oracle_bwd_pins.py): central finite differences of the C
forward oracle on tiny inputs (every input, grouped heads, token lambda,
gate, window and rotary embedding included); torch autograd through
scaled-dot-product attention, rms_norm, sigmoid and complex rotation
(library routines) at the benchmark's head sizes; exact invariants of the
forward (key-shift invariance, the Q/K scaling symmetry, the gain identity).
"""
import numpy as np


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _softmax_rows(z):
    """Row softmax of z (entries of -inf get weight 0; every row has a finite entry)."""
    m = np.max(z, axis=1, keepdims=True)
    w = np.exp(z - m)
    return w / np.sum(w, axis=1, keepdims=True)


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _rotate(x, theta, sign=1.0):
    """Rotary embedding of x [N, d] by token position n: the pair
    (x[2c], x[2c+1]) turned by sign * n * theta^(-2c/d)."""
    N, d = x.shape
    ang = sign * np.arange(N)[:, None] * theta ** (-2.0 * np.arange(d // 2)[None, :] / d)
    cs, sn = np.cos(ang), np.sin(ang)
    y = np.empty_like(x)
    y[:, 0::2] = x[:, 0::2] * cs - x[:, 1::2] * sn
    y[:, 1::2] = x[:, 0::2] * sn + x[:, 1::2] * cs
    return y


def prefill_backward(q1, q2, k1, k2, v, lam, gain, dy, *, scale, eps, causal=True,
                     apply_norm=True, lam_logits=None, gate=None, window=0, rope_theta=0.0):
    """Gradients of sum(dy * Y) for the prefill Y = diffattn(q1, q2, k1, k2, v).

    q1, k1: [B, N, H, d]; q2, k2: [B, N, H_N, d]; v: [B, N, H_V, dv];
    lam: [H] (unused, may be None, with lam_logits); gain: [H, dv] or None
    (then 1); dy: [B, N, H, dv]; lam_logits: [B, N, H] or None; gate:
    [B, N, H, dv] or None; window: 0 or W (causal only); rope_theta: 0 or
    the rotary base.
    Returns a dict of float64 arrays: dq1, dk1 [B, N, H, d]; dq2, dk2
    [B, N, H_N, d]; dv [B, N, H_V, dv]; dlam [H] (zero with lam_logits);
    dgain [H, dv] (zero when the norm is off, since the gain is then
    unused); dlam_logits [B, N, H] and dgate [B, N, H, dv] (zero when the
    input is not given).
    """
    q1, q2, k1, k2, v, lam, gain, dy, lam_logits, gate = map(
        _f64, (q1, q2, k1, k2, v, lam, gain, dy, lam_logits, gate))
    B, N, H, d = q1.shape
    H_N, H_V, dv = q2.shape[2], v.shape[2], v.shape[3]
    assert k1.shape == q1.shape and k2.shape == q2.shape and v.shape[:2] == (B, N)
    assert dy.shape == (B, N, H, dv)
    assert lam_logits is not None or lam.shape == (H,)
    assert H % H_N == 0 and H % H_V == 0
    assert window == 0 or causal
    if gain is None:
        gain = np.ones((H, dv))
    g_n, g_v = H // H_N, H // H_V

    grads = {
        "dq1": np.zeros_like(q1), "dk1": np.zeros_like(k1),
        "dq2": np.zeros_like(q2), "dk2": np.zeros_like(k2),
        "dv": np.zeros_like(v), "dlam": np.zeros(H), "dgain": np.zeros((H, dv)),
        "dlam_logits": np.zeros((B, N, H)), "dgate": np.zeros((B, N, H, dv)),
    }
    # Visible keys: j <= i when causal (and j > i - W under a window), all otherwise.
    i_idx, j_idx = np.arange(N)[:, None], np.arange(N)[None, :]
    visible = (j_idx <= i_idx) if causal else np.ones((N, N), dtype=bool)
    if window > 0:
        visible = visible & (j_idx > i_idx - window)
    rot = (lambda x: _rotate(x, rope_theta)) if rope_theta > 0 else (lambda x: x)
    unrot = (lambda x: _rotate(x, rope_theta, -1.0)) if rope_theta > 0 else (lambda x: x)

    for b in range(B):
        for h in range(H):
            n, hv = h // g_n, h // g_v
            Q = (rot(q1[b, :, h]), rot(q2[b, :, n]))
            K = (rot(k1[b, :, h]), rot(k2[b, :, n]))
            V = v[b, :, hv]
            # forward, kept for the chain rule
            P, A = [], []
            for t in range(2):
                z = np.where(visible, scale * (Q[t] @ K[t].T), -np.inf)
                P.append(_softmax_rows(z))
                A.append(P[t] @ V)
            lam_row = (_sigmoid(lam_logits[b, :, h]) if lam_logits is not None
                       else np.full(N, lam[h]))[:, None]
            D = A[0] - lam_row * A[1]
            if apply_norm:
                r = 1.0 / np.sqrt(np.mean(D * D, axis=1, keepdims=True) + eps)
                Yn = D * r * gain[h]
            else:
                Yn = D
            dY = dy[b, :, h]
            # the output gate
            if gate is not None:
                sg = _sigmoid(gate[b, :, h])
                grads["dgate"][b, :, h] = dY * Yn * sg * (1.0 - sg)
                dYn = dY * sg
            else:
                dYn = dY
            # the norm and gain
            if apply_norm:
                grads["dgain"][h] += np.sum(dYn * D * r, axis=0)
                G = dYn * gain[h]
                dD = r * G - (r ** 3 / dv) * D * np.sum(G * D, axis=1, keepdims=True)
            else:
                dD = dYn
            # the subtraction
            dA = (dD, -lam_row * dD)
            dlam_row = -np.sum(dD * A[1], axis=1)
            if lam_logits is not None:
                s = _sigmoid(lam_logits[b, :, h])
                grads["dlam_logits"][b, :, h] = dlam_row * s * (1.0 - s)
            else:
                grads["dlam"][h] += np.sum(dlam_row)
            # each softmax map
            for t, (dq, dk) in enumerate((("dq1", "dk1"), ("dq2", "dk2"))):
                dP = dA[t] @ V.T
                delta = np.sum(dA[t] * A[t], axis=1, keepdims=True)
                dZ = P[t] * (dP - delta)
                head = h if t == 0 else n
                grads[dq][b, :, head] += unrot(scale * (dZ @ K[t]))
                grads[dk][b, :, head] += unrot(scale * (dZ.T @ Q[t]))
                grads["dv"][b, :, hv] += P[t].T @ dA[t]
    if not apply_norm:
        grads["dgain"][:] = 0.0
    return grads

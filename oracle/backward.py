"""Float64 CPU oracle for the gradient of the differential-attention prefill.

TEST INFRASTRUCTURE ONLY, like the rest of this package: only the tests, the
package's smoke check and the benchmark's CPU-baseline leg may import it.  It
shares no code with the CUDA path.

The pages give the forward pass only (Motif 2.6B explainer, section
"Differential attention" and figure 1; Motif 3 summary, section 2.2, for the
grouped head map); the model is trained with it (Motif 2.6B explainer,
section "A schedule for the data"), so the backward pass is the gradient of
that forward pass, nothing more.  This module writes the chain
rule out step by step, per batch entry and signal head, on whole N x N
matrices (NumPy matmuls are the only library steps):

    Z_t = s Q_t K_t^T                  (masked entries: -inf)
    P_t = softmax_rows(Z_t)            A_t = P_t V
    D   = A_1 - lambda A_2
    Y   = D r gain,  r = (mean_c D^2 + eps)^(-1/2)     (APPLY_NORM; else Y = D)

Given dY (the gradient of a scalar loss with respect to Y):

    dgain_c   = sum_i dY_ic D_ic r_i
    dD        = r (dY gain) - (r^3 / dv) D sum_c (dY gain D)_c   (norm; else dY)
    dA_1 = dD,  dA_2 = -lambda dD,   dlambda = -sum dD A_2
    per map:  dP_t = dA_t V^T,  Delta_t = rowsum(dA_t A_t),
              dZ_t = P_t (dP_t - Delta_t),
              dQ_t = s dZ_t K_t,  dK_t = s dZ_t^T Q_t,  dV += P_t^T dA_t

Grouped head maps accumulate: noise head n(h) = h // (H / H_N) collects the
dQ_2 / dK_2 of all its signal heads, V head h // (H / H_V) the dV.

Pins (tests/test_oracle_bwd_pins.py): central finite differences of the C
forward oracle on tiny inputs (every input, grouped heads included); torch
autograd through scaled-dot-product attention and rms_norm (library
routines) at the benchmark's head sizes; exact invariants of the forward
(key-shift invariance, the Q/K scaling symmetry, the gain identity).
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


def prefill_backward(q1, q2, k1, k2, v, lam, gain, dy, *, scale, eps, causal=True,
                     apply_norm=True):
    """Gradients of sum(dy * Y) for the prefill Y = diffattn(q1, q2, k1, k2, v).

    q1, k1: [B, N, H, d]; q2, k2: [B, N, H_N, d]; v: [B, N, H_V, dv];
    lam: [H]; gain: [H, dv] or None (then 1); dy: [B, N, H, dv].
    Returns a dict of float64 arrays: dq1, dk1 [B, N, H, d]; dq2, dk2
    [B, N, H_N, d]; dv [B, N, H_V, dv]; dlam [H]; dgain [H, dv] (zero when
    the norm is off, since the gain is then unused).
    """
    q1, q2, k1, k2, v, lam, gain, dy = map(_f64, (q1, q2, k1, k2, v, lam, gain, dy))
    B, N, H, d = q1.shape
    H_N, H_V, dv = q2.shape[2], v.shape[2], v.shape[3]
    assert k1.shape == q1.shape and k2.shape == q2.shape and v.shape[:2] == (B, N)
    assert dy.shape == (B, N, H, dv) and lam.shape == (H,)
    assert H % H_N == 0 and H % H_V == 0
    if gain is None:
        gain = np.ones((H, dv))
    g_n, g_v = H // H_N, H // H_V

    grads = {
        "dq1": np.zeros_like(q1), "dk1": np.zeros_like(k1),
        "dq2": np.zeros_like(q2), "dk2": np.zeros_like(k2),
        "dv": np.zeros_like(v), "dlam": np.zeros(H), "dgain": np.zeros((H, dv)),
    }
    # Visible keys: j <= i when causal, all otherwise.
    visible = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)

    for b in range(B):
        for h in range(H):
            n, hv = h // g_n, h // g_v
            Q = (q1[b, :, h], q2[b, :, n])
            K = (k1[b, :, h], k2[b, :, n])
            V = v[b, :, hv]
            # forward, kept for the chain rule
            P, A = [], []
            for t in range(2):
                z = np.where(visible, scale * (Q[t] @ K[t].T), -np.inf)
                P.append(_softmax_rows(z))
                A.append(P[t] @ V)
            D = A[0] - lam[h] * A[1]
            dY = dy[b, :, h]
            # the norm and gain
            if apply_norm:
                r = 1.0 / np.sqrt(np.mean(D * D, axis=1, keepdims=True) + eps)
                grads["dgain"][h] += np.sum(dY * D * r, axis=0)
                G = dY * gain[h]
                dD = r * G - (r ** 3 / dv) * D * np.sum(G * D, axis=1, keepdims=True)
            else:
                dD = dY
            # the subtraction
            dA = (dD, -lam[h] * dD)
            grads["dlam"][h] += -np.sum(dD * A[1])
            # each softmax map
            for t, (dq, dk) in enumerate((("dq1", "dk1"), ("dq2", "dk2"))):
                dP = dA[t] @ V.T
                delta = np.sum(dA[t] * A[t], axis=1, keepdims=True)
                dZ = P[t] * (dP - delta)
                head = h if t == 0 else n
                grads[dq][b, :, head] += scale * (dZ @ K[t])
                grads[dk][b, :, head] += scale * (dZ.T @ Q[t])
                grads["dv"][b, :, hv] += P[t].T @ dA[t]
    if not apply_norm:
        grads["dgain"][:] = 0.0
    return grads

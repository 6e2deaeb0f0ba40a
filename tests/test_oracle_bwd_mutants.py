"""The backward pins must catch plausible mistakes (CPU only).

Each case loads a copy of oracle/backward.py with one planted mistake, swaps
it in for the real function, and checks that at least one pin of
tests/test_oracle_bwd_pins.py fails.  Mistakes are planted in the oracle
only, never in the CUDA path.
"""
import importlib.util
import os

import pytest

import oracle
from . import test_oracle_bwd_pins as pins
from .test_oracle_mutants import _run_pin

SRC = os.path.join(os.path.dirname(oracle.__file__), "backward.py")

MUTANTS = {
    "delta_dropped": ("dZ = P[t] * (dP - delta)", "dZ = P[t] * dP"),
    "noise_gradient_sign": ("dA = (dD, -lam_row * dD)", "dA = (dD, lam_row * dD)"),
    "dk_not_transposed": ("(dZ.T @ Q[t])", "(dZ @ Q[t])"),
    "norm_second_term_dropped": (
        "dD = r * G - (r ** 3 / dv) * D * np.sum(G * D, axis=1, keepdims=True)", "dD = r * G"),
    "norm_second_term_r_squared": ("(r ** 3 / dv)", "(r ** 2 / dv)"),
    "dq_scale_dropped": ("unrot(scale * (dZ @ K[t]))", "unrot((dZ @ K[t]))"),
    "dv_from_map1_weights_only": ('grads["dv"][b, :, hv] += P[t].T @ dA[t]',
                                  'grads["dv"][b, :, hv] += P[0].T @ dA[t]'),
    "dlam_sign": ("dlam_row = -np.sum(dD * A[1], axis=1)", "dlam_row = np.sum(dD * A[1], axis=1)"),
    "dlam_uses_map1": ("dlam_row = -np.sum(dD * A[1], axis=1)",
                       "dlam_row = -np.sum(dD * A[0], axis=1)"),
    "dgain_without_r": ("np.sum(dYn * D * r, axis=0)", "np.sum(dYn * D, axis=0)"),
    "gain_not_in_dD": ("G = dYn * gain[h]", "G = dYn"),
    "noise_head_modulo": ("head = h if t == 0 else n", "head = h if t == 0 else h % H_N"),
    "v_head_modulo": ("n, hv = h // g_n, h // g_v", "n, hv = h // g_n, h % H_V"),
    "mask_not_applied": ("np.where(visible, scale * (Q[t] @ K[t].T), -np.inf)",
                         "scale * (Q[t] @ K[t].T)"),
    "delta_from_map1": ("delta = np.sum(dA[t] * A[t], axis=1, keepdims=True)",
                        "delta = np.sum(dA[t] * A[0], axis=1, keepdims=True)"),
    # token-dependent lambda, output gate, sliding window, rotary embedding
    "gate_derivative_dropped": ("dY * Yn * sg * (1.0 - sg)", "dY * Yn * sg"),
    "gate_grad_before_norm": ("dY * Yn * sg * (1.0 - sg)", "dY * D * sg * (1.0 - sg)"),
    "gate_not_in_dYn": ("dYn = dY * sg", "dYn = dY"),
    "lam_logit_derivative_dropped": ("dlam_row * s * (1.0 - s)", "dlam_row * s"),
    "lam_logit_not_squashed": ("(_sigmoid(lam_logits[b, :, h]) if", "(lam_logits[b, :, h] if"),
    "window_one_key_too_many": ("(j_idx > i_idx - window)", "(j_idx >= i_idx - window)"),
    "rope_gradient_not_rotated_back": ("_rotate(x, rope_theta, -1.0)", "x"),
    "rope_gradient_rotated_forward": ("_rotate(x, rope_theta, -1.0)", "_rotate(x, rope_theta)"),
    "rope_sin_sign": ("y[:, 1::2] = x[:, 0::2] * sn + x[:, 1::2] * cs",
                      "y[:, 1::2] = -x[:, 0::2] * sn + x[:, 1::2] * cs"),
}

PIN_TESTS = [getattr(pins, n) for n in sorted(dir(pins)) if n.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_bwd_pins_catch_mutant(name, tmp_path):
    a, b = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(a) == 1, f"mutation anchor for {name} not found once in the oracle source"
    mpath = tmp_path / "backward_mutant.py"
    mpath.write_text(src.replace(a, b))
    spec = importlib.util.spec_from_file_location("backward_mutant", mpath)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    saved = oracle.prefill_backward
    oracle.prefill_backward = mod.prefill_backward
    failed = []
    try:
        for f in PIN_TESTS:
            try:
                _run_pin(f)
            except (AssertionError, ValueError):
                failed.append(f.__name__)
    finally:
        oracle.prefill_backward = saved
    assert failed, f"no pin caught the planted mistake {name!r}"

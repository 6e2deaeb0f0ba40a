"""The oracle's pins must catch plausible mistakes (CPU only).

Each case compiles a copy of the oracle's C source with one planted mistake
into a temporary directory, swaps it in for the real oracle, and checks that at
least one pin of tests/test_oracle_pins.py fails.  Mistakes are planted in the
oracle only, never in the CUDA path.
"""
import inspect
import os
import subprocess

import pytest

import oracle
from . import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "diffattn_oracle.c")

MUTANTS = {
    "eps_outside_sqrt": ("double r = 1.0 / sqrt(ss / (double)dv + eps);",
                         "double r = 1.0 / (sqrt(ss / (double)dv) + eps);"),
    "plus_instead_of_minus": ("out[c] = a1[c] / l1 - lambda * (a2[c] / l2);",
                              "out[c] = a1[c] / l1 + lambda * (a2[c] / l2);"),
    "diagonal_excluded": ("const int64_t nkeys = causal ? i + 1 : N;",
                          "const int64_t nkeys = causal ? (i > 0 ? i : 1) : N;"),
    "scale_dropped": ("w[j] = scale * dot;", "w[j] = dot;"),
    "noise_head_modulo": ("const int64_t n = h / g, hv = h / gv;",
                          "const int64_t n = h % H_N, hv = h / gv;"),
    "v_head_modulo": ("const int64_t n = h / g, hv = h / gv;",
                      "const int64_t n = h / g, hv = h % H_V;"),
    "map2_uses_map1_weights": ("a2[c] += w2[j] * vj[c];", "a2[c] += w1[j] * vj[c];"),
    "mean_over_dv_minus_1": ("ss / (double)dv", "ss / (double)(dv - 1)"),
    "gain_of_head0": ("lam, gain ? gain + h * dv : NULL, eps, apply_norm, gate,",
                      "lam, gain ? gain : NULL, eps, apply_norm, gate,"),
    "decode_drops_last_key": ("const int64_t nkeys = kv_len ? kv_len[b] : L;",
                              "const int64_t nkeys = kv_len ? kv_len[b] - (kv_len[b] > 1) : L;"),
    "map2_divided_by_l1": ("lambda * (a2[c] / l2)", "lambda * (a2[c] / l1)"),
    "logistic_sign_flipped": ("return 1.0 / (1.0 + exp(-x));", "return 1.0 / (1.0 + exp(x));"),
    "token_lambda_transposed": ("logistic(lambda_logit[row])",
                                "logistic(lambda_logit[(b * H + h) * N + i])"),
    "token_lambda_of_head0": ("logistic(lambda_logit[row])",
                              "logistic(lambda_logit[row - h])"),
    "gate_column_zero": ("logistic(gate_logit[c]) * out[c]", "logistic(gate_logit[0]) * out[c]"),
    "gate_also_before_norm": (
        "    for (int64_t c = 0; c < dv; ++c) out[c] = a1[c] / l1 - lambda * (a2[c] / l2);\n",
        "    for (int64_t c = 0; c < dv; ++c) out[c] = a1[c] / l1 - lambda * (a2[c] / l2);\n"
        "    if (gate_logit) for (int64_t c = 0; c < dv; ++c) out[c] *= logistic(gate_logit[c]);\n"),
    "decode_gate_row_of_batch": ("gate_logit ? gate_logit + r * dv : NULL",
                                 "gate_logit ? gate_logit + b * dv : NULL"),
    "decode_token_lambda_of_head": ("logistic(lambda_logit[r])", "logistic(lambda_logit[h])"),
    "window_one_key_too_many": ("? i + 1 - window : 0;", "? i - window : 0;"),
    "decode_window_one_key_too_few": ("? nkeys - window : 0;", "? nkeys - window + 1 : 0;"),
    "rope_sin_sign": ("yr[2 * c] = xr[2 * c] * cs - xr[2 * c + 1] * sn;",
                      "yr[2 * c] = xr[2 * c] * cs + xr[2 * c + 1] * sn;"),
    "rope_frequency_exponent": ("pow(theta, -2.0 * (double)c / (double)d)",
                                "pow(theta, -1.0 * (double)c / (double)d)"),
    # (A uniform shift of every position is not a mistake: attention with
    # rotary embeddings depends on relative positions only.)
    "rope_keys_not_rotated": ("q1 = rq1; k1 = rk1; q2 = rq2; k2 = rk2;", "q1 = rq1; q2 = rq2;"),
}

PIN_TESTS = [f for name, f in sorted(vars(pins).items())
             if name.startswith("test_") and inspect.isfunction(f)]


def _run_pin(f):
    """Run a pin over every combination of its pytest parametrize values."""
    import itertools
    grids = []
    for mark in getattr(f, "pytestmark", []):
        if mark.name == "parametrize":
            names, values = mark.args[0], mark.args[1]
            names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
            grids.append([dict(zip(names, v if len(names) > 1 else (v,))) for v in values])
    for combo in itertools.product(*grids) if grids else [()]:
        kw = {}
        for part in combo:
            kw.update(part)
        f(**kw)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    a, b = MUTANTS[name]
    src = open(SRC).read()
    assert a in src, f"mutation anchor for {name} not found in the oracle source"
    mpath = tmp_path / "m.c"
    mpath.write_text(src.replace(a, b))
    so = tmp_path / "libm.so"
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-o",
                    str(so), str(mpath), "-lm"], check=True)
    saved = oracle._LIB
    oracle._LIB = oracle.load(str(so))
    failed = []
    try:
        for f in PIN_TESTS:
            try:
                _run_pin(f)
            except (AssertionError, ValueError):
                failed.append(f.__name__)
    finally:
        oracle._LIB = saved
    assert failed, f"no pin caught the planted mistake {name!r}"

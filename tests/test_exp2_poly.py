"""The software exp2 of the prefill and backward kernels (CPU emulation of its exact steps).

The kernels compute part of the softmax exponentials as 2^x = 2^n * p(f)
(range reduction x = n + f by the 1.5*2^23 magic-number add, a degree-3
polynomial p fitted by Remez exchange, 2^n added into the exponent bits).
These tests check that the constants in the CUDA source are the ones the
committed fit script produces and that the float32 / int32 emulation of the
whole sequence stays within 1e-4 relative of exp2 over the inputs the
softmax feeds it (x <= 2^8 after the stale-max threshold, down to -inf).
"""
import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "differential_attention_07_b200", "csrc")


def _kernel_constants():
    src = open(os.path.join(CSRC, "sm100_ptx.cuh")).read()
    c = {}
    for k in range(4):
        m = re.search(rf"constexpr float EXP2_C{k} = (0x[0-9a-fA-Fp.+-]+)f;", src)
        assert m, f"EXP2_C{k} not found"
        c[k] = np.float32(float.fromhex(m.group(1)))
    return [c[k] for k in range(4)]


def _fit_constants():
    sys.path.insert(0, CSRC)
    try:
        import fit_exp2_poly
        return fit_exp2_poly.coefficients(), fit_exp2_poly
    finally:
        sys.path.remove(CSRC)


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _soft_exp2(x, c):
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    rnd = np.float32(12582912.0)
    j = (x + rnd).astype(np.float32)
    n = (j - rnd).astype(np.float32)
    f = _fma32(n, np.float32(-1.0) * np.ones_like(n), x)
    p = _fma32(np.full_like(f, c[3]), f, np.full_like(f, c[2]))
    p = _fma32(p, f, np.full_like(f, c[1]))
    p = _fma32(p, f, np.full_like(f, c[0]))
    bits = p.view(np.int32) + (j.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_kernel_constants_match_fit_script():
    fitted, mod = _fit_constants()
    assert _kernel_constants() == fitted
    assert mod.float32_max_rel_err(fitted) < 8e-5


def test_soft_exp2_relative_error():
    c = _kernel_constants()
    x = np.concatenate([np.linspace(-124.0, 8.0, 2_000_001, dtype=np.float32),
                        np.array([0.0, -0.5, 0.5, -1.0, 1.0, 8.0, -20.25], dtype=np.float32)])
    y = _soft_exp2(x, c).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(y / ref - 1.0)) < 1e-4


def test_soft_exp2_underflow_and_masked():
    c = _kernel_constants()
    x = np.array([-np.inf, -1e30, -200.0, -126.0, -125.0], dtype=np.float32)
    y = _soft_exp2(x, c)
    assert np.all(np.isfinite(y)) and np.all(y >= 0) and np.all(y < 1e-37)
    # fp16 P: all of these round to zero
    assert np.all(y.astype(np.float16) == 0)


def test_fit_script_runs():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "fit_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    assert "EXP2_C3" in out and "max relative error" in out

"""Fit the polynomial of the software exp2 used by the prefill softmax.

Method: Cody-Waite style range reduction x = n + f with n = rint(x), so
f lies in [-1/2, 1/2]; 2^x = 2^n * 2^f, where 2^n goes into the exponent field
by an integer add and 2^f is a degree-3 polynomial.  The coefficients minimise
the maximum RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2]; they are found by
the Remez exchange algorithm (solve for equi-oscillating error on 5 reference
points, move the references to the error's extrema, repeat), then rounded to
float32.

    python differential_attention_07_b200/csrc/fit_exp2_poly.py

prints the coefficients (as C float literals) and the float32 max relative
error; the values are pasted into prefill_sm100.cu (EXP2_C0..EXP2_C3), and a
CPU test checks that the two agree.
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def _solve(ref):
    # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equi-oscillation)
    n = len(ref)
    A = np.zeros((n, n))
    for i, x in enumerate(ref):
        A[i, :DEG + 1] = [x ** k for k in range(DEG + 1)]
        A[i, DEG + 1] = -((-1) ** i) * 2.0 ** x
    sol = np.linalg.solve(A, 2.0 ** ref)
    return sol[:DEG + 1], sol[DEG + 1]


def _rel_err(c, x):
    return np.polyval(c[::-1], x) / 2.0 ** x - 1.0


def fit(iters=30):
    k = np.arange(DEG + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (DEG + 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(ref)
        e = _rel_err(c, grid)
        # extrema: endpoints plus sign-change-bounded local maxima of |e|
        s = np.sign(e)
        idx = [0]
        for i in range(1, len(grid)):
            if s[i] != s[idx[-1]]:
                idx.append(i)
            elif abs(e[i]) > abs(e[idx[-1]]):
                idx[-1] = i
        idx = np.array(idx)
        while len(idx) > DEG + 2:  # drop the smallest end extremum
            if abs(e[idx[0]]) < abs(e[idx[-1]]):
                idx = idx[1:]
            else:
                idx = idx[:-1]
        if len(idx) < DEG + 2:
            break
        ref = grid[idx]
    return c


def float32_max_rel_err(c32, n=400001):
    """Max relative error of the float32 Horner evaluation (fma rounding
    emulated in float64 then rounded to float32) over [-1/2, 1/2]."""
    x = np.linspace(LO, HI, n).astype(np.float32)
    acc = np.float32(c32[DEG]) * np.ones_like(x)
    for k in range(DEG - 1, -1, -1):
        acc = (acc.astype(np.float64) * x.astype(np.float64) + np.float64(c32[k])).astype(np.float32)
    return float(np.max(np.abs(acc.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)))


def coefficients():
    c = fit()
    return [np.float32(v) for v in c]


if __name__ == "__main__":
    c32 = coefficients()
    for k, v in enumerate(c32):
        print(f"EXP2_C{k} = {float(v).hex()}  ({float(v):.9g}f)")
    print(f"float32 max relative error on [-1/2, 1/2]: {float32_max_rel_err(c32):.3e}")

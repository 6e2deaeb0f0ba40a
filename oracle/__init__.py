"""Float64 CPU oracle for the differential-attention forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
benchmark's CPU-baseline leg may import this module.  It shares no code with
the CUDA path (different language, different build, no common helpers) and the
CUDA path never calls it.

The arithmetic lives in ``diffattn_oracle.c`` (plain loops, float64, no tiling,
no online softmax); this module only marshals NumPy arrays.  What it computes:

    Y = Norm( softmax(s Q1 K1^T) V - lambda * softmax(s Q2 K2^T) V )

per batch, signal head and query row, with causal masking (diagonal included),
the noise map of signal head h taken from noise head h // g, and Norm the
per-head RMS normalisation with gain (Motif 2.6B explainer, section
"Differential attention" and figure 1; Motif 3 summary, section 2.2).

With token-dependent lambda logits and output-gate logits (Motif 3 summary,
section 2.2) lambda becomes sigma(logit) per (b, i, h), and the output is
multiplied element-wise by sigma(G) after the norm.

Pins (tests/test_oracle_pins.py): lambda = 0 against torch's scaled-dot-product
attention plus torch's rms_norm; map 2 against the same library routine; the
Q2=Q1, K2=K1 reduction; softmax rows summing to one; causal independence;
SciPy-softmax brute force for N <= 8; the row-0 closed form; exact scale
invariance; the grouped head map against repeat_interleave; decode against the
last prefill row; a hand-derived golden example; for the token-dependent
lambda and the gate: saturated logits reducing to SDPA, sigma(0) = 1/2,
the lambda logits' indexing against SDPA, the gate as the element-wise last
step, decode against the last gated prefill row.  The backward pass
(``oracle/backward.py``) has pins of its own (tests/test_oracle_bwd_pins.py).
Parity unpinned: the choice of
RMS normalisation for the pages' "GroupNorm" and the grouped V layout are
readings of the pages, not facts the pages fix.
"""
import ctypes

import numpy as np

from . import build as _build
from .backward import prefill_backward  # noqa: F401  (gradient of prefill, float64 NumPy)

_LIB = None


def load(path):
    """Load an oracle shared library from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    ip = ctypes.POINTER(ctypes.c_int64)
    i64 = ctypes.c_int64
    lib.diffattn_oracle_prefill.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64,
                                            i64, i64, dp, dp, dp, dp, ctypes.c_double,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_int, i64,
                                            ctypes.c_double, ip, i64, dp]
    lib.diffattn_oracle_prefill.restype = ctypes.c_int
    lib.diffattn_oracle_decode.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64,
                                           ip, dp, dp, dp, dp, ctypes.c_double, ctypes.c_double,
                                           ctypes.c_int, i64, dp]
    lib.diffattn_oracle_decode.restype = ctypes.c_int
    lib.diffattn_oracle_softmax_row.argtypes = [dp, dp, i64, i64, ctypes.c_double, dp]
    lib.diffattn_oracle_softmax_row.restype = None
    lib.diffattn_oracle_threads.argtypes = []
    lib.diffattn_oracle_threads.restype = ctypes.c_int
    return lib


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = load(_build.build())
    return _LIB


def _f64(x):
    """Widen to a contiguous float64 NumPy array (torch tensors accepted)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _dp(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(_lib().diffattn_oracle_threads())


def softmax_row(q, k, scale):
    """Normalised softmax weights of one query row q [d] against keys k [n, d]."""
    q, k = _f64(q), _f64(k)
    out = np.empty(k.shape[0], dtype=np.float64)
    _lib().diffattn_oracle_softmax_row(_dp(q), _dp(k), k.shape[0], k.shape[1], float(scale),
                                       _dp(out))
    return out


def prefill(q1, q2, k1, k2, v, lam, gain=None, *, scale, eps, causal=True, apply_norm=True,
            rows=None, lam_logits=None, gate=None, window=0, rope_theta=0.0):
    """Prefill oracle.

    q1, k1: [B, N, H, d]; q2, k2: [B, N, H_N, d]; v: [B, N, H_V, dv];
    lam: [H] (ignored, may be None, when lam_logits is given); gain: [H, dv]
    or None; lam_logits: token-dependent lambda logits [B, N, H] or None;
    gate: output-gate logits [B, N, H, dv] or None; window: 0, or a causal
    sliding window of that many keys (query i sees keys i-W < j <= i);
    rope_theta: 0, or the base of the rotary embedding applied to Q1, K1,
    Q2, K2 by token position (interleaved pairs).  Returns float64
    [B, N, H, dv].  rows: None (all rows) or an int array [R, 3] of
    (b, i, h); then only those rows are computed and the rest is NaN.
    """
    q1, q2, k1, k2, v = map(_f64, (q1, q2, k1, k2, v))
    lam, gain, lam_logits, gate = map(_f64, (lam, gain, lam_logits, gate))
    B, N, H, d = q1.shape
    H_N, H_V, dv = q2.shape[2], v.shape[2], v.shape[3]
    assert k1.shape == q1.shape and k2.shape == q2.shape and v.shape[:2] == (B, N)
    assert (gain is None or gain.shape == (H, dv))
    assert lam_logits is None or lam_logits.shape == (B, N, H)
    assert gate is None or gate.shape == (B, N, H, dv)
    if lam_logits is None:
        assert lam is not None and lam.shape == (H,)
    out = np.full((B, N, H, dv), np.nan, dtype=np.float64)
    rp, nrows = None, 0
    if rows is not None:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        rp, nrows = rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), rows.shape[0]
    rc = _lib().diffattn_oracle_prefill(_dp(q1), _dp(q2), _dp(k1), _dp(k2), _dp(v), B, N, H,
                                        H_N, H_V, d, dv, _dp(lam), _dp(gain), _dp(lam_logits),
                                        _dp(gate), float(scale),
                                        float(eps), int(bool(causal)), int(bool(apply_norm)),
                                        int(window), float(rope_theta), rp, nrows, _dp(out))
    if rc != 0:
        raise ValueError("oracle prefill: invalid arguments")
    return out


def decode(q1, q2, k1, k2, v, lam, gain=None, *, kv_len=None, scale, eps, apply_norm=True,
           lam_logits=None, gate=None, window=0):
    """Single-query decode oracle.

    q1, q2: [B, H, d]; k1, k2: [B, H, L, d]; v: [B, H, L, dv]; kv_len: [B] or
    None; lam [H] (or None with lam_logits); gain [H, dv] or None;
    lam_logits: [B, H] or None; gate: [B, H, dv] or None; window: 0 or the
    number of most recent cached keys the query sees.  Returns float64
    [B, H, dv].
    """
    q1, q2, k1, k2, v = map(_f64, (q1, q2, k1, k2, v))
    lam, gain, lam_logits, gate = map(_f64, (lam, gain, lam_logits, gate))
    B, H, L, d = k1.shape
    dv = v.shape[3]
    assert lam_logits is None or lam_logits.shape == (B, H)
    assert gate is None or gate.shape == (B, H, dv)
    if lam_logits is None:
        assert lam is not None and lam.shape == (H,)
    kl = None
    if kv_len is not None:
        if hasattr(kv_len, "detach"):
            kv_len = kv_len.detach().cpu().numpy()
        kl = np.ascontiguousarray(np.asarray(kv_len, dtype=np.int64))
        assert kl.shape == (B,)
    out = np.empty((B, H, dv), dtype=np.float64)
    rc = _lib().diffattn_oracle_decode(
        _dp(q1), _dp(q2), _dp(k1), _dp(k2), _dp(v), B, H, L, d, dv,
        kl.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if kl is not None else None,
        _dp(lam), _dp(gain), _dp(lam_logits), _dp(gate), float(scale), float(eps),
        int(bool(apply_norm)), int(window), _dp(out))
    if rc != 0:
        raise ValueError("oracle decode: invalid arguments")
    return out

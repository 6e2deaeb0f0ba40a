"""Host-side checks of the C ABI (no GPU needed).

The library must load on a machine without a GPU, export every function that
include/*.h declares, and reject bad arguments before launching anything.
"""
import ctypes
import glob
import os
import re

import pytest
import torch

from differential_attention_07_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(diffattn_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def test_library_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert "diffattn_fwd" in names and "diffattn_decode" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"
    assert set(ops.EXPORTED) <= set(names)


def test_library_is_sm100a_build():
    src = open(os.path.join(ROOT, "differential_attention_07_b200", "build.py")).read()
    assert "arch=compute_100a,code=sm_100a" in src


def test_status_strings(L):
    for code in range(7):
        assert L.diffattn_status_str(code)
    assert L.diffattn_status_str(6) == b"device wait timed out"


def _fake_fwd_args(B=2, N=300, H=4, H_N=None, H_V=None, d=64, dv=128, base=1 << 20):
    """Argument struct with plausible, 16-byte-aligned fake device addresses.
    Only host validation ever looks at it."""
    H_N = H_N or H
    H_V = H_V or H
    a = ops.FwdArgs()
    a.B, a.N, a.H, a.H_N, a.H_V, a.d, a.dv = B, N, H, H_N, H_V, d, dv
    a.scale, a.eps = 0.125, 1e-5
    a.flags = ops.DIFFATTN_FLAG_CAUSAL | ops.DIFFATTN_FLAG_APPLY_NORM
    for i, (n, h, w) in enumerate((("q1", H, d), ("q2", H_N, d), ("k1", H, d), ("k2", H_N, d),
                                   ("v", H_V, dv), ("out", H, dv))):
        setattr(a, n, base * (i + 1))
        setattr(a, n + "_stride", ops._S3(N * h * w, h * w, w))
    a.lambda_ = base * 16
    return a


def _v(L, a, grouped=0):
    return L.diffattn_fwd_validate(ctypes.byref(a), grouped)


def test_fwd_validation(L):
    assert _v(L, _fake_fwd_args()) == 0
    a = _fake_fwd_args(d=32)
    assert _v(L, a) == 2                          # unsupported head dim
    a = _fake_fwd_args(dv=64)
    assert _v(L, a) == 2
    a = _fake_fwd_args()
    a.q1 = 0
    assert _v(L, a) == 1                          # null pointer
    a = _fake_fwd_args()
    a.k2 = a.k2 + 8
    assert _v(L, a) == 3                          # misaligned
    a = _fake_fwd_args()
    a.v_stride[1] = 130
    assert _v(L, a) == 3                          # stride not a multiple of 8
    a = _fake_fwd_args()
    a.lambda_ = 0
    assert _v(L, a) == 1
    a = _fake_fwd_args()
    a.scale = 0.0
    assert _v(L, a) == 1
    a = _fake_fwd_args()
    a.flags = 8
    assert _v(L, a) == 1
    a = _fake_fwd_args()
    a.gain = (1 << 22) + 4
    assert _v(L, a) == 3                          # gain must be 16-byte aligned
    a = _fake_fwd_args(B=0)
    a.q1 = 0
    assert _v(L, a) == 0                          # empty batch: nothing to check


def test_grouped_validation(L):
    a = _fake_fwd_args(H=24, H_N=8, H_V=8)
    assert _v(L, a, 1) == 0
    assert _v(L, a, 0) == 1                       # ungrouped entry needs H_N == H_V == H
    assert _v(L, _fake_fwd_args(H=24, H_N=7, H_V=8), 1) == 1
    assert _v(L, _fake_fwd_args(H=24, H_N=8, H_V=5), 1) == 1


def test_fwd_rejects_before_launch(L):
    """diffattn_fwd with a bad argument or no workspace returns the error
    without any CUDA call (this machine may have no GPU)."""
    a = _fake_fwd_args(d=32)
    assert L.diffattn_fwd(ctypes.byref(a), None, 0, None) == 2
    a = _fake_fwd_args()
    assert L.diffattn_fwd(ctypes.byref(a), None, 0, None) == 4          # workspace missing
    need = L.diffattn_fwd_workspace_size(ctypes.byref(a))
    assert need == 2 * 300 * 4 * 128 * 2 + 256
    assert L.diffattn_fwd(ctypes.byref(a), ctypes.c_void_p(1 << 30), need - 1, None) == 4
    assert L.diffattn_fwd(ctypes.byref(a), ctypes.c_void_p((1 << 30) + 16), need, None) == 3
    assert L.diffattn_grouped_fwd(ctypes.byref(_fake_fwd_args(H=6, H_N=4)), None, 0, None) == 1
    # groups of 3 signal heads sharing one V head also hold the exported
    # noise outputs (fp32, whole 128-row query tiles: 300 rows take 3) in the
    # workspace, then one ready count per (b, noise head, tile), 256-B aligned
    g = _fake_fwd_args(H=24, H_N=8, H_V=8)
    assert L.diffattn_fwd_workspace_size(ctypes.byref(g)) == (2 * 300 * 8 * 128 * 2 + 256
                                                             + 2 * 8 * 3 * 128 * 128 * 4 + 256)
    g = _fake_fwd_args(H=24, H_N=8, H_V=24)
    assert L.diffattn_fwd_workspace_size(ctypes.byref(g)) == 2 * 300 * 24 * 128 * 2 + 256
    # under a sliding window the kernel reads V itself: no fp16 copy
    w = _fake_fwd_args()
    w.window = 128
    assert L.diffattn_fwd_workspace_size(ctypes.byref(w)) == 256
    assert ops.fwd_workspace_size(2, 300, 4, window=128) == 256


def _fake_decode_args(B=3, H=2, L=1000, base=1 << 20):
    a = ops.DecodeArgs()
    a.B, a.H, a.L, a.d, a.dv = B, H, L, 64, 128
    a.scale, a.eps, a.flags = 0.125, 1e-5, ops.DIFFATTN_FLAG_APPLY_NORM
    a.q1, a.q1_stride = base, ops._S2(H * 64, 64)
    a.q2, a.q2_stride = 2 * base, ops._S2(H * 64, 64)
    a.k1, a.k1_stride = 3 * base, ops._S3(H * L * 64, L * 64, 64)
    a.k2, a.k2_stride = 4 * base, ops._S3(H * L * 64, L * 64, 64)
    a.v, a.v_stride = 5 * base, ops._S3(H * L * 128, L * 128, 128)
    a.out, a.out_stride = 6 * base, ops._S2(H * 128, 128)
    a.lambda_ = 7 * base
    return a


def test_decode_validation_and_workspace(L):
    assert L.diffattn_decode_validate(ctypes.byref(_fake_decode_args())) == 0
    a = _fake_decode_args()
    a.k1 = a.k1 + 2
    assert L.diffattn_decode_validate(ctypes.byref(a)) == 3
    a = _fake_decode_args()
    a.num_splits = -1
    assert L.diffattn_decode_validate(ctypes.byref(a)) == 1
    a = _fake_decode_args()
    assert L.diffattn_decode(ctypes.byref(a), None, 0, None) == 4
    # splits: chunks of at most 2048 keys, a multiple of 64, none empty
    for (B, H, Lk, req) in [(64, 16, 8192, 0), (1, 16, 8192, 0), (3, 2, 1000, 0), (1, 1, 1, 0),
                            (2, 2, 5000, 7), (1, 1, 100000, 0), (4, 4, 130, 3)]:
        s = L.diffattn_decode_num_splits(B, H, Lk, req)
        chunk = ((Lk + s - 1) // s + 63) // 64 * 64
        assert s >= 1 and chunk <= max(2048, 64) and (s - 1) * chunk < Lk <= s * chunk
        ws = L.diffattn_decode_workspace_size(B, H, Lk, req)
        assert ws >= B * H * s * 260 * 4 and ws % 256 == 0
    assert L.diffattn_decode_num_splits(64, 16, 8192, 0) == 4


def test_token_lambda_and_gate_validation(L):
    """Motif 3's token-dependent lambda logits and output gate: the per-head
    lambda may be NULL only when logits are given; the gate follows the
    output's alignment rules; the logits need 4-byte alignment."""
    base = 1 << 20
    a = _fake_fwd_args()
    a.lambda_ = None
    assert _v(L, a) == 1                              # no lambda at all
    a.lambda_logits = 20 * base
    a.lambda_logits_stride = ops._S3(300 * 4, 4, 1)
    assert _v(L, a) == 0                              # logits alone are enough
    a.lambda_logits = 20 * base + 2
    assert _v(L, a) == 3                              # not 4-byte aligned
    a.lambda_logits = 20 * base
    a.lambda_logits_stride = ops._S3(300 * 4, -4, 1)
    assert _v(L, a) == 1
    a = _fake_fwd_args()
    a.gate, a.gate_stride = 21 * base, ops._S3(300 * 4 * 128, 4 * 128, 128)
    assert _v(L, a) == 0
    a.gate = 21 * base + 8
    assert _v(L, a) == 3                              # base not 16-byte aligned
    a.gate = 21 * base
    a.gate_stride = ops._S3(300 * 4 * 128, 4 * 128 + 4, 128)
    assert _v(L, a) == 3                              # stride not a multiple of 8
    a.gate_stride = ops._S3(300 * 4 * 128, -512, 128)
    assert _v(L, a) == 1
    d = _fake_decode_args()
    d.lambda_ = None
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 1
    d.lambda_logits, d.lambda_logits_stride = 8 * base, ops._S2(2, 1)
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 0
    d.gate, d.gate_stride = 9 * base + 2, ops._S2(2 * 128, 128)
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 3
    d.gate = 9 * base
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 0


def test_window_validation(L):
    a = _fake_fwd_args()
    a.window = 128
    assert _v(L, a) == 0
    a.window = -1
    assert _v(L, a) == 1
    a = _fake_fwd_args()
    a.window = 16
    a.flags = ops.DIFFATTN_FLAG_APPLY_NORM          # a window needs the causal mask
    assert _v(L, a) == 1
    d = _fake_decode_args()
    d.window = 100
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 0
    d.window = -5
    assert L.diffattn_decode_validate(ctypes.byref(d)) == 1


def test_rope_validation_and_workspace(L):
    a = _fake_fwd_args(B=2, N=300, H=4)
    base = L.diffattn_fwd_workspace_size(ctypes.byref(a))
    a.rope_theta = 500000.0
    assert _v(L, a) == 0
    # rotated copies of Q1, K1, Q2, K2: 4 x [B, N, H, 64] bf16
    assert L.diffattn_fwd_workspace_size(ctypes.byref(a)) == base + 4 * 2 * 300 * 4 * 64 * 2
    a.rope_theta = -1.0
    assert _v(L, a) == 1
    a.rope_theta = float("inf")
    assert _v(L, a) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ops, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ops, "_LIB", None)
    with pytest.raises(RuntimeError, match="not built"):
        ops.lib()


def test_binding_rejects_cpu_tensor_types():
    x = torch.zeros(1, 4, 1, 64, dtype=torch.float32)
    with pytest.raises(TypeError):
        ops._check_bf16("q1", x, 4)


def _fake_bwd_args(B=2, N=300, H=4, base=1 << 20):
    a = ops.BwdArgs()
    a.B, a.N, a.H, a.d, a.dv = B, N, H, 64, 128
    a.scale, a.eps = 0.125, 1e-5
    a.flags = ops.DIFFATTN_FLAG_CAUSAL | ops.DIFFATTN_FLAG_APPLY_NORM
    for i, (n, w) in enumerate((("q1", 64), ("q2", 64), ("k1", 64), ("k2", 64), ("v", 128),
                                ("dout", 128), ("grad_q1", 64), ("grad_q2", 64), ("grad_k1", 64),
                                ("grad_k2", 64), ("grad_v", 128))):
        setattr(a, n, base * (i + 1))
        setattr(a, n + "_stride", ops._S3(N * H * w, H * w, w))
    a.save, a.lambda_ = base * 20, base * 21
    return a


def test_bwd_rejects_before_launch(L):
    """diffattn_bwd checks its arguments and workspace before any CUDA call.
    (The empty-problem case zeroes dlambda / dgain on the device, so it is
    left to the GPU tests.)"""
    b = lambda a, ws=None, n=0: L.diffattn_bwd(ctypes.byref(a), ws, n, None)
    a = _fake_bwd_args()
    need = L.diffattn_bwd_workspace_size(ctypes.byref(a))
    # fp16 copies of V and dD, then [B, H, 5, 3 tiles * 128] fp32 statistics, then 256 B
    assert need == 2 * (2 * 300 * 4 * 128 * 2) + 2 * 4 * 5 * 384 * 4 + 256
    # grouped heads add fp32 sums of the shared heads' gradients: dK2 and dQ2
    # [B, N, H_N, 64], dV [B, N, H_V, 128]; rope_theta the rotated fp16 copies
    g = _fake_bwd_args()
    g.H_N, g.H_V = 2, 2
    assert L.diffattn_bwd_workspace_size(ctypes.byref(g)) == (
        300 * 2 * 2 * 128 * 2 + 2 * 300 * 4 * 128 * 2 + 2 * 4 * 5 * 384 * 4 + 256
        + 2 * (2 * 300 * 2 * 64 * 4) + 2 * 300 * 2 * 128 * 4)
    g = _fake_bwd_args()
    g.rope_theta = 1e4
    assert L.diffattn_bwd_workspace_size(ctypes.byref(g)) == need + 4 * (2 * 300 * 4 * 64 * 2)
    assert b(a) == 4                                               # workspace missing
    assert b(a, ctypes.c_void_p(1 << 30), need - 1) == 4
    assert b(a, ctypes.c_void_p((1 << 30) + 16), need) == 3         # workspace not 256-aligned
    for field, value, code in (("d", 32, 2), ("dv", 64, 2), ("save", 0, 1), ("dout", 0, 1),
                               ("grad_v", 0, 1), ("lambda_", 0, 1), ("grad_k2", (1 << 20) + 8, 3),
                               ("save", (1 << 20) + 4, 3), ("grad_gain", (1 << 20) + 2, 3),
                               ("flags", 8, 1), ("scale", 0.0, 1), ("H_N", 3, 1), ("H_V", -1, 1),
                               ("window", -1, 1), ("grad_gate", 1 << 27, 1),
                               ("lambda_logits", (1 << 20) + 2, 3)):
        a = _fake_bwd_args()
        setattr(a, field, value)
        assert b(a, ctypes.c_void_p(1 << 30), need) == code, field
    a = _fake_bwd_args()
    a.dout_stride[1] = 130
    assert b(a, ctypes.c_void_p(1 << 30), need) == 3                # stride not a multiple of 8


def test_fwd_save_size_and_support(L):
    a = _fake_fwd_args()
    # per (b, h, 128-row tile): A_1, A_2 (2 x 128 x 128 fp32) and lse_1, lse_2 (2 x 128 fp32)
    assert L.diffattn_fwd_save_size(ctypes.byref(a)) == 2 * 4 * 3 * (2 * 128 * 128 + 2 * 128) * 4
    a.save = 1 << 28
    assert _v(L, a) == 0
    a.save = (1 << 28) + 8
    assert _v(L, a) == 3                                           # 16-byte alignment
    for field, value in (("window", 64), ("rope_theta", 1e4), ("gate", 1 << 27),
                         ("lambda_logits", 1 << 27)):
        a = _fake_fwd_args()
        a.save = 1 << 28
        setattr(a, field, value)
        if field == "gate":
            a.gate_stride = ops._S3(300 * 4 * 128, 4 * 128, 128)
        assert _v(L, a) == 0, field                                # every option saves
    g = _fake_fwd_args(H=24, H_N=8, H_V=8)
    ws = L.diffattn_fwd_workspace_size(ctypes.byref(g))
    g.save = 1 << 28
    assert _v(L, g, 1) == 0                                        # grouped heads too,
    assert L.diffattn_fwd_workspace_size(ctypes.byref(g)) < ws     # one signal head per item

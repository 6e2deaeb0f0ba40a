"""Python binding of libdiffattn (ctypes).  Argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI
declared in include/diffattn.h; this module checks tensor properties, fills
the argument structs with raw device pointers, strides and the current CUDA
stream, and allocates the caller-owned workspace with torch.  There is no CPU
fallback: without the built library or a CUDA device every call raises.

Functions (same names as the C entry points):
    diffattn_fwd(q1, q2, k1, k2, v, lam, gain=None, ...)          -> out
    diffattn_grouped_fwd(q1, q2, k1, k2, v, lam, gain=None, ...)  -> out
    diffattn_decode(q1, q2, k1, k2, v, lam, gain=None, ...)       -> out
    diffattn_bwd(q1, q2, k1, k2, v, lam, gain, dout, save, ...)   -> gradients
and DiffAttention / diff_attention, a torch.autograd.Function over
diffattn_fwd (with the saved state) and diffattn_bwd, for training.
"""
import ctypes
import os

import torch

from . import build as _build

LIB_PATH = _build.LIB

DIFFATTN_FLAG_CAUSAL = 1
DIFFATTN_FLAG_APPLY_NORM = 2
DIFFATTN_FLAG_TEST_WITHHOLD_LOAD = 0x80000000

STATUS = {
    0: "DIFFATTN_OK",
    1: "DIFFATTN_ERR_INVALID_ARG",
    2: "DIFFATTN_ERR_UNSUPPORTED",
    3: "DIFFATTN_ERR_ALIGNMENT",
    4: "DIFFATTN_ERR_WORKSPACE",
    5: "DIFFATTN_ERR_CUDA",
    6: "DIFFATTN_ERR_TIMEOUT",
}

EXPORTED = [
    "diffattn_fwd", "diffattn_grouped_fwd", "diffattn_fwd_workspace_size", "diffattn_fwd_validate",
    "diffattn_decode", "diffattn_decode_workspace_size", "diffattn_decode_num_splits",
    "diffattn_decode_validate", "diffattn_status_str", "diffattn_last_launch_count",
    "diffattn_set_profile_events", "diffattn_last_error", "diffattn_decode_noalloc",
    "diffattn_bwd", "diffattn_bwd_workspace_size", "diffattn_fwd_save_size",
]

_i64 = ctypes.c_int64
_p = ctypes.c_void_p
_S3 = _i64 * 3
_S2 = _i64 * 2


class FwdArgs(ctypes.Structure):
    """Mirror of struct diffattn_fwd_args."""
    _fields_ = [
        ("B", _i64), ("N", _i64), ("H", _i64), ("H_N", _i64), ("H_V", _i64),
        ("d", _i64), ("dv", _i64),
        ("scale", ctypes.c_float), ("eps", ctypes.c_float),
        ("flags", ctypes.c_uint32), ("timeout_ms", ctypes.c_uint32),
        ("q1", _p), ("q1_stride", _S3),
        ("q2", _p), ("q2_stride", _S3),
        ("k1", _p), ("k1_stride", _S3),
        ("k2", _p), ("k2_stride", _S3),
        ("v", _p), ("v_stride", _S3),
        ("out", _p), ("out_stride", _S3),
        ("lambda_", _p), ("gain", _p), ("dev_status", _p),
        ("lambda_logits", _p), ("lambda_logits_stride", _S3),
        ("gate", _p), ("gate_stride", _S3),
        ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
        ("save", _p),
    ]


class BwdArgs(ctypes.Structure):
    """Mirror of struct diffattn_bwd_args."""
    _fields_ = [
        ("B", _i64), ("N", _i64), ("H", _i64),
        ("d", _i64), ("dv", _i64),
        ("scale", ctypes.c_float), ("eps", ctypes.c_float),
        ("flags", ctypes.c_uint32), ("timeout_ms", ctypes.c_uint32),
        ("q1", _p), ("q1_stride", _S3),
        ("q2", _p), ("q2_stride", _S3),
        ("k1", _p), ("k1_stride", _S3),
        ("k2", _p), ("k2_stride", _S3),
        ("v", _p), ("v_stride", _S3),
        ("dout", _p), ("dout_stride", _S3),
        ("save", _p), ("lambda_", _p), ("gain", _p),
        ("grad_q1", _p), ("grad_q1_stride", _S3),
        ("grad_q2", _p), ("grad_q2_stride", _S3),
        ("grad_k1", _p), ("grad_k1_stride", _S3),
        ("grad_k2", _p), ("grad_k2_stride", _S3),
        ("grad_v", _p), ("grad_v_stride", _S3),
        ("grad_lambda", _p), ("grad_gain", _p), ("dev_status", _p),
        ("H_N", _i64), ("H_V", _i64),
        ("lambda_logits", _p), ("lambda_logits_stride", _S3),
        ("gate", _p), ("gate_stride", _S3),
        ("window", ctypes.c_int32), ("rope_theta", ctypes.c_float),
        ("grad_lambda_logits", _p), ("grad_lambda_logits_stride", _S3),
        ("grad_gate", _p), ("grad_gate_stride", _S3),
    ]


class DecodeArgs(ctypes.Structure):
    """Mirror of struct diffattn_decode_args."""
    _fields_ = [
        ("B", _i64), ("H", _i64), ("L", _i64),
        ("d", _i64), ("dv", _i64),
        ("scale", ctypes.c_float), ("eps", ctypes.c_float),
        ("flags", ctypes.c_uint32), ("num_splits", ctypes.c_int32),
        ("q1", _p), ("q1_stride", _S2),
        ("q2", _p), ("q2_stride", _S2),
        ("k1", _p), ("k1_stride", _S3),
        ("k2", _p), ("k2_stride", _S3),
        ("v", _p), ("v_stride", _S3),
        ("out", _p), ("out_stride", _S2),
        ("kv_len", _p), ("lambda_", _p), ("gain", _p), ("dev_status", _p),
        ("lambda_logits", _p), ("lambda_logits_stride", _S2),
        ("gate", _p), ("gate_stride", _S2),
        ("window", ctypes.c_int32),
    ]


class DiffAttnError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if status in (4, 5) and _LIB is not None:
            detail = _LIB.diffattn_last_error()
            if detail:
                msg += f" ({detail.decode(errors='replace')})"
        super().__init__(msg)


_LIB = None


def lib():
    """The loaded libdiffattn (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdiffattn is not built ({LIB_PATH} missing); run "
                               "`python -m differential_attention_07_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        fa, da, ba = ctypes.POINTER(FwdArgs), ctypes.POINTER(DecodeArgs), ctypes.POINTER(BwdArgs)
        for name in ("diffattn_fwd", "diffattn_grouped_fwd"):
            f = getattr(L, name)
            f.argtypes = [fa, _p, ctypes.c_size_t, _p]
            f.restype = ctypes.c_int
        L.diffattn_fwd_workspace_size.argtypes = [fa]
        L.diffattn_fwd_workspace_size.restype = ctypes.c_size_t
        L.diffattn_fwd_save_size.argtypes = [fa]
        L.diffattn_fwd_save_size.restype = ctypes.c_size_t
        L.diffattn_bwd.argtypes = [ba, _p, ctypes.c_size_t, _p]
        L.diffattn_bwd.restype = ctypes.c_int
        L.diffattn_bwd_workspace_size.argtypes = [ba]
        L.diffattn_bwd_workspace_size.restype = ctypes.c_size_t
        L.diffattn_fwd_validate.argtypes = [fa, ctypes.c_int]
        L.diffattn_fwd_validate.restype = ctypes.c_int
        L.diffattn_decode.argtypes = [da, _p, ctypes.c_size_t, _p]
        L.diffattn_decode.restype = ctypes.c_int
        L.diffattn_decode_noalloc.argtypes = [da, _p]
        L.diffattn_decode_noalloc.restype = ctypes.c_int
        L.diffattn_decode_workspace_size.argtypes = [_i64, _i64, _i64, ctypes.c_int32]
        L.diffattn_decode_workspace_size.restype = ctypes.c_size_t
        L.diffattn_decode_num_splits.argtypes = [_i64, _i64, _i64, ctypes.c_int32]
        L.diffattn_decode_num_splits.restype = ctypes.c_int32
        L.diffattn_decode_validate.argtypes = [da]
        L.diffattn_decode_validate.restype = ctypes.c_int
        L.diffattn_status_str.argtypes = [ctypes.c_int]
        L.diffattn_status_str.restype = ctypes.c_char_p
        L.diffattn_last_launch_count.argtypes = []
        L.diffattn_last_launch_count.restype = ctypes.c_int32
        L.diffattn_last_error.argtypes = []
        L.diffattn_last_error.restype = ctypes.c_char_p
        L.diffattn_set_profile_events.argtypes = [_p, _p]
        L.diffattn_set_profile_events.restype = None
        _LIB = L
    return _LIB


def last_launch_count() -> int:
    """Kernels launched by the last successful call on this thread."""
    return int(lib().diffattn_last_launch_count())


def set_profile_events(start=None, stop=None):
    """Record torch.cuda.Event `start` / `stop` around the main kernel of every
    later call on this thread (None, None switches it off)."""
    lib().diffattn_set_profile_events(
        ctypes.c_void_p(start.cuda_event) if start is not None else None,
        ctypes.c_void_p(stop.cuda_event) if stop is not None else None)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_bf16(name, t, ndim):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if t.stride(-1) != 1:
        raise ValueError(f"{name}: last dimension must be contiguous")


def _stream_ptr(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _set_lambda_gate(a, lam, lam_logits, gate, lead, dv, S):
    """Fill lambda (per head), the token-dependent lambda logits and the gate
    logits.  lead: the leading dims (B, N, H) or (B, H); S: the stride type."""
    H = lead[-1]
    if lam_logits is not None:
        if lam_logits.dtype != torch.float32 or tuple(lam_logits.shape) != tuple(lead):
            raise ValueError(f"lam_logits must be float32 {list(lead)}")
        a.lambda_logits = lam_logits.data_ptr()
        a.lambda_logits_stride = S(*lam_logits.stride())
    elif lam is None:
        raise ValueError("lam (per head) or lam_logits (per token) is required")
    if lam is not None:
        if lam.dtype != torch.float32 or lam.shape != (H,):
            raise ValueError("lam must be float32 [H]")
        a.lambda_ = lam.data_ptr()
    if gate is not None:
        _check_bf16("gate", gate, len(lead) + 1)
        if tuple(gate.shape) != tuple(lead) + (dv,):
            raise ValueError(f"gate must be bf16 {list(lead) + [dv]}")
        a.gate = gate.data_ptr()
        a.gate_stride = S(*gate.stride()[:len(lead)])


def _fwd_args(q1, q2, k1, k2, v, lam, gain, out, *, scale, eps, causal, apply_norm,
              timeout_ms, dev_status, test_withhold_load=False, lam_logits=None, gate=None,
              window=0, rope_theta=0.0, save=None):
    for n, t in (("q1", q1), ("q2", q2), ("k1", k1), ("k2", k2), ("v", v), ("out", out)):
        _check_bf16(n, t, 4)
    B, N, H, d = q1.shape
    a = FwdArgs()
    a.B, a.N, a.H, a.H_N, a.H_V = B, N, H, q2.shape[2], v.shape[2]
    a.d, a.dv = d, v.shape[3]
    a.scale, a.eps = float(scale), float(eps)
    a.flags = (DIFFATTN_FLAG_CAUSAL if causal else 0) | (DIFFATTN_FLAG_APPLY_NORM if apply_norm else 0)
    if test_withhold_load:
        a.flags |= DIFFATTN_FLAG_TEST_WITHHOLD_LOAD
    a.timeout_ms = int(timeout_ms)
    a.window = int(window)
    a.rope_theta = float(rope_theta)
    for n, t in (("q1", q1), ("q2", q2), ("k1", k1), ("k2", k2), ("v", v), ("out", out)):
        setattr(a, n, t.data_ptr())
        setattr(a, n + "_stride", _S3(*t.stride()[:3]))
    _set_lambda_gate(a, lam, lam_logits, gate, (B, N, H), a.dv, _S3)
    if gain is not None:
        if gain.dtype != torch.float32 or tuple(gain.shape) != (H, a.dv) or not gain.is_contiguous():
            raise ValueError("gain must be contiguous float32 [H, dv]")
        a.gain = gain.data_ptr()
    a.dev_status = dev_status.data_ptr() if dev_status is not None else None
    if save is not None:
        need = int(lib().diffattn_fwd_save_size(ctypes.byref(a)))
        if not save.is_cuda or save.numel() * save.element_size() < need or not save.is_contiguous():
            raise ValueError(f"save must be a contiguous CUDA buffer of at least {need} bytes")
        a.save = save.data_ptr()
    return a


def _check_shapes_fwd(q1, q2, k1, k2, v):
    B, N, H, d = q1.shape
    if k1.shape != q1.shape:
        raise ValueError("k1 must have q1's shape")
    if q2.shape != k2.shape or q2.shape[:2] != (B, N) or q2.shape[3] != d:
        raise ValueError("q2/k2 must be [B, N, H_N, d]")
    if v.shape[:2] != (B, N):
        raise ValueError("v must be [B, N, H_V, dv]")


def _run_fwd(entry, q1, q2, k1, k2, v, lam, gain, *, scale, eps, causal, apply_norm, out,
             workspace, stream, timeout_ms, dev_status, test_withhold_load=False,
             lam_logits=None, gate=None, window=0, rope_theta=0.0, save=None):
    _check_shapes_fwd(q1, q2, k1, k2, v)
    B, N, H, _ = q1.shape
    if out is None:
        out = torch.empty(B, N, H, v.shape[3], dtype=torch.bfloat16, device=q1.device)
    a = _fwd_args(q1, q2, k1, k2, v, lam, gain, out, scale=scale, eps=eps, causal=causal,
                  apply_norm=apply_norm, timeout_ms=timeout_ms, dev_status=dev_status,
                  test_withhold_load=test_withhold_load, lam_logits=lam_logits, gate=gate,
                  window=window, rope_theta=rope_theta, save=save)
    L = lib()
    need = L.diffattn_fwd_workspace_size(ctypes.byref(a))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q1.device)
    st = getattr(L, entry)(ctypes.byref(a), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if st != 0:
        raise DiffAttnError(st, entry)
    return out


def diffattn_fwd(q1, q2, k1, k2, v, lam, gain=None, *, scale=0.125, eps=1e-5, causal=True,
                 apply_norm=True, out=None, workspace=None, stream=None, timeout_ms=0,
                 dev_status=None, test_withhold_load=False, lam_logits=None, gate=None,
                 window=0, rope_theta=0.0, save=None):
    """Differential-attention prefill.  q1,q2,k1,k2 [B,N,H,64], v [B,N,H,128]
    bf16 CUDA tensors (token-major, last dim contiguous); lam [H] fp32 (or
    None with lam_logits); gain [H,128] fp32 or None; lam_logits: fp32
    [B,N,H] token-dependent lambda logits or None; gate: bf16 [B,N,H,128]
    output-gate logits or None; window: 0, or a causal sliding window of that
    many keys; rope_theta: 0, or the base of the rotary embedding applied to
    Q1, K1, Q2, K2 by token position.  Returns out [B,N,H,128] bf16.
    save: None, or a CUDA buffer of fwd_save_size(B, N, H) bytes that the
    call also fills with the state diffattn_bwd needs.
    test_withhold_load sets the library's failure-path test hook (the call
    then reports a timeout in dev_status)."""
    return _run_fwd("diffattn_fwd", q1, q2, k1, k2, v, lam, gain, scale=scale, eps=eps,
                    causal=causal, apply_norm=apply_norm, out=out, workspace=workspace,
                    stream=stream, timeout_ms=timeout_ms, dev_status=dev_status,
                    test_withhold_load=test_withhold_load, lam_logits=lam_logits, gate=gate,
                    window=window, rope_theta=rope_theta, save=save)


def diffattn_grouped_fwd(q1, q2, k1, k2, v, lam, gain=None, *, scale=0.125, eps=1e-5, causal=True,
                         apply_norm=True, out=None, workspace=None, stream=None, timeout_ms=0,
                         dev_status=None, lam_logits=None, gate=None, window=0, rope_theta=0.0,
                         save=None, test_withhold_load=False):
    """Grouped prefill: q1,k1 [B,N,H,64]; q2,k2 [B,N,H_N,64]; v [B,N,H_V,128];
    signal head h uses noise head h // (H // H_N) and V head h // (H // H_V).
    lam_logits [B,N,H], gate [B,N,H,128] and save as in diffattn_fwd."""
    return _run_fwd("diffattn_grouped_fwd", q1, q2, k1, k2, v, lam, gain, scale=scale, eps=eps,
                    causal=causal, apply_norm=apply_norm, out=out, workspace=workspace,
                    stream=stream, timeout_ms=timeout_ms, dev_status=dev_status,
                    lam_logits=lam_logits, gate=gate, window=window, rope_theta=rope_theta,
                    save=save, test_withhold_load=test_withhold_load)


def fwd_workspace_size(B, N, H, H_V=None, H_N=None, rope_theta=0.0, window=0):
    """Workspace bytes of a prefill call with these sizes."""
    a = FwdArgs()
    a.B, a.N, a.H, a.H_N, a.H_V, a.d, a.dv = B, N, H, H_N or H, H_V or H, 64, 128
    a.rope_theta = float(rope_theta)
    a.window = int(window)
    return int(lib().diffattn_fwd_workspace_size(ctypes.byref(a)))


def decode_workspace_size(B, H, L, num_splits=0):
    return int(lib().diffattn_decode_workspace_size(B, H, L, num_splits))


def decode_num_splits(B, H, L, num_splits=0):
    return int(lib().diffattn_decode_num_splits(B, H, L, num_splits))


def _decode_args(q1, q2, k1, k2, v, lam, gain, out, *, kv_len, num_splits, scale, eps,
                 apply_norm, dev_status, lam_logits=None, gate=None, window=0):
    for n, t, nd in (("q1", q1, 3), ("q2", q2, 3), ("k1", k1, 4), ("k2", k2, 4), ("v", v, 4),
                     ("out", out, 3)):
        _check_bf16(n, t, nd)
    B, H, L, d = k1.shape
    if q1.shape != (B, H, d) or q2.shape != (B, H, d) or k2.shape != k1.shape:
        raise ValueError("decode: q [B,H,d], k [B,H,L,d] expected")
    if v.shape[:3] != (B, H, L):
        raise ValueError("decode: v [B,H,L,dv] expected")
    a = DecodeArgs()
    a.B, a.H, a.L, a.d, a.dv = B, H, L, d, v.shape[3]
    a.scale, a.eps = float(scale), float(eps)
    a.flags = DIFFATTN_FLAG_APPLY_NORM if apply_norm else 0
    a.num_splits = int(num_splits)
    a.window = int(window)
    for n, t in (("q1", q1), ("q2", q2), ("out", out)):
        setattr(a, n, t.data_ptr())
        setattr(a, n + "_stride", _S2(*t.stride()[:2]))
    for n, t in (("k1", k1), ("k2", k2), ("v", v)):
        setattr(a, n, t.data_ptr())
        setattr(a, n + "_stride", _S3(*t.stride()[:3]))
    if kv_len is not None:
        if kv_len.dtype != torch.int32 or kv_len.shape != (B,):
            raise ValueError("kv_len must be int32 [B]")
        a.kv_len = kv_len.data_ptr()
    _set_lambda_gate(a, lam, lam_logits, gate, (B, H), a.dv, _S2)
    if gain is not None:
        if gain.dtype != torch.float32 or tuple(gain.shape) != (H, a.dv) or not gain.is_contiguous():
            raise ValueError("gain must be contiguous float32 [H, dv]")
        a.gain = gain.data_ptr()
    a.dev_status = dev_status.data_ptr() if dev_status is not None else None
    return a


def diffattn_decode(q1, q2, k1, k2, v, lam, gain=None, *, kv_len=None, num_splits=0, scale=0.125,
                    eps=1e-5, apply_norm=True, out=None, workspace=None, stream=None,
                    dev_status=None, lam_logits=None, gate=None, window=0):
    """Single-query decode.  q1,q2 [B,H,64]; k1,k2 [B,H,L,64]; v [B,H,L,128]
    bf16 CUDA tensors; kv_len int32 [B] or None; lam_logits fp32 [B,H] and
    gate bf16 [B,H,128] optional.  Returns out [B,H,128] bf16."""
    B, H, L, _ = k1.shape
    if out is None:
        out = torch.empty(B, H, v.shape[3], dtype=torch.bfloat16, device=q1.device)
    a = _decode_args(q1, q2, k1, k2, v, lam, gain, out, kv_len=kv_len, num_splits=num_splits,
                     scale=scale, eps=eps, apply_norm=apply_norm, dev_status=dev_status,
                     lam_logits=lam_logits, gate=gate, window=window)
    Lb = lib()
    need = Lb.diffattn_decode_workspace_size(B, H, L, int(num_splits))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q1.device)
    st = Lb.diffattn_decode(ctypes.byref(a), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if st != 0:
        raise DiffAttnError(st, "diffattn_decode")
    return out


def diffattn_decode_noalloc(q1, q2, k1, k2, v, lam, gain=None, *, out, kv_len=None, num_splits=0,
                            scale=0.125, eps=1e-5, apply_norm=True, stream=None, dev_status=None,
                            lam_logits=None, gate=None, window=0):
    """Single-query decode that allocates nothing: the caller passes the
    output buffer, and the per-split partial states use the library's fixed
    static scratch (see diffattn_decode_noalloc in include/diffattn.h).  For
    callers that cannot allocate device memory or hand over a workspace."""
    a = _decode_args(q1, q2, k1, k2, v, lam, gain, out, kv_len=kv_len, num_splits=num_splits,
                     scale=scale, eps=eps, apply_norm=apply_norm, dev_status=dev_status,
                     lam_logits=lam_logits, gate=gate, window=window)
    st = lib().diffattn_decode_noalloc(ctypes.byref(a), _stream_ptr(stream))
    if st != 0:
        raise DiffAttnError(st, "diffattn_decode_noalloc")
    return out


def fwd_save_size(B, N, H):
    """Bytes of the state a prefill call with these sizes saves for diffattn_bwd."""
    a = FwdArgs()
    a.B, a.N, a.H, a.H_N, a.H_V, a.d, a.dv = B, N, H, H, H, 64, 128
    return int(lib().diffattn_fwd_save_size(ctypes.byref(a)))


def bwd_workspace_size(B, N, H, H_N=None, H_V=None, rope_theta=0.0):
    """Workspace bytes of a diffattn_bwd call with these sizes."""
    a = BwdArgs()
    a.B, a.N, a.H, a.d, a.dv = B, N, H, 64, 128
    a.H_N, a.H_V = H_N or H, H_V or H
    a.rope_theta = float(rope_theta)
    return int(lib().diffattn_bwd_workspace_size(ctypes.byref(a)))


def _bwd_args(q1, q2, k1, k2, v, lam, gain, dout, save, grads, *, scale, eps, causal, apply_norm,
              timeout_ms, dev_status, lam_logits=None, gate=None, window=0, rope_theta=0.0):
    named = (("q1", q1), ("q2", q2), ("k1", k1), ("k2", k2), ("v", v), ("dout", dout),
             ("grad_q1", grads["dq1"]), ("grad_q2", grads["dq2"]), ("grad_k1", grads["dk1"]),
             ("grad_k2", grads["dk2"]), ("grad_v", grads["dv"]))
    for n, t in named:
        _check_bf16(n, t, 4)
    B, N, H, d = q1.shape
    H_N, H_V = q2.shape[2], v.shape[2]
    heads = {"q1": H, "k1": H, "dout": H, "grad_q1": H, "grad_k1": H, "q2": H_N, "k2": H_N,
             "grad_q2": H_N, "grad_k2": H_N, "v": H_V, "grad_v": H_V}
    for n, t in named:
        if tuple(t.shape[:3]) != (B, N, heads[n]):
            raise ValueError(f"{n} must be [B, N, {heads[n]}, *] (as in the forward call)")
    a = BwdArgs()
    a.B, a.N, a.H, a.d, a.dv = B, N, H, d, v.shape[3]
    a.H_N, a.H_V = H_N, H_V
    a.scale, a.eps = float(scale), float(eps)
    a.flags = (DIFFATTN_FLAG_CAUSAL if causal else 0) | (DIFFATTN_FLAG_APPLY_NORM if apply_norm else 0)
    a.timeout_ms = int(timeout_ms)
    a.window = int(window)
    a.rope_theta = float(rope_theta)
    for n, t in named:
        setattr(a, n, t.data_ptr())
        setattr(a, n + "_stride", _S3(*t.stride()[:3]))
    _set_lambda_gate(a, lam, lam_logits, gate, (B, N, H), a.dv, _S3)
    if gain is not None:
        if gain.dtype != torch.float32 or tuple(gain.shape) != (H, a.dv) or not gain.is_contiguous():
            raise ValueError("gain must be contiguous float32 [H, dv]")
        a.gain = gain.data_ptr()
    if not save.is_cuda or not save.is_contiguous() or save.numel() * save.element_size() < fwd_save_size(B, N, H):
        raise ValueError("save must be the buffer a diffattn_fwd call with these sizes filled")
    a.save = save.data_ptr()
    a.grad_lambda = grads["dlam"].data_ptr() if grads.get("dlam") is not None else None
    a.grad_gain = grads["dgain"].data_ptr() if grads.get("dgain") is not None else None
    if lam_logits is not None and grads.get("dlam_logits") is not None:
        t = grads["dlam_logits"]
        if t.dtype != torch.float32 or tuple(t.shape) != (B, N, H):
            raise ValueError("dlam_logits must be float32 [B, N, H]")
        a.grad_lambda_logits = t.data_ptr()
        a.grad_lambda_logits_stride = _S3(*t.stride())
    if gate is not None and grads.get("dgate") is not None:
        t = grads["dgate"]
        _check_bf16("dgate", t, 4)
        if tuple(t.shape) != (B, N, H, a.dv):
            raise ValueError("dgate must be bf16 [B, N, H, dv]")
        a.grad_gate = t.data_ptr()
        a.grad_gate_stride = _S3(*t.stride()[:3])
    a.dev_status = dev_status.data_ptr() if dev_status is not None else None
    return a


def diffattn_bwd(q1, q2, k1, k2, v, lam, gain, dout, save, *, scale=0.125, eps=1e-5, causal=True,
                 apply_norm=True, grads=None, workspace=None, stream=None, timeout_ms=0,
                 dev_status=None, lam_logits=None, gate=None, window=0, rope_theta=0.0):
    """Backward pass of diffattn_fwd / diffattn_grouped_fwd: gradients of
    sum(dout * out).

    Inputs as in the forward call that filled `save` (same scale, eps,
    causal, apply_norm, lam / lam_logits, gate, window, rope_theta); dout
    [B,N,H,128] bf16.  Returns a dict: dq1, dk1 [B,N,H,64], dq2, dk2
    [B,N,H_N,64], dv [B,N,H_V,128] bf16; dlam [H] and dgain [H,128] fp32;
    with lam_logits also dlam_logits [B,N,H] fp32, with a gate dgate
    [B,N,H,128] bf16.  grads: optional dict of preallocated outputs."""
    B, N, H, d = q1.shape
    H_N, H_V, dv = q2.shape[2], v.shape[2], v.shape[3]
    dev = q1.device
    if grads is None:
        grads = {"dq1": torch.empty(B, N, H, d, dtype=torch.bfloat16, device=dev),
                 "dk1": torch.empty(B, N, H, d, dtype=torch.bfloat16, device=dev),
                 "dq2": torch.empty(B, N, H_N, d, dtype=torch.bfloat16, device=dev),
                 "dk2": torch.empty(B, N, H_N, d, dtype=torch.bfloat16, device=dev),
                 "dv": torch.empty(B, N, H_V, dv, dtype=torch.bfloat16, device=dev),
                 "dlam": torch.empty(H, dtype=torch.float32, device=dev),
                 "dgain": torch.empty(H, dv, dtype=torch.float32, device=dev)}
        if lam_logits is not None:
            grads["dlam_logits"] = torch.empty(B, N, H, dtype=torch.float32, device=dev)
        if gate is not None:
            grads["dgate"] = torch.empty(B, N, H, dv, dtype=torch.bfloat16, device=dev)
    a = _bwd_args(q1, q2, k1, k2, v, lam, gain, dout, save, grads, scale=scale, eps=eps,
                  causal=causal, apply_norm=apply_norm, timeout_ms=timeout_ms,
                  dev_status=dev_status, lam_logits=lam_logits, gate=gate, window=window,
                  rope_theta=rope_theta)
    L = lib()
    need = L.diffattn_bwd_workspace_size(ctypes.byref(a))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    st = L.diffattn_bwd(ctypes.byref(a), _ptr(workspace), workspace.numel(), _stream_ptr(stream))
    if st != 0:
        raise DiffAttnError(st, "diffattn_bwd")
    return grads


class DiffAttention(torch.autograd.Function):
    """Differential attention as an autograd function: the forward runs
    diffattn_fwd (diffattn_grouped_fwd with shared noise or V heads) with the
    saved state, the backward runs diffattn_bwd."""

    @staticmethod
    def forward(ctx, q1, q2, k1, k2, v, lam, gain, lam_logits, gate, scale, eps, causal, apply_norm,
                window, rope_theta):
        B, N, H, _ = q1.shape
        save = torch.empty(max(fwd_save_size(B, N, H), 16), dtype=torch.uint8, device=q1.device)
        grouped = q2.shape[2] != H or v.shape[2] != H
        f = diffattn_grouped_fwd if grouped else diffattn_fwd
        out = f(q1, q2, k1, k2, v, lam, gain, scale=scale, eps=eps, causal=causal,
                apply_norm=apply_norm, save=save, lam_logits=lam_logits, gate=gate, window=window,
                rope_theta=rope_theta)
        ctx.save_for_backward(q1, q2, k1, k2, v, lam, gain, lam_logits, gate, save)
        ctx.cfg = (scale, eps, causal, apply_norm, window, rope_theta)
        return out

    @staticmethod
    def backward(ctx, dout):
        q1, q2, k1, k2, v, lam, gain, lam_logits, gate, save = ctx.saved_tensors
        scale, eps, causal, apply_norm, window, rope_theta = ctx.cfg
        dout = dout.to(torch.bfloat16)
        if dout.stride(-1) != 1:
            dout = dout.contiguous()
        g = diffattn_bwd(q1, q2, k1, k2, v, lam, gain, dout, save, scale=scale, eps=eps,
                         causal=causal, apply_norm=apply_norm, lam_logits=lam_logits, gate=gate,
                         window=window, rope_theta=rope_theta)
        dlam = g["dlam"] if lam is not None else None
        dgain = g["dgain"] if gain is not None else None
        return (g["dq1"], g["dq2"], g["dk1"], g["dk2"], g["dv"], dlam, dgain, g.get("dlam_logits"),
                g.get("dgate"), None, None, None, None, None, None)


def diff_attention(q1, q2, k1, k2, v, lam, gain=None, *, scale=0.125, eps=1e-5, causal=True,
                   apply_norm=True, lam_logits=None, gate=None, window=0, rope_theta=0.0):
    """Differentiable differential attention (bf16 q1, k1 [B,N,H,64], q2, k2
    [B,N,H_N,64], v [B,N,H_V,128]; fp32 lam [H] and gain [H,128]; optional
    lambda logits fp32 [B,N,H], gate logits bf16 [B,N,H,128], a causal
    window, a rotary base); gradients flow to every tensor input."""
    return DiffAttention.apply(q1, q2, k1, k2, v, lam, gain, lam_logits, gate, scale, eps, causal,
                               apply_norm, window, rope_theta)

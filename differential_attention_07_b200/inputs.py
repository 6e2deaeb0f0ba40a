"""Seeded synthetic inputs for the differential-attention forward pass.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic, so both the CUDA path's tests and the float64 oracle can
be fed from it.  Tensors are created on the CPU; callers move them.

Recipe (the same for every workload):

* A CPU ``torch.Generator`` seeded with the workload's seed.
* Draw order: Q1, Q2, K1, K2, V as float32 ``randn`` in logical
  ``[B, heads, N, dim]`` order, each rounded to bf16 (round to nearest even);
  then lambda (float32 uniform per signal head); then the RMS gain
  (float32 ``1 + 0.1 * randn`` of shape ``[H, dv]``, or ones).
* Gated workloads (Motif 3's token-dependent lambda and output gate) draw,
  from a second generator seeded with seed + 1000, lambda logits (float32
  ``1.5 * randn``, [B, N, H]) and gate logits (``2 * randn`` rounded to
  bf16, [B, N, H, 128]); see ``gate_inputs``.
* The tensors handed out are permuted to the token-major layout
  ``[B, N, heads, dim]`` (``.contiguous()``), which is what the prefill entry
  points read.  Decode tensors stay head-major: q ``[B, H, d]``, K/V
  ``[B, H, L, dim]``.

Shapes follow Motif 2.6B's attention (hidden 2048, 16 heads, no GQA; context
4,096 and 16,384; Motif 2.6B explainer, section "The block"; edgentiq blog),
split per head into two 64-wide Q/K maps and one 128-wide V.
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """One named workload: shapes, lambda / gain recipe and seed."""
    name: str
    kind: str                      # "prefill" | "grouped" | "decode"
    B: int
    N: int                         # query length (prefill) or KV-cache length (decode)
    H: int                         # signal heads
    H_N: int                       # noise heads (== H unless grouped)
    H_V: int                       # V heads (== H unless grouped)
    d: int = 64
    dv: int = 128
    scale: float = 0.125
    eps: float = 1e-5
    lam: Tuple[float, float] = (0.8, 0.8)   # uniform range per signal head
    lam_head0: Optional[float] = None        # overrides lambda of head 0
    gain_std: float = 0.0                    # 0 => gain of ones
    seed: int = 0
    causal: bool = True
    gated: bool = False            # token-dependent lambda logits and output-gate logits
    apply_norm: bool = True
    window: int = 0                # causal sliding window in keys (0 = none)
    rope_theta: float = 0.0        # rotary embedding base (0 = none)


WORKLOADS = {
    "tiny": Workload("tiny", "prefill", B=1, N=128, H=2, H_N=2, H_V=2, lam=(0.8, 0.8),
                     gain_std=0.0, seed=0),
    "motif4k": Workload("motif4k", "prefill", B=4, N=4096, H=16, H_N=16, H_V=16,
                        lam=(0.2, 0.8), gain_std=0.1, seed=1),
    "lc16k": Workload("lc16k", "prefill", B=1, N=16384, H=16, H_N=16, H_V=16, lam=(0.0, 0.8),
                      lam_head0=0.0, gain_std=0.1, seed=2),
    "grouped": Workload("grouped", "grouped", B=2, N=4096, H=24, H_N=8, H_V=8, lam=(0.2, 0.8),
                        gain_std=0.0, seed=3),
    "decode": Workload("decode", "decode", B=64, N=8192, H=16, H_N=16, H_V=16, lam=(0.2, 0.8),
                       gain_std=0.1, seed=4),
    # Motif-3-style attention output (Motif 3 summary, section 2.2): grouped
    # heads, token-dependent lambda, output gate, no norm.
    "gated": Workload("gated", "grouped", B=2, N=4096, H=24, H_N=8, H_V=8, lam=(0.2, 0.8),
                      gain_std=0.0, seed=5, gated=True, apply_norm=False),
    # A sliding-window layer (Motif 3 summary: 128-token windows) over the
    # long-context shape.
    "swa16k": Workload("swa16k", "prefill", B=1, N=16384, H=16, H_N=16, H_V=16, lam=(0.2, 0.8),
                       gain_std=0.1, seed=6, window=128),
    # The 4K shape with Motif 2.6B's rotary embedding (theta = 500,000)
    # applied by the library.
    "rope4k": Workload("rope4k", "prefill", B=4, N=4096, H=16, H_N=16, H_V=16, lam=(0.2, 0.8),
                       gain_std=0.1, seed=7, rope_theta=500000.0),
}


def _lam_gain(g: torch.Generator, H: int, dv: int, lam, lam_head0, gain_std):
    lo, hi = lam
    lamv = lo + (hi - lo) * torch.rand(H, generator=g, dtype=torch.float32)
    if lam_head0 is not None:
        lamv[0] = lam_head0
    if gain_std > 0:
        gain = 1.0 + gain_std * torch.randn(H, dv, generator=g, dtype=torch.float32)
    else:
        gain = torch.ones(H, dv, dtype=torch.float32)
    return lamv, gain


def _randn_bf16(g, shape):
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def prefill_inputs(B, N, H, H_N=None, H_V=None, d=64, dv=128, *, seed=0, lam=(0.8, 0.8),
                   lam_head0=None, gain_std=0.0):
    """Q1,K1 [B,N,H,d]; Q2,K2 [B,N,H_N,d]; V [B,N,H_V,dv] bf16; lam [H]; gain [H,dv]."""
    H_N = H if H_N is None else H_N
    H_V = H if H_V is None else H_V
    g = torch.Generator().manual_seed(seed)
    q1 = _randn_bf16(g, (B, H, N, d))
    q2 = _randn_bf16(g, (B, H_N, N, d))
    k1 = _randn_bf16(g, (B, H, N, d))
    k2 = _randn_bf16(g, (B, H_N, N, d))
    v = _randn_bf16(g, (B, H_V, N, dv))
    lamv, gain = _lam_gain(g, H, dv, lam, lam_head0, gain_std)
    tok = lambda t: t.permute(0, 2, 1, 3).contiguous()
    return dict(q1=tok(q1), q2=tok(q2), k1=tok(k1), k2=tok(k2), v=tok(v), lam=lamv, gain=gain)


def decode_inputs(B, L, H, d=64, dv=128, *, seed=0, lam=(0.2, 0.8), lam_head0=None,
                  gain_std=0.0):
    """q1,q2 [B,H,d]; K1,K2 [B,H,L,d]; V [B,H,L,dv] bf16; lam [H]; gain [H,dv]."""
    g = torch.Generator().manual_seed(seed)
    q1 = _randn_bf16(g, (B, H, d))
    q2 = _randn_bf16(g, (B, H, d))
    k1 = _randn_bf16(g, (B, H, L, d))
    k2 = _randn_bf16(g, (B, H, L, d))
    v = _randn_bf16(g, (B, H, L, dv))
    lamv, gain = _lam_gain(g, H, dv, lam, lam_head0, gain_std)
    return dict(q1=q1, q2=q2, k1=k1, k2=k2, v=v, lam=lamv, gain=gain)


def gate_inputs(B, N, H, dv=128, *, seed=0, lam_logit_std=1.5, gate_std=2.0):
    """Token-dependent lambda logits and output-gate logits (random draws).

    A generator seeded with ``seed + 1000``: lambda logits float32 ``randn *
    lam_logit_std`` of shape [B, N, H] (prefill) or [B, H] (N = None,
    decode), then gate logits ``randn * gate_std`` rounded to bf16, [B, N, H,
    dv] or [B, H, dv].  These stand for the outputs of the projections
    x_t W^lambda and c_t^Q W^G."""
    g = torch.Generator().manual_seed(seed + 1000)
    lead = (B, H) if N is None else (B, N, H)
    lam_logits = lam_logit_std * torch.randn(*lead, generator=g, dtype=torch.float32)
    gate = (gate_std * torch.randn(*lead, dv, generator=g, dtype=torch.float32)).to(torch.bfloat16)
    return dict(lam_logits=lam_logits, gate=gate)


def grad_output(B, N, H, dv=128, *, seed=0, std=1.0):
    """Gradient of a loss with respect to the prefill output, dY [B, N, H, dv]
    bf16: a generator seeded with ``seed + 2000``, ``randn * std`` rounded to
    bf16 (the upstream gradient a training step hands the backward pass)."""
    g = torch.Generator().manual_seed(seed + 2000)
    return (std * torch.randn(B, N, H, dv, generator=g, dtype=torch.float32)).to(torch.bfloat16)


def workload_inputs(w: Workload):
    """Inputs of a named workload (CPU tensors)."""
    if w.kind == "decode":
        x = decode_inputs(w.B, w.N, w.H, w.d, w.dv, seed=w.seed, lam=w.lam,
                          lam_head0=w.lam_head0, gain_std=w.gain_std)
        if w.gated:
            x.update(gate_inputs(w.B, None, w.H, w.dv, seed=w.seed))
        return x
    x = prefill_inputs(w.B, w.N, w.H, w.H_N, w.H_V, w.d, w.dv, seed=w.seed, lam=w.lam,
                       lam_head0=w.lam_head0, gain_std=w.gain_std)
    if w.gated:
        x.update(gate_inputs(w.B, w.N, w.H, w.dv, seed=w.seed))
    return x


def sample_rows(B, N, H, count, seed=0, tile=128):
    """(b, i, h) triples for sampled parity checks at full size.

    Always includes the first and last query rows and rows on each side of the
    first few tile boundaries; the rest are drawn uniformly.  Returns an int64
    tensor [R, 3].
    """
    g = torch.Generator().manual_seed(seed + 12345)
    fixed = []
    for i in {0, 1, tile - 1, tile, tile + 1, 2 * tile - 1, N // 2, N - 2, N - 1}:
        if 0 <= i < N:
            fixed.append((0, i, 0))
            fixed.append((B - 1, i, H - 1))
    n_rand = max(0, count - len(fixed))
    b = torch.randint(0, B, (n_rand,), generator=g)
    i = torch.randint(0, N, (n_rand,), generator=g)
    h = torch.randint(0, H, (n_rand,), generator=g)
    rows = torch.tensor(fixed, dtype=torch.int64).reshape(-1, 3)
    rnd = torch.stack([b, i, h], dim=1).to(torch.int64)
    return torch.cat([rows, rnd], dim=0)

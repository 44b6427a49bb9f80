"""Seeded synthetic inputs for the delta-rule sequence mixer.

This module only draws random numbers in the shapes and distributions of the
workloads; it holds none of the method's arithmetic, and both the CUDA path
and the CPU oracle are fed from it.

Recipe (draw order fixed: q, k, v, beta, alpha):
  q, v  ~ N(0, 1)
  k     ~ N(0, 1), then L2-normalised per (token, head) in float32
  beta  = sigmoid(N(0, 1))                 float32, one per (b, h, t)
  alpha = exp(-softplus(N(0, 1)))          float32 in (0, 1), one per (b, h, t)
                                           (per-dimension gate: one per (b, h, t, i))
Inputs of the calls that apply the layer's pre-step themselves ("raw"): k is
left unnormalised and beta is the N(0, 1) logit itself.
q, k, v are stored in ``dtype`` (float32 or bfloat16) after the float32 draw.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    Dk: int
    Dv: int
    dtype: torch.dtype
    C: int = 64
    gated: bool = False


# The workloads the library is measured and checked on (sizes as named).
TINY = Workload("tiny DeltaNet forward B1 H2 T256 D64 fp32 C64", 1, 2, 256, 64, 64, torch.float32)
PREFILL = Workload("prefill DeltaNet forward B4 H16 T4096 D128 bf16 C64", 4, 16, 4096, 128, 128,
                   torch.bfloat16)
PREFILL_LINEAR = Workload("prefill ELU+1 linear attention B4 H16 T4096 D128 bf16 C64", 4, 16, 4096,
                          128, 128, torch.bfloat16)
LONG64 = Workload("long-context DeltaNet forward B1 H32 T65536 D128 bf16 C64", 1, 32, 65536, 128,
                  128, torch.bfloat16, C=64)
LONG128 = Workload("long-context DeltaNet forward B1 H32 T65536 D128 bf16 C128", 1, 32, 65536, 128,
                   128, torch.bfloat16, C=128)
FORGET = Workload("gated (forgetting) DeltaNet forward B8 H16 T8192 D128 bf16 C64", 8, 16, 8192,
                  128, 128, torch.bfloat16, gated=True)
# Batched decode: 256 sequences x 32 heads, D128, fp32 state from a 512-token
# prefill, then single-token steps with fresh q, k, v, beta each step.
DECODE_SEQS, DECODE_HEADS, DECODE_PREFILL, DECODE_STEPS = 256, 32, 512, 1024


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(B, H, T, Dk, Dv, dtype=torch.bfloat16, gated=False, seed=0, device="cpu",
                raw=False, gate_per_dim=False):
    """Return dict(q, k, v, beta, alpha) drawn with the recipe above.

    ``alpha`` is None unless ``gated``; with ``gate_per_dim`` it has one decay
    per key dimension, shape (B,H,T,Dk), drawn the same way.  ``raw`` leaves k
    unnormalised and beta as its N(0,1) logit (the inputs of the call that
    applies the layer's maps itself).  All tensors are contiguous on ``device``.
    """
    g = _gen(seed, device)
    q = torch.randn(B, H, T, Dk, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(B, H, T, Dk, generator=g, device=device, dtype=torch.float32)
    if not raw:
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    v = torch.randn(B, H, T, Dv, generator=g, device=device, dtype=torch.float32)
    beta = torch.randn(B, H, T, generator=g, device=device, dtype=torch.float32)
    if not raw:
        beta = torch.sigmoid(beta)
    alpha = None
    if gated:
        shape = (B, H, T, Dk) if gate_per_dim else (B, H, T)
        x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
        alpha = torch.exp(-torch.nn.functional.softplus(x))
    return dict(q=q.to(dtype).contiguous(), k=k.to(dtype).contiguous(),
                v=v.to(dtype).contiguous(), beta=beta.contiguous(),
                alpha=None if alpha is None else alpha.contiguous())


def make_workload(w: Workload, seed=0, device="cpu"):
    return make_inputs(w.B, w.H, w.T, w.Dk, w.Dv, w.dtype, w.gated, seed, device)


def make_decode_step_inputs(B, H, Dk, Dv, dtype=torch.bfloat16, gated=False, seed=0,
                            device="cpu", raw=False, gate_per_dim=False):
    """One decode step's q, k, v (B,H,D), beta (B,H) and optional alpha (B,H)
    (or (B,H,Dk) with ``gate_per_dim``)."""
    d = make_inputs(B, H, 1, Dk, Dv, dtype, gated, seed, device, raw, gate_per_dim)
    return {n: (None if t is None else t.reshape(t.shape[:2] + t.shape[3:]).contiguous())
            for n, t in d.items()}

"""Seeded synthetic inputs for the GLA / GSA operators.

This module only draws random numbers; it holds none of the operator's arithmetic.  The
same draws feed the CUDA library and the fp64 oracle used by the tests.

Recipe (fixed draw order from one CPU ``torch.Generator`` seeded with ``seed``):
    q, k, v, x, [phi], [dO]   each ~ N(0, 1) in float32
    q *= d_k ** -0.5                       (queries pre-scaled; the operator has no scale)
    x += gate_mu                           (gate-bias sweep; 0 by default)
    g  = logsigmoid(x) / gate_tau          (log-decay, alpha = exp(g) in (0, 1))
Then every tensor is rounded once to the compute dtype (bf16 or fp32).  The oracle receives
the rounded values widened to float64, so both sides see identical inputs.

Gate temperatures: tau = 16 for GLA (alpha = sigmoid(x)^(1/16)), tau = 8 for GSA's per-slot
forget gate (alpha = sigmoid(x)^(1/8)).
"""
from __future__ import annotations

import dataclasses

import torch

__all__ = ["GLAShape", "GSAShape", "CONFIGS", "make_gla_inputs", "make_gsa_inputs"]


@dataclasses.dataclass(frozen=True)
class GLAShape:
    B: int
    H: int
    T: int
    dk: int
    dv: int
    chunk: int = 64
    dtype: torch.dtype = torch.bfloat16
    gate_mu: float = 0.0


@dataclasses.dataclass(frozen=True)
class GSAShape:
    B: int
    H: int
    T: int
    dk: int
    dv: int
    m: int
    chunk: int = 64
    dtype: torch.dtype = torch.bfloat16


# The five workloads: a small fp32 forward, the 340M- and 1.3B-model layer shapes, a long
# sequence (32768 tokens, then 256 decode steps) and GSA with 64 slots.
CONFIGS = {
    "gla_fwd_fp32_small": GLAShape(1, 2, 256, 64, 64, 64, torch.float32),
    "gla_340m": GLAShape(8, 4, 2048, 128, 256, 64, torch.bfloat16),
    "gla_1p3b": GLAShape(8, 4, 2048, 256, 512, 64, torch.bfloat16),
    "gla_long": GLAShape(1, 4, 32768, 128, 256, 64, torch.bfloat16),
    "gsa_64slots": GSAShape(4, 4, 4096, 128, 128, 64, 64, torch.bfloat16),
}


def _randn(gen, shape):
    return torch.randn(shape, generator=gen, dtype=torch.float32)


def make_gla_inputs(B, H, T, dk, dv, dtype=torch.bfloat16, seed=0, gate_mu=0.0,
                    gate_tau=16.0, with_do=True, with_h0=False, with_dhT=False):
    """CPU tensors q, k, g [B,H,T,dk], v [B,H,T,dv] (and dO, h0, dhT) in ``dtype``.

    h0 / dhT, when requested, are float32 [B,H,dk,dv] drawn after dO.
    """
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, H, T, dk)) * dk ** -0.5
    k = _randn(gen, (B, H, T, dk))
    v = _randn(gen, (B, H, T, dv))
    x = _randn(gen, (B, H, T, dk)) + gate_mu
    out = {"q": q, "k": k, "v": v, "g": torch.nn.functional.logsigmoid(x) / gate_tau}
    if with_do:
        out["do"] = _randn(gen, (B, H, T, dv))
    out = {n: t.to(dtype) for n, t in out.items()}
    if with_h0:
        out["h0"] = _randn(gen, (B, H, dk, dv))
    if with_dhT:
        out["dhT"] = _randn(gen, (B, H, dk, dv))
    return out


def make_gsa_inputs(B, H, T, dk, dv, m, dtype=torch.bfloat16, seed=0, gate_tau=8.0,
                    with_do=True):
    """CPU tensors q, k [B,H,T,dk], v [B,H,T,dv], phi, g [B,H,T,m] (and dO) in ``dtype``."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn(gen, (B, H, T, dk)) * dk ** -0.5
    k = _randn(gen, (B, H, T, dk))
    v = _randn(gen, (B, H, T, dv))
    x = _randn(gen, (B, H, T, m))
    phi = _randn(gen, (B, H, T, m))
    out = {"q": q, "k": k, "v": v, "g": torch.nn.functional.logsigmoid(x) / gate_tau,
           "phi": phi}
    if with_do:
        out["do"] = _randn(gen, (B, H, T, dv))
    return {n: t.to(dtype) for n, t in out.items()}

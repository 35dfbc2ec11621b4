"""Plain fp64 CPU oracle for the elementwise pieces around the GLA operator.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs use it.  It shares no code with
the CUDA library and never calls it.

* Raw-logit gate.  The GLA gate is data dependent and taken in log space, g = log(alpha) <= 0
  ("MS-GLA: Multi-Scale Gated Linear Attention ...", section 2.1: a data-dependent forget gate;
  "Gated Slot Attention ...", "Approach": per-slot forget gates from a sigmoid).  The benchmark
  shapes build it as g = logsigmoid(x) / tau (tau = 16 for GLA, 8 for GSA, where
  alpha = sigmoid(x)^(1/8)).  ``gate_logsigmoid`` is that definition; ``gate_logsigmoid_bwd`` is
  its derivative d g / d x = sigmoid(-x) / tau applied to an upstream gradient.
* MS-GLA temporal pooling and causal hold ("MS-GLA ...", sections 3.1 and 3.3).  A scale s
  averages non-overlapping blocks of s tokens (the last block may be short: padding positions
  are masked out of the mean), giving ceil(T / s) pooled tokens.  The pooled branch's outputs
  are brought back to token resolution by a causal hold: a block's output becomes visible once
  every token of the block has been seen, i.e. token t receives block floor((t + 1) / s) - 1
  (nothing, i.e. zeros, before the first block completes).  The backward passes are the
  adjoints (transposes) of these two linear maps.

All arrays are [B, H, T, D] (pooled: [B, H, ceil(T/s), D]).  Everything is float64.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = ["gate_logsigmoid", "gate_logsigmoid_bwd", "msgla_pool", "msgla_pool_bwd", "msgla_hold",
           "msgla_hold_bwd"]


def gate_logsigmoid(x, tau):
    """g = log(sigmoid(x)) / tau, element by element (stable for large |x|)."""
    x = np.asarray(x, dtype=np.float64)
    return (np.minimum(x, 0.0) - np.log1p(np.exp(-np.abs(x)))) / tau


def gate_logsigmoid_bwd(x, dg, tau):
    """dx = dg * sigmoid(-x) / tau  (d/dx log sigmoid(x) = 1 - sigmoid(x) = sigmoid(-x))."""
    x = np.asarray(x, dtype=np.float64)
    dg = np.asarray(dg, dtype=np.float64)
    sig_neg = np.where(x >= 0, np.exp(-np.abs(x)) / (1.0 + np.exp(-np.abs(x))), 1.0 / (1.0 + np.exp(-np.abs(x))))
    return dg * sig_neg / tau


def _blocks(T, s):
    return [(p * s, min(T, (p + 1) * s)) for p in range(math.ceil(T / s))]


def msgla_pool(x, s):
    """Average of each block of s tokens (a short last block averages only its real tokens)."""
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[-2]
    out = np.zeros(x.shape[:-2] + (math.ceil(T / s), x.shape[-1]))
    for p, (a, b) in enumerate(_blocks(T, s)):
        out[..., p, :] = x[..., a:b, :].mean(axis=-2)
    return out


def msgla_pool_bwd(dy, T, s):
    """Adjoint of msgla_pool: each token of block p receives dy_p / (tokens in block p)."""
    dy = np.asarray(dy, dtype=np.float64)
    dx = np.zeros(dy.shape[:-2] + (T, dy.shape[-1]))
    for p, (a, b) in enumerate(_blocks(T, s)):
        dx[..., a:b, :] = dy[..., p : p + 1, :] / (b - a)
    return dx


def msgla_hold(y, T, s):
    """Token t gets pooled output floor((t + 1) / s) - 1, or zeros before the first full block."""
    y = np.asarray(y, dtype=np.float64)
    out = np.zeros(y.shape[:-2] + (T, y.shape[-1]))
    for t in range(T):
        p = (t + 1) // s - 1
        if p >= 0:
            out[..., t, :] = y[..., p, :]
    return out


def msgla_hold_bwd(dout, s):
    """Adjoint of msgla_hold: pooled output p collects the gradients of the tokens that read it."""
    dout = np.asarray(dout, dtype=np.float64)
    T = dout.shape[-2]
    dy = np.zeros(dout.shape[:-2] + (math.ceil(T / s), dout.shape[-1]))
    for t in range(T):
        p = (t + 1) // s - 1
        if p >= 0:
            dy[..., p, :] += dout[..., t, :]
    return dy

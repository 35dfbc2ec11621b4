"""Plain fp64 CPU oracle for chunkwise Gated Linear Attention (GLA) and Gated Slot Attention (GSA).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module: only the
tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` use it.  It shares no code with the CUDA library and never calls it.

What it computes, and where each piece comes from
-------------------------------------------------
* GLA is a linear recurrence over a matrix-valued memory with a data-dependent,
  per-key-dimension ("row-wise") forget gate:

      S_t = diag(alpha_t) . S_{t-1} + k_t^T v_t ,    o_t = q_t . S_t ,    alpha_t = exp(g_t)

  with q_t, k_t, g_t in R^{d_k}, v_t in R^{d_v}, S_t in R^{d_k x d_v}.
  Source: "Gated Linear Attention for Efficient Long Sequences", panels "Core move"
  (gated recurrent memory updates replace softmax attention) and "Step-by-step memory
  update: plain linear attention vs GLA" (the gate keeps, decays or overwrites features of a
  matrix memory); "MS-GLA: Multi-Scale Gated Linear Attention ...", section 2.1 (GLA adds a
  data-dependent forget gate to the linear-attention recurrence; the gate scales rows).
  The recurrence is the operator's definition, so the oracle is that definition written out
  step by step (``gla_fwd``).
* Chunkwise form: "MS-GLA", section 2.1 (chunks processed with sequential inter-chunk updates
  and parallel intra-chunk computation) and section 3.4.  ``gla_chunked_fwd`` is the plain
  textbook chunk form, used only to check that chunking leaves the result unchanged.
* Recurrent inference, O(1) memory per token: "MS-GLA", section 1; "Gated Slot Attention for
  Efficient Linear-Time Sequence Modeling", abstract.  ``gla_decode_step``.
* GSA: "Gated Slot Attention ...", abstract (a two-layer GLA linked through a softmax) and
  "Approach" (two-pass linear attention with a softmax in between, data-dependent forget gates
  per memory slot).  ``gsa_fwd`` / ``gsa_bwd``.
* Backward passes are reverse-mode recurrences derived by hand from the forward recurrences;
  the derivation is given in each docstring.  They are pinned by finite differences.

Readings taken where the pages are silent (each is listed in the design doc):
  1. o_t reads S_t after token t has been written (inclusive causal readout).
  2. alpha_t multiplies S_{t-1} before k_t^T v_t is added.
  3. The gate acts on the key axis (rows of S) for GLA; for GSA pass 1 it acts on the slot
     axis, which is the value axis of that pass, and for pass 2 on the slot axis, which is the
     key axis of that pass.
  4. The operator takes the log-gate g (alpha = exp g); no scale is applied inside.
  5. GSA pass 2 uses queries p = softmax(o1) over the m slots and keys phi.

All arrays are laid out [B, H, T, D]; states are [B, H, d_k, d_v].  Everything is float64.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "gla_fwd",
    "gla_bwd",
    "gla_chunked_fwd",
    "gla_decode_step",
    "gla_value_gated_fwd",
    "gla_value_gated_bwd",
    "softmax",
    "gsa_fwd",
    "gsa_bwd",
    "dg_from_identity",
]


def _f64(x):
    return None if x is None else np.array(x, dtype=np.float64, copy=True)


def _zeros_state(q, dv):
    B, H, _, dk = q.shape
    return np.zeros((B, H, dk, dv), dtype=np.float64)


# ----------------------------------------------------------------------------------------
# GLA (gate on the key axis)
# ----------------------------------------------------------------------------------------
def gla_fwd(q, k, v, g, h0=None):
    """Step-by-step GLA recurrence (the operator's definition).

    S_0 = h0 (zeros if None); for t = 1..T:
        S_t[i, j] = exp(g_t[i]) * S_{t-1}[i, j] + k_t[i] * v_t[j]
        o_t[j]    = sum_i q_t[i] * S_t[i, j]
    Returns (o [B,H,T,dv], hT = S_T [B,H,dk,dv]).
    Follows "Gated Linear Attention for Efficient Long Sequences", "Step-by-step memory update",
    and "MS-GLA", section 2.1 (row-wise data-dependent forget gate).
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    T, dv = q.shape[2], v.shape[3]
    S = _zeros_state(q, dv) if h0 is None else _f64(h0)
    o = np.empty(q.shape[:3] + (dv,), dtype=np.float64)
    for t in range(T):
        alpha = np.exp(g[:, :, t, :])
        S = alpha[..., :, None] * S + k[:, :, t, :, None] * v[:, :, t, None, :]
        o[:, :, t, :] = np.einsum("bhi,bhij->bhj", q[:, :, t, :], S)
    return o, S


def gla_bwd(q, k, v, g, h0, do, dhT=None, ckpt=32):
    """Reverse-mode recurrence for ``gla_fwd``, derived by hand.

    With D_t = dL/dS_t (all paths): D_T = dhT + q_T^T do_T and
        D_t   = q_t^T do_t + diag(alpha_{t+1}) D_{t+1}
        dq_t  = S_t do_t^T            (dq_t[i] = sum_j S_t[i,j] do_t[j])
        dk_t  = D_t v_t^T             (dk_t[i] = sum_j D_t[i,j] v_t[j])
        dv_t  = k_t D_t               (dv_t[j] = sum_i k_t[i] D_t[i,j])
        dg_t  = alpha_t * dalpha_t,   dalpha_t[i] = sum_j D_t[i,j] S_{t-1}[i,j]
        dh0   = diag(alpha_1) D_1
    States are re-derived forward from checkpoints every ``ckpt`` steps, so memory stays
    O(ckpt) states.  Returns (dq, dk, dv, dg, dh0).
    """
    q, k, v, g, do = _f64(q), _f64(k), _f64(v), _f64(g), _f64(do)
    T, dv = q.shape[2], v.shape[3]
    S = _zeros_state(q, dv) if h0 is None else _f64(h0)
    alpha = np.exp(g)
    ckpts = {}
    for t in range(T):
        if t % ckpt == 0:
            ckpts[t] = S.copy()
        S = alpha[:, :, t, :, None] * S + k[:, :, t, :, None] * v[:, :, t, None, :]
    D = np.zeros_like(S) if dhT is None else _f64(dhT)
    dq, dk, dg = np.zeros_like(q), np.zeros_like(k), np.zeros_like(g)
    dvv = np.zeros_like(v)
    for s0 in reversed(range(0, T, ckpt)):
        s1 = min(s0 + ckpt, T)
        S = ckpts[s0].copy()
        prev = []
        for t in range(s0, s1):
            prev.append(S)
            S = alpha[:, :, t, :, None] * S + k[:, :, t, :, None] * v[:, :, t, None, :]
        for t in reversed(range(s0, s1)):
            S_prev = prev[t - s0]
            S_t = alpha[:, :, t, :, None] * S_prev + k[:, :, t, :, None] * v[:, :, t, None, :]
            D = D + q[:, :, t, :, None] * do[:, :, t, None, :]
            dq[:, :, t, :] = np.einsum("bhij,bhj->bhi", S_t, do[:, :, t, :])
            dk[:, :, t, :] = np.einsum("bhij,bhj->bhi", D, v[:, :, t, :])
            dvv[:, :, t, :] = np.einsum("bhi,bhij->bhj", k[:, :, t, :], D)
            dg[:, :, t, :] = alpha[:, :, t, :] * np.einsum("bhij,bhij->bhi", D, S_prev)
            D = alpha[:, :, t, :, None] * D
    return dq, dk, dvv, dg, D


def dg_from_identity(q, k, dq, dk, hT, dhT=None):
    """Gate gradient from the cumulative-sum identity instead of the direct d(alpha) route.

    With b_t = sum_{s<=t} g_s, o depends on b through exp(b_t - b_s) factors, so
    dL/db_t = q_t*dq_t - k_t*dk_t (+ sum_j dhT[i,j] hT[i,j] at t = T), and
    dg_t = sum_{s>=t} dL/db_s.  Used only as an independent cross-check of ``gla_bwd``.
    """
    db = _f64(q) * _f64(dq) - _f64(k) * _f64(dk)
    if dhT is not None:
        db[:, :, -1, :] += np.einsum("bhij,bhij->bhi", _f64(dhT), _f64(hT))
    return np.flip(np.cumsum(np.flip(db, axis=2), axis=2), axis=2)


def gla_chunked_fwd(q, k, v, g, h0=None, chunk=64):
    """Textbook chunkwise form of ``gla_fwd`` (no sub-chunking), for the invariance check.

    For each chunk of L <= chunk tokens with local inclusive cumulative log-gates
    Bc_j = sum_{r<=j} g_r and gamma = Bc_L:
        o_j   = (q_j * exp(Bc_j)) S_in + sum_{r<=j} [sum_d q_jd k_rd exp(Bc_jd - Bc_rd)] v_r
        S_out = diag(exp(gamma)) S_in + sum_r (k_r * exp(gamma - Bc_r))^T v_r
    "MS-GLA", section 2.1: sequential across chunks, parallel inside a chunk.
    """
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    T, dv = q.shape[2], v.shape[3]
    S = _zeros_state(q, dv) if h0 is None else _f64(h0)
    o = np.empty(q.shape[:3] + (dv,), dtype=np.float64)
    for s0 in range(0, T, chunk):
        s1 = min(s0 + chunk, T)
        L = s1 - s0
        qc, kc, vc = q[:, :, s0:s1], k[:, :, s0:s1], v[:, :, s0:s1]
        Bc = np.cumsum(g[:, :, s0:s1], axis=2)
        gamma = Bc[:, :, -1, :]
        causal = np.tril(np.ones((L, L), dtype=bool))
        diff = Bc[:, :, :, None, :] - Bc[:, :, None, :, :]  # [B,H,j,r,d]
        decay = np.exp(np.where(causal[None, None, :, :, None], diff, -np.inf))
        A = np.einsum("bhjd,bhrd,bhjrd->bhjr", qc, kc, decay)
        o[:, :, s0:s1] = np.einsum("bhjd,bhdv->bhjv", qc * np.exp(Bc), S) + np.einsum(
            "bhjr,bhrv->bhjv", A, vc
        )
        S = np.exp(gamma)[..., None] * S + np.einsum(
            "bhrd,bhrv->bhdv", kc * np.exp(gamma[:, :, None, :] - Bc), vc
        )
    return o, S


def gla_decode_step(q, k, v, g, S):
    """One recurrent-inference step: S <- diag(exp g) S + k^T v ;  o = q S.

    q, k, g: [B,H,dk]; v: [B,H,dv]; S: [B,H,dk,dv].  Returns (o [B,H,dv], S_new).
    "MS-GLA", section 1 (O(1) inference memory); "Gated Slot Attention ...", abstract
    (efficient recurrent inference).
    """
    q, k, v, g, S = _f64(q), _f64(k), _f64(v), _f64(g), _f64(S)
    S = np.exp(g)[..., :, None] * S + k[..., :, None] * v[..., None, :]
    return np.einsum("bhi,bhij->bhj", q, S), S


# ----------------------------------------------------------------------------------------
# Value-gated GLA (GSA pass 1: gate on the slot axis, which is the value axis of the pass)
# ----------------------------------------------------------------------------------------
def gla_value_gated_fwd(q, k, phi, g, h0=None):
    """S_t = S_{t-1} diag(alpha_t) + k_t^T phi_t ;  o1_t = q_t S_t ;  alpha_t = exp(g_t).

    q, k: [B,H,T,dk]; phi, g: [B,H,T,m]; S: [B,H,dk,m].  Returns (o1 [B,H,T,m], hT).
    "Gated Slot Attention ...", "Approach": each memory slot has its own data-dependent
    forget gate; the slots are written with the slot weights phi.
    """
    q, k, phi, g = _f64(q), _f64(k), _f64(phi), _f64(g)
    T, m = q.shape[2], phi.shape[3]
    S = _zeros_state(q, m) if h0 is None else _f64(h0)
    o = np.empty(q.shape[:3] + (m,), dtype=np.float64)
    for t in range(T):
        alpha = np.exp(g[:, :, t, :])
        S = S * alpha[..., None, :] + k[:, :, t, :, None] * phi[:, :, t, None, :]
        o[:, :, t, :] = np.einsum("bhi,bhis->bhs", q[:, :, t, :], S)
    return o, S


def gla_value_gated_bwd(q, k, phi, g, h0, do1, dhT=None):
    """Reverse mode of ``gla_value_gated_fwd``, derived by hand.

    D_t = dL/dS_t:  D_T = dhT + q_T^T do1_T,  D_t = q_t^T do1_t + D_{t+1} diag(alpha_{t+1})
        dq_t[i]   = sum_s S_t[i,s] do1_t[s]
        dk_t[i]   = sum_s D_t[i,s] phi_t[s]
        dphi_t[s] = sum_i k_t[i] D_t[i,s]
        dg_t[s]   = alpha_t[s] * sum_i D_t[i,s] S_{t-1}[i,s]
        dh0       = D_1 diag(alpha_1)
    Returns (dq, dk, dphi, dg, dh0).
    """
    q, k, phi, g, do1 = _f64(q), _f64(k), _f64(phi), _f64(g), _f64(do1)
    T, m = q.shape[2], phi.shape[3]
    S = _zeros_state(q, m) if h0 is None else _f64(h0)
    alpha = np.exp(g)
    states = [S]
    for t in range(T):
        S = S * alpha[:, :, t, None, :] + k[:, :, t, :, None] * phi[:, :, t, None, :]
        states.append(S)
    D = np.zeros_like(S) if dhT is None else _f64(dhT)
    dq, dk = np.zeros_like(q), np.zeros_like(k)
    dphi, dg = np.zeros_like(phi), np.zeros_like(g)
    for t in reversed(range(T)):
        S_prev, S_t = states[t], states[t + 1]
        D = D + q[:, :, t, :, None] * do1[:, :, t, None, :]
        dq[:, :, t, :] = np.einsum("bhis,bhs->bhi", S_t, do1[:, :, t, :])
        dk[:, :, t, :] = np.einsum("bhis,bhs->bhi", D, phi[:, :, t, :])
        dphi[:, :, t, :] = np.einsum("bhi,bhis->bhs", k[:, :, t, :], D)
        dg[:, :, t, :] = alpha[:, :, t, :] * np.einsum("bhis,bhis->bhs", D, S_prev)
        D = D * alpha[:, :, t, None, :]
    return dq, dk, dphi, dg, D


# ----------------------------------------------------------------------------------------
# GSA: two GLA passes joined by a softmax over the m slots
# ----------------------------------------------------------------------------------------
def softmax(x, axis=-1):
    x = _f64(x)
    z = np.exp(x - x.max(axis=axis, keepdims=True))
    return z / z.sum(axis=axis, keepdims=True)


def gsa_fwd(q, k, v, phi, g, h0_1=None, h0_2=None):
    """Gated Slot Attention forward.

    pass 1 (value-gated GLA, d_k -> m):  o1 = GLA_v(q, k, phi, g)
    slot softmax:                         p  = softmax_m(o1)
    pass 2 (key-gated GLA, m -> d_v):     o  = GLA(p, phi, v, g)   (same slot gates)
    Returns (o, p, hT1 [B,H,dk,m], hT2 [B,H,m,dv]).
    "Gated Slot Attention ...", abstract (two-layer GLA linked via softmax) and "Approach".
    """
    o1, hT1 = gla_value_gated_fwd(q, k, phi, g, h0_1)
    p = softmax(o1, axis=-1)
    o, hT2 = gla_fwd(p, phi, v, g, h0_2)
    return o, p, hT1, hT2


def gsa_bwd(q, k, v, phi, g, h0_1, h0_2, do, dhT1=None, dhT2=None):
    """Gated Slot Attention backward: pass-2 reverse mode, softmax Jacobian, pass-1 reverse mode.

    dp, dphi2, dv, dg2, dh0_2 = GLA reverse mode of pass 2
    do1 = p * (dp - <p, dp>)                       (softmax Jacobian over the m slots)
    dq, dk, dphi1, dg1, dh0_1 = value-gated reverse mode of pass 1
    dphi = dphi1 + dphi2 ;  dg = dg1 + dg2
    Returns (dq, dk, dv, dphi, dg, dh0_1, dh0_2).
    """
    o1, _ = gla_value_gated_fwd(q, k, phi, g, h0_1)
    p = softmax(o1, axis=-1)
    dp, dphi2, dv, dg2, dh0_2 = gla_bwd(p, phi, v, g, h0_2, do, dhT2)
    do1 = p * (dp - np.sum(p * dp, axis=-1, keepdims=True))
    dq, dk, dphi1, dg1, dh0_1 = gla_value_gated_bwd(q, k, phi, g, h0_1, do1, dhT1)
    return dq, dk, dv, dphi1 + dphi2, dg1 + dg2, dh0_1, dh0_2

"""The chunk-local form of the gate gradient that the fused backward evaluates, checked in fp64
against the oracle's dg (CPU; no CUDA involved).  For token t at local position tau of chunk i,
with B the chunk-local inclusive cumulative log-gate, gamma = B at the chunk's last token,
Qt = q e^B, Kh = k e^{gamma - B}, X_t = dO_t S_i^T, Z_t = v_t G_{i+1}^T (S_i the state entering
chunk i, G_{i+1} = dL/dS at its end):

    dg_t = c_i + sum_{r<tau} Kh_r Z_r + sum_{j>=tau} Qt_j X_j + sum_{r<tau} (k_r dk^intra_r - q_r dq^intra_r)
    c_i  = e^{gamma_i} rowsum(G_{i+1} * S_i)

and the carry runs backwards inside a segment of chunks [a, b] as
c_b = rowsum(G_{b+1} * S_{b+1}) - K_b, c_i = c_{i+1} + Q_{i+1} - K_i (Q, K the chunk sums of Qt X
and Kh Z).  The unsplit walk is the single segment; the sequence split restarts the carry at every
segment's last chunk.  The decomposition follows from the reverse-mode recurrence of
"MS-GLA", section 2.1 (row-wise gate, sequential across chunks)."""
import numpy as np
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs

C = 64


def _chunk_terms(q, k, v, g, h0, do, dhT):
    """fp64 states at chunk boundaries and the per-token pieces of the decomposition (one head)."""
    T, dk = q.shape
    NC = -(-T // C)
    S = [h0.copy()]
    for i in range(NC):  # forward: state entering each chunk, and after the last one
        s = S[-1].copy()
        for t in range(i * C, min(T, (i + 1) * C)):
            s = np.exp(g[t])[:, None] * s + np.outer(k[t], v[t])
        S.append(s)
    B = np.zeros_like(g)
    for i in range(NC):
        acc = np.zeros(dk)
        for t in range(i * C, min(T, (i + 1) * C)):
            acc = acc + g[t]
            B[t] = acc
    gam = [B[min(T, (i + 1) * C) - 1] for i in range(NC)]
    G = [None] * (NC + 1)
    G[NC] = dhT.copy()
    for i in range(NC - 1, -1, -1):  # reverse: dL/dS entering chunk i
        ts = range(i * C, min(T, (i + 1) * C))
        G[i] = np.exp(gam[i])[:, None] * G[i + 1] + sum(np.outer(q[t] * np.exp(B[t]), do[t]) for t in ts)
    return S, G, B, gam


@pytest.mark.parametrize("segments", [[(0, 2)], [(0, 0), (1, 2)], [(0, 0), (1, 1), (2, 2)]])
def test_chunk_local_gate_gradient_with_segment_carries(segments):
    inp = make_gla_inputs(1, 2, 150, 4, 3, torch.float32, seed=5, with_h0=True, with_dhT=True)
    a = {n: np.asarray(inp[n], dtype=np.float64) for n in ["q", "k", "v", "g", "do", "h0", "dhT"]}
    dq, dk, _, dg_ref, _ = O.gla_bwd(a["q"], a["k"], a["v"], a["g"], a["h0"], a["do"], a["dhT"])
    T = a["q"].shape[2]
    NC = -(-T // C)
    for h in range(2):
        q, k, v, g, do = (a[n][0, h] for n in ["q", "k", "v", "g", "do"])
        S, G, B, gam = _chunk_terms(q, k, v, g, a["h0"][0, h], do, a["dhT"][0, h])
        E1 = np.exp(B)
        E2 = np.stack([np.exp(gam[t // C] - B[t]) for t in range(T)])
        X = np.stack([S[t // C] @ do[t] for t in range(T)])        # X_t[d] = sum_v S_i[d, v] dO_t[v]
        Z = np.stack([G[t // C + 1] @ v[t] for t in range(T)])    # Z_t[d] = sum_v G_{i+1}[d, v] v_t[v]
        dq_intra = dq[0, h] - E1 * X
        dk_intra = dk[0, h] - E2 * Z
        QX, KZ = q * E1 * X, k * E2 * Z
        Qsum = [QX[i * C:(i + 1) * C].sum(0) for i in range(NC)]
        Ksum = [KZ[i * C:(i + 1) * C].sum(0) for i in range(NC)]
        c = [None] * NC
        for a0, b0 in segments:  # the carry restarts at each segment's last chunk
            c[b0] = (G[b0 + 1] * S[b0 + 1]).sum(1) - Ksum[b0]
            for i in range(b0 - 1, a0 - 1, -1):
                c[i] = c[i + 1] + Qsum[i + 1] - Ksum[i]
        for i in range(NC):  # every carry is e^{gamma_i} rowsum(G_{i+1} * S_i)
            np.testing.assert_allclose(c[i], np.exp(gam[i]) * (G[i + 1] * S[i]).sum(1), rtol=1e-10, atol=1e-12)
        dg = np.empty_like(q)
        for i in range(NC):
            ts = list(range(i * C, min(T, (i + 1) * C)))
            for tau, t in enumerate(ts):
                pre = sum((KZ[r] + k[r] * dk_intra[r] - q[r] * dq_intra[r] for r in ts[:tau]), np.zeros(q.shape[1]))
                suf = QX[ts[tau:]].sum(0)
                dg[t] = c[i] + pre + suf
        scale = np.abs(dg_ref[0, h]).max()
        np.testing.assert_allclose(dg, dg_ref[0, h], rtol=0, atol=1e-10 * scale)


def test_segment_scans_reproduce_the_boundary_states():
    """The sequence split's two affine scans: segment-local states from zero (the forward one from
    h0 in the first segment, the reverse one from dhT in the last) and the segments' decay
    products Gamma compose to the exact state entering every segment and the exact dL/dS at the
    end of every segment."""
    inp = make_gla_inputs(1, 1, 64 * 7 + 9, 4, 3, torch.float32, seed=6, with_h0=True, with_dhT=True)
    a = {n: np.asarray(inp[n], dtype=np.float64)[0, 0] for n in ["q", "k", "v", "g", "do", "h0", "dhT"]}
    T = a["q"].shape[0]
    NC = -(-T // C)
    S, G, B, gam = _chunk_terms(a["q"], a["k"], a["v"], a["g"], a["h0"], a["do"], a["dhT"])
    per = 3
    segs = [(s0, min(NC, s0 + per)) for s0 in range(0, NC, per)]  # chunk ranges [s0, s1)
    ns = len(segs)
    Gam = [np.prod([np.exp(gam[i]) for i in range(s0, s1)], axis=0) for s0, s1 in segs]

    def walk_fwd(s0, s1, start):
        s = start.copy()
        for t in range(s0 * C, min(T, s1 * C)):
            s = np.exp(a["g"][t])[:, None] * s + np.outer(a["k"][t], a["v"][t])
        return s

    def walk_rev(s0, s1, end):
        x = end.copy()
        for i in range(s1 - 1, s0 - 1, -1):
            ts = range(i * C, min(T, (i + 1) * C))
            x = np.exp(gam[i])[:, None] * x + sum(np.outer(a["q"][t] * np.exp(B[t]), a["do"][t]) for t in ts)
        return x

    zero = np.zeros_like(a["h0"])
    s_in = [a["h0"]]
    for s in range(ns - 1):  # S_in(s+1) = Gamma_s * S_in(s) + S_local(s), S_local(0) from h0
        local = walk_fwd(*segs[s], a["h0"] if s == 0 else zero)
        s_in.append(local if s == 0 else Gam[s][:, None] * s_in[s] + local)
    g_end = [None] * ns
    g_end[ns - 1] = a["dhT"]
    for s in range(ns - 2, -1, -1):  # G_end(s) = Gamma_{s+1} * G_end(s+1) + G_local(s+1)
        local = walk_rev(*segs[s + 1], a["dhT"] if s + 1 == ns - 1 else zero)
        g_end[s] = local if s + 1 == ns - 1 else Gam[s + 1][:, None] * g_end[s + 1] + local
    for s, (s0, s1) in enumerate(segs):
        np.testing.assert_allclose(s_in[s], S[s0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(g_end[s], G[s1], rtol=1e-12, atol=1e-12)

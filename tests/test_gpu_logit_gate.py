"""The raw-logit entries gla_chunk_fwd_logit / gla_chunk_bwd_logit: the gate arrives as logits x and
the kernels form g = logsigmoid(x) / tau themselves.

Two checks per case: (1) against the library's own two-step route, gla_gate_logsigmoid then
gla_chunk_fwd / gla_chunk_bwd: the kernels form the same bf16 log-gates, so o, hT, dq, dk, dv and
dh0 must agree bit for bit, and dx (formed from the log-gate instead of x) within the bf16 bound;
(2) against the fp64 oracle: oracle.gate_logsigmoid composed with oracle.gla_fwd / gla_bwd, and
dx = oracle.gate_logsigmoid_bwd of the oracle's dg.  Shapes cover the fused kernels (with the
sequence split and a ragged tail), the blocked 1.3B-model shape and the fp32 generic kernels."""
import numpy as np
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import CONFIGS
from helpers import TOL_BF16, assert_close, cuda, f64, tol_for

pytestmark = pytest.mark.gpu


def _inputs(B, H, T, dk, dv, dtype, seed, tau, states):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, T, dk, generator=gen) * dk ** -0.5
    k = torch.randn(B, H, T, dk, generator=gen)
    v = torch.randn(B, H, T, dv, generator=gen)
    x = torch.randn(B, H, T, dk, generator=gen)
    do = torch.randn(B, H, T, dv, generator=gen)
    d = {n: t.to(dtype) for n, t in dict(q=q, k=k, v=v, x=x, do=do).items()}
    if states:
        d["h0"] = torch.randn(B, H, dk, dv, generator=gen)
        d["dhT"] = torch.randn(B, H, dk, dv, generator=gen)
    return d


def _run(B, H, T, dk, dv, dtype, seed, tau, states, idx=None):
    inp = _inputs(B, H, T, dk, dv, dtype, seed, tau, states)
    d = cuda(inp)
    h0, dhT = d.get("h0"), d.get("dhT")
    o, hT = gla.chunk_fwd_logit(d["q"], d["k"], d["v"], d["x"], tau, h0=h0)
    dq, dk_, dv_, dx, dh0 = gla.chunk_bwd_logit(d["q"], d["k"], d["v"], d["x"], tau, d["do"], h0=h0, dhT=dhT)
    # (1) the two-step route through the standalone gate entry
    g = gla.gate_logsigmoid(d["x"], tau)
    o2, hT2 = gla.chunk_fwd(d["q"], d["k"], d["v"], g, h0=h0)
    dq2, dk2, dv2, dg2, dh02 = gla.chunk_bwd(d["q"], d["k"], d["v"], g, d["do"], h0=h0, dhT=dhT)
    dx2 = gla.gate_logsigmoid_bwd(d["x"], dg2, tau)
    torch.cuda.synchronize()
    for name, a, b in [("o", o, o2), ("hT", hT, hT2), ("dq", dq, dq2), ("dk", dk_, dk2), ("dv", dv_, dv2),
                       ("dh0", dh0, dh02)]:
        assert torch.equal(a, b), f"{name}: the raw-logit entry differs from the two-step route"
    tol = tol_for(dtype)
    assert_close("dx vs two-step", dx, dx2, tol)
    # (2) the oracle, on all heads or a sample
    sel = (lambda t: t) if idx is None else (lambda t: torch.stack([t[b, h] for b, h in idx])[:, None])
    a = {n: f64(sel(inp[n])) for n in inp}
    ga = O.gate_logsigmoid(a["x"], tau)
    ro, rhT = O.gla_fwd(a["q"], a["k"], a["v"], ga, a.get("h0"))
    assert_close("o", f64(sel(o.cpu())), ro, tol)
    assert_close("hT", f64(sel(hT.cpu())), rhT, tol)
    rq, rk, rv, rg, rh0 = O.gla_bwd(a["q"], a["k"], a["v"], ga, a.get("h0"), a["do"], a.get("dhT"))
    rx = O.gate_logsigmoid_bwd(a["x"], rg, tau)
    for name, x, r in [("dq", dq, rq), ("dk", dk_, rk), ("dv", dv_, rv), ("dx", dx, rx), ("dh0", dh0, rh0)]:
        assert_close(name, f64(sel(x.cpu())), r, tol)
    assert gla.device_error() == 0


@pytest.mark.parametrize("shape", [(1, 2, 200, 128, 256), (2, 2, 130, 128, 128), (1, 2, 150, 64, 128)])
def test_logit_entry_fused_shapes(shape):
    """bf16 fused shapes with a ragged tail; few heads, so the sequence is split into segments."""
    B, H, T, dk, dv = shape
    _run(B, H, T, dk, dv, torch.bfloat16, seed=31, tau=16.0, states=True)


def test_logit_entry_blocked_shape():
    """d_k = 256, d_v = 512 runs as 128-wide key blocks on the fused kernels."""
    _run(1, 2, 130, 256, 512, torch.bfloat16, seed=32, tau=16.0, states=True)


def test_logit_entry_generic_fp32():
    """fp32 runs on the generic kernels behind the standalone gate pass."""
    _run(1, 2, 100, 64, 64, torch.float32, seed=33, tau=8.0, states=True)


def test_logit_entry_340m_shape():
    """The 340M-model layer shape (B=8, H=4, T=2048, d_k=128, d_v=256, tau = 16), first and last
    head against the oracle's composition."""
    cfg = CONFIGS["gla_340m"]
    _run(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=34, tau=16.0, states=False,
         idx=[(0, 0), (cfg.B - 1, cfg.H - 1)])

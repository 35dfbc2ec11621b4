"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The GPU runs every head of the workload; the fp64 oracle recomputes a sample of heads (it is a
step-by-step recurrence, so each sampled head is checked exactly, element by element)."""
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import CONFIGS, make_gla_inputs, make_gsa_inputs
from helpers import TOL_BF16, assert_close, cuda, f64

pytestmark = pytest.mark.gpu


def _heads(x, idx):
    return f64(torch.stack([x[b, h] for b, h in idx])[:, None])


def _check_gla(cfg, idx, mu=0.0, seed=0, check_bwd=True):
    inp = make_gla_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=seed, gate_mu=mu)
    d = cuda(inp)
    o, hT = gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], chunk=cfg.chunk)
    sub = {n: _heads(inp[n], idx) for n in ["q", "k", "v", "g", "do"]}
    ro, rhT = O.gla_fwd(sub["q"], sub["k"], sub["v"], sub["g"])
    assert_close("o", _heads(o.cpu(), idx), ro, TOL_BF16)
    assert_close("hT", _heads(hT.cpu(), idx), rhT, TOL_BF16)
    if check_bwd:
        grads = gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], chunk=cfg.chunk)
        ref = O.gla_bwd(sub["q"], sub["k"], sub["v"], sub["g"], None, sub["do"])
        for name, x, r in zip(["dq", "dk", "dv", "dg", "dh0"], grads, ref):
            assert_close(name, _heads(x.cpu(), idx), r, TOL_BF16)
    assert gla.device_error() == 0


def _ends(cfg):
    """The first and the last head of the grid, so that an off-by-one head or tile index at either
    end cannot hide."""
    return [(0, 0), (cfg.B - 1, cfg.H - 1)]


def test_gla_340m_shape_fwd_bwd():
    _check_gla(CONFIGS["gla_340m"], _ends(CONFIGS["gla_340m"]))


@pytest.mark.parametrize("mu", [-2.0, 0.0, 3.0])
def test_gla_1p3b_shape_gate_sweep(mu):
    _check_gla(CONFIGS["gla_1p3b"], _ends(CONFIGS["gla_1p3b"]), mu=mu)


def test_gla_long_sequence_then_decode():
    cfg = CONFIGS["gla_long"]
    n = 256
    inp = make_gla_inputs(cfg.B, cfg.H, cfg.T + n, cfg.dk, cfg.dv, cfg.dtype, seed=0, with_do=False)
    d = cuda(inp)
    o_full, hT_full = gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], chunk=cfg.chunk)
    head = {n_: v[:, :, :cfg.T].contiguous() for n_, v in d.items()}
    _, S = gla.chunk_fwd(head["q"], head["k"], head["v"], head["g"], chunk=cfg.chunk)
    outs = [gla.recurrent_step(*(d[nm][:, :, t].contiguous() for nm in ["q", "k", "v", "g"]), S)
            for t in range(cfg.T, cfg.T + n)]
    o_dec = torch.stack(outs, 2)
    # GPU decode against the GPU chunked run over T + 256 tokens
    assert_close("decode vs chunked o", o_dec, o_full[:, :, cfg.T:], TOL_BF16)
    assert_close("decode vs chunked hT", S, hT_full, TOL_BF16)
    # and both against the oracle on the first and the last head
    idx = _ends(cfg)
    sub = {nm: _heads(inp[nm], idx) for nm in ["q", "k", "v", "g"]}
    ro, rhT = O.gla_fwd(sub["q"], sub["k"], sub["v"], sub["g"])
    assert_close("o (oracle)", _heads(o_full.cpu(), idx), ro, TOL_BF16)
    assert_close("decode o (oracle)", _heads(o_dec.cpu(), idx), ro[:, :, cfg.T:], TOL_BF16)
    assert_close("hT (oracle)", _heads(hT_full.cpu(), idx), rhT, TOL_BF16)


def test_gsa_64_slots_fwd_bwd():
    cfg = CONFIGS["gsa_64slots"]
    inp = make_gsa_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.m, cfg.dtype, seed=0)
    d = cuda(inp)
    o, p, hT1, hT2 = gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], chunk=cfg.chunk, save_p=True)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], chunk=cfg.chunk)
    idx = _ends(cfg)
    sub = [_heads(inp[nm], idx) for nm in ["q", "k", "v", "phi", "g"]]
    ro, rp, rhT1, rhT2 = O.gsa_fwd(*sub)
    for name, x, r in [("o", o, ro), ("p", p, rp), ("hT1", hT1, rhT1), ("hT2", hT2, rhT2)]:
        assert_close(name, _heads(x.cpu(), idx), r, TOL_BF16)
    ref = O.gsa_bwd(*sub, None, None, _heads(inp["do"], idx))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg", "dh0_1", "dh0_2"], grads, ref):
        assert_close(name, _heads(x.cpu(), idx), r, TOL_BF16)
    assert gla.device_error() == 0

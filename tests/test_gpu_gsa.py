"""GPU parity of the GSA entry points (two GLA passes joined by a slot softmax) against the
fp64 oracle, at small sizes with ragged tails, both dtypes, and the GSA decode step."""
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import make_gsa_inputs
from helpers import assert_close, cuda, f64, tol_for

pytestmark = pytest.mark.gpu


def _states(B, H, dk, dv, m, seed):
    gen = torch.Generator().manual_seed(seed)
    return [torch.randn(s, generator=gen) * 0.5 for s in
            [(B, H, dk, m), (B, H, m, dv), (B, H, dk, m), (B, H, m, dv)]]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 2, 130, 64, 64, 32), (2, 1, 70, 128, 64, 64)])
def test_gsa_fwd_bwd(dtype, shape):
    B, H, T, dk, dv, m = shape
    tol = tol_for(dtype)
    inp = make_gsa_inputs(B, H, T, dk, dv, m, dtype, seed=11)
    h1, h2, d1, d2 = _states(B, H, dk, dv, m, 12)
    d = cuda(inp)
    o, p, hT1, hT2 = gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], h0_1=h1.cuda(), h0_2=h2.cuda(),
                                 save_p=True)
    a = [f64(inp[n]) for n in ["q", "k", "v", "phi", "g"]]
    ro, rp, rhT1, rhT2 = O.gsa_fwd(*a, f64(h1), f64(h2))
    assert_close("o", o, ro, tol)
    assert_close("p", p, rp, tol)
    assert_close("hT1", hT1, rhT1, tol)
    assert_close("hT2", hT2, rhT2, tol)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], h0_1=h1.cuda(), h0_2=h2.cuda(),
                        dhT1=d1.cuda(), dhT2=d2.cuda())
    ref = O.gsa_bwd(*a, f64(h1), f64(h2), f64(inp["do"]), f64(d1), f64(d2))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg", "dh0_1", "dh0_2"], grads, ref):
        assert_close(name, x, r, tol)
    assert gla.device_error() == 0


@pytest.mark.parametrize("shape", [(1, 2, 150, 128, 128, 64), (2, 1, 100, 64, 256, 32)])
def test_gsa_bwd_second_pass_on_fused_kernels(shape):
    """bf16, d_v in {128, 256}: the second pass's backward runs on the fused kernels with its m slots
    zero-padded to a 128-wide key block; every gradient against the oracle, with initial and final
    states for both passes."""
    B, H, T, dk, dv, m = shape
    tol = tol_for(torch.bfloat16)
    inp = make_gsa_inputs(B, H, T, dk, dv, m, torch.bfloat16, seed=19)
    h1, h2, d1, d2 = _states(B, H, dk, dv, m, 20)
    d = cuda(inp)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], h0_1=h1.cuda(), h0_2=h2.cuda(),
                        dhT1=d1.cuda(), dhT2=d2.cuda())
    a = [f64(inp[n]) for n in ["q", "k", "v", "phi", "g"]]
    ref = O.gsa_bwd(*a, f64(h1), f64(h2), f64(inp["do"]), f64(d1), f64(d2))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg", "dh0_1", "dh0_2"], grads, ref):
        assert_close(name, x, r, tol)
    assert gla.device_error() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gsa_decode_continues_forward(dtype):
    B, H, T, n, dk, dv, m = 1, 2, 100, 12, 64, 64, 32
    inp = make_gsa_inputs(B, H, T + n, dk, dv, m, dtype, seed=13, with_do=False)
    d = cuda(inp)
    sl = {k: v[:, :, :T].contiguous() for k, v in d.items()}
    _, _, S1, S2 = gla.gsa_fwd(sl["q"], sl["k"], sl["v"], sl["phi"], sl["g"])
    outs = [gla.gsa_recurrent_step(*(d[nm][:, :, t].contiguous() for nm in ["q", "k", "v", "phi", "g"]), S1, S2)
            for t in range(T, T + n)]
    ro, _, rhT1, rhT2 = O.gsa_fwd(*(f64(inp[nm]) for nm in ["q", "k", "v", "phi", "g"]))
    tol = tol_for(dtype)
    assert_close("o", torch.stack(outs, 2), ro[:, :, T:], tol)
    assert_close("S1", S1, rhT1, tol)
    assert_close("S2", S2, rhT2, tol)


@pytest.mark.parametrize("variant", ["abc_no_gate", "data_independent_gate"])
def test_gsa_gate_variants(variant):
    """The ABC form (no forget gate, g = 0) and a data-independent gate (one log-decay per slot,
    the same at every step) run through the same kernels."""
    B, H, T, dk, dv, m = 1, 2, 150, 64, 64, 32
    dtype = torch.bfloat16
    inp = make_gsa_inputs(B, H, T, dk, dv, m, dtype, seed=17)
    if variant == "abc_no_gate":
        inp["g"] = torch.zeros_like(inp["g"])
    else:
        per_slot = inp["g"][:, :, :1, :].float()  # one value per (batch, head, slot)
        inp["g"] = per_slot.expand(B, H, T, m).contiguous().to(dtype)
    d = cuda(inp)
    o, p, hT1, hT2 = gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], save_p=True)
    a = [f64(inp[n]) for n in ["q", "k", "v", "phi", "g"]]
    ro, rp, rhT1, rhT2 = O.gsa_fwd(*a)
    tol = tol_for(dtype)
    assert_close("o", o, ro, tol)
    assert_close("hT2", hT2, rhT2, tol)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"])
    ref = O.gsa_bwd(*a, None, None, f64(inp["do"]))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg"], grads, ref):
        assert_close(name, x, r, tol)


def test_gsa_fused_near_reset_slots():
    """bf16 at the fused shape (d_k = 128, m = 64, d_v = 128), with a few slots that forget (g = -30)
    over a whole chunk or a short stretch: those chunks take the first pass's exact path (its
    intra-chunk terms formed in fp32 from products of the decays).  Initial and final states on
    both passes; every output and gradient against the oracle."""
    B, H, T, dk, dv, m = 1, 2, 200, 128, 128, 64
    tol = tol_for(torch.bfloat16)
    inp = make_gsa_inputs(B, H, T, dk, dv, m, torch.bfloat16, seed=21)
    g = inp["g"].float()
    g[:, :, 64:128, 5] = -30.0
    g[:, 1, 150:160, 40] = -30.0
    inp["g"] = g.to(torch.bfloat16)
    h1, h2, d1, d2 = _states(B, H, dk, dv, m, 22)
    d = cuda(inp)
    o, p, hT1, hT2 = gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], h0_1=h1.cuda(), h0_2=h2.cuda(),
                                 save_p=True)
    a = [f64(inp[n]) for n in ["q", "k", "v", "phi", "g"]]
    ro, rp, rhT1, rhT2 = O.gsa_fwd(*a, f64(h1), f64(h2))
    for name, x, r in [("o", o, ro), ("p", p, rp), ("hT1", hT1, rhT1), ("hT2", hT2, rhT2)]:
        assert_close(name, x, r, tol)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], h0_1=h1.cuda(), h0_2=h2.cuda(),
                        dhT1=d1.cuda(), dhT2=d2.cuda())
    ref = O.gsa_bwd(*a, f64(h1), f64(h2), f64(inp["do"]), f64(d1), f64(d2))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg", "dh0_1", "dh0_2"], grads, ref):
        assert_close(name, x, r, tol)
    assert gla.device_error() == 0


def test_gsa_fused_many_heads_unsplit():
    """80 heads fill the SMs, so the first pass runs one CTA per head over the whole sequence (no
    sequence split); the first and the last head against the oracle."""
    B, H, T, dk, dv, m = 4, 20, 130, 128, 128, 64
    tol = tol_for(torch.bfloat16)
    inp = make_gsa_inputs(B, H, T, dk, dv, m, torch.bfloat16, seed=23)
    d = cuda(inp)
    o, p, hT1, hT2 = gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], save_p=True)
    grads = gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"])
    idx = [(0, 0), (B - 1, H - 1)]

    def heads(x):
        return f64(torch.stack([x[b, h].cpu() for b, h in idx])[:, None])

    sub = [heads(inp[n]) for n in ["q", "k", "v", "phi", "g"]]
    ro, rp, rhT1, rhT2 = O.gsa_fwd(*sub)
    for name, x, r in [("o", o, ro), ("p", p, rp), ("hT1", hT1, rhT1), ("hT2", hT2, rhT2)]:
        assert_close(name, heads(x), r, tol)
    ref = O.gsa_bwd(*sub, None, None, heads(inp["do"]))
    for name, x, r in zip(["dq", "dk", "dv", "dphi", "dg", "dh0_1", "dh0_2"], grads, ref):
        assert_close(name, heads(x), r, tol)
    assert gla.device_error() == 0

"""GPU parity of the GLA entry points against the fp64 oracle at sizes the oracle finishes in
seconds: several tiles in every dimension, ragged tails, all chunk sizes, both dtypes, and the
degenerate cases (T = 0, T = 1, T < chunk, a near-reset gate, zero gate)."""
import numpy as np
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs
from helpers import assert_close, cuda, f64, tol_for

pytestmark = pytest.mark.gpu


def _run_fwd_bwd(inp, chunk, with_state=True, check_bwd=True):
    dt = inp["q"].dtype
    tol = tol_for(dt)
    d = cuda(inp)
    h0 = d.get("h0") if with_state else None
    dhT = d.get("dhT") if with_state else None
    o, hT = gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], h0=h0, chunk=chunk)
    ro, rhT = O.gla_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                        f64(inp["h0"]) if h0 is not None else None)
    errs = {"o": assert_close("o", o, ro, tol), "hT": assert_close("hT", hT, rhT, tol)}
    if check_bwd:
        dq, dk, dv, dg, dh0 = gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], h0=h0, dhT=dhT, chunk=chunk)
        ref = O.gla_bwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]),
                        f64(inp["h0"]) if h0 is not None else None, f64(inp["do"]),
                        f64(inp["dhT"]) if dhT is not None else None)
        for name, x, r in zip(["dq", "dk", "dv", "dg", "dh0"], [dq, dk, dv, dg, dh0], ref):
            errs[name] = assert_close(name, x, r, tol)
    torch.cuda.synchronize()
    assert gla.device_error() == 0
    return errs


def test_config_fwd_fp32_small():
    """B=1, H=2, T=256, d_k=d_v=64, chunk 64, fp32: o and hT within 1e-4."""
    inp = make_gla_inputs(1, 2, 256, 64, 64, torch.float32, seed=0, with_do=False)
    _run_fwd_bwd(inp, 64, with_state=False, check_bwd=False)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(2, 2, 200, 128, 192), (1, 3, 77, 64, 64), (1, 1, 130, 24, 40)])
def test_fwd_bwd_multi_tile_ragged(dtype, shape):
    B, H, T, dk, dv = shape
    inp = make_gla_inputs(B, H, T, dk, dv, dtype, seed=1, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, 64)


@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_every_chunk_size_gives_the_same_result(chunk):
    inp = make_gla_inputs(1, 2, 100, 64, 64, torch.float32, seed=2, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, chunk)


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65])
def test_short_sequences(T):
    inp = make_gla_inputs(2, 1, T, 64, 128, torch.float32, seed=3, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, 64)


def test_empty_sequence():
    B, H, dk, dv = 2, 2, 64, 64
    z = torch.empty(B, H, 0, dk, device="cuda")
    h0 = torch.randn(B, H, dk, dv, device="cuda")
    o, hT = gla.chunk_fwd(z, z, torch.empty(B, H, 0, dv, device="cuda"), z, h0=h0)
    assert o.shape == (B, H, 0, dv)
    torch.testing.assert_close(hT, h0, rtol=0, atol=0)
    dq, dk_, dv_, dg, dh0 = gla.chunk_bwd(z, z, torch.empty(B, H, 0, dv, device="cuda"), z,
                                          torch.empty(B, H, 0, dv, device="cuda"), h0=h0, dhT=h0)
    torch.testing.assert_close(dh0, h0, rtol=0, atol=0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_zero_gates(dtype):
    inp = make_gla_inputs(1, 2, 150, 64, 64, dtype, seed=4, with_h0=True, with_dhT=True)
    inp["g"] = torch.zeros_like(inp["g"])
    _run_fwd_bwd(inp, 64)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_near_reset_gates(dtype):
    """g = -30 everywhere: o_t = (q_t . k_t) v_t.  Every output but dg is checked as usual.

    The true dg is O(alpha) ~ 1e-13 here, while the chunked gate gradient is a reverse cumulative
    sum of q*dq - k*dk whose terms are O(1) and cancel (the final-state term against the last
    token's dk), so dg is checked in absolute terms against the scale of those terms."""
    inp = make_gla_inputs(1, 2, 150, 64, 64, dtype, seed=4, with_h0=True, with_dhT=True)
    inp["g"] = torch.full_like(inp["g"], -30.0)
    tol = tol_for(dtype)
    d = cuda(inp)
    o, hT = gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], h0=d["h0"])
    a = {n: f64(inp[n]) for n in ["q", "k", "v", "g", "h0", "do", "dhT"]}
    ro, rhT = O.gla_fwd(a["q"], a["k"], a["v"], a["g"], a["h0"])
    assert_close("o", o, ro, tol)
    assert_close("hT", hT, rhT, tol)
    grads = gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], h0=d["h0"], dhT=d["dhT"])
    ref = O.gla_bwd(a["q"], a["k"], a["v"], a["g"], a["h0"], a["do"], a["dhT"])
    for name, x, r in zip(["dq", "dk", "dv", "dh0"], [grads[i] for i in (0, 1, 2, 4)], [ref[i] for i in (0, 1, 2, 4)]):
        assert_close(name, x, r, tol)
    scale = np.sqrt(np.mean((a["q"] * ref[0]) ** 2)) + np.sqrt(np.mean((a["k"] * ref[1]) ** 2))
    scale += np.sqrt(np.mean((a["dhT"] * rhT) ** 2)) * a["dhT"].shape[-1]
    assert np.max(np.abs(f64(grads[3]) - ref[3])) <= tol * scale


@pytest.mark.parametrize("mu", [-2.0, 0.0, 3.0])
def test_gate_bias_sweep_bf16(mu):
    inp = make_gla_inputs(1, 2, 192, 128, 128, torch.bfloat16, seed=5, gate_mu=mu)
    _run_fwd_bwd(inp, 64, with_state=False)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_steps_continue_chunked_forward(dtype):
    B, H, T, n, dk, dv = 1, 2, 130, 20, 64, 128
    inp = make_gla_inputs(B, H, T + n, dk, dv, dtype, seed=6, with_do=False)
    d = cuda(inp)
    o_full, hT_full = gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"])
    _, S = gla.chunk_fwd(d["q"][:, :, :T].contiguous(), d["k"][:, :, :T].contiguous(),
                         d["v"][:, :, :T].contiguous(), d["g"][:, :, :T].contiguous())
    steps = []
    for t in range(T, T + n):
        steps.append(gla.recurrent_step(d["q"][:, :, t].contiguous(), d["k"][:, :, t].contiguous(),
                                        d["v"][:, :, t].contiguous(), d["g"][:, :, t].contiguous(), S))
    ro, rhT = O.gla_fwd(f64(inp["q"]), f64(inp["k"]), f64(inp["v"]), f64(inp["g"]))
    tol = tol_for(dtype)
    assert_close("decode o", torch.stack(steps, 2), ro[:, :, T:], tol)
    assert_close("decode S", S, rhT, tol)
    assert_close("chunked o", o_full[:, :, T:], ro[:, :, T:], tol)
    assert_close("chunked hT", hT_full, rhT, tol)


def test_decode_step_matches_oracle_step():
    B, H, dk, dv = 2, 2, 64, 96
    gen = torch.Generator().manual_seed(7)
    q, k, g = (torch.randn(B, H, dk, generator=gen) for _ in range(3))
    g = -torch.nn.functional.softplus(g)
    v = torch.randn(B, H, dv, generator=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen)
    S = S0.cuda()
    o = gla.recurrent_step(q.cuda(), k.cuda(), v.cuda(), g.cuda(), S)
    ro, rS = O.gla_decode_step(f64(q), f64(k), f64(v), f64(g), f64(S0))
    assert_close("o", o, ro, 1e-5)
    assert_close("S", S, rS, 1e-5)


def test_deterministic_repeat():
    inp = cuda(make_gla_inputs(2, 2, 300, 128, 256, torch.bfloat16, seed=8))
    a = gla.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"])
    b = gla.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["g"])
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    ga = gla.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["do"])
    gb = gla.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["do"])
    for x, y in zip(ga, gb):
        assert torch.equal(x, y)


def test_fused_forward_is_selected_for_bf16_shapes():
    """bf16, chunk 64, d_k in {64, 128}, d_v a multiple of 64: the fused kernel runs.  With enough
    heads to fill the GPU it needs no workspace; with few heads it splits the sequence and keeps one
    fp32 state and one decay vector per (head, segment)."""
    assert gla.workspace_bytes("gla_chunk_fwd", 8, 4, 2048, 128, 256, 64, 1) == 0
    nseg = 2  # 2 chunks, one head: one segment per chunk
    expect = -(-nseg * 64 * 64 * 4 // 256) * 256 + -(-nseg * 64 * 4 // 256) * 256
    assert gla.workspace_bytes("gla_chunk_fwd", 1, 1, 100, 64, 64, 64, 1) == expect
    assert gla.workspace_bytes("gla_chunk_fwd", 1, 1, 100, 64, 64, 64, 0) > 0  # fp32: generic passes


@pytest.mark.parametrize("dk,dv,T", [(128, 64, 64 * 23 + 5), (64, 128, 64 * 9), (128, 256, 64 * 40 + 63),
                                     (128, 128, 64 * 2)])
def test_fused_forward_sequence_split(dk, dv, T):
    """Few heads and many chunks: the forward runs as segments (state-only pass, scan of the segment
    entry states, full pass per segment).  o and hT against the oracle, with an initial state."""
    inp = make_gla_inputs(1, 2, T, dk, dv, torch.bfloat16, seed=40 + dk + T, with_h0=True, with_do=False)
    _run_fwd_bwd(inp, 64, check_bwd=False)


@pytest.mark.parametrize("dv", [128, 256])
@pytest.mark.parametrize("T", [1, 40, 64, 150, 300])
def test_fused_shapes_fwd_bwd(dv, T):
    """d_k = 128 bf16 shapes served by the fused kernels, with initial and final state gradients."""
    inp = make_gla_inputs(2, 2, T, 128, dv, torch.bfloat16, seed=20 + T, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, 64)


def test_fused_shapes_mixed_strong_gates():
    """Some chunks keep less than e^-40 of their state (exact fp32 intra-chunk path), others do not."""
    inp = make_gla_inputs(1, 2, 320, 128, 256, torch.bfloat16, seed=31, with_h0=True, with_dhT=True)
    g = inp["g"].float()
    g[:, :, 64:128] -= 2.0      # chunk 1: ~ -128 over the chunk in every dimension
    g[:, 1, 200:210, :7] = -9.0  # part of chunk 3, a few dimensions
    inp["g"] = g.to(torch.bfloat16)
    _run_fwd_bwd(inp, 64)


def _bwd_workspace_bytes(BH, T, dk, dv, nseg):
    """Size of the fused backward's workspace: six parts, the segment states when split, and per
    (head, chunk) the masked dA block (bf16 hi and lo 64 x 64 tiles and the fp32 diagonal)."""
    NC = -(-T // 64)
    parts = [BH * NC * dk, BH * NC * 64 * dk, BH * nseg * dk, BH * (dv // 128) * NC * dk * 64,
             BH * (dv // 128) * NC * 2 * dk, BH * NC * dk]
    if nseg > 1:
        parts += [BH * nseg * dk * dv, BH * nseg * dk * dv, BH * nseg * dk]
    parts += [BH * NC * (2 * 64 * 64 * 2 + 64 * 4) // 4]
    return sum(-(-4 * p // 256) * 256 for p in parts)


@pytest.mark.parametrize("B,H,T,dv,nseg", [(2, 4, 64 * 40 + 17, 256, 4), (1, 4, 64 * 30, 128, 10)])
def test_fused_backward_sequence_split(B, H, T, dv, nseg):
    """Few heads: the backward's walks run as segments of several chunks (state entry from the
    forward's segment scan, state gradient from the reverse one, the dg carry restarting per
    segment).  Every gradient against the oracle, with initial and final states."""
    assert gla.workspace_bytes("gla_chunk_bwd", B, H, T, 128, dv, 64, 1) == \
        _bwd_workspace_bytes(B * H, T, 128, dv, nseg)
    inp = make_gla_inputs(B, H, T, 128, dv, torch.bfloat16, seed=70 + dv, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, 64)


def test_fused_backward_unsplit_workspace():
    """Enough heads to fill the GPU: one segment, no segment states."""
    assert gla.workspace_bytes("gla_chunk_bwd", 8, 4, 2048, 128, 256, 64, 1) == \
        _bwd_workspace_bytes(32, 2048, 128, 256, 1)


@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128)])
def test_fused_forward_long_walk(dk, dv):
    """Enough heads to fill the GPU (no sequence split), so one CTA walks every chunk of its head:
    exercises the pipelined forward's ring buffers and barrier phases over many chunks."""
    H = 80 if dv == 64 else 40
    inp = make_gla_inputs(1, H, 64 * 9 + 7, dk, dv, torch.bfloat16, seed=50 + dk, with_h0=True, with_do=False)
    assert gla.workspace_bytes("gla_chunk_fwd", 1, H, 64 * 9 + 7, dk, dv, 64, 1) == 0  # no split
    _run_fwd_bwd(inp, 64, check_bwd=False)


@pytest.mark.parametrize("shape", [(1, 2, 150, 256, 512), (1, 2, 100, 128, 384), (2, 1, 70, 384, 128)])
def test_wide_shapes_run_as_fused_blocks(shape):
    """bf16 shapes wider than the fused kernels run as key-block / value-block sub-problems whose
    outputs add up (GLA is linear in a split of the key axis, its loss in a split of the value
    axis); checked against the oracle with initial and final states."""
    B, H, T, dk, dv = shape
    inp = make_gla_inputs(B, H, T, dk, dv, torch.bfloat16, seed=60 + dk + dv, with_h0=True, with_dhT=True)
    _run_fwd_bwd(inp, 64)

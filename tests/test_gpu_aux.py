"""GPU parity of the raw-logit gate entry and the MS-GLA pooling / causal hold against the fp64
oracle, both dtypes, ragged lengths (a short last block, vector tails of the gate)."""
import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from helpers import assert_close, f64, tol_for

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("n", [1, 7, 8, 4099, 1 << 20])
@pytest.mark.parametrize("tau", [16.0, 8.0])
def test_gate_logsigmoid(dtype, n, tau):
    gen = torch.Generator().manual_seed(n)
    x = (torch.randn(n, generator=gen) * 4).to(dtype)
    dg = torch.randn(n, generator=gen).to(dtype)
    g = gla.gate_logsigmoid(x.cuda(), tau)
    dx = gla.gate_logsigmoid_bwd(x.cuda(), dg.cuda(), tau)
    torch.cuda.synchronize()
    tol = tol_for(dtype)
    assert_close("g", g, O.gate_logsigmoid(f64(x), tau), tol)
    assert_close("dx", dx, O.gate_logsigmoid_bwd(f64(x), f64(dg), tau), tol)


def test_gate_logsigmoid_extremes():
    x = torch.tensor([-80.0, -20.0, -1e-3, 0.0, 1e-3, 20.0, 80.0] + [0.0], dtype=torch.float32)
    g = gla.gate_logsigmoid(x.cuda(), 1.0).cpu()
    dx = gla.gate_logsigmoid_bwd(x.cuda(), torch.ones_like(x).cuda(), 1.0).cpu()
    assert torch.isfinite(g).all() and torch.isfinite(dx).all()
    assert_close("g", g, O.gate_logsigmoid(f64(x), 1.0), 1e-6)
    assert_close("dx", dx, O.gate_logsigmoid_bwd(f64(x), f64(torch.ones_like(x)), 1.0), 1e-6)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("T,s,D", [(1, 1, 8), (13, 4, 64), (64, 64, 128), (130, 3, 16), (200, 8, 256),
                                   (5, 9, 8)])
def test_msgla_pool_hold(dtype, T, s, D):
    gen = torch.Generator().manual_seed(T * 1000 + s)
    B, H = 2, 3
    P = -(-T // s)
    x = torch.randn(B, H, T, D, generator=gen).to(dtype)
    dy = torch.randn(B, H, P, D, generator=gen).to(dtype)
    dz = torch.randn(B, H, T, D, generator=gen).to(dtype)
    tol = tol_for(dtype)
    y = gla.msgla_pool(x.cuda(), s)
    dx = gla.msgla_pool_bwd(dy.cuda(), T, s)
    z = gla.msgla_hold(dy.cuda(), T, s)
    dyh = gla.msgla_hold_bwd(dz.cuda(), s)
    torch.cuda.synchronize()
    assert_close("pool", y, O.msgla_pool(f64(x), s), tol)
    assert_close("pool_bwd", dx, O.msgla_pool_bwd(f64(dy), T, s), tol)
    assert_close("hold", z, O.msgla_hold(f64(dy), T, s), 0.0 if dtype == torch.float32 else tol)
    assert_close("hold_bwd", dyh, O.msgla_hold_bwd(f64(dz), s), tol)

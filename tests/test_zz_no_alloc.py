"""gla_chunk_bwd_noalloc: the backward for callers that cannot provide a workspace.

Those callers (a plain C host without a device allocator, a runtime that hands out pre-carved
device memory only for tensors, code that must not let cudaMalloc synchronise the device) get a
variant whose scratch is a fixed array compiled into the library.  It runs the same kernels as
gla_chunk_bwd, which takes a caller-provided workspace, and those kernels are deterministic (no
atomics), so the two must agree bit for bit.  The test calls it through the C ABI several times in
a row: first at the 340M-model layer shape (close to the array's limit; also checked against the
fp64 oracle on its first and last head), then on smaller inputs that reuse the array with the
larger call's contents still in it, so that stale or aliased scratch would show.  It is collected
last so that a run stopping at the first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import oracle as O
from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import CONFIGS, make_gla_inputs
from helpers import TOL_BF16, assert_close, cuda, f64

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 128 << 20


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc_bwd(d, h0, dhT):
    lib = gla.load_library()
    B, H, T, dk = d["q"].shape
    dv = d["v"].shape[-1]
    dq, dkk, dg = (torch.empty_like(d["q"]) for _ in range(3))
    dvv = torch.empty_like(d["v"])
    dh0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device="cuda")
    status = lib.gla_chunk_bwd_noalloc(
        _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["g"]), _ptr(h0), _ptr(d["do"]), _ptr(dhT),
        _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(dh0), B, H, T, dk, dv, 64, 1,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert status == 0, gla.status_string(status)
    return dq, dkk, dvv, dg, dh0


def _check_equal(d, h0, dhT):
    got = _noalloc_bwd(d, h0, dhT)
    ref = gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], h0=h0, dhT=dhT)
    torch.cuda.synchronize()
    for name, x, r in zip(["dq", "dk", "dv", "dg", "dh0"], got, ref):
        assert torch.equal(x, r), f"{name}: the scratch-array backward differs from the workspace backward"
    return got


def test_noalloc_backward_equals_workspace_backward():
    cfg = CONFIGS["gla_340m"]
    lib = gla.load_library()
    need = lib.gla_chunk_bwd_workspace(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.chunk, 1)
    assert 0 < need <= SCRATCH_BYTES
    # 1) the 340M-model layer shape, also against the oracle on its first and last head
    inp = make_gla_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=40)
    d = cuda(inp)
    got = _check_equal(d, None, None)
    idx = [(0, 0), (cfg.B - 1, cfg.H - 1)]
    sub = {n: f64(torch.stack([inp[n][b, h] for b, h in idx])[:, None]) for n in ["q", "k", "v", "g", "do"]}
    ref = O.gla_bwd(sub["q"], sub["k"], sub["v"], sub["g"], None, sub["do"])
    for name, x, r in zip(["dq", "dk", "dv", "dg", "dh0"], got, ref):
        assert_close(name, f64(torch.stack([x[b, h].cpu() for b, h in idx])[:, None]), r, TOL_BF16)
    del d, got
    # 2) two smaller calls in a row, each after a larger one left its contents in the array
    cases = [
        dict(B=2, H=2, T=300, dv=256, states=True, seed=41),
        dict(B=1, H=3, T=150, dv=128, states=False, seed=42),
    ]
    for c in cases:
        inp = make_gla_inputs(c["B"], c["H"], c["T"], 128, c["dv"], torch.bfloat16, seed=c["seed"],
                              with_h0=c["states"], with_dhT=c["states"])
        d = cuda(inp)
        _check_equal(d, d.get("h0"), d.get("dhT"))
    assert gla.device_error() == 0

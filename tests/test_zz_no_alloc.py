"""gla_chunk_bwd_noalloc: the backward for callers that cannot provide a workspace.

Those callers (a plain C host without a device allocator, a runtime that hands out pre-carved
device memory only for tensors, code that must not let cudaMalloc synchronise the device) get a
variant whose scratch is a fixed array compiled into the library.  This test calls it through the
C ABI twice in a row, on different inputs so that the shared scratch is reused with new contents,
and checks each result against gla_chunk_bwd (which takes a caller-provided workspace) within the
bf16 tolerance of the other parity tests.  It is collected last so that a run stopping at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs
from helpers import TOL_BF16, assert_close, cuda

pytestmark = pytest.mark.gpu


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


def test_noalloc_backward_matches_workspace_backward_twice():
    cases = [
        dict(B=2, H=2, T=300, dv=256, states=True, seed=41),
        dict(B=1, H=3, T=150, dv=128, states=False, seed=42),
    ]
    for c in cases:
        inp = make_gla_inputs(c["B"], c["H"], c["T"], 128, c["dv"], torch.bfloat16, seed=c["seed"],
                              with_h0=c["states"], with_dhT=c["states"])
        d = cuda(inp)
        h0, dhT = d.get("h0"), d.get("dhT")
        got = _noalloc_bwd(d, h0, dhT)
        ref = gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], h0=h0, dhT=dhT)
        torch.cuda.synchronize()
        for name, x, r in zip(["dq", "dk", "dv", "dg", "dh0"], got, ref):
            assert_close(name, x, r, TOL_BF16)
    assert gla.device_error() == 0

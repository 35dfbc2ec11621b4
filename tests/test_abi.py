"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every function the
header declares, answers workspace queries, and rejects invalid arguments before any launch."""
import ctypes

import pytest

from chunkwise_linear_rnn_02_b200 import binding
from chunkwise_linear_rnn_02_b200.build_lib import build

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 3
P = 0x7F0000000000  # a 16-byte aligned fake device address: never dereferenced by these tests
BAD = P + 8         # misaligned


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def test_every_header_symbol_is_exported(lib):
    names = binding.header_symbols()
    expected = {"gla_status_string", "gla_version", "gla_chunk_fwd_workspace", "gla_chunk_fwd",
                "gla_chunk_bwd_workspace", "gla_chunk_bwd", "gla_recurrent_step", "gsa_fwd_workspace",
                "gsa_fwd", "gsa_bwd_workspace", "gsa_bwd", "gsa_recurrent_step", "gla_device_error"}
    assert expected <= set(names)
    for n in names:
        assert hasattr(lib, n), n
        assert n in binding._SIGNATURES, n


def test_status_strings_and_version(lib):
    for code in range(6):
        assert binding.status_string(code).startswith("GLA_")
    assert "unknown" in binding.status_string(99)
    assert lib.gla_version() >= 10000


# fp32 (dtype 0) keeps every call below on the workspace-using path, so that a call which
# passes the other checks still fails the workspace check and never reaches a launch.
def _fwd(lib, q=P, k=P, v=P, g=P, h0=None, o=P, hT=None, B=1, H=1, T=64, dk=64, dv=64, chunk=64, dtype=0,
         ws=P, nb=1 << 40):
    return lib.gla_chunk_fwd(q, k, v, g, h0, o, hT, B, H, T, dk, dv, chunk, dtype, ws, nb, None)


def test_fwd_argument_checks(lib):
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, o=None) == INVALID
    assert _fwd(lib, k=BAD) == INVALID
    assert _fwd(lib, h0=BAD) == INVALID
    assert _fwd(lib, B=0) == INVALID
    assert _fwd(lib, T=-1) == INVALID
    assert _fwd(lib, dk=0) == INVALID
    assert _fwd(lib, dk=12) == UNSUPPORTED
    assert _fwd(lib, dv=1024) == UNSUPPORTED
    assert _fwd(lib, chunk=48) == UNSUPPORTED
    assert _fwd(lib, dtype=7) == UNSUPPORTED
    need = lib.gla_chunk_fwd_workspace(1, 1, 64, 64, 64, 64, 0)
    assert need > 0
    assert _fwd(lib, ws=None) == WORKSPACE
    assert _fwd(lib, nb=need - 1) == WORKSPACE
    assert _fwd(lib, ws=BAD) == WORKSPACE


def test_bwd_and_gsa_argument_checks(lib):
    # every call below is invalid: none may reach a launch with these fake pointers
    args = [P] * 5 + [P, None] + [P] * 4 + [None]
    bad = list(args)
    bad[8] = None  # dv output missing
    assert lib.gla_chunk_bwd(*bad, 1, 1, 64, 64, 64, 64, 0, P, 1 << 40, None) == INVALID
    assert lib.gla_chunk_bwd(*args, 1, 1, 64, 64, 64, 64, 0, P, 8, None) == WORKSPACE
    g11 = [P] * 5 + [None, None, P, None, None, None]
    assert lib.gsa_fwd(*g11, 1, 1, 64, 64, 64, 20, 64, 1, P, 1 << 40, None) == UNSUPPORTED
    assert lib.gsa_fwd(*g11, 1, 1, 64, 64, 64, 0, 64, 1, P, 1 << 40, None) == INVALID
    assert lib.gsa_fwd(*g11, 1, 1, 64, 64, 64, 64, 64, 0, P, 16, None) == WORKSPACE
    assert lib.gla_recurrent_step(P, P, P, P, None, P, 1, 1, 64, 64, 1, None) == INVALID
    assert lib.gla_recurrent_step(P, P, P, P, P, P, 1, 1, 64, 64, 3, None) == UNSUPPORTED
    assert lib.gsa_recurrent_step(P, P, P, P, P, P, BAD, P, 1, 1, 64, 64, 64, 1, None) == INVALID
    assert lib.gla_device_error(None, 0, None) == INVALID
    # the workspace-free backward rejects what it cannot run before touching the device
    nb = [P] * 5 + [P, None] + [P] * 4 + [None]
    assert lib.gla_chunk_bwd_noalloc(*nb, 1, 1, 64, 128, 256, 64, 0, None) == UNSUPPORTED   # fp32
    assert lib.gla_chunk_bwd_noalloc(*nb, 1, 1, 64, 64, 256, 64, 1, None) == UNSUPPORTED    # d_k
    assert lib.gla_chunk_bwd_noalloc(*nb, 1, 1, 0, 128, 256, 64, 1, None) == INVALID        # T = 0
    bad_nb = list(nb)
    bad_nb[0] = None
    assert lib.gla_chunk_bwd_noalloc(*bad_nb, 1, 1, 64, 128, 256, 64, 1, None) == INVALID
    # a supported shape whose scratch exceeds the fixed 128 MiB: B=8, H=8, T=2048, d_v=256 needs
    # (66 + 256/2 + 256/64) * 64 * 32 * 128 * 4 bytes (six parts, each a multiple of 256 bytes)
    need = (66 + 128 + 4) * 64 * 32 * 128 * 4 + 64 * 128 * 4
    assert need > 128 << 20
    assert lib.gla_chunk_bwd_noalloc(*nb, 8, 8, 2048, 128, 256, 64, 1, None) == WORKSPACE


def test_workspace_queries(lib):
    # generic passes: fp32 per-chunk states (and, for bwd, state gradients, db and hT)
    B, H, T, dk, dv, C = 2, 3, 130, 64, 128, 64
    NC = 3
    fwd_f32 = lib.gla_chunk_fwd_workspace(B, H, T, dk, dv, C, 0)
    assert fwd_f32 >= B * H * NC * dk * dv * 4
    assert fwd_f32 % 256 == 0
    assert lib.gla_chunk_bwd_workspace(B, H, T, dk, dv, C, 0) >= 2 * fwd_f32
    assert lib.gla_chunk_fwd_workspace(B, H, 0, dk, dv, C, 1) == 0
    assert lib.gla_chunk_fwd_workspace(B, H, T, 7, dv, C, 1) == 0
    assert lib.gsa_bwd_workspace(B, H, T, dk, dv, 64, C, 1) > lib.gsa_fwd_workspace(B, H, T, dk, dv, 64, C, 1)


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 8, 8)
    with pytest.raises(binding.GLAError):
        binding.chunk_fwd(x, x, x, x)


def test_gate_and_msgla_argument_checks(lib):
    """Every call here fails a check (or has nothing to do) before any launch."""
    vp = ctypes.c_void_p
    # gate: tau must be positive, dtype known, pointers non-NULL and aligned when n > 0
    assert lib.gla_gate_logsigmoid(vp(P), vp(P), 16, 0.0, 1, None) == INVALID
    assert lib.gla_gate_logsigmoid(vp(P), vp(P), 16, float("nan"), 1, None) == INVALID
    assert lib.gla_gate_logsigmoid(vp(P), vp(P), 16, 16.0, 5, None) == UNSUPPORTED
    assert lib.gla_gate_logsigmoid(None, vp(P), 16, 16.0, 1, None) == INVALID
    assert lib.gla_gate_logsigmoid(vp(P), vp(BAD), 16, 16.0, 1, None) == INVALID
    assert lib.gla_gate_logsigmoid(None, None, 0, 16.0, 1, None) == OK  # nothing to do
    assert lib.gla_gate_logsigmoid_bwd(vp(P), None, vp(P), 16, 8.0, 0, None) == INVALID
    for name in ("gla_msgla_pool", "gla_msgla_pool_bwd", "gla_msgla_hold", "gla_msgla_hold_bwd"):
        f = getattr(lib, name)
        assert f(vp(P), vp(P), 1, 1, 10, 12, 2, 1, None) == UNSUPPORTED   # D not a multiple of 8
        assert f(vp(P), vp(P), 1, 1, 10, 16, 0, 1, None) == INVALID       # s = 0
        assert f(vp(P), vp(P), 0, 1, 10, 16, 2, 1, None) == INVALID       # B = 0
        assert f(None, vp(P), 1, 1, 10, 16, 2, 1, None) == INVALID        # NULL input
        assert f(vp(P), vp(BAD), 1, 1, 10, 16, 2, 1, None) == INVALID     # misaligned output
        assert f(vp(P), vp(P), 1, 1, 10, 16, 2, 3, None) == UNSUPPORTED   # dtype
        assert f(None, None, 1, 1, 0, 16, 2, 1, None) == OK               # T = 0: nothing to do

"""Thin Python binding of the C ABI in ``include/gla.h`` (ctypes; argument marshalling only).

PyTorch supplies device memory and the current CUDA stream.  Every step of every operator runs
in the CUDA library ``lib/libgla_b200.so``; if that library is missing or the tensors are not
CUDA tensors, the calls raise instead of computing anything elsewhere.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

__all__ = [
    "GLAError", "load_library", "library_path", "header_symbols", "status_string", "version",
    "chunk_fwd", "chunk_bwd", "chunk_fwd_logit", "chunk_bwd_logit", "recurrent_step", "gsa_fwd", "gsa_bwd", "gsa_recurrent_step",
    "device_error", "workspace_bytes",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_HEADER = os.path.join(os.path.dirname(_HERE), "include", "gla.h")
_LIB = None

DTYPE_CODE = {torch.float32: 0, torch.bfloat16: 1}

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_SIGNATURES = {
    "gla_status_string": (ctypes.c_char_p, [_i]),
    "gla_version": (_i, []),
    "gla_chunk_fwd_workspace": (_sz, [_i] * 7),
    "gla_chunk_fwd": (_i, [_vp] * 7 + [_i] * 7 + [_vp, _sz, _vp]),
    "gla_chunk_bwd_workspace": (_sz, [_i] * 7),
    "gla_chunk_bwd": (_i, [_vp] * 12 + [_i] * 7 + [_vp, _sz, _vp]),
    "gla_chunk_fwd_logit_workspace": (_sz, [_i] * 7),
    "gla_chunk_fwd_logit": (_i, [_vp] * 4 + [ctypes.c_float] + [_vp] * 3 + [_i] * 7 + [_vp, _sz, _vp]),
    "gla_chunk_bwd_logit_workspace": (_sz, [_i] * 7),
    "gla_chunk_bwd_logit": (_i, [_vp] * 4 + [ctypes.c_float] + [_vp] * 8 + [_i] * 7 + [_vp, _sz, _vp]),
    "gla_recurrent_step": (_i, [_vp] * 6 + [_i] * 5 + [_vp]),
    "gsa_fwd_workspace": (_sz, [_i] * 8),
    "gsa_fwd": (_i, [_vp] * 11 + [_i] * 8 + [_vp, _sz, _vp]),
    "gsa_bwd_workspace": (_sz, [_i] * 8),
    "gsa_bwd": (_i, [_vp] * 17 + [_i] * 8 + [_vp, _sz, _vp]),
    "gsa_recurrent_step": (_i, [_vp] * 8 + [_i] * 6 + [_vp]),
    "gla_device_error": (_i, [_vp, _i, ctypes.POINTER(_i)]),
    "gla_chunk_bwd_noalloc": (_i, [_vp] * 12 + [_i] * 7 + [_vp]),
    "gla_gate_logsigmoid": (_i, [_vp, _vp, ctypes.c_size_t, ctypes.c_float, _i, _vp]),
    "gla_gate_logsigmoid_bwd": (_i, [_vp, _vp, _vp, ctypes.c_size_t, ctypes.c_float, _i, _vp]),
    "gla_msgla_pool": (_i, [_vp, _vp] + [_i] * 6 + [_vp]),
    "gla_msgla_pool_bwd": (_i, [_vp, _vp] + [_i] * 6 + [_vp]),
    "gla_msgla_hold": (_i, [_vp, _vp] + [_i] * 6 + [_vp]),
    "gla_msgla_hold_bwd": (_i, [_vp, _vp] + [_i] * 6 + [_vp]),
}


class GLAError(RuntimeError):
    pass


def library_path() -> str:
    return os.path.join(_HERE, "lib", "libgla_b200.so")


def header_symbols(path: str = _HEADER):
    """Names of the functions declared in include/gla.h."""
    text = open(path).read()
    return re.findall(r"^\s*(?:const\s+char\s*\*|size_t|int)\s+(\w+)\s*\(", text, flags=re.M)


def load_library():
    """Load the CUDA library once; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            raise GLAError(f"{path} is missing: build it with `python -m chunkwise_linear_rnn_02_b200.build_lib`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype, fn.argtypes = res, args
        _LIB = lib
    return _LIB


def status_string(code: int) -> str:
    return load_library().gla_status_string(int(code)).decode()


def version() -> int:
    return load_library().gla_version()


def _check(code: int, what: str):
    if code != 0:
        raise GLAError(f"{what}: {status_string(code)}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise GLAError("tensors must be CUDA tensors: this library has no CPU path")
        if not t.is_contiguous():
            raise GLAError("tensors must be contiguous")


def _dtype_code(t):
    if t.dtype not in DTYPE_CODE:
        raise GLAError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")
    return DTYPE_CODE[t.dtype]


def _state(t, shape, device):
    if t is None:
        return None
    if t.dtype != torch.float32 or tuple(t.shape) != tuple(shape):
        raise GLAError(f"state tensors must be float32 of shape {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")
    _need_cuda(t)
    return t


def workspace_bytes(kind: str, *args) -> int:
    lib = load_library()
    return int(getattr(lib, f"{kind}_workspace")(*[int(a) for a in args]))


def _workspace(nbytes: int, device):
    if nbytes == 0:
        return None, 0
    return torch.empty(nbytes, dtype=torch.uint8, device=device), nbytes


# ------------------------------------------------------------------------------------------
def chunk_fwd(q, k, v, g, h0=None, chunk: int = 64, output_final_state: bool = True):
    """GLA forward: returns (o [B,H,T,dv], hT [B,H,dk,dv] fp32 or None)."""
    _need_cuda(q, k, v, g)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0 = _state(h0, (B, H, dk, dv), dev)
    o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    hT = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if output_final_state else None
    ws, nb = _workspace(lib.gla_chunk_fwd_workspace(B, H, T, dk, dv, chunk, dt), dev)
    _check(lib.gla_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(h0), _ptr(o), _ptr(hT),
                             B, H, T, dk, dv, chunk, dt, _ptr(ws), nb, _stream(dev)), "gla_chunk_fwd")
    return o, hT


def chunk_bwd(q, k, v, g, do, h0=None, dhT=None, chunk: int = 64, need_dh0: bool = True):
    """GLA backward: returns (dq, dk, dv, dg, dh0 or None)."""
    _need_cuda(q, k, v, g, do)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0 = _state(h0, (B, H, dk, dv), dev)
    dhT = _state(dhT, (B, H, dk, dv), dev)
    dq, dkk, dg = (torch.empty_like(q) for _ in range(3))
    dvv = torch.empty_like(v)
    dh0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if need_dh0 else None
    ws, nb = _workspace(lib.gla_chunk_bwd_workspace(B, H, T, dk, dv, chunk, dt), dev)
    _check(lib.gla_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(h0), _ptr(do), _ptr(dhT),
                             _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dg), _ptr(dh0), B, H, T, dk, dv, chunk, dt,
                             _ptr(ws), nb, _stream(dev)), "gla_chunk_bwd")
    return dq, dkk, dvv, dg, dh0


def chunk_fwd_logit(q, k, v, x, tau: float, h0=None, chunk: int = 64, output_final_state: bool = True):
    """GLA forward from raw gate logits x (g = logsigmoid(x) / tau formed inside the kernels)."""
    _need_cuda(q, k, v, x)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0 = _state(h0, (B, H, dk, dv), dev)
    o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    hT = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if output_final_state else None
    ws, nb = _workspace(lib.gla_chunk_fwd_logit_workspace(B, H, T, dk, dv, chunk, dt), dev)
    _check(lib.gla_chunk_fwd_logit(_ptr(q), _ptr(k), _ptr(v), _ptr(x), float(tau), _ptr(h0), _ptr(o), _ptr(hT),
                                   B, H, T, dk, dv, chunk, dt, _ptr(ws), nb, _stream(dev)), "gla_chunk_fwd_logit")
    return o, hT


def chunk_bwd_logit(q, k, v, x, tau: float, do, h0=None, dhT=None, chunk: int = 64, need_dh0: bool = True):
    """Backward of chunk_fwd_logit: returns (dq, dk, dv, dx, dh0 or None)."""
    _need_cuda(q, k, v, x, do)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0 = _state(h0, (B, H, dk, dv), dev)
    dhT = _state(dhT, (B, H, dk, dv), dev)
    dq, dkk, dx = (torch.empty_like(q) for _ in range(3))
    dvv = torch.empty_like(v)
    dh0 = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev) if need_dh0 else None
    ws, nb = _workspace(lib.gla_chunk_bwd_logit_workspace(B, H, T, dk, dv, chunk, dt), dev)
    _check(lib.gla_chunk_bwd_logit(_ptr(q), _ptr(k), _ptr(v), _ptr(x), float(tau), _ptr(h0), _ptr(do), _ptr(dhT),
                                   _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dx), _ptr(dh0), B, H, T, dk, dv, chunk, dt,
                                   _ptr(ws), nb, _stream(dev)), "gla_chunk_bwd_logit")
    return dq, dkk, dvv, dx, dh0


def recurrent_step(q, k, v, g, S):
    """One decode step; q, k, g [B,H,dk], v [B,H,dv]; S [B,H,dk,dv] fp32 updated in place.  Returns o."""
    _need_cuda(q, k, v, g, S)
    B, H, dk = q.shape
    dv = v.shape[-1]
    _state(S, (B, H, dk, dv), q.device)
    o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _check(load_library().gla_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(S), _ptr(o), B, H, dk, dv,
                                             _dtype_code(q), _stream(q.device)), "gla_recurrent_step")
    return o


def gsa_fwd(q, k, v, phi, g, h0_1=None, h0_2=None, chunk: int = 64, save_p: bool = False,
            output_final_state: bool = True):
    """GSA forward: returns (o, p or None, hT1 or None, hT2 or None)."""
    _need_cuda(q, k, v, phi, g)
    B, H, T, dk = q.shape
    dv, m = v.shape[-1], phi.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0_1 = _state(h0_1, (B, H, dk, m), dev)
    h0_2 = _state(h0_2, (B, H, m, dv), dev)
    o = torch.empty(B, H, T, dv, dtype=q.dtype, device=dev)
    p = torch.empty(B, H, T, m, dtype=q.dtype, device=dev) if save_p else None
    hT1 = torch.empty(B, H, dk, m, dtype=torch.float32, device=dev) if output_final_state else None
    hT2 = torch.empty(B, H, m, dv, dtype=torch.float32, device=dev) if output_final_state else None
    ws, nb = _workspace(lib.gsa_fwd_workspace(B, H, T, dk, dv, m, chunk, dt), dev)
    _check(lib.gsa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(phi), _ptr(g), _ptr(h0_1), _ptr(h0_2), _ptr(o), _ptr(p),
                       _ptr(hT1), _ptr(hT2), B, H, T, dk, dv, m, chunk, dt, _ptr(ws), nb, _stream(dev)), "gsa_fwd")
    return o, p, hT1, hT2


def gsa_bwd(q, k, v, phi, g, do, h0_1=None, h0_2=None, dhT1=None, dhT2=None, chunk: int = 64,
            need_dh0: bool = True):
    """GSA backward: returns (dq, dk, dv, dphi, dg, dh0_1, dh0_2)."""
    _need_cuda(q, k, v, phi, g, do)
    B, H, T, dk = q.shape
    dv, m = v.shape[-1], phi.shape[-1]
    dt = _dtype_code(q)
    lib = load_library()
    dev = q.device
    h0_1 = _state(h0_1, (B, H, dk, m), dev)
    h0_2 = _state(h0_2, (B, H, m, dv), dev)
    dhT1 = _state(dhT1, (B, H, dk, m), dev)
    dhT2 = _state(dhT2, (B, H, m, dv), dev)
    dq, dkk = torch.empty_like(q), torch.empty_like(k)
    dvv, dphi, dg = torch.empty_like(v), torch.empty_like(phi), torch.empty_like(g)
    dh01 = torch.empty(B, H, dk, m, dtype=torch.float32, device=dev) if need_dh0 else None
    dh02 = torch.empty(B, H, m, dv, dtype=torch.float32, device=dev) if need_dh0 else None
    ws, nb = _workspace(lib.gsa_bwd_workspace(B, H, T, dk, dv, m, chunk, dt), dev)
    _check(lib.gsa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(phi), _ptr(g), _ptr(h0_1), _ptr(h0_2), _ptr(do),
                       _ptr(dhT1), _ptr(dhT2), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dphi), _ptr(dg), _ptr(dh01),
                       _ptr(dh02), B, H, T, dk, dv, m, chunk, dt, _ptr(ws), nb, _stream(dev)), "gsa_bwd")
    return dq, dkk, dvv, dphi, dg, dh01, dh02


def gsa_recurrent_step(q, k, v, phi, g, S1, S2):
    """One GSA decode step; S1 [B,H,dk,m], S2 [B,H,m,dv] fp32 updated in place.  Returns o [B,H,dv]."""
    _need_cuda(q, k, v, phi, g, S1, S2)
    B, H, dk = q.shape
    dv, m = v.shape[-1], phi.shape[-1]
    _state(S1, (B, H, dk, m), q.device)
    _state(S2, (B, H, m, dv), q.device)
    o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _check(load_library().gsa_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(phi), _ptr(g), _ptr(S1), _ptr(S2),
                                             _ptr(o), B, H, dk, dv, m, _dtype_code(q), _stream(q.device)),
           "gsa_recurrent_step")
    return o


def device_error(reset: bool = True, device=None) -> int:
    """Synchronise the current stream and return the device error latch (0 = no error)."""
    code = ctypes.c_int(0)
    dev = device or torch.device("cuda", torch.cuda.current_device())
    _check(load_library().gla_device_error(_stream(dev), int(reset), ctypes.byref(code)), "gla_device_error")
    return code.value


# ------------------------------------------------------------------------------------------
def gate_logsigmoid(x, tau: float):
    """Raw-logit gate: g = logsigmoid(x) / tau (same shape and dtype as x)."""
    _need_cuda(x)
    g = torch.empty_like(x)
    _check(load_library().gla_gate_logsigmoid(_ptr(x), _ptr(g), x.numel(), float(tau), _dtype_code(x),
                                             _stream(x.device)), "gla_gate_logsigmoid")
    return g


def gate_logsigmoid_bwd(x, dg, tau: float):
    """dx = dg * sigmoid(-x) / tau."""
    _need_cuda(x, dg)
    dx = torch.empty_like(x)
    _check(load_library().gla_gate_logsigmoid_bwd(_ptr(x), _ptr(dg), _ptr(dx), x.numel(), float(tau),
                                                 _dtype_code(x), _stream(x.device)), "gla_gate_logsigmoid_bwd")
    return dx


def _msgla(name, inp, rows_out, T, s):
    _need_cuda(inp)
    B, H, _, D = inp.shape
    out = torch.empty(B, H, rows_out, D, dtype=inp.dtype, device=inp.device)
    _check(getattr(load_library(), name)(_ptr(inp), _ptr(out), B, H, T, D, int(s), _dtype_code(inp),
                                         _stream(inp.device)), name)
    return out


def msgla_pool(x, s: int):
    """Average pooling of non-overlapping blocks of s tokens: [B,H,T,D] -> [B,H,ceil(T/s),D]."""
    T = x.shape[2]
    return _msgla("gla_msgla_pool", x, -(-T // s), T, s)


def msgla_pool_bwd(dy, T: int, s: int):
    return _msgla("gla_msgla_pool_bwd", dy, T, T, s)


def msgla_hold(y, T: int, s: int):
    """Causal hold back to T tokens: token t gets pooled row (t+1)//s - 1 (zeros before that)."""
    return _msgla("gla_msgla_hold", y, T, T, s)


def msgla_hold_bwd(dout, s: int):
    T = dout.shape[2]
    return _msgla("gla_msgla_hold_bwd", dout, -(-T // s), T, s)

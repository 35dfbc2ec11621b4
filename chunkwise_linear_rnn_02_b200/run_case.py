"""Run the GLA operators on one synthetic case, e.g. to profile a single kernel.

    python -m chunkwise_linear_rnn_02_b200.run_case --op fwd --B 8 --H 4 --T 2048 --dk 128 --dv 256 --iters 3

Inputs follow the seeded recipe of ``inputs.py``.  Prints the mean time per call measured with
CUDA events (not meaningful under a profiler).
"""
from __future__ import annotations

import argparse

import torch

from . import binding as gla
from .inputs import make_gla_inputs, make_gsa_inputs


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--op", choices=["fwd", "bwd", "fwdbwd", "decode", "gsa_fwd", "gsa_bwd"], default="fwdbwd")
    ap.add_argument("--B", type=int, default=8)
    ap.add_argument("--H", type=int, default=4)
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--dk", type=int, default=128)
    ap.add_argument("--dv", type=int, default=256)
    ap.add_argument("--m", type=int, default=64)
    ap.add_argument("--chunk", type=int, default=64)
    ap.add_argument("--dtype", choices=["bf16", "fp32"], default="bf16")
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args(argv)
    dt = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    if a.op.startswith("gsa"):
        d = {k: v.cuda() for k, v in make_gsa_inputs(a.B, a.H, a.T, a.dk, a.dv, a.m, dt).items()}
    else:
        d = {k: v.cuda() for k, v in make_gla_inputs(a.B, a.H, a.T, a.dk, a.dv, dt).items()}

    def call():
        if a.op in ("fwd", "fwdbwd"):
            gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], chunk=a.chunk)
        if a.op in ("bwd", "fwdbwd"):
            gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], chunk=a.chunk)
        if a.op == "decode":
            S = torch.zeros(a.B, a.H, a.dk, a.dv, device="cuda")
            gla.recurrent_step(d["q"][:, :, 0].contiguous(), d["k"][:, :, 0].contiguous(),
                               d["v"][:, :, 0].contiguous(), d["g"][:, :, 0].contiguous(), S)
        if a.op == "gsa_fwd":
            gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], chunk=a.chunk)
        if a.op == "gsa_bwd":
            gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], chunk=a.chunk)

    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(a.iters):
        call()
    e1.record()
    torch.cuda.synchronize()
    print(f"{a.op} B={a.B} H={a.H} T={a.T} dk={a.dk} dv={a.dv}: {e0.elapsed_time(e1) / a.iters:.4f} ms/call "
          f"(device error latch {gla.device_error()})")


if __name__ == "__main__":
    main()

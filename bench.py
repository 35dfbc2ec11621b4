#!/usr/bin/env python
"""Benchmark of the chunkwise GLA operator: forward + backward on one B200 per rank.

One step = gla_chunk_fwd then gla_chunk_bwd (the whole hot path) over one synthetic batch of the
340M-model layer shape (B=8, H=4, T=2048, d_k=128, d_v=256, chunk 64, bf16), inputs resident in
HBM.  L2 is flushed (256 MiB memset) between steps, outside the per-step CUDA events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  With N > 1 (torchrun, one rank per GPU) every rank runs the same
per-GPU workload on its own batch (weak scaling; the heads are independent, so there is no data
exchange); the step time is the max over ranks and `value` counts the tokens of all ranks.
`--impl reference` times the fp64 CPU oracle (the only other implementation of this operator)
on rank 0, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GLA chunk fwd+bwd tokens/s and % of roofline, 1 B200, vs host oracle"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
E2E_PARTS = 4  # batch slices (each on its own stream) in the end-to-end measurement


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gla_340m", choices=["gla_340m", "gla_1p3b"])
    ap.add_argument("--cpu-heads", type=int, default=24, help="heads in the oracle's CPU sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-slices", type=int, default=E2E_PARTS,
                    help="batch slices, each on its own stream, in the end-to-end measurement")
    ap.add_argument("--no-launch-count", action="store_true", help="skip the CUDA-profiler launch count")
    return ap.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    p = dict(FALLBACK_PEAKS)
    p["source"] = "fallback"
    return p


def algorithmic(cfg):
    """Compulsory bytes and algorithmic FLOPs of one fwd and one bwd call (per call, all heads)."""
    e = 2 if cfg.dtype.is_floating_point and cfg.dtype.itemsize == 2 else 4
    th = cfg.B * cfg.H * cfg.T
    dk, dv, C = cfg.dk, cfg.dv, cfg.chunk
    fwd_bytes = th * (3 * dk + dv) * e + th * dv * e + cfg.B * cfg.H * dk * dv * 4
    bwd_bytes = th * (3 * dk + 2 * dv) * e + th * (3 * dk + dv) * e
    fwd_flops = th * (4 * dk * dv + C * (dk + dv))
    bwd_flops = th * (8 * dk * dv + C * (3 * dk + 2 * dv))
    return fwd_bytes, bwd_bytes, fwd_flops, bwd_flops


def workload_desc(cfg, name):
    return {"workload": f"{name}: GLA fwd+bwd B={cfg.B} H={cfg.H} T={cfg.T} d_k={cfg.dk} d_v={cfg.dv} "
                        f"chunk={cfg.chunk} bf16, q,k,v,dO~N(0,1), q*d_k^-0.5, g=logsigmoid(N(0,1))/16, h0=0",
            "B": cfg.B, "H": cfg.H, "T": cfg.T, "d_k": cfg.dk, "d_v": cfg.dv, "chunk": cfg.chunk,
            "tokens_per_step_per_gpu": cfg.B * cfg.T,
            "l2": "flushed between steps (256 MiB memset outside the per-step events)"}


# ---------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=timestamp," + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "nvidia-smi unavailable"}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 1 + len(self.FIELDS):
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            rows.append((ts, parts[1:]))
        inside = [r for t, r in rows if self.t0 is not None and self.t0 - 0.15 <= t <= self.t1 + 0.15]
        use = inside if inside else [r for _, r in rows]
        sm = [float(r[0]) for r in use if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in use if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in use for n, v in zip(names, r[3:]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(use), "samples_inside_timed_region": len(inside)}


def gpu_id_for_smi(dev_index):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if dev_index < len(ids):
            return ids[dev_index]
    return dev_index


# ---------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------
def time_oracle(cfg, n_heads, seed=0):
    """Time the fp64 oracle fwd + bwd on the first n_heads heads of the workload; 1 thread."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    import oracle as O
    from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs

    nb = max(1, (n_heads + cfg.H - 1) // cfg.H)
    inp = make_gla_inputs(nb, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=seed)
    a = {k: v.reshape(nb * cfg.H, 1, cfg.T, -1)[:n_heads].double().numpy() for k, v in inp.items()}
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        O.gla_fwd(a["q"], a["k"], a["v"], a["g"])
        O.gla_bwd(a["q"], a["k"], a["v"], a["g"], None, a["do"])
        dt = time.perf_counter() - t0
    tokens = n_heads * cfg.T / cfg.H  # a token of the workload carries H heads
    return dt, tokens / dt, np


def run_reference(args, cfg, name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = []
    for i in range(args.warmup + args.steps):
        dt, _, _ = time_oracle(cfg, 1, seed=i)
        if i >= args.warmup:
            steps.append(dt)
    ms = 1e3 * statistics.mean(steps)
    tokens = cfg.T / cfg.H
    value = tokens / (ms / 1e3)
    sample = f"1 of {cfg.B * cfg.H} heads per step (T={cfg.T}), fwd+bwd, float64 numpy, 1 thread"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_desc(cfg, name),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------------------------
def count_launches(step_fn):
    """Kernels of this library launched by one step, counted with the CUDA profiler."""
    import torch
    from torch.profiler import ProfilerActivity, profile

    try:
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step_fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
        return sum(1 for n in names if "gla::" in n), sorted({n.split("<")[0].split("(")[0] for n in names
                                                               if "gla::" in n})
    except Exception as exc:  # profiler unavailable
        return None, [f"profiler unavailable: {exc}"]


def traffic_from_profiles(kernel_key):
    """Per-launch DRAM bytes recorded in profiles/*.md lines 'traffic_bytes_per_call[<key>]: N'."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    tag = f"traffic_bytes_per_call[{kernel_key}]:"
    for fn in sorted(os.listdir(pdir)):
        if not fn.endswith((".md", ".txt")):
            continue
        for line in open(os.path.join(pdir, fn)):
            if line.strip().startswith(tag):
                try:
                    return float(line.strip()[len(tag):].split()[0])
                except (ValueError, IndexError):
                    return None
    return None


def run_ours(args, cfg, name):
    import torch
    import torch.distributed as dist

    from chunkwise_linear_rnn_02_b200 import binding as gla
    from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs
    from chunkwise_linear_rnn_02_b200.ranks import batch_seed, max_over_ranks, rank_env, sum_over_ranks

    world, rank, local = rank_env()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    gla.load_library()

    inp = make_gla_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=batch_seed(1000, rank))
    d = {k: v.to(dev) for k, v in inp.items()}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def fwd():
        return gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], chunk=cfg.chunk)

    def bwd():
        return gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], chunk=cfg.chunk)

    def step():
        fwd()
        bwd()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    sampler = ClockSampler(gpu_id_for_smi(dev.index))
    sampler.start()
    for _ in range(max(3, args.warmup)):
        step()
        flush.zero_()
    barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler.mark("t0")
    for i in range(args.steps):
        evs[i][0].record()
        fwd()
        evs[i][1].record()
        bwd()
        evs[i][2].record()
        flush.zero_()
    barrier()
    sampler.mark("t1")
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    step_ms = fwd_ms + bwd_ms
    clocks = sampler.stop()
    step_ms, fwd_ms, bwd_ms = max_over_ranks([step_ms, fwd_ms, bwd_ms], dev)

    # end-to-end through the public API with host buffers: H2D inputs, fwd, bwd, D2H results.
    # The batch goes through in --e2e-slices slices of whole sequences, each on its own stream, so
    # that one slice's host->device copy, another's kernels and a third's device->host copy
    # overlap (the sequences are independent; every byte still crosses PCIe inside the region).
    names_in = ["q", "k", "v", "g", "do"]
    host_in = {k: inp[k].pin_memory() for k in names_in}
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    parts = args.e2e_slices if args.e2e_slices > 0 and cfg.B % args.e2e_slices == 0 else 1
    rows = cfg.B // parts
    streams = [torch.cuda.Stream(device=dev) for _ in range(parts)]
    e2e_times = []
    outs_host = None
    for i in range(args.e2e_steps + 2):
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        done = []
        for p_i, s_i in enumerate(streams):
            s_i.wait_event(e0)
            sl = slice(p_i * rows, (p_i + 1) * rows)
            with torch.cuda.stream(s_i):
                dd = {k: v[sl].to(dev, non_blocking=True) for k, v in host_in.items()}
                o, hT = gla.chunk_fwd(dd["q"], dd["k"], dd["v"], dd["g"], chunk=cfg.chunk)
                grads = gla.chunk_bwd(dd["q"], dd["k"], dd["v"], dd["g"], dd["do"], chunk=cfg.chunk,
                                      need_dh0=False)
                results = [o, hT] + [x for x in grads if x is not None]
                if outs_host is None:
                    outs_host = [torch.empty((cfg.B,) + tuple(x.shape[1:]), dtype=x.dtype, pin_memory=True)
                                 for x in results]
                for hbuf, x in zip(outs_host, results):
                    hbuf[sl].copy_(x, non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_i)
                done.append(ev)
        for ev in done:
            torch.cuda.current_stream().wait_event(ev)
        e1.record()
        torch.cuda.synchronize()
        flush.zero_()
        if i >= 2:
            e2e_times.append(e0.elapsed_time(e1))
    d2h = sum(x.numel() * x.element_size() for x in outs_host)
    e2e_ms = statistics.mean(e2e_times)
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)

    launches_per_step, kernel_names = (None, ["not counted"]) if args.no_launch_count else count_launches(step)
    peaks = load_peaks()
    fb, bb, ff, bf = algorithmic(cfg)
    (tokens,) = sum_over_ranks([cfg.B * cfg.T], dev)
    t_roof = max((fb + bb) / (peaks["hbm_gbs"] * 1e9), (ff + bf) / (peaks["bf16_tflops"] * 1e12))
    # dominant call: the larger of the fwd and bwd device times
    if bwd_ms >= fwd_ms:
        key, byt, ms, fl = "gla_chunk_bwd", bb, bwd_ms, bf
    else:
        key, byt, ms, fl = "gla_chunk_fwd", fb, fwd_ms, ff
    achieved = byt / (ms / 1e3) / 1e9
    traffic = traffic_from_profiles(f"{key}:{name}")
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "kernel": key,
                "algorithmic_bytes_per_call": byt, "call_ms": ms,
                "tensor_tflops_achieved": fl / (ms / 1e3) / 1e12,
                "peak_source": f"{peaks['source']} (HBM copy bandwidth)"}
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        n = min(args.cpu_heads, cfg.B * cfg.H)
        dt, val, _ = time_oracle(cfg, n)
        cpu = {"value": val, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"{n} of {cfg.B * cfg.H} heads, T={cfg.T}, fwd+bwd, float64 numpy, 1 thread, "
                         f"{dt:.1f} s; tokens = heads*T/H"}
    line = {"metric": METRIC, "value": tokens / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_desc(cfg, name), parallelism=f"replicas x{world} (independent heads)"),
            "pct_of_roofline": 100.0 * t_roof / (step_ms / 1e3), "roofline_step_ms": t_roof * 1e3,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "batch_slices_on_streams": parts},
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
            "launches_per_step": launches_per_step, "kernels": kernel_names, "clocks": clocks}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse_args()
    from chunkwise_linear_rnn_02_b200.inputs import CONFIGS

    cfg = CONFIGS[args.workload]
    if args.impl == "reference":
        run_reference(args, cfg, args.workload)
    else:
        run_ours(args, cfg, args.workload)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the chunkwise GLA operator: forward + backward on one B200 per rank.

One step = gla_chunk_fwd then gla_chunk_bwd (the whole hot path) over one synthetic batch of the
1.3B-model layer shape (B=8, H=4, T=2048, d_k=256, d_v=512, chunk 64, bf16; the largest
forward+backward workload), inputs resident in HBM.  L2 is flushed (256 MiB memset) between
steps, outside the per-step CUDA events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Prints ONE JSON line on rank 0.  With N > 1 (torchrun, one rank per GPU) every rank runs the same
per-GPU workload on its own batch (weak scaling; the heads are independent, so there is no data
exchange); the step time is the max over ranks and `value` counts the tokens of all ranks.
At N = 1 the line also carries, under `extra`, the other timed workloads: the 340M-model shape
(forward + backward), the long sequence (forward over 32768 tokens, then the microseconds per
gla_recurrent_step call over 256 decode steps) and GSA with 64 slots (forward + backward).
`--impl reference` times the fp64 CPU oracle (the only other implementation of this operator)
on rank 0, on a bounded sample of the same workload, spread over the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import json
import multiprocessing
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
GATE_DESC = {"gla": "g=logsigmoid(N(0,1))/16", "gsa": "g=logsigmoid(N(0,1))/8"}


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gla_1p3b", choices=["gla_1p3b", "gla_340m"])
    ap.add_argument("--cpu-tokens", type=int, default=512,
                    help="tokens per head (a prefix of the sequence) in the oracle's cpu_baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=128,
                    help="tokens per head in each step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' figures")
    ap.add_argument("--extra-steps", type=int, default=10)
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
    """Compulsory bytes and algorithmic FLOPs of one GLA fwd and one bwd call (per call, all heads).

    Bytes: the forward reads q, k, g, v and writes o and the fp32 final state; the backward reads
    q, k, g, v, dO and writes dq, dk, dg, dv.  FLOPs: the chunk form's contractions (causal half of
    the intra-chunk products)."""
    e = 2 if cfg.dtype.is_floating_point and cfg.dtype.itemsize == 2 else 4
    th = cfg.B * cfg.H * cfg.T
    dk, dv, C = cfg.dk, cfg.dv, cfg.chunk
    fwd_bytes = th * (3 * dk + dv) * e + th * dv * e + cfg.B * cfg.H * dk * dv * 4
    bwd_bytes = th * (3 * dk + 2 * dv) * e + th * (3 * dk + dv) * e
    fwd_flops = th * (4 * dk * dv + C * (dk + dv))
    bwd_flops = th * (8 * dk * dv + C * (3 * dk + 2 * dv))
    return fwd_bytes, bwd_bytes, fwd_flops, bwd_flops


def gsa_algorithmic(cfg):
    """Compulsory bytes and FLOPs of one GSA fwd and bwd call: both passes' contractions; the
    forward reads q, k, v, phi, g and writes o and both fp32 final states, the backward reads
    q, k, v, phi, g, dO and writes dq, dk, dv, dphi, dg."""
    th = cfg.B * cfg.H * cfg.T
    dk, dv, m, C = cfg.dk, cfg.dv, cfg.m, cfg.chunk
    fwd_bytes = th * (2 * dk + dv + 2 * m) * 2 + th * dv * 2 + cfg.B * cfg.H * (dk * m + m * dv) * 4
    bwd_bytes = th * (2 * dk + 2 * dv + 2 * m) * 2 + th * (2 * dk + dv + 2 * m) * 2

    def f(a, b):
        return 4 * a * b + C * (a + b), 8 * a * b + C * (3 * a + 2 * b)

    (f1, b1), (f2, b2) = f(dk, m), f(m, dv)
    return fwd_bytes, bwd_bytes, th * (f1 + f2), th * (b1 + b2)


def roofline_ms(nbytes, flops, peaks):
    return 1e3 * max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peaks["bf16_tflops"] * 1e12))


def workload_desc(cfg, name):
    return {"workload": f"{name}: GLA fwd+bwd B={cfg.B} H={cfg.H} T={cfg.T} d_k={cfg.dk} d_v={cfg.dv} "
                        f"chunk={cfg.chunk} bf16, q,k,v,dO~N(0,1), q*d_k^-0.5, {GATE_DESC['gla']}, h0=0",
            "B": cfg.B, "H": cfg.H, "T": cfg.T, "d_k": cfg.dk, "d_v": cfg.dv, "chunk": cfg.chunk,
            "tokens_per_step_per_gpu": cfg.B * cfg.T,
            "l2": "flushed between steps (256 MiB memset outside the per-step events)"}


def config_desc(cfg, name, world):
    """The `config` object of both arms' JSON lines (identical for the same workload and N)."""
    return dict(workload_desc(cfg, name), parallelism=f"replicas x{world} (independent heads)")


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
# CPU oracle timing (cpu_baseline leg and the reference arm), over the host cores
# ---------------------------------------------------------------------------------------------
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_piece(a):
    """One head of the oracle's fp64 fwd + bwd, single-threaded (runs in a pool worker)."""
    from threadpoolctl import threadpool_limits

    import oracle as O
    with threadpool_limits(limits=1):
        if a is None:  # warm-up: imports done, nothing timed
            return 0.0
        t0 = time.perf_counter()
        O.gla_fwd(a["q"], a["k"], a["v"], a["g"])
        O.gla_bwd(a["q"], a["k"], a["v"], a["g"], None, a["do"])
        return time.perf_counter() - t0


class OraclePool:
    """A spawn-started process pool (safe next to a CUDA context) running oracle head pieces."""

    def __init__(self, workers):
        self.workers = max(1, workers)
        self.pool = multiprocessing.get_context("spawn").Pool(self.workers)
        self.pool.map(_oracle_piece, [None] * self.workers)

    def pieces(self, cfg, n_heads, tokens, seed):
        from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs

        inp = make_gla_inputs(n_heads, 1, tokens, cfg.dk, cfg.dv, cfg.dtype, seed=seed)
        return [{n: inp[n][h:h + 1].double().numpy() for n in ["q", "k", "v", "g", "do"]} for h in range(n_heads)]

    def time(self, pieces):
        """Wall time of all pieces spread over the workers, and the summed single-thread times."""
        t0 = time.perf_counter()
        per = self.pool.map(_oracle_piece, pieces, chunksize=1)
        return time.perf_counter() - t0, sum(per)

    def close(self):
        self.pool.close()
        self.pool.join()


def cpu_baseline(cfg, name, tokens):
    """The oracle on min(B*H, host cores) heads x the first `tokens` tokens, one process per core."""
    heads = min(cfg.B * cfg.H, host_cores())
    tokens = min(tokens, cfg.T)
    pool = OraclePool(heads)
    try:
        wall, cpu_s = pool.time(pool.pieces(cfg, heads, tokens, seed=7))
    finally:
        pool.close()
    tok = heads * tokens / cfg.H  # a token of the workload carries H heads
    return {"value": tok / wall, "unit": "tokens/s", "cores": heads, "kind": "oracle",
            "sample": f"{heads} of {cfg.B * cfg.H} heads x the first {tokens} of {cfg.T} tokens of {name}, "
                      f"fwd+bwd, float64 numpy, one spawn process per core (1 BLAS thread each), wall {wall:.2f} s, "
                      f"{cpu_s:.1f} CPU-s; tokens = heads*tokens/H",
            "single_thread_value": tok / cpu_s, "host_cores": host_cores()}


def run_reference(args, cfg, name):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    heads = min(cfg.B * cfg.H, host_cores())
    tokens = min(args.ref_tokens, cfg.T)
    pool = OraclePool(heads)
    steps = []
    try:
        for i in range(args.warmup + args.steps):
            wall, _ = pool.time(pool.pieces(cfg, heads, tokens, seed=100 + i))
            if i >= args.warmup:
                steps.append(wall)
    finally:
        pool.close()
    ms = 1e3 * statistics.mean(steps)
    value = heads * tokens / cfg.H / (ms / 1e3)
    sample = (f"{heads} of {cfg.B * cfg.H} heads x {tokens} of {cfg.T} tokens per step, fwd+bwd, float64 numpy, "
              f"one spawn process per core (1 BLAS thread each); tokens = heads*tokens/H")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_desc(cfg, name, world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": heads, "kind": "oracle", "sample": sample},
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


def time_pair(first, second, steps, warmup, flush):
    """Mean CUDA-event times (ms) of first() and second() over `steps` steps, L2 flushed between."""
    import torch

    for _ in range(max(3, warmup)):
        first()
        second()
        flush.zero_()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        evs[i][0].record()
        first()
        evs[i][1].record()
        second()
        evs[i][2].record()
        flush.zero_()
    torch.cuda.synchronize()
    a = sum(e[0].elapsed_time(e[1]) for e in evs) / steps
    b = sum(e[1].elapsed_time(e[2]) for e in evs) / steps
    return a, b


def extra_workloads(args, dev, flush, peaks):
    """The other timed workloads, each with its own roofline (same device-timing rules)."""
    import torch

    from chunkwise_linear_rnn_02_b200 import binding as gla
    from chunkwise_linear_rnn_02_b200.inputs import CONFIGS, make_gla_inputs, make_gsa_inputs

    out = {}
    steps = args.extra_steps
    # the 340M-model shape (or the 1.3B one when that is not the main workload)
    other = "gla_340m" if args.workload != "gla_340m" else "gla_1p3b"
    cfg = CONFIGS[other]
    d = {k: v.to(dev) for k, v in make_gla_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.dtype, seed=1).items()}
    f_ms, b_ms = time_pair(lambda: gla.chunk_fwd(d["q"], d["k"], d["v"], d["g"], chunk=cfg.chunk),
                           lambda: gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], chunk=cfg.chunk),
                           steps, 3, flush)
    fb, bb, ff, bf = algorithmic(cfg)
    roof = roofline_ms(fb + bb, ff + bf, peaks)
    out[other] = {"what": workload_desc(cfg, other)["workload"], "fwd_ms": f_ms, "bwd_ms": b_ms,
                  "step_ms": f_ms + b_ms, "tokens_per_s": cfg.B * cfg.T / ((f_ms + b_ms) / 1e3),
                  "roofline_ms": roof, "pct_of_roofline": 100 * roof / (f_ms + b_ms), "steps": steps}
    del d
    # the long sequence: forward over T tokens, then 256 decode steps from its final state
    cfg = CONFIGS["gla_long"]
    n_dec = 256
    inp = make_gla_inputs(cfg.B, cfg.H, cfg.T + n_dec, cfg.dk, cfg.dv, cfg.dtype, seed=2, with_do=False)
    d = {k: v.to(dev) for k, v in inp.items()}
    head = {k: v[:, :, :cfg.T].contiguous() for k, v in d.items()}
    toks = [{k: v[:, :, t].contiguous() for k, v in d.items()} for t in range(cfg.T, cfg.T + n_dec)]
    state = {}

    def long_fwd():
        state["S"] = gla.chunk_fwd(head["q"], head["k"], head["v"], head["g"], chunk=cfg.chunk)[1]

    def decode():
        S = state["S"]
        for t in toks:
            gla.recurrent_step(t["q"], t["k"], t["v"], t["g"], S)

    f_ms, dec_ms = time_pair(long_fwd, decode, max(3, steps // 2), 3, flush)
    # the same 256 steps captured once as a CUDA graph and replayed: the device time per step
    # without the host's per-call overhead (the state is rewritten in place by every replay)
    graph_us = None
    try:
        S0 = state["S"].clone()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            decode()  # warm-up on the capturing stream
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode()
        reps = 10
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        state["S"].copy_(S0)
        graph.replay()
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        graph_us = 1e3 * e0.elapsed_time(e1) / (reps * n_dec)
        del graph
    except Exception as exc:  # capture unavailable: keep the eager figure only
        graph_us = f"not captured: {exc}"
    fb, _, ff, _ = algorithmic(cfg)
    roof = roofline_ms(fb, ff, peaks)
    dec_bytes = cfg.B * cfg.H * (2 * cfg.dk * cfg.dv * 4 + (3 * cfg.dk + 2 * cfg.dv) * 2)
    out["gla_long"] = {"what": f"gla_long: GLA fwd B={cfg.B} H={cfg.H} T={cfg.T} d_k={cfg.dk} d_v={cfg.dv} bf16, "
                               f"then {n_dec} gla_recurrent_step calls from its final state",
                       "fwd_ms": f_ms, "fwd_tokens_per_s": cfg.B * cfg.T / (f_ms / 1e3), "fwd_roofline_ms": roof,
                       "fwd_pct_of_roofline": 100 * roof / f_ms,
                       "decode_us_per_step": 1e3 * dec_ms / n_dec,
                       "decode_graph_us_per_step": graph_us,
                       "decode_roofline_us_per_step": 1e6 * dec_bytes / (peaks["hbm_gbs"] * 1e9),
                       "decode_note": "one launch per token; decode_us_per_step from eager calls (host-bound: "
                                      "Python and ctypes per call), decode_graph_us_per_step from a CUDA-graph "
                                      "replay of the 256 calls; L2 not flushed between decode steps (the 0.5 MB "
                                      "state stays resident, as in serving)"}
    del d, head, toks, state
    # GSA with 64 slots
    cfg = CONFIGS["gsa_64slots"]
    d = {k: v.to(dev) for k, v in make_gsa_inputs(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.m, cfg.dtype,
                                                  seed=3).items()}
    f_ms, b_ms = time_pair(lambda: gla.gsa_fwd(d["q"], d["k"], d["v"], d["phi"], d["g"], chunk=cfg.chunk),
                           lambda: gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"], chunk=cfg.chunk),
                           steps, 3, flush)
    fb, bb, ff, bf = gsa_algorithmic(cfg)
    roof = roofline_ms(fb + bb, ff + bf, peaks)
    out["gsa_64slots"] = {"what": f"gsa_64slots: GSA fwd+bwd B={cfg.B} H={cfg.H} T={cfg.T} d_k={cfg.dk} "
                                  f"d_v={cfg.dv} m={cfg.m} bf16, {GATE_DESC['gsa']}",
                          "fwd_ms": f_ms, "bwd_ms": b_ms, "step_ms": f_ms + b_ms,
                          "tokens_per_s": cfg.B * cfg.T / ((f_ms + b_ms) / 1e3), "roofline_ms": roof,
                          "pct_of_roofline": 100 * roof / (f_ms + b_ms), "steps": steps}
    del d
    torch.cuda.synchronize()
    return out


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
    del host_in, outs_host, streams

    launches_per_step, kernel_names = (None, ["not counted"]) if args.no_launch_count else count_launches(step)
    peaks = load_peaks()
    fb, bb, ff, bf = algorithmic(cfg)
    (tokens,) = sum_over_ranks([cfg.B * cfg.T], dev)
    t_roof = roofline_ms(fb + bb, ff + bf, peaks) / 1e3
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
                "flop_roofline_ms": 1e3 * fl / (peaks["bf16_tflops"] * 1e12),
                "peak_source": f"{peaks['source']} (HBM copy bandwidth)"}
    extra = None
    if world == 1 and not args.no_extra:
        del d
        extra = extra_workloads(args, dev, flush, peaks)
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(cfg, name, args.cpu_tokens)
    line = {"metric": METRIC, "value": tokens / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_desc(cfg, name, world),
            "pct_of_roofline": 100.0 * t_roof / (step_ms / 1e3), "roofline_step_ms": t_roof * 1e3,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "roofline": roofline, "cpu_baseline": cpu,
            "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "batch_slices_on_streams": parts},
            "gpu_launches": None if launches_per_step is None else launches_per_step * args.steps,
            "launches_per_step": launches_per_step, "kernels": kernel_names, "clocks": clocks,
            "extra": extra}
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

"""Host-side pieces of bench.py (CPU only): the compulsory byte counts behind the roofline, the
per-call DRAM traffic read back from the committed ncu summaries, and the reference arm's JSON
line (the fp64 oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import bench
from chunkwise_linear_rnn_02_b200.inputs import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_compulsory_bytes_of_the_benchmark_workload():
    """gla_340m (B=8, H=4, T=2048, d_k=128, d_v=256, bf16): forward reads q, k, g, v and writes o and
    the fp32 final state; backward reads q, k, g, v, dO and writes dq, dk, dg, dv."""
    cfg = CONFIGS["gla_340m"]
    fb, bb, ff, bf = bench.algorithmic(cfg)
    th = 8 * 4 * 2048
    assert fb == th * 2 * (3 * 128 + 2 * 256) + 8 * 4 * 128 * 256 * 4
    assert bb == th * 3072 == 201_326_592
    assert ff > 0 and bf > ff


def test_gsa_compulsory_bytes_and_flops():
    """gsa_64slots (B=4, H=4, T=4096, d_k=d_v=128, m=64): 3,600 bytes per token-head in all (reads of
    q, k, v, phi, g (+ dO) and writes of o (+ dq, dk, dv, dphi, dg)), plus the two fp32 final
    states; FLOPs are both passes' chunk-form contractions (d_k x m, then m x d_v)."""
    cfg = CONFIGS["gsa_64slots"]
    fb, bb, ff, bf = bench.gsa_algorithmic(cfg)
    th = 4 * 4 * 4096
    assert fb == th * 1280 + 16 * (128 * 64 + 64 * 128) * 4
    assert bb == th * 2304
    assert ff == th * 90112 and bf == th * 192512


def test_traffic_is_read_from_the_profile_summaries():
    """The roofline's `traffic` comes from a line of the committed ncu summary; it must parse to a
    byte count of the same order as the compulsory bytes (above them: workspace and re-reads)."""
    t = bench.traffic_from_profiles("gla_chunk_bwd:gla_340m")
    assert t is not None
    _, bb, _, _ = bench.algorithmic(CONFIGS["gla_340m"])
    assert bb < t < 5 * bb
    assert bench.traffic_from_profiles("no_such_call:gla_340m") is None


def test_reference_arm_prints_one_json_line():
    """`--impl reference` times the oracle on a sample of heads per step, spread over the host cores,
    and prints the contract's line."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"].startswith("gla_1p3b")
    # the same config object as the GPU arm's line for this workload and GPU count
    assert d["config"] == bench.config_desc(CONFIGS["gla_1p3b"], "gla_1p3b", 1)
    assert d["cpu_baseline"]["cores"] >= 1

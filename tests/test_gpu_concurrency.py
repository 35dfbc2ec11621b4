"""Concurrent callers of the entry points that fork onto the library's per-device side streams: the
blocked backward (wide shapes run as sub-problems on two streams), the GSA backward (its dq
forwards beside the first pass's backward) and the split backward (its two segment-state passes
side by side).  Two host threads, each on a CUDA stream of its own, run them at the same time; every
result must equal, bit for bit, the same call made alone (the kernels are deterministic)."""
import threading

import pytest
import torch

from chunkwise_linear_rnn_02_b200 import binding as gla
from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs, make_gsa_inputs
from helpers import cuda

pytestmark = pytest.mark.gpu


def _gla_bwd(d):
    return gla.chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["do"], h0=d["h0"], dhT=d["dhT"])


def _gsa_bwd(d):
    return gla.gsa_bwd(d["q"], d["k"], d["v"], d["phi"], d["g"], d["do"])


def _run_together(jobs):
    """Run each (fn, inputs) three times in its own thread and stream; return the last results."""
    results, errors = [None] * len(jobs), []

    def worker(j):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(3):
                    out = jobs[j][0](jobs[j][1])
            s.synchronize()
            results[j] = out
        except Exception as e:  # reported in the main thread
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(j,)) for j in range(len(jobs))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads), "a worker thread did not finish"
    assert not errors, errors
    return results


@pytest.mark.parametrize("second", ["blocked", "gsa", "split"])
def test_concurrent_callers_match_single_calls(second):
    wide = cuda(make_gla_inputs(2, 2, 300, 256, 512, torch.bfloat16, seed=81, with_h0=True, with_dhT=True))
    if second == "blocked":
        other = (_gla_bwd, cuda(make_gla_inputs(1, 3, 260, 256, 512, torch.bfloat16, seed=82, with_h0=True,
                                                with_dhT=True)))
    elif second == "gsa":
        other = (_gsa_bwd, cuda(make_gsa_inputs(1, 4, 700, 128, 128, 64, torch.bfloat16, seed=83)))
    else:  # two heads over 2,000 tokens: the backward splits the sequence into segments
        other = (_gla_bwd, cuda(make_gla_inputs(1, 2, 2000, 128, 256, torch.bfloat16, seed=84, with_h0=True,
                                                with_dhT=True)))
    jobs = [(_gla_bwd, wide), other]
    alone = [fn(d) for fn, d in jobs]
    torch.cuda.synchronize()
    together = _run_together(jobs)
    for j, (a, r) in enumerate(zip(alone, together)):
        for n, (x, y) in enumerate(zip(a, r)):
            if x is None:
                assert y is None
                continue
            assert torch.equal(x, y), f"job {j}, output {n}: differs when another caller runs at the same time"
    assert gla.device_error() == 0

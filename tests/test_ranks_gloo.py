"""Multi-rank host logic on CPU: two gloo ranks, no GPU.

Covers what a multi-GPU run of the operator adds to the single-GPU path: each rank owns whole
sequences (shard_rows), seeds its own batch (batch_seed), and the step time / token count combine
as max / sum over ranks.  The data-parallel claim itself is checked by having each rank run the
fp64 oracle on its shard of a tiny batch and gathering the shards: the result must equal the
oracle on the whole batch, since sequences do not interact.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from chunkwise_linear_rnn_02_b200.inputs import make_gla_inputs
from chunkwise_linear_rnn_02_b200.ranks import batch_seed, max_over_ranks, shard_rows, sum_over_ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    import datetime

    from oracle import gla_oracle as ora

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        res["max"] = max_over_ranks([rank + 1.0, 10.0 - rank])
        res["sum"] = sum_over_ranks([1000.0 * (rank + 1)])
        # data parallel: the oracle on this rank's rows of one shared tiny batch
        d = make_gla_inputs(3, 2, 40, 8, 8, torch.float32, seed=7)
        lo, hi = shard_rows(3, world, rank)
        o, hT = ora.gla_fwd(d["q"][lo:hi].numpy(), d["k"][lo:hi].numpy(), d["v"][lo:hi].numpy(),
                            d["g"][lo:hi].numpy())
        shards = [None] * world
        dist.all_gather_object(shards, (lo, hi, o, hT))
        res["shards"] = shards
        torch.save(res, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_shard_rows_partition():
    for n in range(0, 11):
        for world in range(1, 5):
            spans = [shard_rows(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(4, 2, 2)


def test_batch_seed_distinct():
    assert len({batch_seed(1000, r) for r in range(8)}) == 8


def test_single_process_reductions_are_identity():
    assert max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
    assert sum_over_ranks([3.0]) == [3.0]


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    from oracle import gla_oracle as ora

    d = make_gla_inputs(3, 2, 40, 8, 8, torch.float32, seed=7)
    o_ref, hT_ref = ora.gla_fwd(d["q"].numpy(), d["k"].numpy(), d["v"].numpy(), d["g"].numpy())
    for rank in range(world):
        res = torch.load(os.path.join(tmp_path, f"rank{rank}.pt"), weights_only=False)
        assert res["max"] == [2.0, 10.0]
        assert res["sum"] == [3000.0]
        o = np.concatenate([s[2] for s in res["shards"]], axis=0)
        hT = np.concatenate([s[3] for s in res["shards"]], axis=0)
        assert [s[:2] for s in res["shards"]] == [(0, 2), (2, 3)]
        np.testing.assert_array_equal(o, o_ref)
        np.testing.assert_array_equal(hT, hT_ref)

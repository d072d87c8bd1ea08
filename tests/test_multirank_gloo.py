"""The multi-GPU host logic on CPU: two gloo ranks (spawned processes).

The hot path needs no data-path collective; what runs across ranks is the
work assignment (independent seeded batches, or slices of one batch) and the
timing reduction (max over ranks). Both are checked here with world size 2.
"""

import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_softmax_attention_causal_b200 import sharding, workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # 1. independent batches: every rank draws from its own seed
        x = workloads.prefill_inputs(1, 2, 1, 16, 8, sharding.rank_seed(0, rank))
        mine = x.q.float().sum().reshape(1)
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, mine)
        # 2. slices of one global batch cover it exactly once
        sl = list(sharding.batch_slice(7, world, rank))
        lens = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(lens, torch.tensor([len(sl)]))
        # 3. the step time is the maximum over ranks
        t = sharding.max_over_ranks([10.0 + rank, 5.0 * (world - rank)])
        results[rank] = {"sums": [float(g) for g in gathered], "slice": sl,
                         "lens": [int(v) for v in lens], "max": t}
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
        res = dict(results)
    assert sorted(res) == [0, 1]
    # identical views on every rank, distinct batches per rank
    assert res[0]["sums"] == res[1]["sums"]
    assert res[0]["sums"][0] != res[0]["sums"][1]
    # rank 0's batch is the single-process batch of the same seed
    solo = workloads.prefill_inputs(1, 2, 1, 16, 8, 0).q.float().sum().item()
    assert res[0]["sums"][0] == pytest.approx(solo, abs=0)
    # the slices partition range(7)
    assert sorted(res[0]["slice"] + res[1]["slice"]) == list(range(7))
    assert res[0]["lens"] == [4, 3]
    # max over ranks: [max(10, 11), max(10, 5)]
    assert res[0]["max"] == res[1]["max"] == [11.0, 10.0]


@pytest.mark.parametrize("n,world", [(0, 3), (1, 4), (64, 8), (5, 2)])
def test_batch_slices_partition(n, world):
    got = [list(sharding.batch_slice(n, world, r)) for r in range(world)]
    assert sum(got, []) == list(range(n))
    assert max(map(len, got)) - min(map(len, got)) <= 1


def test_job_throughput_counts_all_ranks():
    # 2 ranks x 3 steps x 1e12 FLOP in 1.5 s (the slowest rank) = 4 TFLOP/s
    assert sharding.job_throughput(1e12, 2, 3, 1500.0) == pytest.approx(4e12)
    with pytest.raises(ValueError):
        sharding.job_throughput(1.0, 1, 1, 0.0)

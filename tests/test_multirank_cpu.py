"""The N > 1 path of the benchmark on CPU: two gloo ranks.

Every (sequence, head) of the CPR layer is independent, so more GPUs means
more sequences, one shard per rank, and no data-path collective.  The only
collectives are the timing reduction (max over ranks) and barriers.  These
tests run that host logic with world_size 2 over gloo and check:
* the shards are disjoint;
* the maximum is taken over ranks;
* the whole-job throughput counts every rank's tokens.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ids = list(bench.rank_sequence_ids(rank, 4))
        gathered = [None] * world
        dist.all_gather_object(gathered, ids)
        my_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(my_ms, world, device="cpu")
        thr = bench.job_throughput(4 * 4096, world, mx, steps=2)
        out[rank] = (gathered, mx, thr)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_shard_and_time():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        gathered, mx, thr = out[rank]
        assert set(gathered[0]).isdisjoint(gathered[1])
        assert sorted(gathered[0] + gathered[1]) == list(range(8))
        assert mx == 15.0
        # 2 ranks x 4 sequences x 4096 tokens x 2 steps over the slowest 15 ms
        assert thr == pytest.approx(2 * 4 * 4096 * 2 / 0.015)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert list(bench.rank_sequence_ids(0, 3)) == [0, 1, 2]
    assert bench.job_throughput(100, 1, 1000.0, 1) == pytest.approx(100.0)

"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The codec shards over units with no data-path collective: every rank compresses its own batch of
the same shape (weak scaling); the only collectives are the barrier and the MAX of the timed
region over ranks.  These tests run that host logic in two gloo processes.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from dct_transform_coding_b200.workloads import WORKLOADS, make_batch


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.rank_workload(WORKLOADS["tiny"], rank)
        x = make_batch(w)                                  # this rank's batch
        my_ms = 10.0 + 5.0 * rank                          # a stand-in for the rank's timed region
        dist.barrier()
        ms = bench.max_over_ranks(my_ms, dist, torch.device("cpu"))
        out[rank] = (float(x.double().sum()), tuple(x.shape), ms,
                     bench.job_gbs(world, x.numel() * x.element_size(), ms))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_units_and_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    (s0, shape0, ms0, v0), (s1, shape1, ms1, v1) = out[0], out[1]
    assert shape0 == shape1                                # same work per rank (weak scaling)
    assert s0 != s1                                        # independent seeds: different batches
    assert ms0 == ms1 == 15.0                              # both ranks report the slowest rank
    assert v0 == v1
    nbytes = 1
    for d in shape0:
        nbytes *= d
    nbytes *= 4                                            # the tiny workload is fp32
    assert v0 == pytest.approx(2 * nbytes / 15e-3 / 1e9)


def test_single_rank_workload_is_the_configured_one():
    w = WORKLOADS["med4b"]
    assert bench.rank_workload(w, 0) == w
    assert bench.rank_workload(w, 1).seed != w.seed

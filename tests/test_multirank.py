"""The N > 1 benchmark path, on CPU: replicas only (no data-path
collective), device times reduced to the maximum over ranks, throughput
aggregated over all ranks. Two gloo ranks on 127.0.0.1."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" (1 + r) ms and (10 + 3r) ms end to end
        got = bench.max_over_ranks([1.0 + rank, 10.0 + 3 * rank], world, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
        res = dict(out)
    # every rank ends with the slowest rank's times
    assert res[0] == res[1] == [2.0, 13.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 7.0], 1, "cpu") == [3.5, 7.0]


def test_whole_job_value_aggregates_ranks():
    # 4 ranks x 100 steps x 2 MB in 1 ms -> 800 GB/s whole job
    assert bench.whole_job_value(4, 100, 2e6, 1.0, 1e9) == pytest.approx(800.0)
    assert bench.whole_job_value(1, 100, 2e6, 1.0, 1e9) == pytest.approx(200.0)


def test_replicas_get_distinct_inputs_except_the_seeded_copy():
    assert bench.replica_seed(2, 0, 0) == bench.replica_seed(2, 0, 3) == 2
    seeds = {bench.replica_seed(2, c, r) for c in range(1, 128) for r in range(8)}
    assert len(seeds) == 127 * 8

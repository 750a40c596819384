"""Host logic of the multi-GPU run (bench.py --gpus N): the layers are
independent problems, so each rank quantizes its own layer and the only
cross-rank step is taking the slowest rank's step time.  Exercised here with
two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        local_ms = 5.0 + 3.0 * rank            # rank 1 is the slower one
        got = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        off = bench.replica_seed_offset(rank)
        # each rank draws a different layer from the same workload recipe
        w = workloads.gaussian_weights(4, 8, 0.02, seed=workloads.BASE_SEED + 104729 * off)
        gathered = [torch.zeros_like(w) for _ in range(world)]
        dist.all_gather(gathered, w)
        out[rank] = (got, off, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step_and_distinct_layers():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    assert out[0][0] == out[1][0] == 8.0          # max over ranks on both ranks
    assert {out[0][1], out[1][1]} == {0, 1}        # one layer per rank
    assert out[0][2] is False and out[1][2] is False  # the layers differ


def test_job_throughput_counts_every_rank():
    import bench
    one = bench.job_weights_per_s(1, 4096, 4096, 8.0)
    eight = bench.job_weights_per_s(8, 4096, 4096, 8.0)
    assert eight == pytest.approx(8 * one)
    assert one == pytest.approx(4096 * 4096 / 8e-3)
    assert bench.max_over_ranks(3.5) == 3.5

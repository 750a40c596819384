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


def test_stage_rooflines_use_the_closed_forms():
    """The bench line's per-stage bounds: the lazy update of a d_col that is a
    whole number of blocks does r d (d - B) flop (each block updates the
    columns after it), the Hessian n d (d + 1), the inverse factor 2/3 d^3 and
    pack r d (1 + b/8) bytes; the layer's bound is their sum plus the column
    walk's r d B flop on the FFMA pipe."""
    import bench
    import workloads
    wl = workloads.WORKLOADS["llama7b_q_proj"]
    r, d, n, B, b = wl.d_row, wl.d_col, wl.n_tokens, wl.block_size, wl.bits
    pk = {"bf16_tflops": 1600.0, "hbm_gbs": 6400.0}
    ms = {"hessian": 3.0, "prepare_hinv": 1.4, "quantize_layer": 1.1, "pack": 0.01}
    out = bench.stage_rooflines(wl, pk, "measured", ms, 5.6)
    st = out["stages"]
    tf32x3 = 1600.0 * 1.1 / 2.25 / 3
    assert st["hessian"]["bound_ms"] == pytest.approx(n * d * (d + 1) / 1600e12 * 1e3)
    assert st["prepare_hinv"]["bound_ms"] == pytest.approx(2 * d ** 3 / 3 / (tf32x3 * 1e12) * 1e3)
    lazy = r * d * (d - B)
    walk = r * d * B
    assert st["quantize_layer"]["bound_ms"] == pytest.approx(
        (lazy / (tf32x3 * 1e12) + walk / (148 * 128 * 2 * 1.965e9)) * 1e3)
    assert st["pack"]["bound_ms"] == pytest.approx(r * d * (1 + b / 8) / 6400e9 * 1e3)
    total = sum(v["bound_ms"] for v in st.values())
    assert out["sum_bound_ms"] == pytest.approx(total)
    assert out["layer_frac_of_summed_bound"] == pytest.approx(total / 5.6)
    for name, v in st.items():
        assert v["frac"] == pytest.approx(v["bound_ms"] / ms[name])
    # a ragged layer (d_col = 300): block 0 updates the 172 columns after it,
    # block 1 the last 44, the partial block 2 nothing
    import dataclasses
    rag = dataclasses.replace(wl, d_col=300)
    out = bench.stage_rooflines(rag, pk, "measured", ms, 5.6)
    assert f"lazy update {2.0 * r * B * (172 + 44):.3e} flop" in out["stages"]["quantize_layer"]["work"]

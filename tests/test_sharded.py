"""Host logic of one layer spread over several ranks (package module
``sharded``): token and row shards, the all-reduce of the partial Hessians,
the status combination and the gather of the row slices.  Exercised with gloo
ranks on the CPU, the per-rank arithmetic done by the float64 oracle: the
sharded result must be the unsharded one (H to rounding, the quantized rows
bit for bit, since rows are independent given H^-1)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_gptq_b200 import sharded


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("n,world,quantum", [(0, 2, 64), (1, 2, 64), (64, 3, 64), (1000, 2, 64),
                                             (5 * 64 + 7, 4, 64), (262144, 8, 32768),
                                             (40000, 3, 32768), (100, 5, 64)])
def test_token_shards_cover_the_tokens_on_quantum_boundaries(n, world, quantum):
    spans = [sharded.token_range(n, k, world, quantum) for k in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a0, a1), (b0, b1) in zip(spans[:-1], spans[1:]):
        assert a1 == b0                                   # contiguous, no overlap
    for t0, t1 in spans:
        assert 0 <= t0 <= t1 <= n
        assert t0 % quantum == 0 or t0 == n               # every shard starts on a boundary
    units = [-(-(t1 - t0) // quantum) for t0, t1 in spans]
    assert max(units) - min(units) <= 1                   # balanced to one unit


@pytest.mark.parametrize("d_row,world", [(0, 2), (1, 2), (7, 3), (4096, 8), (11008, 3), (5, 8)])
def test_row_shards_are_balanced_and_contiguous(d_row, world):
    spans = [sharded.row_range(d_row, k, world) for k in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == d_row
    assert all(a[1] == b[0] for a, b in zip(spans[:-1], spans[1:]))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_bad_ranks_are_rejected():
    with pytest.raises(ValueError):
        sharded.token_range(10, 2, 2)
    with pytest.raises(ValueError):
        sharded.row_range(10, -1, 2)
    with pytest.raises(ValueError):
        sharded.token_range(-1, 0, 1)


def _worker(rank, world, port, case, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    import workloads
    from post_weight_quantization_gptq_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        n, d, r, quantum, bits, g, desc_act = case
        W, X = workloads.small_layer(r, d, n, seed=workloads.BASE_SEED + 11)
        t0, t1 = sh.token_range(n, rank, world, quantum)
        H = torch.from_numpy(oracle.hessian(X[t0:t1]) if t1 > t0 else np.zeros((d, d)))
        sh.allreduce_hessian(H)
        H = H.numpy()
        r0, r1 = sh.row_range(r, rank, world)
        res = oracle.quantize_layer(H, W[r0:r1], bits=bits, group_size=g, desc_act=desc_act)
        packed = torch.from_numpy(oracle.pack(res["codes"], bits).view(np.int32))
        p, s, z = sh.gather_quantized(packed, torch.from_numpy(res["scales"]),
                                      torch.from_numpy(res["zeros"]), r)
        # a device error on one rank reaches every rank
        status = sh.combine_status(3 if rank == world - 1 else 0, torch.device("cpu"))
        out[rank] = dict(H=H, packed=p.numpy(), scales=s.numpy(), zeros=z.numpy(),
                         perm=res["perm"], status=status)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,case", [
    (2, (300, 24, 37, 64, 4, 8, False)),      # ragged tokens and rows
    (3, (100, 16, 5, 64, 3, -1, True)),       # a rank with no tokens, act-order, 3-bit
    (2, (256, 16, 1, 64, 4, 8, False)),       # a rank with no rows
])
def test_gloo_ranks_reproduce_the_unsharded_layer(world, case):
    import oracle
    import workloads
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), case, out), nprocs=world,
                       start_method="spawn", join=True)
    n, d, r, quantum, bits, g, desc_act = case
    W, X = workloads.small_layer(r, d, n, seed=workloads.BASE_SEED + 11)
    H = oracle.hessian(X)
    Hs = out[0]["H"]
    # the shard sums differ from the one-pass sum only in float64 rounding
    assert np.allclose(Hs, H, rtol=1e-12, atol=1e-12 * np.abs(H).max())
    ref = oracle.quantize_layer(Hs, W, bits=bits, group_size=g, desc_act=desc_act)
    for k in range(world):
        o = out[k]
        assert o["status"] == 3
        assert np.array_equal(o["H"], Hs)                 # every rank holds the same sum
        assert np.array_equal(o["perm"], ref["perm"])
        # rows are independent given H^-1: the gathered slices are the layer
        assert np.array_equal(o["packed"].view(np.uint32), oracle.pack(ref["codes"], bits))
        assert np.array_equal(o["scales"], ref["scales"])
        assert np.array_equal(o["zeros"], ref["zeros"])


def _bad_shape_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import post_weight_quantization_gptq_b200 as g
    from post_weight_quantization_gptq_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        d_row, d_col = 10, 16
        r0, r1 = sh.row_range(d_row, rank, world)
        X = torch.zeros(4, d_col, dtype=torch.bfloat16)
        W = torch.zeros(r1 - r0 + 1, d_col)  # one row too many: rejected before any device work
        try:
            sh.quantize_layer_sharded(X, W, d_row, g.GPTQConfig())
            out[rank] = "accepted"
        except ValueError as e:
            out[rank] = "rows [%d, %d)" % (r0, r1) in str(e)
    finally:
        dist.destroy_process_group()


def test_a_wrong_row_slice_is_rejected_on_the_host():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_bad_shape_worker, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    assert out[0] is True and out[1] is True

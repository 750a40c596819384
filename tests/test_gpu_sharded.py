"""One layer spread over two processes through the CUDA library
(``sharded.quantize_layer_sharded``): each process accumulates its token
shard, the partial Hessians are summed, both build U, and each quantizes its
row slice.  The two processes share one GPU and talk through gloo (host
staging), so no kernel waits on another process; the NCCL form differs only
in the transport of the same collectives.  Checked against the float64
oracle on the summed H, as the single-process parity tests are."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gptq_testlib import compare_quantization, lower_rel_err

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, case, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import workloads
    import post_weight_quantization_gptq_b200 as g
    from post_weight_quantization_gptq_b200 import sharded as sh
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        n, d, r, bits, gs, desc_act = case
        W, X = workloads.small_layer(r, d, n, seed=workloads.BASE_SEED + 21)
        t0, t1 = sh.token_range(n, rank, world)
        r0, r1 = sh.row_range(r, rank, world)
        cfg = g.GPTQConfig(bits=bits, group_size=gs, desc_act=desc_act)
        Wl = W[r0:r1].contiguous().cuda()
        res = sh.quantize_layer_sharded(X[t0:t1].cuda(), Wl, r, cfg)
        # the summed H the ranks factorized, for the oracle comparison
        H = torch.zeros(d, d, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        g.gptq_hessian_accumulate(X[t0:t1].cuda(), H, st)
        sh.allreduce_hessian(H)
        out[rank] = dict(rows=res["rows"], codes=res["codes"].cpu().numpy(),
                         w=res["w_at_quant"].cpu().numpy(),
                         perm=res["perm"].cpu().numpy(), dead=res["dead"].cpu().numpy(),
                         packed_all=res["packed_all"].cpu().numpy(),
                         scales_all=res["scales_all"].cpu().numpy(),
                         zeros_all=res["zeros_all"].cpu().numpy(),
                         H=H.cpu().numpy(), status=g.gptq_sync_status(st))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", [
    (3 * 32768 + 1000, 512, 300, 4, 128, False),   # ragged token shard and row slices
    (40000, 384, 257, 4, 32, True),                # act-order, g32
])
def test_two_processes_quantize_one_layer(case):
    import oracle
    import workloads
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), case, out), nprocs=world,
                       start_method="spawn", join=True)
    n, d, r, bits, gs, desc_act = case
    W, X = workloads.small_layer(r, d, n, seed=workloads.BASE_SEED + 21)
    o0, o1 = out[0], out[1]
    assert o0["status"] == o1["status"] == 0
    assert np.array_equal(o0["H"], o1["H"])
    # per-drain accumulation drift of the tensor cores (32768-token drains);
    # the H bar of the parity rules is 1e-3
    assert lower_rel_err(o0["H"], oracle.hessian(X)) <= 3e-4
    for k in ("perm", "dead", "packed_all", "scales_all", "zeros_all"):
        assert np.array_equal(o0[k], o1[k]), k           # both ranks hold the same layer
    codes = np.concatenate([o0["codes"], o1["codes"]])
    w = np.concatenate([o0["w"], o1["w"]])
    assert np.array_equal(o0["packed_all"].view(np.uint32), oracle.pack(codes, bits))
    gpu = dict(status=0, perm=o0["perm"], dead=o0["dead"].astype(bool), codes=codes,
               scales=o0["scales_all"], zeros=o0["zeros_all"], w_at_quant=w,
               packed=o0["packed_all"].view(np.uint32))
    Hl = np.tril(o0["H"].astype(np.float64))            # the kernel writes the lower triangle
    compare_quantization(Hl + np.tril(Hl, -1).T, W, gpu, bits, gs, desc_act)

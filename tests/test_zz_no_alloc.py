"""gptq_quantize_layer_noalloc: the column walk for callers that cannot
allocate device memory (an enqueue call that may not allocate, a memory pool
already holding nearly all of HBM, a path that cannot afford the device
synchronization of cudaMalloc / cudaFree).  Its scratch is a fixed array
inside the library instead of a caller workspace.

Checked through the C ABI against gptq_quantize_layer (which takes a
workspace) on the same inputs, for two calls in a row: the shared scratch
keeps the previous call's contents, and the second call must not depend on
them.  Collected last (file name) so that a stop-at-first-failure run has
already run every other test."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_gptq_b200 as pkg
    return pkg


def _prepared(g, d_row, d_col, bits, group, desc_act, seed):
    W, X = workloads.small_layer(d_row, d_col, 4 * d_col, seed=seed, kind="student_t")
    H = torch.from_numpy(oracle.hessian(X).astype(np.float32)).cuda()
    cfg = g.GPTQConfig(bits=bits, group_size=group, desc_act=desc_act)
    ws = torch.empty(g.gptq_workspace_size(cfg, d_row, d_col), dtype=torch.uint8, device="cuda")
    U = torch.empty(d_col, d_col, device="cuda")
    perm = torch.empty(d_col, dtype=torch.int32, device="cuda")
    dead = torch.empty(d_col, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    return W, cfg, ws, U, perm, dead, st


def _outputs(g, d_row, d_col, group):
    ng = g.n_groups(d_col, group)
    return (torch.empty(d_row, d_col, dtype=torch.uint8, device="cuda"),
            torch.empty(ng, d_row, dtype=torch.float32, device="cuda"),
            torch.empty(ng, d_row, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("d_row,d_col,bits,group,desc_act",
                         [(300, 1024, 4, 128, True), (77, 640, 3, 32, False)])
def test_noalloc_matches_the_workspace_entry_point_twice(g, d_row, d_col, bits, group, desc_act):
    W, cfg, ws, U, perm, dead, st = _prepared(g, d_row, d_col, bits, group, desc_act,
                                              seed=d_row + d_col)
    Wref = W.cuda().contiguous()
    ref = _outputs(g, d_row, d_col, group)
    g.gptq_quantize_layer(Wref, U, perm, dead, cfg, *ref, st, ws)
    assert g.gptq_sync_status(st) == 0
    for call in range(2):
        Wn = W.cuda().contiguous()
        out = _outputs(g, d_row, d_col, group)
        for t in out:
            t.fill_(0xFF if t.dtype == torch.uint8 else 7)
        g.gptq_quantize_layer_noalloc(Wn, U, perm, dead, cfg, *out, st)
        assert g.gptq_sync_status(st) == 0, call
        # same kernels, same inputs: identical results (well inside the
        # parity tolerances: codes exact, scales 1e-4 relative)
        assert torch.equal(out[0], ref[0]), call
        assert torch.equal(out[2], ref[2]), call
        assert torch.allclose(out[1], ref[1], rtol=1e-4, atol=0), call
        assert torch.equal(out[1], ref[1]), call
        assert torch.equal(Wn, Wref), call


def test_noalloc_rejects_layers_beyond_its_scratch(g):
    assert g.gptq_noalloc_scratch_bytes() == 16 << 20
    d_row, d_col = 40000, 128   # needs d_row * 512 bytes > 16 MiB
    cfg = g.GPTQConfig(bits=4, group_size=128)
    W = torch.zeros(d_row, d_col, device="cuda")
    U = torch.eye(d_col, device="cuda")
    perm = torch.arange(d_col, dtype=torch.int32, device="cuda")
    dead = torch.zeros(d_col, dtype=torch.uint8, device="cuda")
    out = _outputs(g, d_row, d_col, 128)
    with pytest.raises(g.GPTQError) as e:
        g.gptq_quantize_layer_noalloc(W, U, perm, dead, cfg, *out, None)
    assert e.value.status == 6

"""gptq_quantize_layer_noalloc: the column walk for callers that cannot
allocate device memory (an enqueue call that may not allocate, a memory pool
already holding nearly all of HBM, a path that cannot afford the device
synchronization of cudaMalloc / cudaFree).  Its scratch is a fixed array
inside the library instead of a caller workspace.

Checked through the C ABI against gptq_quantize_layer (which takes a
workspace) on the same inputs, for two calls in a row, each preceded by a
noalloc call on a different layer (other d_row, other d_col and so another
error-buffer pitch, weights 1000x larger) so that the shared scratch holds
another call's leftovers: a call must not depend on them.  Collected last
(file name) so that a stop-at-first-failure run has already run every other
test."""
import ctypes

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


def _prepared(g, d_row, d_col, bits, group, desc_act, seed, scale=1.0):
    W, X = workloads.small_layer(d_row, d_col, 4 * d_col, seed=seed, kind="student_t")
    H = torch.from_numpy(oracle.hessian(X).astype(np.float32)).cuda()
    cfg = g.GPTQConfig(bits=bits, group_size=group, desc_act=desc_act)
    ws = torch.empty(g.gptq_workspace_size(cfg, d_row, d_col), dtype=torch.uint8, device="cuda")
    U = torch.empty(d_col, d_col, device="cuda")
    perm = torch.empty(d_col, dtype=torch.int32, device="cuda")
    dead = torch.empty(d_col, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    assert g.gptq_sync_status(st) == 0
    return W * scale, X, cfg, ws, U, perm, dead, st


def _outputs(g, d_row, d_col, group):
    ng = g.n_groups(d_col, group)
    out = (torch.empty(d_row, d_col, dtype=torch.uint8, device="cuda"),
           torch.empty(ng, d_row, dtype=torch.float32, device="cuda"),
           torch.empty(ng, d_row, dtype=torch.int32, device="cuda"))
    for t in out:
        t.fill_(0xFF if t.dtype == torch.uint8 else 7)
    return out


def _other_layer(g, d_row, d_col):
    """A noalloc call on a different layer: it leaves its own errors (with
    its own pitch, 1000x larger) in the shared scratch."""
    W, _, cfg, _, U, perm, dead, st = _prepared(g, d_row, d_col, 4, 128, False, seed=d_row + 5,
                                                scale=1000.0)
    out = _outputs(g, d_row, d_col, 128)
    g.gptq_quantize_layer_noalloc(W.cuda().contiguous(), U, perm, dead, cfg, *out, st)
    assert g.gptq_sync_status(st) == 0


@pytest.mark.parametrize("d_row,d_col,bits,group,desc_act,other",
                         [(300, 1024, 4, 128, True, (1000, 640)),
                          (77, 640, 3, 32, False, (513, 1536))])
def test_noalloc_matches_the_workspace_entry_point_twice(g, d_row, d_col, bits, group, desc_act,
                                                         other):
    W, _, cfg, ws, U, perm, dead, st = _prepared(g, d_row, d_col, bits, group, desc_act,
                                                 seed=d_row + d_col)
    Wref = W.cuda().contiguous()
    ref = _outputs(g, d_row, d_col, group)
    g.gptq_quantize_layer(Wref, U, perm, dead, cfg, *ref, st, ws)
    assert g.gptq_sync_status(st) == 0
    for call in range(2):
        _other_layer(g, *other)
        Wn = W.cuda().contiguous()
        out = _outputs(g, d_row, d_col, group)
        g.gptq_quantize_layer_noalloc(Wn, U, perm, dead, cfg, *out, st)
        assert g.gptq_sync_status(st) == 0, call
        # same kernels, same schedule, same inputs: bitwise the same results
        # (well inside the parity tolerances: codes exact, scales 1e-4)
        assert torch.equal(out[0], ref[0]), call
        assert torch.equal(out[1], ref[1]), call
        assert torch.equal(out[2], ref[2]), call
        assert torch.equal(Wn, Wref), call


def test_noalloc_large_layer_runs_the_shortened_schedule(g):
    """d_row = 8192: eight deferred blocks would need 32 MiB, so the 16 MiB
    scratch holds four and the lazy update runs in shorter products.  The
    result equals gptq_quantize_layer given a 16 MiB workspace bit for bit,
    and the oracle on sampled rows (teacher-forced checks)."""
    from gptq_testlib import compare_quantization
    d_row, d_col, bits, group = 8192, 1024, 4, 128
    W, X, cfg, _, U, perm, dead, st = _prepared(g, d_row, d_col, bits, group, False, seed=81)
    ws16 = torch.empty(16 << 20, dtype=torch.uint8, device="cuda")
    Wref = W.cuda().contiguous()
    ref = _outputs(g, d_row, d_col, group)
    g.gptq_quantize_layer(Wref, U, perm, dead, cfg, *ref, st, ws16)
    assert g.gptq_sync_status(st) == 0
    for call in range(2):
        _other_layer(g, 640, 768)
        Wn = W.cuda().contiguous()
        out = _outputs(g, d_row, d_col, group)
        g.gptq_quantize_layer_noalloc(Wn, U, perm, dead, cfg, *out, st)
        assert g.gptq_sync_status(st) == 0, call
        for a, b in zip(out, ref):
            assert torch.equal(a, b), call
        assert torch.equal(Wn, Wref), call
    packed = torch.empty(d_row, g.packed_words(d_col, bits), dtype=torch.int32, device="cuda")
    g.gptq_pack(out[0], bits, packed)
    res = dict(status=g.gptq_sync_status(st), perm=perm.cpu().numpy(),
               dead=dead.cpu().numpy().astype(bool), codes=out[0].cpu().numpy(),
               scales=out[1].cpu().numpy(), zeros=out[2].cpu().numpy(),
               w_at_quant=Wn.cpu().numpy(), packed=packed.cpu().numpy().view(np.uint32))
    rows = np.array([0, 1, 4095, 4096, 6000, 8191])
    compare_quantization(oracle.hessian(X).astype(np.float32).astype(np.float64), W, res, bits,
                         group, False, rows=rows, strict_free=False)


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


def test_noalloc_rejects_buffers_off_the_current_device(g):
    """The scratch belongs to the current device, so every buffer must too: a
    W in host memory is refused through the C ABI before anything runs (the
    outputs keep their fill), and the binding refuses a U that is not on W's
    device."""
    d_row, d_col = 16, 256
    cfg = g.GPTQConfig(bits=4, group_size=128)
    U = torch.eye(d_col, device="cuda")
    perm = torch.arange(d_col, dtype=torch.int32, device="cuda")
    dead = torch.zeros(d_col, dtype=torch.uint8, device="cuda")
    out = _outputs(g, d_row, d_col, 128)
    W_host = np.zeros((d_row, d_col), dtype=np.float32)
    lib = ctypes.CDLL(g.library_path())
    fn = lib.gptq_quantize_layer_noalloc
    P, i64 = ctypes.c_void_p, ctypes.c_int64
    fn.argtypes = [P, i64, i64, i64, P, P, P, ctypes.POINTER(g.GPTQConfig), P, P, P, P, P]
    fn.restype = ctypes.c_int
    rc = fn(W_host.ctypes.data, d_row, d_col, d_col, U.data_ptr(), perm.data_ptr(),
            dead.data_ptr(), ctypes.byref(cfg), out[0].data_ptr(), out[1].data_ptr(),
            out[2].data_ptr(), None, None)
    assert rc == 1
    torch.cuda.synchronize()
    assert bool((out[0] == 0xFF).all()) and bool((out[2] == 7).all())
    with pytest.raises(ValueError):
        g.gptq_quantize_layer_noalloc(torch.zeros(d_row, d_col, device="cuda"), U.cpu(), perm,
                                      dead, cfg, *out, None)

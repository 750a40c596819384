"""The bounded device-side waits, exercised without a faulty GPU.

Every spin-wait in the tensor-core kernels is bounded; on expiry the kernel
lets its issued copies and MMAs land, frees its tensor memory, writes
GPTQ_ERR_TIMEOUT to the call's status word and returns.  The test hook
gptq_debug_arm_wait_probe makes the next launch's MMA-issuing thread wait,
with a short limit, on a barrier that nothing ever completes (a flag nothing
sets); the wind-down waits keep the normal limit.  Each test sees the timeout
in the status word and then a normal call on the same stream succeeding with
the reference result.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

PROBE_NS = 200_000  # 0.2 ms


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_gptq_b200 as pkg
    return pkg


def test_hessian_wait_expiry_is_reported_and_the_next_call_runs(g):
    _, X = workloads.small_layer(4, 384, 5000, seed=31, kind="student_t")
    Xd = X.cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref = torch.zeros(384, 384, device="cuda")
    g.gptq_hessian_accumulate(Xd, ref, st)
    assert g.gptq_sync_status(st) == 0
    H = torch.zeros(384, 384, device="cuda")
    g.gptq_debug_arm_wait_probe(1, PROBE_NS)
    g.gptq_hessian_accumulate(Xd, H, st)
    assert g.gptq_sync_status(st) == 4  # GPTQ_ERR_TIMEOUT
    st.zero_()
    H.zero_()
    g.gptq_hessian_accumulate(Xd, H, st)
    assert g.gptq_sync_status(st) == 0
    L = torch.tril(torch.ones_like(H, dtype=torch.bool))
    assert torch.equal(H[L], ref[L])


def test_gemm_wait_expiry_is_reported_and_the_next_call_runs(g):
    """The first fp32-accurate GEMM of prepare_hinv (its first panel solve)
    times out; the call reports GPTQ_ERR_TIMEOUT; the same call again on the
    same stream gives the reference U bit for bit."""
    d = 512
    _, X = workloads.small_layer(4, d, 4 * d, seed=32, kind="student_t")
    H = oracle.hessian(X).astype(np.float32)
    cfg = g.GPTQConfig(bits=4, group_size=128)
    ws = torch.empty(g.gptq_workspace_size(cfg, 8, d), dtype=torch.uint8, device="cuda")

    def prepare():
        U = torch.empty(d, d, device="cuda")
        perm = torch.empty(d, dtype=torch.int32, device="cuda")
        dead = torch.empty(d, dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        g.gptq_prepare_hinv(torch.from_numpy(H).cuda(), cfg, U, perm, dead, st, ws)
        return U, g.gptq_sync_status(st)

    ref, status = prepare()
    assert status == 0
    g.gptq_debug_arm_wait_probe(2, PROBE_NS)
    _, status = prepare()
    assert status == 4
    again, status = prepare()
    assert status == 0
    assert torch.equal(again, ref)

"""Host logic of the streaming calibration hook (CPU): input checks, empty
batches, and the forward pre-hook's attach / detach.  The accumulation itself
runs on the GPU (tests/test_gpu_parity.py)."""
import pytest
import torch


@pytest.fixture(scope="module")
def calib():
    from post_weight_quantization_gptq_b200 import calibration
    return calibration


def test_inputs_are_checked_before_any_device_work(calib):
    acc = calib.HessianAccumulator(16, device="cpu")
    assert acc.H.shape == (16, 16) and acc.H.dtype == torch.float32
    with pytest.raises(TypeError):
        acc.add(torch.zeros(4, 16))                      # the Hessian's input precision is bf16
    with pytest.raises(ValueError):
        acc.add(torch.zeros(4, 15, dtype=torch.bfloat16))  # wrong feature count
    acc.add(torch.zeros(0, 16, dtype=torch.bfloat16))     # an empty batch adds nothing
    acc.add(torch.zeros(2, 0, 16, dtype=torch.bfloat16))
    assert acc.tokens == 0


def test_a_batch_on_another_device_is_refused(calib):
    acc = calib.HessianAccumulator(8, device="cpu")
    x = torch.zeros(3, 8, dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError):
        acc.add(x)


def test_the_pre_hook_sees_each_forward_call_until_detached(calib):
    acc = calib.HessianAccumulator(8, device="cpu")
    seen = []
    acc.add = lambda x: seen.append(tuple(x.shape))      # record instead of accumulating
    lin = torch.nn.Linear(8, 4, bias=False, dtype=torch.bfloat16)
    other = torch.nn.Linear(8, 4, bias=False, dtype=torch.bfloat16)
    assert acc.attach(lin, other) is acc
    x = torch.zeros(2, 5, 8, dtype=torch.bfloat16)
    with torch.no_grad():
        lin(x)
        other(x[0])
    assert seen == [(2, 5, 8), (5, 8)]
    acc.detach()
    with torch.no_grad():
        lin(x)
    assert len(seen) == 2

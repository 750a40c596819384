"""Streaming calibration: H = 2 X^T X accumulated from a layer's inputs as a
model's forward pass produces them.

GPTQ quantizes a model one layer after another, each from the Hessian of its
own calibration inputs ("GPTQ" article: the layers are processed
sequentially; "GPTQ (GPT Quantization)", "Fondation theorique : OBQ":
H = 2 X^T X, a sum over tokens).  Because H is a sum over tokens it can be
built chunk by chunk while the calibration batches flow through the model:
``HessianAccumulator`` owns a layer's H and adds every batch of inputs it is
given, and ``attach`` registers it as a forward pre-hook on the modules whose
inputs it should see (one accumulator per distinct input: q/k/v projections
share one, gate/up another).

Only marshalling happens here: each batch (any leading shape, last dimension
d, bf16 on the accumulator's device) is viewed as an n x d matrix and handed
to ``gptq_hessian_accumulate``; the tensor-core kernel does the arithmetic.
"""
from __future__ import annotations

import torch

from . import gptq_hessian_accumulate, gptq_sync_status


class HessianAccumulator:
    """H += 2 X^T X over every batch added, for one d-wide layer input.

    H is d x d fp32 on ``device``; only its lower triangle is valid (the
    kernel writes tiles that touch it).  Errors detected on the device land in
    ``status`` (read with ``check``)."""

    def __init__(self, d: int, device=None, stream=None):
        self.d = int(d)
        self.device = torch.device(device if device is not None else "cuda")
        if self.device.type == "cuda" and self.device.index is None:
            self.device = torch.device("cuda", torch.cuda.current_device())
        self.H = torch.zeros(self.d, self.d, dtype=torch.float32, device=self.device)
        self.status = torch.zeros(1, dtype=torch.int32, device=self.device)
        self.tokens = 0
        self.stream = stream
        self._handles = []

    def add(self, x: torch.Tensor) -> None:
        """Accumulate one batch of activations (..., d) in bf16."""
        if not isinstance(x, torch.Tensor) or x.dtype != torch.bfloat16:
            raise TypeError("activations must be a bf16 tensor (the Hessian's input precision)")
        if x.device != self.device:
            raise ValueError(f"activations are on {x.device}, the accumulator on {self.device}")
        if x.shape[-1] != self.d:
            raise ValueError(f"activations have {x.shape[-1]} features, expected {self.d}")
        x2 = x.reshape(-1, self.d)
        if x2.shape[0] == 0:
            return
        if x2.stride(1) != 1 or (x2.stride(0) % 8) != 0 or (x2.data_ptr() % 16) != 0:
            # the kernel reads rows by TMA (16-byte aligned rows): copy into a
            # row pitch rounded up to 8 elements and pass the d-wide view
            ld = (self.d + 7) // 8 * 8
            buf = torch.empty(x2.shape[0], ld, dtype=torch.bfloat16, device=self.device)
            buf[:, :self.d].copy_(x2)
            if self.stream is not None:
                buf.record_stream(self.stream)  # freed only after the GEMM read it
            x2 = buf[:, :self.d]
        gptq_hessian_accumulate(x2, self.H, self.status, stream=self.stream)
        self.tokens += x2.shape[0]

    def _hook(self, module, args, kwargs=None):
        x = args[0] if args else (kwargs or {}).get("input")
        self.add(x.detach())

    def attach(self, *modules: torch.nn.Module) -> "HessianAccumulator":
        """Accumulate the first positional input of every forward call of the
        given modules (register each shared input once)."""
        for m in modules:
            self._handles.append(m.register_forward_pre_hook(self._hook))
        return self

    def detach(self) -> None:
        for h in self._handles:
            h.remove()
        self._handles.clear()

    def check(self) -> None:
        """Wait for the accumulations and raise on a device-side error."""
        st = gptq_sync_status(self.status, stream=self.stream)
        if st != 0:
            from . import GPTQError
            raise GPTQError(st, "HessianAccumulator")

    def reset(self) -> None:
        self.H.zero_()
        self.status.zero_()
        self.tokens = 0

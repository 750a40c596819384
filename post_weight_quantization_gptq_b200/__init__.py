"""Python binding of the sm_100a GPTQ layer quantizer (libgptq_b200.so).

Argument marshalling only: every function below forwards torch CUDA tensors
as raw device pointers (and the current CUDA stream) to the C ABI declared in
``include/gptq.h`` under the same name.  All arithmetic runs in the library's
CUDA kernels; there is no CPU path.  Importing this package fails loudly when
the library has not been built (``python
post_weight_quantization_gptq_b200/build.py``).

Stages (see the header for the exact contracts):

* ``gptq_hessian_accumulate``  H += 2 X^T X            (tcgen05 bf16 GEMM)
* ``gptq_hessian_accumulate_host``  the same with X in host memory, copies
  overlapped with the GEMM through a two-slot device staging buffer
* ``gptq_prepare_hinv``        dead columns, act-order, damping, U = chol-inverse factor
* ``gptq_quantize_layer``      column walk with OBQ error feedback and lazy updates
* ``gptq_pack``                codes -> uint32 bit stream (8 codes per word at 4 bits)
* ``gptq_dequant_matmul``      Y = X W_hat^T from the packed layer (decode form)
* ``gptq_dequant_gemm``        the same for many tokens on the tensor cores (bf16 W_hat)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "GPTQConfig", "GPTQError", "gptq_hessian_accumulate", "gptq_hessian_accumulate_host",
    "gptq_hessian_staging_size", "gptq_prepare_hinv", "gptq_dequant_matmul", "gptq_dequant_matmul_workspace_size",
    "gptq_dequant_gemm", "gptq_dequant_gemm_workspace_size",
    "gptq_quantize_layer", "gptq_quantize_layer_noalloc", "gptq_noalloc_scratch_bytes", "gptq_pack", "gptq_workspace_size", "gptq_sync_status",
    "gptq_status_string", "gptq_version", "gptq_launch_counter", "gptq_debug_arm_wait_probe",
    "library_path", "n_groups", "packed_words",
    "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgptq_b200.so")

STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_UNSUPPORTED",
          3: "GPTQ_ERR_NOT_PD", 4: "GPTQ_ERR_TIMEOUT", 5: "GPTQ_ERR_CUDA",
          6: "GPTQ_ERR_WORKSPACE"}


class GPTQConfig(ctypes.Structure):
    """Mirror of ``gptq_config``: bits, group_size (-1 = one group per row),
    block_size (128), desc_act, damp (lambda = damp * mean(diag H)),
    pure_minmax (each group's own [min, max] instead of the range widened to
    contain 0)."""
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("desc_act", ctypes.c_int32),
                ("damp", ctypes.c_float), ("pure_minmax", ctypes.c_int32)]

    def __init__(self, bits=4, group_size=128, desc_act=False, damp=0.01, block_size=128,
                 pure_minmax=False):
        super().__init__(int(bits), int(group_size), int(block_size), int(bool(desc_act)),
                         float(damp), int(bool(pure_minmax)))


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS.get(self.status, self.status)} "
                         f"({gptq_status_string(self.status)})")


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is missing: build the CUDA library first "
            "(python post_weight_quantization_gptq_b200/build.py)")
    lib = ctypes.CDLL(_LIB_PATH)
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
    cfgp = ctypes.POINTER(GPTQConfig)
    sig = {
        "gptq_status_string": ([i32], ctypes.c_char_p),
        "gptq_version": ([], i32),
        "gptq_launch_counter": ([], ctypes.c_int64),
        "gptq_workspace_size": ([cfgp, i64, i64, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
        "gptq_hessian_accumulate": ([P, i64, i64, i64, P, i64, P, P, ctypes.c_size_t, P],
                                    ctypes.c_int),
        "gptq_hessian_accumulate_host": ([P, i64, i64, i64, P, i64, P, P, ctypes.c_size_t, P],
                                         ctypes.c_int),
        "gptq_hessian_staging_size": ([i64, i64], ctypes.c_size_t),
        "gptq_prepare_hinv": ([P, i64, i64, cfgp, P, P, P, P, P, ctypes.c_size_t, P],
                              ctypes.c_int),
        "gptq_quantize_layer": ([P, i64, i64, i64, P, P, P, cfgp, P, P, P, P, P,
                                 ctypes.c_size_t, P], ctypes.c_int),
        "gptq_pack": ([P, i64, i64, i32, P, P], ctypes.c_int),
        "gptq_dequant_matmul": ([P, i64, i64, i64, P, P, P, P, i64, i32, i32, P, i64, P,
                                 ctypes.c_size_t, P], ctypes.c_int),
        "gptq_dequant_matmul_workspace_size": ([i64, i64], ctypes.c_size_t),
        "gptq_dequant_gemm": ([P, i64, i64, i64, P, P, P, P, i64, i32, i32, P, i64, P, P,
                               ctypes.c_size_t, P], ctypes.c_int),
        "gptq_dequant_gemm_workspace_size": ([i64, i64], ctypes.c_size_t),
        "gptq_quantize_layer_noalloc": ([P, i64, i64, i64, P, P, P, cfgp, P, P, P, P, P],
                                        ctypes.c_int),
        "gptq_noalloc_scratch_bytes": ([], ctypes.c_size_t),
        "gptq_sync_status": ([P, P, ctypes.POINTER(i32)], ctypes.c_int),
        "gptq_debug_arm_wait_probe": ([i32, i64], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


_lib = _load()


def library_path() -> str:
    return _LIB_PATH


def gptq_status_string(status: int) -> str:
    return _lib.gptq_status_string(int(status)).decode()


def gptq_version() -> int:
    return int(_lib.gptq_version())


def gptq_launch_counter() -> int:
    """Kernels launched by the library in this process so far."""
    return int(_lib.gptq_launch_counter())


def n_groups(d_col: int, group_size: int) -> int:
    g = d_col if group_size == -1 or group_size > d_col else group_size
    return -(-d_col // g)


def packed_words(d_col: int, bits: int) -> int:
    return -(-(d_col * bits) // 32)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return getattr(stream, "cuda_stream", stream)


def _check(status: int, where: str) -> None:
    if status != 0:
        raise GPTQError(status, where)


def _cuda(t: torch.Tensor, name: str, dtype=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _row_major(t: torch.Tensor, name: str) -> int:
    """Leading dimension of a 2-D tensor with unit column stride."""
    if t.dim() != 2 or (t.stride(1) != 1 and t.shape[1] > 1):
        raise ValueError(f"{name} must be 2-D with contiguous rows")
    return t.stride(0) if t.shape[0] > 1 else max(t.shape[1], t.stride(0))


def _same_device(ref: torch.Tensor, ref_name: str, *others) -> None:
    """Every (tensor, name, dtype) of ``others`` that is given lives on ref's
    device, and that device is the current one: the library launches on the
    current device and its kernels dereference every pointer there, so a
    buffer elsewhere (host memory, another GPU) is refused here instead of
    being read by a kernel.  dtype None accepts any element type."""
    for t, name, dtype in others:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != ref.device:
            where = t.device if isinstance(t, torch.Tensor) else type(t).__name__
            raise ValueError(f"{name} must be on {ref.device} like {ref_name}, not on {where}")
        if dtype is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ref.device.index != torch.cuda.current_device():
        raise ValueError(f"{ref_name} is on {ref.device} but cuda:{torch.cuda.current_device()} "
                         "is current: make its device current (torch.cuda.device(...))")


def gptq_workspace_size(cfg: GPTQConfig, d_row: int, d_col: int) -> int:
    out = ctypes.c_size_t(0)
    _check(_lib.gptq_workspace_size(ctypes.byref(cfg), int(d_row), int(d_col), ctypes.byref(out)),
           "gptq_workspace_size")
    return int(out.value)


def gptq_hessian_accumulate(X: torch.Tensor, H: torch.Tensor, dev_status: torch.Tensor | None = None,
                            ws: torch.Tensor | None = None, stream=None) -> None:
    """H += 2 X^T X (X: n x d bf16, H: d x d fp32, both CUDA, row-major)."""
    _cuda(X, "X", torch.bfloat16)
    _cuda(H, "H", torch.float32)
    _same_device(X, "X", (H, "H", torch.float32), (dev_status, "dev_status", torch.int32),
                 (ws, "ws", None))
    n, d = X.shape
    ldx = _row_major(X, "X")
    ldh = _row_major(H, "H")
    _check(_lib.gptq_hessian_accumulate(_ptr(X), n, d, ldx, _ptr(H), ldh, _ptr(dev_status),
                                        _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                        _stream(stream)), "gptq_hessian_accumulate")


def gptq_hessian_accumulate_host(X: torch.Tensor, H: torch.Tensor, staging: torch.Tensor,
                                 dev_status: torch.Tensor | None = None, stream=None) -> None:
    """H += 2 X^T X with X (n x d bf16) in HOST memory, streamed through the
    device buffer ``staging`` (two slots; copies overlap the GEMM when X is
    pinned).  X must stay unchanged until the stream has run the call."""
    if not isinstance(X, torch.Tensor) or X.is_cuda or X.dtype != torch.bfloat16:
        raise TypeError("X must be a host bf16 tensor")
    _cuda(H, "H", torch.float32)
    _cuda(staging, "staging")
    _same_device(H, "H", (staging, "staging", None), (dev_status, "dev_status", torch.int32))
    n, d = X.shape
    ldx = _row_major(X, "X")
    _check(_lib.gptq_hessian_accumulate_host(_ptr(X), n, d, ldx, _ptr(H), _row_major(H, "H"),
                                             _ptr(dev_status), _ptr(staging),
                                             staging.numel() * staging.element_size(),
                                             _stream(stream)), "gptq_hessian_accumulate_host")


def gptq_hessian_staging_size(d: int, chunk_tokens: int) -> int:
    """Bytes of staging gptq_hessian_accumulate_host needs for chunk_tokens-token chunks."""
    return int(_lib.gptq_hessian_staging_size(int(d), int(chunk_tokens)))


def gptq_prepare_hinv(H: torch.Tensor, cfg: GPTQConfig, U: torch.Tensor, perm: torch.Tensor,
                      dead: torch.Tensor, dev_status: torch.Tensor | None, ws: torch.Tensor,
                      stream=None) -> None:
    """Consumes H (lower triangle); writes U (d x d upper, quantization
    order), perm (int32) and dead (uint8)."""
    _cuda(H, "H", torch.float32)
    _cuda(U, "U", torch.float32)
    _cuda(perm, "perm", torch.int32)
    _cuda(dead, "dead", torch.uint8)
    if ws is None:
        raise ValueError("gptq_prepare_hinv needs a workspace (gptq_workspace_size bytes)")
    _same_device(H, "H", (U, "U", torch.float32), (perm, "perm", torch.int32),
                 (dead, "dead", torch.uint8), (dev_status, "dev_status", torch.int32),
                 (ws, "ws", None))
    d = H.shape[0]
    if not U.is_contiguous() or tuple(U.shape) != (d, d):
        raise ValueError("U must be a contiguous d x d tensor")
    _check(_lib.gptq_prepare_hinv(_ptr(H), d, _row_major(H, "H"), ctypes.byref(cfg), _ptr(U),
                                  _ptr(perm), _ptr(dead), _ptr(dev_status), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)),
           "gptq_prepare_hinv")


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor, dead: torch.Tensor,
                        cfg: GPTQConfig, codes: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor, dev_status: torch.Tensor | None, ws: torch.Tensor,
                        stream=None) -> None:
    """W (d_row x d_col fp32, original order; overwritten) -> codes (uint8,
    quantization order), scales (fp32 [groups][d_row]), zeros (int32)."""
    _cuda(W, "W", torch.float32)
    _cuda(codes, "codes", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    _cuda(zeros, "zeros", torch.int32)
    if ws is None:
        raise ValueError("gptq_quantize_layer needs a workspace (gptq_workspace_size bytes)")
    _same_device(W, "W", (U, "U", torch.float32), (perm, "perm", torch.int32),
                 (dead, "dead", torch.uint8), (codes, "codes", None), (scales, "scales", None),
                 (zeros, "zeros", None), (dev_status, "dev_status", torch.int32), (ws, "ws", None))
    d_row, d_col = W.shape
    for t, name in ((codes, "codes"), (scales, "scales"), (zeros, "zeros"), (U, "U")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _check(_lib.gptq_quantize_layer(_ptr(W), d_row, d_col, _row_major(W, "W"), _ptr(U), _ptr(perm),
                                    _ptr(dead), ctypes.byref(cfg), _ptr(codes), _ptr(scales),
                                    _ptr(zeros), _ptr(dev_status), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
           "gptq_quantize_layer")


def gptq_quantize_layer_noalloc(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor,
                                dead: torch.Tensor, cfg: GPTQConfig, codes: torch.Tensor,
                                scales: torch.Tensor, zeros: torch.Tensor,
                                dev_status: torch.Tensor | None, stream=None) -> None:
    """gptq_quantize_layer without a workspace, for callers that cannot
    allocate device memory (an enqueue call that may not allocate, a memory
    pool that already holds nearly all of HBM, a path that cannot afford the
    device synchronization of cudaMalloc / cudaFree).  The scratch is a fixed
    array inside the library (gptq_noalloc_scratch_bytes() per device), shared
    by every call: calls that overlap on the GPU race on it."""
    _cuda(W, "W", torch.float32)
    _cuda(codes, "codes", torch.uint8)
    _cuda(scales, "scales", torch.float32)
    _cuda(zeros, "zeros", torch.int32)
    d_row, d_col = W.shape
    for t, name in ((codes, "codes"), (scales, "scales"), (zeros, "zeros"), (U, "U")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    # the scratch array used is the current device's: every buffer must be on
    # W's device, and the call runs with that device current
    for t, name in ((U, "U"), (perm, "perm"), (dead, "dead"), (codes, "codes"),
                    (scales, "scales"), (zeros, "zeros"), (dev_status, "dev_status")):
        if t is not None and (not t.is_cuda or t.device != W.device):
            raise ValueError(f"{name} must be on {W.device}, like W")
    for t, name, dtype in ((U, "U", torch.float32), (perm, "perm", torch.int32),
                           (dead, "dead", torch.uint8), (dev_status, "dev_status", torch.int32)):
        if t is not None and t.dtype != dtype:
            raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    with torch.cuda.device(W.device):
        _check(_lib.gptq_quantize_layer_noalloc(_ptr(W), d_row, d_col, _row_major(W, "W"),
                                                _ptr(U), _ptr(perm), _ptr(dead),
                                                ctypes.byref(cfg), _ptr(codes), _ptr(scales),
                                                _ptr(zeros), _ptr(dev_status), _stream(stream)),
               "gptq_quantize_layer_noalloc")


def gptq_noalloc_scratch_bytes() -> int:
    return int(_lib.gptq_noalloc_scratch_bytes())


def gptq_pack(codes: torch.Tensor, bits: int, packed: torch.Tensor, stream=None) -> None:
    """codes (d_row x d_col uint8) -> packed (d_row x ceil(d_col*bits/32) int32 view of uint32)."""
    _cuda(codes, "codes", torch.uint8)
    _cuda(packed, "packed")
    _same_device(codes, "codes", (packed, "packed", None))
    if not codes.is_contiguous() or not packed.is_contiguous():
        raise ValueError("codes and packed must be contiguous")
    d_row, d_col = codes.shape
    _check(_lib.gptq_pack(_ptr(codes), d_row, d_col, int(bits), _ptr(packed), _stream(stream)),
           "gptq_pack")


def gptq_dequant_matmul(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor, perm: torch.Tensor | None, bits: int,
                        group_size: int, Y: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """Y = X W_hat^T for a quantized layer (decode form): X (tokens x d_col bf16,
    original column order), packed / scales / zeros / perm as the quantizer
    wrote them, Y (tokens x d_row fp32) overwritten, ws a device workspace of
    gptq_dequant_matmul_workspace_size(tokens, d_col) bytes."""
    _cuda(X, "X", torch.bfloat16)
    _cuda(packed, "packed")
    _cuda(scales, "scales", torch.float32)
    _cuda(zeros, "zeros", torch.int32)
    _cuda(Y, "Y", torch.float32)
    _cuda(ws, "ws")
    if perm is not None:
        _cuda(perm, "perm", torch.int32)
    _same_device(X, "X", (packed, "packed", None), (scales, "scales", None),
                 (zeros, "zeros", None), (perm, "perm", None), (Y, "Y", None), (ws, "ws", None))
    for t, name in ((packed, "packed"), (scales, "scales"), (zeros, "zeros")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    n_tok, d_col = X.shape
    d_row = packed.shape[0]
    _check(_lib.gptq_dequant_matmul(_ptr(X), n_tok, d_col, _row_major(X, "X"), _ptr(packed),
                                    _ptr(scales), _ptr(zeros), _ptr(perm), d_row, int(bits),
                                    int(group_size), _ptr(Y), _row_major(Y, "Y"), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)),
           "gptq_dequant_matmul")


def gptq_dequant_matmul_workspace_size(n_tok: int, d_col: int) -> int:
    return int(_lib.gptq_dequant_matmul_workspace_size(int(n_tok), int(d_col)))


def gptq_dequant_gemm(X: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor,
                      zeros: torch.Tensor, perm: torch.Tensor | None, bits: int, group_size: int,
                      Y: torch.Tensor, ws: torch.Tensor | None = None,
                      dev_status: torch.Tensor | None = None, stream=None) -> None:
    """Y = X W_hat^T for a quantized layer, many-token form on the tensor
    cores (W_hat dequantized to bf16 per stage): X (tokens x d_col bf16,
    original column order), packed / scales / zeros / perm as the quantizer
    wrote them, Y (tokens x d_row fp32) overwritten; ws (bytes of
    gptq_dequant_gemm_workspace_size) is needed with a permutation."""
    _cuda(X, "X", torch.bfloat16)
    _cuda(packed, "packed")
    _cuda(scales, "scales", torch.float32)
    _cuda(zeros, "zeros", torch.int32)
    _cuda(Y, "Y", torch.float32)
    if perm is not None:
        _cuda(perm, "perm", torch.int32)
    _same_device(X, "X", (packed, "packed", None), (scales, "scales", None),
                 (zeros, "zeros", None), (perm, "perm", None), (Y, "Y", None), (ws, "ws", None),
                 (dev_status, "dev_status", torch.int32))
    for t, name in ((packed, "packed"), (scales, "scales"), (zeros, "zeros")):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    n_tok, d_col = X.shape
    d_row = packed.shape[0]
    _check(_lib.gptq_dequant_gemm(_ptr(X), n_tok, d_col, _row_major(X, "X"), _ptr(packed),
                                  _ptr(scales), _ptr(zeros), _ptr(perm), d_row, int(bits),
                                  int(group_size), _ptr(Y), _row_major(Y, "Y"), _ptr(dev_status),
                                  _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                  _stream(stream)), "gptq_dequant_gemm")


def gptq_dequant_gemm_workspace_size(n_tok: int, d_col: int) -> int:
    return int(_lib.gptq_dequant_gemm_workspace_size(int(n_tok), int(d_col)))


def gptq_debug_arm_wait_probe(kernel: int, limit_ns: int) -> None:
    """Test hook: the next launch of kernel kind 1 (Hessian) or 2 (the next
    fp32-accurate tensor-core GEMM) waits once, bounded by limit_ns, on a
    barrier nothing completes, and reports GPTQ_ERR_TIMEOUT."""
    _check(_lib.gptq_debug_arm_wait_probe(int(kernel), int(limit_ns)),
           "gptq_debug_arm_wait_probe")


def gptq_sync_status(dev_status: torch.Tensor, stream=None) -> int:
    """Wait for the stream and return the device status word."""
    out = ctypes.c_int32(0)
    _check(_lib.gptq_sync_status(_stream(stream), _ptr(dev_status), ctypes.byref(out)),
           "gptq_sync_status")
    return int(out.value)

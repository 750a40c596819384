"""Seeded synthetic inputs for the GPTQ layer quantizer.

This module only draws random numbers: weight matrices W and calibration
activations X shaped like the workloads the GPTQ pages quantize (Llama-style
linear layers calibrated on a few hundred sequences).  It holds none of the
quantizer's arithmetic, so the CUDA library, the float64 oracle, the tests and
the benchmark can all consume the same tensors.

Every generator is a pure function of (shape, seed, device): the same call
returns the same tensor.  The CPU and CUDA random streams differ, so a caller
that compares two implementations generates once and hands the same tensor to
both sides.

Recipes (the pages' calibration set is C4 text, 128 samples; no dataset or
trained weights exist here, so these distributions stand in for them):

* weights: i.i.d. N(0, std^2), fp32.
* "correlated" activations: X = Z L with Z ~ N(0, 1) and L lower-triangular,
  diagonal log-spaced from 1 down to 10^-cond_exp, strict lower part
  N(0, (0.1/sqrt(d))^2); a few seeded outlier channels are scaled up.
* "student_t" activations: i.i.d. Student-t with 4 degrees of freedom, drawn as
  Z / sqrt(chi2_4 / 4) with chi2_4 = -2 ln(U1 U2); a seeded fraction of the
  channels is scaled up (heavy-tailed LLM activations with outlier channels).
* "half_normal" activations: |N(0, 1)| (post-SiLU-like), with outlier channels.

Activations are returned as bfloat16, the precision the Hessian consumes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BASE_SEED = 1234


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def gaussian_weights(rows: int, cols: int, std: float, seed: int,
                     device="cpu") -> torch.Tensor:
    """W ~ N(0, std^2), fp32, rows x cols, row-major."""
    g = _gen(seed, device)
    return torch.randn(rows, cols, generator=g, device=device,
                       dtype=torch.float32) * std


def outlier_channels(d: int, frac: float, seed: int, count: int | None = None) -> torch.Tensor:
    """Seeded choice of outlier channel indices (CPU int64, sorted)."""
    k = count if count is not None else max(1, int(round(frac * d)))
    g = _gen(seed ^ 0x5EED, "cpu")
    return torch.sort(torch.randperm(d, generator=g)[:k]).values


def correlated_activations(n: int, d: int, seed: int, cond_exp: float = 3.0,
                           n_outliers: int = 4, outlier_scale: float = 20.0,
                           device="cpu") -> torch.Tensor:
    """X = Z L (bf16, n x d): correlated channels with a controlled spread."""
    g = _gen(seed, device)
    z = torch.randn(n, d, generator=g, device=device, dtype=torch.float64)
    low = torch.randn(d, d, generator=g, device=device, dtype=torch.float64)
    low = torch.tril(low, diagonal=-1) * (0.1 / math.sqrt(d))
    diag = torch.logspace(0.0, -cond_exp, d, dtype=torch.float64, device=device)
    low = low + torch.diag(diag)
    x = z @ low
    idx = outlier_channels(d, 0.0, seed, count=n_outliers).to(device)
    x[:, idx] *= outlier_scale
    return x.to(torch.bfloat16)


def _scale_outliers(x: torch.Tensor, frac: float, scale: float, seed: int) -> None:
    if frac <= 0.0:
        return
    idx = outlier_channels(x.shape[1], frac, seed).to(x.device)
    x[:, idx] *= scale


def student_t_activations(n: int, d: int, seed: int, outlier_frac: float = 0.01,
                          outlier_scale: float = 50.0, device="cpu",
                          chunk_rows: int = 16384) -> torch.Tensor:
    """i.i.d. Student-t(4) activations (bf16, n x d) with outlier channels."""
    g = _gen(seed, device)
    out = torch.empty(n, d, dtype=torch.bfloat16, device=device)
    idx = outlier_channels(d, outlier_frac, seed).to(device) if outlier_frac > 0 else None
    for r0 in range(0, n, chunk_rows):
        m = min(chunk_rows, n - r0)
        z = torch.randn(m, d, generator=g, device=device, dtype=torch.float32)
        u1 = 1.0 - torch.rand(m, d, generator=g, device=device, dtype=torch.float32)
        u2 = 1.0 - torch.rand(m, d, generator=g, device=device, dtype=torch.float32)
        t = z / torch.sqrt(-0.5 * torch.log(u1 * u2))
        if idx is not None:
            t[:, idx] *= outlier_scale
        out[r0:r0 + m] = t.to(torch.bfloat16)
    return out


def half_normal_activations(n: int, d: int, seed: int, outlier_frac: float = 0.005,
                            outlier_scale: float = 30.0, device="cpu",
                            chunk_rows: int = 16384) -> torch.Tensor:
    """|N(0,1)| activations (bf16, n x d) with outlier channels."""
    g = _gen(seed, device)
    out = torch.empty(n, d, dtype=torch.bfloat16, device=device)
    idx = outlier_channels(d, outlier_frac, seed).to(device) if outlier_frac > 0 else None
    for r0 in range(0, n, chunk_rows):
        m = min(chunk_rows, n - r0)
        t = torch.randn(m, d, generator=g, device=device, dtype=torch.float32).abs_()
        if idx is not None:
            t[:, idx] *= outlier_scale
        out[r0:r0 + m] = t.to(torch.bfloat16)
    return out


@dataclass(frozen=True)
class Workload:
    """One quantization problem: a weight shape, its calibration source and
    the quantizer settings (bits, group size, act-order, damping)."""
    name: str
    d_row: int
    d_col: int
    n_tokens: int
    activations: str          # "correlated" | "student_t" | "half_normal"
    w_std: float
    bits: int
    group_size: int
    desc_act: bool
    damp: float = 0.01
    block_size: int = 128
    outlier_frac: float = 0.01
    outlier_scale: float = 50.0
    seed: int = BASE_SEED
    shares: tuple = field(default=())   # extra weight rows sharing the same H


# The five workloads: a tiny layer the oracle finishes in seconds, the
# Llama-7B-shaped q_proj (128 sequences x 2048 tokens), the Llama-7B MLP
# down_proj, one full Llama-7B block and the two largest Llama-70B layers.
WORKLOADS = {
    "tiny": Workload("tiny", 256, 512, 2048, "correlated", 0.02, 4, 128, False,
                     outlier_frac=4 / 512, outlier_scale=20.0, seed=BASE_SEED + 0),
    "llama7b_q_proj": Workload("llama7b_q_proj", 4096, 4096, 128 * 2048, "student_t",
                               0.02, 4, 128, False, seed=BASE_SEED + 1),
    "llama7b_down_proj": Workload("llama7b_down_proj", 4096, 11008, 128 * 2048,
                                  "half_normal", 0.015, 4, 32, True,
                                  outlier_frac=0.005, outlier_scale=30.0,
                                  seed=BASE_SEED + 2),
    "llama70b_q_proj": Workload("llama70b_q_proj", 8192, 8192, 128 * 2048, "student_t",
                                0.01, 4, 128, True, seed=BASE_SEED + 4),
    "llama70b_down_proj": Workload("llama70b_down_proj", 8192, 28672, 128 * 2048,
                                   "student_t", 0.01, 4, 128, True, seed=BASE_SEED + 4),
}

# Full Llama-7B block: (weight name, rows, cols, calibration source, w_std).
# q/k/v share the attention-input H; gate/up share the MLP-input H.
LLAMA7B_BLOCK = [
    ("q_proj", 4096, 4096, "attn_in", 0.02),
    ("k_proj", 4096, 4096, "attn_in", 0.02),
    ("v_proj", 4096, 4096, "attn_in", 0.02),
    ("o_proj", 4096, 4096, "o_in", 0.02),
    ("gate_proj", 11008, 4096, "mlp_in", 0.02),
    ("up_proj", 11008, 4096, "mlp_in", 0.02),
    ("down_proj", 4096, 11008, "down_in", 0.015),
]
LLAMA7B_BLOCK_SOURCES = {"attn_in": 4096, "o_in": 4096, "mlp_in": 4096, "down_in": 11008}
LLAMA7B_BLOCK_QUANT = dict(bits=3, group_size=128, desc_act=False, damp=0.01)
_BLOCK_SOURCE_SEED = {"attn_in": 3, "o_in": 5, "mlp_in": 6, "down_in": 8}


def block_activations(source: str, n_tokens: int = 128 * 2048, device="cpu") -> torch.Tensor:
    """Calibration input of one Llama-7B block source (Student-t(4), 1 % of
    the channels x50): attn_in feeds q/k/v, o_in o_proj, mlp_in gate/up,
    down_in down_proj."""
    d = LLAMA7B_BLOCK_SOURCES[source]
    return student_t_activations(n_tokens, d, seed=BASE_SEED + _BLOCK_SOURCE_SEED[source],
                                 device=device)


def block_weights(name: str, device="cpu") -> torch.Tensor:
    """W of one Llama-7B block weight (LLAMA7B_BLOCK row), N(0, std^2)."""
    j = [b[0] for b in LLAMA7B_BLOCK].index(name)
    _, rows, cols, _, std = LLAMA7B_BLOCK[j]
    return gaussian_weights(rows, cols, std, seed=BASE_SEED + 3 + 101 * j, device=device)


def activations(w: Workload, device="cpu", n_tokens: int | None = None,
                seed_offset: int = 0) -> torch.Tensor:
    n = w.n_tokens if n_tokens is None else n_tokens
    seed = w.seed + 7919 * (seed_offset + 1)
    if w.activations == "correlated":
        n_out = max(1, int(round(w.outlier_frac * w.d_col)))
        return correlated_activations(n, w.d_col, seed, n_outliers=n_out,
                                      outlier_scale=w.outlier_scale, device=device)
    if w.activations == "student_t":
        return student_t_activations(n, w.d_col, seed, w.outlier_frac,
                                     w.outlier_scale, device=device)
    if w.activations == "half_normal":
        return half_normal_activations(n, w.d_col, seed, w.outlier_frac,
                                       w.outlier_scale, device=device)
    raise ValueError(w.activations)


def weights(w: Workload, device="cpu", seed_offset: int = 0) -> torch.Tensor:
    return gaussian_weights(w.d_row, w.d_col, w.w_std, w.seed + 104729 * seed_offset,
                            device=device)


def small_layer(d_row: int, d_col: int, n_tokens: int, seed: int, kind: str = "student_t",
                device="cpu") -> tuple[torch.Tensor, torch.Tensor]:
    """A small (W, X) pair of arbitrary shape for parity and edge-case tests."""
    w = gaussian_weights(d_row, d_col, 0.02, seed, device=device)
    if kind == "correlated":
        x = correlated_activations(n_tokens, d_col, seed + 1,
                                   n_outliers=max(1, d_col // 128), device=device)
    elif kind == "half_normal":
        x = half_normal_activations(n_tokens, d_col, seed + 1, device=device)
    else:
        x = student_t_activations(n_tokens, d_col, seed + 1, device=device)
    return w, x

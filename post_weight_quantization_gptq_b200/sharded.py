"""One layer quantized by several processes (one per GPU, torch.distributed).

Two facts of the method let a single layer spread over ranks:

* H = 2 X^T X is a sum over calibration tokens ("GPTQ (GPT Quantization)",
  "Algorithme complet (pseudo-code)", step 1), so each rank accumulates the
  tokens of its own shard and one all-reduce (sum) of the d x d fp32 matrix
  joins the partial Hessians.
* The OBQ feedback W_F <- W_F - e / (H^-1)_ii * (H^-1)_{i,F} ("GPTQ (GPT
  Quantization)", "Fondation theorique : OBQ") moves each weight row using
  only that row's own errors and H^-1, so rows are independent given H^-1:
  each rank runs the column walk on a contiguous slice of W's rows.

Every rank builds U from the same all-reduced H.  The library's kernels are
deterministic (no atomics, a fixed reduction order for a given GPU model), so
every rank gets the same U without exchanging it; recomputing it costs less
than broadcasting d^2 floats for the layer sizes this targets.

The module is plumbing: it slices, calls the C-ABI through the binding and
moves finished tensors with torch.distributed.  With the gloo backend, CUDA
tensors are staged through host memory for each collective.  Ranks take the
same collectives in the same order on every path, errors included: a device
status is combined over ranks (max) before any rank raises.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (GPTQConfig, GPTQError, gptq_hessian_accumulate, gptq_pack, gptq_prepare_hinv,
               gptq_quantize_layer, gptq_sync_status, gptq_workspace_size, n_groups,
               packed_words)

# The Hessian kernel adds its fp32 partial sums into H every 32,768 tokens.
# Token shards that start on such a boundary keep each rank's partial sums
# those of the single-process call; only the order of the cross-rank
# additions differs.
TOKEN_QUANTUM = 32768


def token_range(n_tokens: int, rank: int, world: int, quantum: int = TOKEN_QUANTUM):
    """[t0, t1) of the calibration tokens this rank accumulates: contiguous
    shards of whole `quantum`-token units, the first n_units % world ranks one
    unit longer; the last unit may be ragged and a rank may get none."""
    _check_rank(rank, world)
    if n_tokens < 0 or quantum <= 0:
        raise ValueError("n_tokens must be >= 0 and quantum > 0")
    units = -(-n_tokens // quantum)
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(n_tokens, u0 * quantum), min(n_tokens, u1 * quantum)


def row_range(d_row: int, rank: int, world: int):
    """[r0, r1) of W's rows this rank quantizes (balanced contiguous slices)."""
    _check_rank(rank, world)
    if d_row < 0:
        raise ValueError("d_row must be >= 0")
    return rank * d_row // world, (rank + 1) * d_row // world


def _check_rank(rank: int, world: int) -> None:
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")


def _staged(t: torch.Tensor, group) -> bool:
    return t.is_cuda and dist.get_backend(group) == "gloo"


def allreduce_hessian(H: torch.Tensor, group=None) -> None:
    """Sum the ranks' partial Hessians in place (fp32, every rank gets H)."""
    if _staged(H, group):
        h = H.cpu()
        dist.all_reduce(h, op=dist.ReduceOp.SUM, group=group)
        H.copy_(h)
    else:
        dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)


def combine_status(status: int, device, group=None) -> int:
    """The largest device status over all ranks (0 when every rank is OK)."""
    t = torch.tensor([int(status)], dtype=torch.int32,
                     device="cpu" if dist.get_backend(group) == "gloo" else device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return int(t.item())


def _all_gather_rows(local: torch.Tensor, d_row: int, world: int, group) -> torch.Tensor:
    """Concatenate every rank's row slice (row_range order) into d_row rows."""
    cap = -(-d_row // world)
    stage = _staged(local, group)
    src = local.cpu() if stage else local
    pad = torch.zeros((cap,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    pad[: src.shape[0]] = src
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    rows = [parts[k][: row_range(d_row, k, world)[1] - row_range(d_row, k, world)[0]]
            for k in range(world)]
    out = torch.cat(rows, dim=0)
    return out.to(local.device) if stage else out


def gather_quantized(packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                     d_row: int, group=None):
    """All ranks' row slices -> the whole layer on every rank.

    packed: rows x words (int32 view of uint32); scales / zeros: groups x rows
    (group-major, as the quantizer writes them).  Returns (packed, scales,
    zeros) for all d_row rows, in the same layouts."""
    world = dist.get_world_size(group)
    p = _all_gather_rows(packed.contiguous(), d_row, world, group)
    s = _all_gather_rows(scales.t().contiguous(), d_row, world, group).t().contiguous()
    z = _all_gather_rows(zeros.t().contiguous(), d_row, world, group).t().contiguous()
    return p, s, z


def quantize_layer_sharded(X_local: torch.Tensor, W_local: torch.Tensor, d_row: int,
                           cfg: GPTQConfig, group=None, gather: bool = True) -> dict:
    """Quantize one layer spread over the ranks of `group`.

    X_local: this rank's calibration tokens (token_range(n, rank, world) of
    the layer's n x d_col bf16 activations; any count, zero included), CUDA.
    W_local: this rank's rows (row_range(d_row, rank, world)) of the d_row x
    d_col fp32 weights, original column order, CUDA; overwritten (as by
    gptq_quantize_layer).  Returns perm and dead (same on every rank), this
    rank's packed / scales / zeros, and with gather=True the whole layer's
    packed_all / scales_all / zeros_all on every rank.

    The library calls and the NCCL collectives are all issued on torch's
    current stream, which orders them; with gloo the host staging copies
    synchronize that stream before each collective."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    r0, r1 = row_range(d_row, rank, world)
    d_col = W_local.shape[1]
    if W_local.shape[0] != r1 - r0 or X_local.shape[1] != d_col:
        raise ValueError(f"rank {rank}: W_local must hold rows [{r0}, {r1}) and X_local "
                         f"{d_col} columns")
    dev = W_local.device
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    H = torch.zeros(d_col, d_col, dtype=torch.float32, device=dev)
    gptq_hessian_accumulate(X_local, H, st)
    allreduce_hessian(H, group)

    ws = torch.empty(gptq_workspace_size(cfg, max(1, r1 - r0), d_col), dtype=torch.uint8,
                     device=dev)
    U = torch.empty(d_col, d_col, dtype=torch.float32, device=dev)
    perm = torch.empty(d_col, dtype=torch.int32, device=dev)
    dead = torch.empty(d_col, dtype=torch.uint8, device=dev)
    gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    ng = n_groups(d_col, cfg.group_size)
    rows = r1 - r0
    codes = torch.empty(rows, d_col, dtype=torch.uint8, device=dev)
    scales = torch.empty(ng, rows, dtype=torch.float32, device=dev)
    zeros = torch.empty(ng, rows, dtype=torch.int32, device=dev)
    packed = torch.empty(rows, packed_words(d_col, cfg.bits), dtype=torch.int32, device=dev)
    if rows > 0:
        gptq_quantize_layer(W_local, U, perm, dead, cfg, codes, scales, zeros, st, ws)
        gptq_pack(codes, cfg.bits, packed)
    status = combine_status(gptq_sync_status(st), dev, group)
    if status != 0:
        raise GPTQError(status, "quantize_layer_sharded")
    out = dict(perm=perm, dead=dead, rows=(r0, r1), packed=packed, scales=scales,
               zeros=zeros, codes=codes, w_at_quant=W_local)
    if gather:
        out["packed_all"], out["scales_all"], out["zeros_all"] = gather_quantized(
            packed, scales, zeros, d_row, group)
    return out

"""GPU parity of the product with a quantized layer (gptq_dequant_matmul)
against the float64 oracle, through the C ABI.

Inputs are seeded random packed words (random bits are random codes), scales,
zero points, act-order permutations and bf16 activations; the oracle unpacks
and dequantizes them itself.  Tolerance: the kernel forms each weight with one
fp32 FMA and sums in fp32, so each output may differ from the float64 value by
a few fp32 rounding steps per partial sum; the bound below is relative to
sum_k |x_k| |w_k| (the conditioning of the sum), growing with the number of
sequential fp32 additions per lane.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _case(n_tok, d_col, d_row, bits, g, with_perm, seed):
    rng = np.random.default_rng(seed)
    words = d_col * bits // 32
    packed = rng.integers(0, 1 << 32, size=(d_row, words), dtype=np.uint64).astype(np.uint32)
    gg = d_col if g == -1 or g > d_col else g
    ng = -(-d_col // gg)
    scales = (rng.random((ng, d_row)) * 0.02 + 1e-3).astype(np.float32)
    zeros = rng.integers(0, 1 << bits, size=(ng, d_row)).astype(np.int32)
    perm = rng.permutation(d_col).astype(np.int32) if with_perm else None
    X = torch.from_numpy(rng.standard_normal((n_tok, d_col)).astype(np.float32)).to(torch.bfloat16)
    return X, packed, scales, zeros, perm


def _run(X, packed, scales, zeros, perm, bits, g, d_row, ldy=None):
    import post_weight_quantization_gptq_b200 as gq
    n_tok = X.shape[0]
    Yfull = torch.full((n_tok, ldy or d_row), float("nan"), dtype=torch.float32, device="cuda")
    Y = Yfull[:, :d_row]
    ws = torch.empty(gq.gptq_dequant_matmul_workspace_size(n_tok, X.shape[1]), dtype=torch.uint8,
                     device="cuda")
    gq.gptq_dequant_matmul(X.cuda(), torch.from_numpy(packed.view(np.int32)).cuda(),
                           torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(),
                           None if perm is None else torch.from_numpy(perm).cuda(), bits, g, Y, ws)
    torch.cuda.synchronize()
    return Yfull.cpu().numpy()


@pytest.mark.parametrize("n_tok,d_col,d_row,bits,g,with_perm", [
    (1, 4096, 100, 4, 128, True),     # decode, act-order, ragged row block
    (3, 1000, 33, 4, 32, False),      # ragged K tile (1000 = 1024 - 24)
    (2, 2048, 64, 2, 64, True),
    (8, 512, 40, 8, -1, True),        # one group per row, 8 tokens in one launch
    (13, 3072, 70, 4, 256, True),     # two launches (8 + 5 tokens), groups across K tiles
    (2, 512, 17, 4, 8, False),        # smallest groups: 8 codes, one word each
    (1, 28672, 96, 4, 128, True),     # Llama-70B down_proj width
])
def test_dequant_matmul_matches_oracle(n_tok, d_col, d_row, bits, g, with_perm):
    X, packed, scales, zeros, perm = _case(n_tok, d_col, d_row, bits, g, with_perm,
                                           seed=d_col + d_row + bits)
    Yg = _run(X, packed, scales, zeros, perm, bits, g, d_row)
    Yo = oracle.dequant_matmul(X, packed, scales, zeros, perm, bits, g, d_col)
    Xq = np.abs(X.to(torch.float64).numpy())
    if perm is not None:
        Xq = Xq[:, perm]
    Qa = np.abs(oracle.dequantize(oracle.unpack(packed, d_col, bits), scales, zeros, g))
    scale = Xq @ Qa.T
    tol = 1e-6 * (8 + d_col / 256) * scale
    err = np.abs(Yg - Yo)
    print(f"max |err| / bound {np.max(err / (tol + 1e-30)):.3f}")
    assert np.all(err <= tol)


def test_dequant_matmul_leaves_padding_and_is_deterministic():
    X, packed, scales, zeros, perm = _case(5, 768, 50, 4, 128, True, seed=9)
    a = _run(X, packed, scales, zeros, perm, 4, 128, 50, ldy=64)
    b = _run(X, packed, scales, zeros, perm, 4, 128, 50, ldy=64)
    assert np.all(np.isnan(a[:, 50:]))                      # columns past d_row untouched
    assert np.array_equal(a[:, :50], b[:, :50])             # no atomics: same bits every call

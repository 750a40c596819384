"""GPU parity of the many-token product with a quantized layer
(gptq_dequant_gemm, tcgen05) against the float64 oracle, through the C ABI.

The kernel dequantizes each weight to bf16 (one fp32 product, rounded to
nearest-even) and multiplies on the tensor cores; the oracle forms the same
bf16 weights (oracle.dequant_matmul with weights_bf16) and sums in float64.
The products of two bf16 values are exact, so the outputs differ only by the
fp32 accumulation: at most one rounding of the running sum per 16-term MMA
step (K / 16 of them) plus the sum inside each step, each within 2^-23 of
sum_k |x_k w_k|; the bound below allows twice that.
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
    zeros = rng.integers(-2, (1 << bits) + 2, size=(ng, d_row)).astype(np.int32)
    perm = rng.permutation(d_col).astype(np.int32) if with_perm else None
    X = torch.from_numpy(rng.standard_normal((n_tok, d_col)).astype(np.float32)).to(torch.bfloat16)
    return X, packed, scales, zeros, perm


def _run(X, packed, scales, zeros, perm, bits, g, d_row, ldy=None, ldx=None):
    import post_weight_quantization_gptq_b200 as gq
    n_tok, d_col = X.shape
    Yfull = torch.full((n_tok, ldy or d_row), float("nan"), dtype=torch.float32, device="cuda")
    Y = Yfull[:, :d_row]
    Xs = torch.zeros(n_tok, ldx or d_col, dtype=torch.bfloat16)
    Xs[:, :d_col] = X
    Xd = Xs.cuda()[:, :d_col]
    ws = torch.empty(gq.gptq_dequant_gemm_workspace_size(n_tok, d_col), dtype=torch.uint8,
                     device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq.gptq_dequant_gemm(Xd, torch.from_numpy(packed.view(np.int32)).cuda(),
                         torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(),
                         None if perm is None else torch.from_numpy(perm).cuda(), bits, g, Y, ws, st)
    assert gq.gptq_sync_status(st) == 0
    return Yfull.cpu().numpy()


@pytest.mark.parametrize("n_tok,d_col,d_row,bits,g,with_perm,ldx", [
    (256, 512, 256, 4, 128, True, None),     # one whole tile, act-order
    (300, 1024, 300, 4, 128, False, None),   # ragged token and output tails
    (1000, 4096, 520, 4, 128, True, None),
    (64, 768, 1000, 2, 64, True, None),
    (130, 2048, 257, 8, -1, False, None),    # one group per row
    (512, 1024, 128, 4, 8, True, None),      # smallest groups (8 codes)
    (77, 512, 96, 4, 32, False, 516),        # X rows not 16-byte aligned: gathered
    (2048, 8192, 1024, 4, 128, True, None),
    (16, 82048, 128, 4, 128, True, None),    # rows too wide to stage: gathered through L1
])
def test_dequant_gemm_matches_oracle(n_tok, d_col, d_row, bits, g, with_perm, ldx):
    X, packed, scales, zeros, perm = _case(n_tok, d_col, d_row, bits, g, with_perm,
                                           seed=n_tok + d_col + d_row + bits)
    Yg = _run(X, packed, scales, zeros, perm, bits, g, d_row, ldx=ldx)
    Yo = oracle.dequant_matmul(X, packed, scales, zeros, perm, bits, g, d_col, weights_bf16=True)
    Xa = np.abs(X.to(torch.float64).numpy())
    if perm is not None:
        Xa = Xa[:, perm]
    codes = oracle.unpack(packed, d_col, bits)
    gg = d_col if g == -1 else g
    gi = np.arange(d_col) // gg
    Wa = np.abs(oracle.bf16_round(scales[gi, :].T * (codes.astype(np.float32)
                                                     - zeros[gi, :].T.astype(np.float32))))
    bound = 2 * (d_col / 16 + 16) * 2.0 ** -23 * (Xa @ Wa.T)
    err = np.abs(Yg[:, :d_row] - Yo)
    print(f"max |err| / bound {np.max(err / (bound + 1e-30)):.3f}")
    assert np.all(err <= bound)


def test_dequant_gemm_leaves_padding_and_is_deterministic():
    X, packed, scales, zeros, perm = _case(300, 1024, 200, 4, 128, True, seed=9)
    a = _run(X, packed, scales, zeros, perm, 4, 128, 200, ldy=260)
    b = _run(X, packed, scales, zeros, perm, 4, 128, 200, ldy=260)
    assert np.all(np.isnan(a[:, 200:]))          # columns past d_row untouched
    assert np.array_equal(a[:, :200], b[:, :200])  # no atomics: same bits every call


def test_dequant_gemm_agrees_with_the_decode_form():
    """Both forms of the product on the same packed layer: the decode form
    keeps the weights exact (fp32), the many-token form rounds them to bf16,
    so they agree within the bf16 rounding of the weights."""
    import post_weight_quantization_gptq_b200 as gq
    X, packed, scales, zeros, perm = _case(8, 1024, 256, 4, 128, True, seed=5)
    zeros = np.clip(zeros, 0, 15).astype(np.int32)
    Yg = _run(X, packed, scales, zeros, perm, 4, 128, 256)
    Y = torch.empty(8, 256, dtype=torch.float32, device="cuda")
    ws = torch.empty(gq.gptq_dequant_matmul_workspace_size(8, 1024), dtype=torch.uint8,
                     device="cuda")
    gq.gptq_dequant_matmul(X.cuda(), torch.from_numpy(packed.view(np.int32)).cuda(),
                           torch.from_numpy(scales).cuda(), torch.from_numpy(zeros).cuda(),
                           torch.from_numpy(perm).cuda(), 4, 128, Y, ws)
    Yd = Y.cpu().numpy()
    Xa = np.abs(X.to(torch.float64).numpy())[:, perm]
    Qa = np.abs(oracle.dequantize(oracle.unpack(packed, 1024, 4), scales, zeros, 128))
    assert np.all(np.abs(Yg - Yd) <= 2.0 ** -8 * (Xa @ Qa.T) + 1e-6)

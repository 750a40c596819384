"""Parity at the workloads' full sizes, on sampled outputs the oracle can
compute one by one (rows of H; rows of W, which are independent given U),
plus properties that hold at any size where a float64 inverse is out of
reach on the host.

* Llama-7B q_proj (the benchmark workload): H over all 262,144 tokens in the
  launch configuration the benchmark times; the column walk on 4096 x 4096.
* Llama-7B down_proj (d = 11,008, g32, act-order), Llama-70B q_proj
  (d = 8192): H rows on a 65,536-token slice, the column walk at full size.
* One Llama-7B block: q/k/v share one H and one U (3-bit g128).
* Llama-70B down_proj (d = 28,672): H rows, and U^T U (H + lambda I) v = v.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gptq_testlib import compare_quantization, gpu

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _sample(d, k, seed, extra=()):
    rng = np.random.default_rng(seed)
    idx = set(int(i) for i in rng.choice(d, size=k, replace=False))
    idx.update(int(e) for e in extra if 0 <= e < d)
    return np.array(sorted(idx))


def _gpu_H(X):
    g = gpu()
    d = X.shape[1]
    H = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    st = _status()
    g.gptq_hessian_accumulate(X, H, st)
    assert g.gptq_sync_status(st) == 0
    return H


def _lower_rows(H, idx):
    """Rows idx of a symmetric H of which the lower triangle is valid."""
    rows = []
    for i in idx:
        i = int(i)
        left = H[i, : i + 1]
        below = H[i + 1:, i]
        rows.append(torch.cat([left, below]).double().cpu().numpy())
    return np.stack(rows)


@pytest.mark.parametrize("name,tokens,k", [("llama7b_q_proj", None, 32),
                                           ("llama7b_down_proj", 65536, 24),
                                           ("llama70b_q_proj", 65536, 24),
                                           ("llama70b_down_proj", 32768, 12)])
def test_hessian_rows_at_full_width(name, tokens, k):
    wl = workloads.WORKLOADS[name]
    X = workloads.activations(wl, device=DEV, n_tokens=tokens)
    H = _gpu_H(X)
    out_idx = workloads.outlier_channels(wl.d_col, wl.outlier_frac, wl.seed + 7919).numpy()
    idx = _sample(wl.d_col, k, seed=wl.d_col, extra=(0, wl.d_col - 1, *out_idx[:2]))
    Hg = _lower_rows(H, idx)
    del H
    Xh = X.cpu()
    del X
    torch.cuda.empty_cache()
    Ho = oracle.hessian_rows(Xh, idx, chunk=4096)
    errs = [np.linalg.norm(Hg[j] - Ho[j]) / np.linalg.norm(Ho[j]) for j in range(len(idx))]
    print(f"{name}: {len(idx)} rows of H, max row rel err {max(errs):.2e}")
    assert max(errs) <= 1e-3


def _quantize_on_gpu(H32, W, bits, group, desc_act, damp=0.01, prepared=None):
    g = gpu()
    d_row, d_col = W.shape
    cfg = g.GPTQConfig(bits=bits, group_size=group, desc_act=desc_act, damp=damp)
    ws = torch.empty(g.gptq_workspace_size(cfg, d_row, d_col), dtype=torch.uint8, device=DEV)
    st = _status()
    if prepared is None:
        U = torch.empty(d_col, d_col, dtype=torch.float32, device=DEV)
        perm = torch.empty(d_col, dtype=torch.int32, device=DEV)
        dead = torch.empty(d_col, dtype=torch.uint8, device=DEV)
        g.gptq_prepare_hinv(torch.from_numpy(H32).to(DEV), cfg, U, perm, dead, st, ws)
        prepared = (U, perm, dead)
    U, perm, dead = prepared
    Wd = W.to(DEV).contiguous()
    ng = g.n_groups(d_col, group)
    codes = torch.empty(d_row, d_col, dtype=torch.uint8, device=DEV)
    scales = torch.empty(ng, d_row, dtype=torch.float32, device=DEV)
    zeros = torch.empty(ng, d_row, dtype=torch.int32, device=DEV)
    g.gptq_quantize_layer(Wd, U, perm, dead, cfg, codes, scales, zeros, st, ws)
    packed = torch.empty(d_row, g.packed_words(d_col, bits), dtype=torch.int32, device=DEV)
    g.gptq_pack(codes, bits, packed)
    status = g.gptq_sync_status(st)
    out = dict(status=status, perm=perm.cpu().numpy(), dead=dead.cpu().numpy().astype(bool),
               codes=codes.cpu().numpy(), scales=scales.cpu().numpy(), zeros=zeros.cpu().numpy(),
               w_at_quant=Wd.cpu().numpy(), packed=packed.cpu().numpy().view(np.uint32))
    return out, prepared


@pytest.mark.parametrize("name,h_tokens,rows", [("llama7b_q_proj", 8192, 48),
                                                ("llama7b_down_proj", 16384, 24),
                                                ("llama70b_q_proj", 8192, 24)])
def test_column_walk_at_full_size_sampled_rows(name, h_tokens, rows):
    """The full d_row x d_col layer on the GPU; the oracle replays sampled rows
    (rows are independent given U) from the same float32 H.  H is taken from
    a slice of the calibration tokens so that the host can form it in float64."""
    wl = workloads.WORKLOADS[name]
    Xs = workloads.activations(wl, n_tokens=h_tokens)
    H64 = oracle.hessian(Xs)
    H32 = H64.astype(np.float32)
    W = workloads.weights(wl)
    out, _ = _quantize_on_gpu(H32, W, wl.bits, wl.group_size, wl.desc_act, wl.damp)
    sel = _sample(wl.d_row, rows, seed=wl.d_row + 1, extra=(0, wl.d_row - 1))
    res = compare_quantization(H32.astype(np.float64), W, out, wl.bits, wl.group_size,
                               wl.desc_act, wl.damp, rows=sel)
    assert res["loss_gpu"] < res["loss_rtn"]


def test_llama7b_block_qkv_share_one_inverse_factor():
    """q, k and v see the same input, so one H and one U serve all three
    (3-bit g128, the block workload's quantizer)."""
    q = workloads.LLAMA7B_BLOCK_QUANT
    d = 4096
    Xs = workloads.student_t_activations(8192, d, seed=workloads.BASE_SEED + 3)
    H64 = oracle.hessian(Xs)
    H32 = H64.astype(np.float32)
    prepared = None
    for j, name in enumerate(("q_proj", "k_proj", "v_proj")):
        W = workloads.gaussian_weights(d, d, 0.02, seed=workloads.BASE_SEED + 3 + 101 * j)
        out, prepared = _quantize_on_gpu(H32, W, q["bits"], q["group_size"], q["desc_act"],
                                         q["damp"], prepared=prepared)
        sel = _sample(d, 16, seed=17 + j)
        compare_quantization(H32.astype(np.float64), W, out, q["bits"], q["group_size"],
                             q["desc_act"], q["damp"], rows=sel)


def test_llama70b_down_proj_inverse_factor_property():
    """d = 28,672: the inverse factor satisfies U^T U (P^T H P + lambda I) v = v
    for random v (float64 on the host, from the GPU's H and U), U is upper
    with a positive diagonal, and act-order is a stable descending sort."""
    g = gpu()
    wl = workloads.WORKLOADS["llama70b_down_proj"]
    d = wl.d_col
    X = workloads.activations(wl, device=DEV, n_tokens=32768)
    H = _gpu_H(X)
    del X
    Hl = torch.tril(H).cpu()  # lower triangle, as the GPU guarantees
    Hsym = (Hl + Hl.T - torch.diag(torch.diag(Hl))).double()
    cfg = g.GPTQConfig(bits=4, group_size=128, desc_act=True, damp=wl.damp)
    ws = torch.empty(g.gptq_workspace_size(cfg, 8, d), dtype=torch.uint8, device=DEV)
    U = torch.empty(d, d, dtype=torch.float32, device=DEV)
    perm = torch.empty(d, dtype=torch.int32, device=DEV)
    dead = torch.empty(d, dtype=torch.uint8, device=DEV)
    st = _status()
    g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    assert g.gptq_sync_status(st) == 0
    del H
    p = perm.cpu().numpy()
    diag = np.diag(Hsym.numpy())
    assert np.array_equal(p, np.argsort(-diag, kind="stable"))
    lam = wl.damp * diag.mean()
    Uh = U.cpu()
    del U
    torch.cuda.empty_cache()
    pt = torch.from_numpy(p.astype(np.int64))
    Hp = Hsym[pt][:, pt]
    del Hsym
    Hp.diagonal().add_(lam)
    assert torch.all(torch.diagonal(Uh) > 0)
    assert float(torch.tril(Uh[:2048, :2048], -1).abs().max()) == 0.0
    Ud = Uh.double()
    rng = np.random.default_rng(5)
    v = torch.from_numpy(rng.standard_normal((d, 3)))
    y = Ud.T @ (Ud @ (Hp @ v))
    rel = float((y - v).norm() / v.norm())
    print(f"d={d}: |U^T U H v - v| / |v| = {rel:.2e}")
    assert rel <= 5e-2

"""GPU parity of every stage against the float64 oracle, through the C ABI.

Sizes span several tiles and ragged tails; the tiny workload (256 x 512,
2048 tokens) runs in full.  See gptq_testlib for the comparison rules.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from gptq_testlib import compare_quantization, gpu, gpu_hessian, gpu_quantize, lower_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


# ------------------------------------------------------------------ stage 1
@pytest.mark.parametrize("n,d,kind", [(2048, 512, "correlated"), (1000, 200, "student_t"),
                                      (63, 72, "student_t"), (1, 8, "student_t"),
                                      (4100, 520, "half_normal"), (777, 384, "student_t"),
                                      (3000, 1040, "student_t")])
def test_hessian_matches_oracle(n, d, kind):
    _, X = workloads.small_layer(4, d, n, seed=n + d, kind=kind)
    Hg = gpu_hessian(X)
    Ho = oracle.hessian(X)
    err = lower_rel_err(Hg, Ho)
    print(f"H rel Frobenius error {err:.3e}")
    assert err <= 1e-3
    # elementwise: fp32 summation of exact products
    L = np.tril(np.ones_like(Ho, dtype=bool))
    scale = np.sqrt(np.outer(np.diag(Ho), np.diag(Ho)))[L] + 1e-30
    assert np.max(np.abs(Hg - Ho)[L] / scale) <= 1e-4


def test_hessian_tiny_workload_and_strided_x():
    w = workloads.WORKLOADS["tiny"]
    X = workloads.activations(w)
    Ho = oracle.hessian(X)
    assert lower_rel_err(gpu_hessian(X), Ho) <= 1e-5
    assert lower_rel_err(gpu_hessian(X, ldx=520), Ho) <= 1e-5


def test_hessian_accumulates_over_token_chunks():
    _, X = workloads.small_layer(4, 256, 3000, seed=11)
    one = gpu_hessian(X)
    three = gpu_hessian(X, chunks=3)
    L = np.tril(np.ones_like(one, dtype=bool))
    assert np.max(np.abs(one - three)[L]) <= 1e-5 * np.max(np.abs(one))
    assert lower_rel_err(three, oracle.hessian(X)) <= 1e-5


@pytest.mark.parametrize("n,d,ldx,chunk", [(70000, 256, 256, 32768), (40000, 256, 256, 16384),
                                            (3000, 200, 203, 500),
                                            (777, 384, 384, 64), (100, 8, 8, 1 << 20)])
def test_hessian_from_host_memory(n, d, ldx, chunk):
    """X streamed from pinned host memory through the two-slot staging buffer:
    bitwise equal to the device-resident call when the chunk is a multiple
    of 32768 tokens (the GEMM's own accumulation chunk), else within fp32
    summation-order error plus, past one chunk, the accumulation drift of
    differently placed drains; ragged last chunk, padded host rows, d not a
    multiple of 8 included."""
    import post_weight_quantization_gptq_b200 as g
    _, X = workloads.small_layer(4, d, n, seed=n + d + 5, kind="student_t")
    dev = torch.device("cuda")
    Xh = torch.zeros(n, ldx, dtype=torch.bfloat16).pin_memory()
    Xh[:, :d] = X
    if ldx > d:
        Xh[:, d:] = 7.0  # never read: only the first d channels of a row are X
    staging = torch.empty(g.gptq_hessian_staging_size(d, min(chunk, n)), dtype=torch.uint8,
                          device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    H = torch.zeros(d, d, dtype=torch.float32, device=dev)
    g.gptq_hessian_accumulate_host(Xh[:, :d], H, staging, st)
    assert g.gptq_sync_status(st) == 0
    Hh = H.cpu().numpy()
    Hd = gpu_hessian(X)
    L = np.tril(np.ones_like(Hd, dtype=bool))
    if chunk % 32768 == 0:
        assert np.array_equal(Hh[L], Hd[L])
    elif n <= 32768:
        # both sides drain once, at the end of each call: summation order only
        assert np.max(np.abs(Hh - Hd)[L]) <= 1e-5 * np.max(np.abs(Hd))
    else:
        # different drain points: the tensor cores' accumulation drift (up to
        # ~1.8e-4 per 32768-token drain) differs as well
        assert np.max(np.abs(Hh - Hd)[L]) <= 2e-4 * np.max(np.abs(Hd))
    # the tensor cores' fp32 accumulation drifts within each 32768-token
    # drain (measured 1.4e-4 here, up to 1.8e-4 on full-size rows); the H bar
    # of the parity rules is 1e-3
    assert lower_rel_err(Hh, oracle.hessian(X)) <= 3e-4


# ------------------------------------------------------------------ stage 2
@pytest.mark.parametrize("d,desc_act,n_dead", [(512, False, 0), (512, True, 0), (200, True, 3),
                                               (132, False, 2), (1024, True, 0), (64, False, 0)])
def test_prepare_hinv_matches_oracle_elimination(d, desc_act, n_dead):
    rng = np.random.default_rng(d + n_dead)
    _, X = workloads.small_layer(4, d, 4 * d, seed=d, kind="correlated")
    Xf = X.to(torch.float32)
    dead_idx = rng.choice(d, size=n_dead, replace=False)
    Xf[:, dead_idx] = 0.0
    H = oracle.hessian(Xf.to(torch.bfloat16)).astype(np.float32)
    W = workloads.gaussian_weights(8, d, 0.02, seed=1)
    out = gpu_quantize(H, W, 4, 128 if d % 128 == 0 else -1, desc_act)
    assert out["status"] == 0
    prep = oracle.prepare(H.astype(np.float64), W, damp=0.01, desc_act=desc_act)
    assert np.array_equal(out["perm"], prep["perm"])
    assert np.array_equal(out["dead"], prep["dead"])
    _, Uo = oracle.eliminate(oracle.inverse(prep["H_damped"]))
    Ug = out["U"]
    rel = np.max(np.abs(Ug - Uo)) / np.max(np.abs(Uo))
    cond = np.linalg.cond(prep["H_damped"])
    print(f"d={d} cond={cond:.2e} U max rel err {rel:.3e}")
    assert np.all(np.tril(Ug, -1) == 0.0)
    assert rel <= 2e-3
    # U^T U Hd = I (a property of the output at any size)
    resid = np.max(np.abs(Ug.T @ (Ug @ prep["H_damped"]) - np.eye(d)))
    assert resid <= 5e-2


@pytest.mark.parametrize("fill", [float("nan"), 123.0])
def test_prepare_hinv_ignores_prior_output_contents(fill):
    """12 panels (side streams, lookahead and early-started launches all in
    play) with U pre-filled: nothing the caller left in U may leak into it,
    and every panel must see every update before it is factored."""
    g = gpu()
    d = 1536
    _, X = workloads.small_layer(4, d, 3 * d, seed=77, kind="student_t")
    H = oracle.hessian(X)
    cfg = g.GPTQConfig(bits=4, group_size=128)
    ws = torch.empty(g.gptq_workspace_size(cfg, 8, d), dtype=torch.uint8, device="cuda")
    prep = oracle.prepare(H, torch.zeros(1, d), damp=0.01, desc_act=False)
    Uo = oracle.upper_factor(prep["H_damped"])
    for _ in range(3):
        U = torch.full((d, d), fill, device="cuda")
        perm = torch.empty(d, dtype=torch.int32, device="cuda")
        dead = torch.empty(d, dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        g.gptq_prepare_hinv(torch.from_numpy(H.astype(np.float32)).cuda(), cfg, U, perm, dead, st, ws)
        assert g.gptq_sync_status(st) == 0
        Ug = U.cpu().numpy().astype(np.float64)
        assert np.isfinite(Ug).all()
        rel = np.max(np.abs(Ug - Uo)) / np.max(np.abs(Uo))
        print(f"fill={fill} U max rel err {rel:.3e}")
        assert rel <= 1e-4


def test_not_positive_definite_is_reported():
    g = gpu()
    d = 96
    cfg = g.GPTQConfig(bits=4, group_size=32, damp=0.0)
    H = -torch.eye(d, dtype=torch.float32, device="cuda")
    ws = torch.empty(g.gptq_workspace_size(cfg, 4, d), dtype=torch.uint8, device="cuda")
    U = torch.empty(d, d, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    assert g.gptq_sync_status(st) == 3
    assert torch.isfinite(U).all()


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_non_finite_diagonal_is_reported_and_perm_stays_a_permutation(bad):
    """A non-finite diagonal entry of H (e.g. a NaN in the calibration data)
    is reported as not positive definite; the act-order permutation is still a
    permutation (NaN columns ranked last, as a stable sort of -diag does), so
    nothing downstream indexes outside the matrix."""
    g = gpu()
    d = 256
    _, X = workloads.small_layer(4, d, 4 * d, seed=3, kind="student_t")
    H = oracle.hessian(X).astype(np.float32)
    for i in (5, 77, 200):
        H[i, i] = bad
    cfg = g.GPTQConfig(bits=4, group_size=128, desc_act=True)
    ws = torch.empty(g.gptq_workspace_size(cfg, 4, d), dtype=torch.uint8, device="cuda")
    U = torch.empty(d, d, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.gptq_prepare_hinv(torch.from_numpy(H).cuda(), cfg, U, perm, dead, st, ws)
    assert g.gptq_sync_status(st) == 3
    p = perm.cpu().numpy()
    assert np.array_equal(np.sort(p), np.arange(d))
    assert np.array_equal(p, np.argsort(-np.diag(H).astype(np.float64), kind="stable"))


def test_out_of_range_permutation_entry_is_reported():
    """quantize_layer with act-order reads perm; an entry outside [0, d_col)
    is reported as an invalid argument on the device and no access leaves
    the row (the entry is read as the identity)."""
    g = gpu()
    d, r = 256, 8
    W, X = workloads.small_layer(r, d, 4 * d, seed=4, kind="student_t")
    H = oracle.hessian(X).astype(np.float32)
    cfg = g.GPTQConfig(bits=4, group_size=128, desc_act=True)
    ws = torch.empty(g.gptq_workspace_size(cfg, r, d), dtype=torch.uint8, device="cuda")
    U = torch.empty(d, d, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g.gptq_prepare_hinv(torch.from_numpy(H).cuda(), cfg, U, perm, dead, st, ws)
    assert g.gptq_sync_status(st) == 0
    perm[10] = d + 1000
    perm[11] = -7
    codes = torch.empty(r, d, dtype=torch.uint8, device="cuda")
    scales = torch.empty(2, r, device="cuda")
    zeros = torch.empty(2, r, dtype=torch.int32, device="cuda")
    g.gptq_quantize_layer(W.cuda().contiguous(), U, perm, dead, cfg, codes, scales, zeros, st, ws)
    assert g.gptq_sync_status(st) == 1


# ------------------------------------------------------------ stages 3 + 4
QUANT_CASES = [
    # d_row, d_col, tokens, kind, bits, group, desc_act
    (256, 512, 2048, "correlated", 4, 128, False),
    (256, 512, 2048, "correlated", 4, 32, True),
    (64, 384, 2048, "student_t", 3, 128, False),
    (40, 256, 1024, "half_normal", 2, 64, True),
    (33, 512, 2048, "student_t", 4, -1, False),
    (16, 512, 2048, "student_t", 4, 256, True),
    (7, 200, 800, "student_t", 4, 8, False),
    (5, 132, 700, "correlated", 8, 128, True),
    (1, 64, 256, "student_t", 4, 32, False),
    (300, 1024, 4096, "student_t", 4, 128, True),
]


@pytest.mark.parametrize("d_row,d_col,n,kind,bits,g,desc_act", QUANT_CASES)
def test_quantize_layer_matches_oracle(d_row, d_col, n, kind, bits, g, desc_act):
    W, X = workloads.small_layer(d_row, d_col, n, seed=d_row * 7 + d_col, kind=kind)
    H = oracle.hessian(X).astype(np.float32)
    out = gpu_quantize(H, W, bits, g, desc_act)
    compare_quantization(H.astype(np.float64), W, out, bits, g, desc_act)


@pytest.mark.parametrize("d_row,d_col,n,kind,bits,g,desc_act,offset",
                         [(256, 512, 2048, "correlated", 4, 128, False, 0.0),
                          (64, 384, 2048, "student_t", 3, 32, True, 0.03),
                          (40, 256, 1024, "half_normal", 2, 8, True, 0.0),
                          (33, 512, 2048, "student_t", 4, -1, False, -0.12),
                          (16, 1024, 4096, "student_t", 8, 256, False, 0.12)])
def test_pure_minmax_range_matches_oracle(d_row, d_col, n, kind, bits, g, desc_act, offset):
    """The pure min-max option (each group's own [min, max]): weights
    shifted off zero so that many groups are one-signed and get zero points
    outside the code range; small groups (8) make one-signed groups common
    without a shift."""
    W, X = workloads.small_layer(d_row, d_col, n, seed=d_row * 5 + d_col, kind=kind)
    W = W + offset
    H = oracle.hessian(X).astype(np.float32)
    out = gpu_quantize(H, W, bits, g, desc_act, pure=True)
    # at 8 bits a level is 16 times finer than at 4, so the same fp32 drift
    # puts 16 times more codes on ties: the free-running rate is reported only
    res = compare_quantization(H.astype(np.float64), W, out, bits, g, desc_act, pure=True,
                               strict_free=bits < 8)
    if offset != 0.0:
        z = out["zeros"]
        assert z.min() < 0 or z.max() > (1 << bits) - 1  # one-signed groups occurred
    assert res["loss_gpu"] < res["loss_rtn"]


@pytest.mark.parametrize("d_row,d_col,g,damp,desc_act", [(24, 2048, 1024, 0.01, False),
                                                         (24, 2048, 1024, 0.005, True),
                                                         (48, 768, 32, 0.005, True)])
def test_quantize_layer_wide_groups_and_light_damping(d_row, d_col, g, damp, desc_act):
    """The guide's other knobs: groups of 1024 columns (eight blocks share one
    scale and zero point, the deferred lazy-update schedule shortens its runs
    so the group's later columns are complete when it opens) and its
    high-accuracy damping of 0.005."""
    W, X = workloads.small_layer(d_row, d_col, 3 * d_col, seed=d_col + g, kind="student_t")
    H = oracle.hessian(X).astype(np.float32)
    out = gpu_quantize(H, W, 4, g, desc_act, damp)
    compare_quantization(H.astype(np.float64), W, out, 4, g, desc_act, damp)


@pytest.mark.parametrize("g,desc_act", [(128, True), (128, False), (256, False), (32, False)])
def test_dead_columns_are_zero_weight(g, desc_act):
    """Dead input channels quantize to exact zeros, whether the act-order pass
    zeroes them (desc_act) or the column walk does as it loads its block
    (including the later columns a group wider than a block reads)."""
    W, X = workloads.small_layer(24, 512, 2048, seed=5)
    Xf = X.to(torch.float32)
    Xf[:, [3, 100, 255, 300]] = 0.0
    H = oracle.hessian(Xf.to(torch.bfloat16)).astype(np.float32)
    out = gpu_quantize(H, W, 4, g, desc_act)
    compare_quantization(H.astype(np.float64), W, out, 4, g, desc_act)
    pos = np.nonzero(np.isin(out["perm"], [3, 100, 255, 300]))[0]
    Q = oracle.dequantize(out["codes"], out["scales"], out["zeros"], g)
    assert np.all(Q[:, pos] == 0.0)


def test_identity_hessian_gives_round_to_nearest():
    d = 256
    W = workloads.gaussian_weights(32, d, 0.03, seed=2)
    H = (5.0 * np.eye(d)).astype(np.float32)
    out = gpu_quantize(H, W, 4, 64, False)
    rc, rs, rz = oracle.rtn(W.numpy().astype(np.float64), 4, 64)
    assert np.array_equal(out["codes"], rc)
    assert np.array_equal(out["zeros"], rz)
    assert np.max(np.abs(out["scales"] - rs) / rs) <= 1e-6


def test_end_to_end_tiny_workload_from_activations():
    """X -> H (GPU) -> U -> codes -> packed, checked against the oracle run
    from the same X (its own float64 H)."""
    w = workloads.WORKLOADS["tiny"]
    W, X = workloads.weights(w), workloads.activations(w)
    g = gpu()
    cfg = g.GPTQConfig(bits=w.bits, group_size=w.group_size, desc_act=w.desc_act, damp=w.damp)
    Hg = gpu_hessian(X)
    Ho = oracle.hessian(X)
    assert lower_rel_err(Hg, Ho) <= 1e-3
    out = gpu_quantize(np.tril(Hg), W, w.bits, w.group_size, w.desc_act, w.damp)
    res = compare_quantization(Ho, W, out, w.bits, w.group_size, w.desc_act, w.damp)
    assert res["loss_gpu"] < res["loss_rtn"]
    del cfg


# ------------------------------------------------------------------ stage 5
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("d", [8, 64, 100, 4096])
def test_pack_is_bit_exact(bits, d):
    g = gpu()
    rng = np.random.default_rng(bits * d)
    c = rng.integers(0, 1 << bits, size=(37, d), dtype=np.uint8)
    cd = torch.from_numpy(c).cuda()
    packed = torch.empty(37, g.packed_words(d, bits), dtype=torch.int32, device="cuda")
    g.gptq_pack(cd, bits, packed)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(c, bits))


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_pack_is_bit_exact_from_unaligned_codes(bits):
    """Codes that do not start on a 16-byte boundary take the word-at-a-time
    kernel instead of the 16-code chunks; same bits."""
    g = gpu()
    d = 256
    rng = np.random.default_rng(bits + 7)
    c = rng.integers(0, 1 << bits, size=(50, d), dtype=np.uint8)
    buf = torch.zeros(50 * d + 16, dtype=torch.uint8, device="cuda")
    cd = buf[3:3 + 50 * d].view(50, d)
    cd.copy_(torch.from_numpy(c))
    packed = torch.empty(50, g.packed_words(d, bits), dtype=torch.int32, device="cuda")
    g.gptq_pack(cd, bits, packed)
    torch.cuda.synchronize()
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack(c, bits))


def test_stages_replay_from_a_cuda_graph_bit_exactly():
    """The four stages captured once in CUDA graphs (the library's side streams
    join the capture through its events) and replayed twice give the same bits
    as the stream-launched calls: U, perm, codes, scales, zeros, packed words."""
    g = gpu()
    r, d, n = 96, 640, 2560
    W, X = workloads.small_layer(r, d, n, seed=31, kind="correlated")
    cfg = g.GPTQConfig(bits=4, group_size=128, desc_act=True, damp=0.01)
    dev = torch.device("cuda")
    Xd, W0 = X.to(dev), W.to(dev).contiguous()
    bufs = dict(H=torch.zeros(d, d, device=dev), U=torch.empty(d, d, device=dev),
                perm=torch.empty(d, dtype=torch.int32, device=dev),
                dead=torch.empty(d, dtype=torch.uint8, device=dev), W=torch.empty_like(W0),
                codes=torch.empty(r, d, dtype=torch.uint8, device=dev),
                scales=torch.empty(g.n_groups(d, 128), r, device=dev),
                zeros=torch.empty(g.n_groups(d, 128), r, dtype=torch.int32, device=dev),
                packed=torch.empty(r, g.packed_words(d, 4), dtype=torch.int32, device=dev),
                ws=torch.empty(g.gptq_workspace_size(cfg, r, d), dtype=torch.uint8, device=dev),
                st=torch.zeros(1, dtype=torch.int32, device=dev))
    b = bufs

    def stages():
        return [lambda: (b["H"].zero_(), g.gptq_hessian_accumulate(Xd, b["H"], b["st"])),
                lambda: g.gptq_prepare_hinv(b["H"], cfg, b["U"], b["perm"], b["dead"], b["st"], b["ws"]),
                lambda: (b["W"].copy_(W0), g.gptq_quantize_layer(b["W"], b["U"], b["perm"], b["dead"], cfg,
                                                                  b["codes"], b["scales"], b["zeros"],
                                                                  b["st"], b["ws"])),
                lambda: g.gptq_pack(b["codes"], 4, b["packed"])]

    for fn in stages():  # stream launches (also the one-time set-up of the side streams)
        fn()
    assert g.gptq_sync_status(b["st"]) == 0
    ref = {k: b[k].clone() for k in ("U", "perm", "codes", "scales", "zeros", "packed")}
    graphs = []
    for fn in stages():
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, capture_error_mode="thread_local"):
            fn()
        graphs.append(gr)
    for _ in range(2):
        for k in ("U", "codes", "packed"):
            b[k].zero_()
        for gr in graphs:
            gr.replay()
        assert g.gptq_sync_status(b["st"]) == 0
        for k, v in ref.items():
            assert torch.equal(b[k], v), k


@pytest.mark.parametrize("d_row,d_col,bits,g,desc_act", [(300, 1536, 4, 128, True),
                                                     (130, 2048, 3, 32, False)])
def test_lazy_update_presplit_is_bit_identical(d_row, d_col, bits, g, desc_act):
    """The full workspace makes the lazy update read its operands' low parts,
    split once by the column walk (errors) and one pass over U; a workspace
    that only holds the eight deferred blocks' errors makes it split in the
    GEMM.  Same schedule, same split values: codes, scales, zeros and the
    pre-quantization weights agree bit for bit."""
    g_ = gpu()
    W, X = workloads.small_layer(d_row, d_col, 4 * d_col, seed=d_row + d_col, kind="student_t")
    H = torch.from_numpy(oracle.hessian(X).astype(np.float32)).cuda()
    cfg = g_.GPTQConfig(bits=bits, group_size=g, desc_act=desc_act)
    full = g_.gptq_workspace_size(cfg, d_row, d_col)
    errs_only = (d_row * 128 * min(8, -(-d_col // 128)) * 4 + 255) // 256 * 256
    assert errs_only < full
    ws = torch.empty(full, dtype=torch.uint8, device="cuda")
    U = torch.empty(d_col, d_col, device="cuda")
    perm = torch.empty(d_col, dtype=torch.int32, device="cuda")
    dead = torch.empty(d_col, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    g_.gptq_prepare_hinv(H, cfg, U, perm, dead, st, ws)
    outs = []
    for nbytes in (full, errs_only):
        Wd = W.cuda().contiguous()
        ng = g_.n_groups(d_col, g)
        o = (torch.empty(d_row, d_col, dtype=torch.uint8, device="cuda"),
             torch.empty(ng, d_row, dtype=torch.float32, device="cuda"),
             torch.empty(ng, d_row, dtype=torch.int32, device="cuda"))
        g_.gptq_quantize_layer(Wd, U, perm, dead, cfg, *o, st, ws[:nbytes])
        assert g_.gptq_sync_status(st) == 0
        outs.append((*o, Wd))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


@pytest.mark.parametrize("pad,offset", [(3, 0), (3, 1), (1, 3)])
def test_quantize_layer_on_strided_and_offset_weights(pad, offset):
    """W as a view into a wider buffer: a row pitch that is not a multiple of
    4 floats, or a base that is not 16-byte aligned.  The lazy update cannot
    address such rows with a tensor map and drains through shared memory, the
    column walk moves W element by element; the result must be the contiguous
    call's bit for bit, and the buffer outside the view stays untouched."""
    g = gpu()
    d_row, d_col, bits, gs = 96, 512, 4, 128
    W, X = workloads.small_layer(d_row, d_col, 2048, seed=pad * 10 + offset, kind="student_t")
    H = oracle.hessian(X).astype(np.float32)
    ref = gpu_quantize(H, W, bits, gs, False)
    cfg = g.GPTQConfig(bits=bits, group_size=gs, desc_act=False)
    Hd = torch.from_numpy(H).cuda()
    U = torch.empty(d_col, d_col, device="cuda")
    perm = torch.empty(d_col, dtype=torch.int32, device="cuda")
    dead = torch.empty(d_col, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(g.gptq_workspace_size(cfg, d_row, d_col), dtype=torch.uint8, device="cuda")
    g.gptq_prepare_hinv(Hd, cfg, U, perm, dead, st, ws)
    buf = torch.full((d_row, offset + d_col + pad), 7.0, device="cuda")
    Wv = buf[:, offset:offset + d_col]
    Wv.copy_(W.cuda())
    ng = g.n_groups(d_col, gs)
    codes = torch.empty(d_row, d_col, dtype=torch.uint8, device="cuda")
    scales = torch.empty(ng, d_row, device="cuda")
    zeros = torch.empty(ng, d_row, dtype=torch.int32, device="cuda")
    g.gptq_quantize_layer(Wv, U, perm, dead, cfg, codes, scales, zeros, st, ws)
    assert g.gptq_sync_status(st) == 0
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(scales.cpu().numpy(), ref["scales"])
    assert np.array_equal(zeros.cpu().numpy(), ref["zeros"])
    assert np.array_equal(Wv.cpu().numpy(), ref["w_at_quant"])
    outside = torch.cat([buf[:, :offset], buf[:, offset + d_col:]], dim=1)
    assert bool((outside == 7.0).all())


# ------------------------------------------------ streaming calibration (hook)
@pytest.mark.parametrize("d,shapes", [(384, [(2, 700), (3, 128), (1, 5000)]),
                                      (200, [(4, 33), (1, 1), (2, 900)])])
def test_forward_hook_accumulates_the_layer_inputs(d, shapes):
    """HessianAccumulator attached to a Linear layer as a forward pre-hook
    sums H = 2 X^T X over every calibration batch that flows through it, in
    any leading shape (d = 200: rows copied into a 16-byte pitch); compared
    with the oracle on all the tokens seen."""
    from post_weight_quantization_gptq_b200.calibration import HessianAccumulator
    lin = torch.nn.Linear(d, 48, bias=False, dtype=torch.bfloat16, device="cuda")
    acc = HessianAccumulator(d).attach(lin)
    seen = []
    for i, (b, t) in enumerate(shapes):
        _, X = workloads.small_layer(1, d, b * t, seed=100 + i, kind="student_t")
        x = X.reshape(b, t, d).cuda()
        with torch.no_grad():
            lin(x)
        seen.append(X)
    acc.detach()
    with torch.no_grad():
        lin(torch.ones(3, d, dtype=torch.bfloat16, device="cuda"))  # not accumulated
    acc.check()
    Xall = torch.cat(seen)
    assert acc.tokens == Xall.shape[0]
    # separate calls, each drained into H once (fp32 sums; the tensor cores'
    # accumulation drifts by ~2^-25 per step within a call): well inside 1e-3
    assert lower_rel_err(acc.H.cpu().numpy(), oracle.hessian(Xall)) <= 1e-4

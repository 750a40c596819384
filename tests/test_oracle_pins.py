"""Pins of the float64 oracle against what the GPTQ pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a
hand-computed worked example (tests/golden/), a closed form, a brute-force
solve, an invariant, or a textbook identity checked through an independent
library routine.  Page citations: "GPTQ (GPT Quantization)" sections
"Fondation theorique : OBQ" and "Algorithme complet (pseudo-code)"; the
AutoGPTQ guide "Optimization Gptq", "Quantizacao group-wise"; the "GPTQ"
article, "Desempenho e Precisao".
"""
import itertools
import os

import numpy as np
import pytest

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _spd(d, seed, n=None, cond_spread=1.0):
    rng = np.random.default_rng(seed)
    n = n or 4 * d
    X = rng.standard_normal((n, d)) * np.exp(cond_spread * rng.standard_normal(d))
    return 2.0 * X.T @ X


def _rows(path):
    out = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        out.append([f.strip() for f in line.split("|")])
    return out


# ---------------------------------------------------------------- quantizer
def test_quantizer_worked_examples():
    """Hand-computed scale / zero / codes / dequantized values (golden file)."""
    for name, bits, ws, s, z, codes, what in _rows(os.path.join(GOLDEN, "quantizer_worked_example.txt")):
        bits = int(bits)
        w = np.array([float(v) for v in ws.split()])
        scale, _, zero = oracle.quant_params(w, bits)
        assert scale == pytest.approx(float(s), rel=1e-15), name
        assert zero == int(z), name
        got = [oracle.quantize_code(x, scale, zero, bits) for x in w]
        assert got == [int(c) for c in codes.split()], name
        deq = oracle.dequantize(np.array([got], dtype=np.uint8), np.array([[scale]]),
                                np.array([[zero]]), -1)[0]
        assert np.allclose(deq, [float(v) for v in what.split()], atol=1e-15), name


def test_pure_minmax_quantizer_worked_examples():
    """The pure min-max range (the group's own [min, max]): hand-computed
    scale / zero / codes / dequantized values (golden file), zero points
    outside [0, 2^b - 1] included, and the two fall-backs to the widened
    range."""
    path = os.path.join(GOLDEN, "quantizer_pure_minmax_worked_example.txt")
    for name, bits, ws, s, z, codes, what in _rows(path):
        bits = int(bits)
        w = np.array([float(v) for v in ws.split()])
        scale, _, zero = oracle.quant_params(w, bits, pure=True)
        assert scale == pytest.approx(float(s), rel=1e-15), name
        assert zero == int(z), name
        got = [oracle.quantize_code(x, scale, zero, bits) for x in w]
        assert got == [int(c) for c in codes.split()], name
        deq = scale * (np.array(got, dtype=np.float64) - zero)
        assert np.allclose(deq, [float(v) for v in what.split()], rtol=1e-15, atol=1e-15), name


def test_pure_minmax_is_the_default_when_the_range_holds_zero():
    """A group whose values straddle 0 has the same range either way, so the
    two rules agree exactly; a one-signed group gets a finer scale."""
    rng = np.random.default_rng(12)
    for bits in (2, 3, 4, 8):
        w = rng.standard_normal(64)
        w[0], w[1] = -abs(w[0]), abs(w[1])
        assert oracle.quant_params(w, bits, pure=True) == oracle.quant_params(w, bits)
        pos = np.abs(w) + 0.5
        sp, _, zp = oracle.quant_params(pos, bits, pure=True)
        sd, _, _ = oracle.quant_params(pos, bits)
        assert sp < sd and zp < 0
        q = np.array([oracle.quantize_code(x, sp, zp, bits) for x in pos])
        assert q.min() >= 0 and q.max() <= (1 << bits) - 1
        assert np.abs(sp * (q - zp) - pos).max() <= 0.5 * sp * (1 + 1e-12)


def test_quantizer_roundtrip_bound():
    """|w_hat - w| <= s/2 for every weight inside the group's range."""
    rng = np.random.default_rng(3)
    for bits in (2, 3, 4, 8):
        for _ in range(50):
            w = rng.standard_normal(32) * rng.uniform(0.01, 3)
            s, _, z = oracle.quant_params(w, bits)
            q = np.array([oracle.quantize_code(x, s, z, bits) for x in w])
            assert q.min() >= 0 and q.max() <= (1 << bits) - 1
            assert 0 <= z <= (1 << bits) - 1
            err = np.abs(s * (q - z) - w)
            assert err.max() <= 0.5 * s * (1 + 1e-12) + 1e-15


# ------------------------------------------------------------------ packing
def test_pack_worked_examples():
    for bits, codes, words in _rows(os.path.join(GOLDEN, "pack_worked_example.txt")):
        bits = int(bits)
        c = np.array([[int(v) for v in codes.split()]], dtype=np.uint8)
        p = oracle.pack(c, bits)
        assert [int(v) for v in p[0]] == [int(v, 16) for v in words.split()]
        assert np.array_equal(oracle.unpack(p, c.shape[1], bits), c)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_roundtrip_and_size(bits):
    rng = np.random.default_rng(bits)
    for d in (1, 7, 8, 32, 33, 96, 130):
        c = rng.integers(0, 1 << bits, size=(5, d), dtype=np.uint8)
        p = oracle.pack(c, bits)
        assert p.shape == (5, -(-(d * bits) // 32))
        assert np.array_equal(oracle.unpack(p, d, bits), c)
        if (d * bits) % 32 == 0:
            assert p.nbytes == 5 * d * bits // 8


def test_memory_and_group_arithmetic_from_the_pages():
    """175e9 weights at 4 bits -> 87.5e9 bytes ("GPTQ" article, "Desempenho e
    Precisao"); a [1024, 4096] matrix with group size 128 has 32768 groups
    (AutoGPTQ guide, "Quantizacao group-wise", worked example)."""
    assert 175e9 * 4 / 8 == 87.5e9
    c = np.zeros((1, 4096), dtype=np.uint8)
    assert oracle.pack(c, 4).nbytes == 4096 // 2
    assert 1024 * oracle.n_groups(4096, 128) == 32768
    assert oracle.n_groups(4096, -1) == 1
    assert oracle.n_groups(130, 32) == 5


# ------------------------------------------------------------------ Hessian
def test_hessian_one_hot_rows_closed_form():
    """X made of unit rows e_k -> H = 2 diag(count_k)."""
    rng = np.random.default_rng(0)
    d = 16
    ks = rng.integers(0, d, size=200)
    X = np.zeros((200, d))
    X[np.arange(200), ks] = 1.0
    H = oracle.hessian(X, chunk=37)
    assert np.array_equal(H, 2.0 * np.diag(np.bincount(ks, minlength=d).astype(float)))


def test_hessian_brute_force_outer_products():
    rng = np.random.default_rng(1)
    n, d = 9, 5
    X = rng.standard_normal((n, d))
    H = oracle.hessian(X, chunk=4)
    ref = [[0.0] * d for _ in range(d)]
    for t in range(n):
        for a in range(d):
            for b in range(d):
                ref[a][b] += 2.0 * X[t, a] * X[t, b]
    assert np.allclose(H, np.array(ref), rtol=1e-13, atol=1e-13)
    assert np.array_equal(H, H.T)
    rows = oracle.hessian_rows(X, [4, 0, 2], chunk=4)
    assert np.allclose(rows, H[[4, 0, 2]], rtol=1e-13, atol=1e-13)


def test_hessian_of_bf16_inputs_is_exact_in_float64():
    """bf16 values are exact in float64, and so is every product of two of
    them; only the float64 sum rounds."""
    import torch
    x = workloads.student_t_activations(512, 24, seed=5)
    H = oracle.hessian(x)
    xf = x.to(torch.float64).numpy()
    ref = 2.0 * np.einsum("ta,tb->ab", xf, xf)
    assert np.allclose(H, ref, rtol=1e-13)


# ---------------------------------------------- inverse and its elimination
@pytest.mark.parametrize("d", [9, 33, 64])
def test_reduced_inverse_invariant(d):
    """After k elimination steps the trailing block equals inv(H[k:, k:])."""
    H = _spd(d, d, cond_spread=0.7)
    Minv = oracle.inverse(H)
    assert np.allclose(Minv @ H, np.eye(d), atol=1e-9)
    for k in (1, 2, d // 3, d - 1):
        M, _ = oracle.eliminate(Minv, steps=k)
        ref = np.linalg.inv(H[k:, k:])
        got = np.triu(M[k:, k:]) + np.triu(M[k:, k:], 1).T
        assert np.abs(got - ref).max() <= 1e-10 * np.abs(ref).max()


@pytest.mark.parametrize("d", [9, 40, 128])
def test_elimination_rows_are_the_upper_cholesky_factor_of_the_inverse(d):
    """U from the elimination rows: U^T U = H^-1, U = chol(H^-1)^T, and the
    flip route U = J inv(chol(J H J)) J (J the exchange matrix)."""
    H = _spd(d, 100 + d, cond_spread=0.5)
    _, U = oracle.eliminate(oracle.inverse(H))
    Hi = np.linalg.inv(H)
    scale = np.abs(Hi).max()
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.abs(U.T @ U - Hi).max() <= 1e-10 * scale
    assert np.abs(U - np.linalg.cholesky(Hi).T).max() <= 1e-10 * np.abs(U).max()
    J = np.eye(d)[::-1]
    flip = J @ np.linalg.inv(np.linalg.cholesky(J @ H @ J)) @ J
    assert np.abs(U - flip).max() <= 1e-10 * np.abs(U).max()
    # the oracle's two library routes to U
    assert np.abs(U - oracle.upper_factor(H)).max() <= 1e-10 * np.abs(U).max()
    assert np.abs(U - oracle.upper_factor_flip(H)).max() <= 1e-10 * np.abs(U).max()
    assert np.all(np.tril(oracle.upper_factor_flip(H), -1) == 0.0)


# ------------------------------------------------------------- the OBQ step
def _kkt_loop(W0, Hd, bits, g):
    """Independent restatement of the loop: at step i the remaining columns
    move by the minimiser of D H[i:, i:] D^T subject to D_i = q_i - w_i,
    found by a direct linear solve of the stationarity condition (no inverse,
    no elimination)."""
    W = W0.copy()
    r, d = W.shape
    codes = np.zeros((r, d), dtype=np.uint8)
    s = np.zeros(r)
    z = np.zeros(r, dtype=np.int64)
    for i in range(d):
        if i % g == 0:
            for row in range(r):
                s[row], _, z[row] = oracle.quant_params(W[row, i:i + g], bits)
        for row in range(r):
            codes[row, i] = oracle.quantize_code(W[row, i], s[row], int(z[row]), bits)
        if i + 1 < d:
            dq = s * (codes[:, i].astype(float) - z) - W[:, i]
            step = np.linalg.solve(Hd[i + 1:, i + 1:], Hd[i + 1:, i])
            W[:, i + 1:] -= np.outer(dq, step)
    return codes, W


@pytest.mark.parametrize("d,g", [(2, 2), (3, 3), (4, 2), (4, 4), (8, 4), (16, 8)])
def test_obq_step_matches_a_direct_kkt_solve(d, g):
    rng = np.random.default_rng(10 * d + g)
    H = _spd(d, 7 * d + g, cond_spread=0.8)
    W0 = rng.standard_normal((12, d)) * 0.05
    res = oracle.gptq_columns(W0, oracle.inverse(H), 3, g)
    codes, Wk = _kkt_loop(W0, H, 3, g)
    assert np.array_equal(res.codes, codes)
    assert np.abs(res.w_at_quant - Wk).max() <= 1e-12


def test_gptq_loss_is_not_below_the_exhaustive_optimum():
    """d = 4, 2 bits, one group: enumerate all 4^4 code vectors at the group's
    fixed scale / zero; GPTQ's loss is never below the optimum, and across
    many rows GPTQ's mean loss is below round-to-nearest's."""
    rng = np.random.default_rng(42)
    d, bits = 4, 2
    H = _spd(d, 77, n=6, cond_spread=0.3)
    W0 = rng.standard_normal((200, d))
    res = oracle.gptq_columns(W0, oracle.inverse(H), bits, d)
    rc, rs, rz = oracle.rtn(W0, bits, d)
    assert np.allclose(res.scales, rs) and np.array_equal(res.zeros, rz)
    allc = np.array(list(itertools.product(range(4), repeat=d)), dtype=float)
    tot_g = tot_r = 0.0
    for row in range(W0.shape[0]):
        s, z = res.scales[0, row], res.zeros[0, row]
        D = W0[row] - s * (allc - z)
        best = np.min(np.einsum("ka,ab,kb->k", D, H, D))
        Dg = W0[row] - s * (res.codes[row].astype(float) - z)
        Dr = W0[row] - s * (rc[row].astype(float) - z)
        lg, lr = Dg @ H @ Dg, Dr @ H @ Dr
        assert lg >= best - 1e-12
        tot_g += lg
        tot_r += lr
    assert tot_g < tot_r


# ------------------------------------------------------ lazy batch update
@pytest.mark.parametrize("B,g", [(1, 16), (2, 16), (4, 16), (8, 16), (128, 16),
                                 (8, 8), (16, 64), (32, 96), (128, 192), (7, 192)])
@pytest.mark.parametrize("pure", [False, True])
def test_lazy_block_update_equals_the_unbatched_loop(B, g, pure):
    """The pages' batched loop with its lazy update equals the one-column-at-
    a-time OBQ loop: same codes, same weights to 1e-10 (either group range)."""
    rng = np.random.default_rng(B * 1000 + g)
    d, r = 192, 24
    H = _spd(d, B + g, cond_spread=0.6)
    W0 = rng.standard_normal((r, d)) * 0.02 + (0.01 if pure else 0.0)
    res = oracle.gptq_columns(W0, oracle.inverse(H), 4, g, want_U=True, pure=pure)
    codes, scales, zeros, Wb = oracle.gptq_blocked(W0, res.U, 4, g, B, pure=pure)
    assert np.array_equal(codes, res.codes)
    assert np.array_equal(zeros, res.zeros)
    assert np.allclose(scales, res.scales, rtol=1e-12, atol=0)
    assert np.abs(Wb - res.w_at_quant).max() <= 1e-10 * np.abs(W0).max()


# --------------------------------------------------- special cases of GPTQ
@pytest.mark.parametrize("g", [8, 32, -1])
@pytest.mark.parametrize("pure", [False, True])
def test_identity_hessian_gives_round_to_nearest_exactly(g, pure):
    """H proportional to I: H^-1 has no off-diagonal terms, so there is no
    feedback and GPTQ equals round-to-nearest exactly (also after damping,
    since H + lambda I is still proportional to I), with either group range."""
    rng = np.random.default_rng(abs(g))
    d = 64
    W = rng.standard_normal((16, d)) * 0.03 + (0.02 if pure else 0.0)
    H = 3.7 * np.eye(d)
    out = oracle.quantize_layer(H, W, bits=4, group_size=g, damp=0.01, pure=pure)
    rc, rs, rz = oracle.rtn(out["W0"], 4, g, pure=pure)
    assert np.array_equal(out["codes"], rc)
    assert np.array_equal(out["scales"], rs)
    assert np.array_equal(out["zeros"], rz)
    assert out["loss"] == out["loss_rtn"]


def test_proxy_loss_closed_form():
    """tr((W - Q) H (W - Q)^T) with H = 2 X^T X equals 2 ||(W - Q) X^T||_F^2."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((50, 12))
    W = rng.standard_normal((7, 12))
    Q = W + 0.01 * rng.standard_normal((7, 12))
    H = oracle.hessian(X)
    assert oracle.proxy_loss(W, Q, H) == pytest.approx(2.0 * np.sum(((W - Q) @ X.T) ** 2), rel=1e-12)


def test_gptq_beats_round_to_nearest_on_the_tiny_layer():
    """GPTQ's proxy loss stays below round-to-nearest's on the tiny workload
    ("GPTQ" article, "Desempenho e Precisao": GPTQ consistently reduces the
    error of rounding to nearest).  Per-row violations are allowed (the
    method is greedy) but the layer aggregate must hold."""
    w = workloads.WORKLOADS["tiny"]
    W = workloads.weights(w)
    X = workloads.activations(w)
    H = oracle.hessian(X)
    out = oracle.quantize_layer(H, W, bits=w.bits, group_size=w.group_size, damp=w.damp)
    assert out["loss"] < out["loss_rtn"]
    assert out["loss_damped"] >= out["loss"]


def test_act_order_dead_columns_and_damping():
    H = np.diag([3.0, 0.0, 5.0, 3.0, 1.0])
    H[0, 2] = H[2, 0] = 0.5
    W = np.arange(10, dtype=float).reshape(2, 5) + 1.0
    assert list(oracle.dead_columns(H)) == [False, True, False, False, False]
    prep = oracle.prepare(H, W, damp=0.1, desc_act=True)
    # dead column 1 -> H_11 = 1; descending diag 5, 3, 3, 1, 1 with ties in index order
    assert list(prep["perm"]) == [2, 0, 3, 1, 4]
    assert np.all(prep["W0"][:, 3] == 0.0)           # dead column zeroed (now at position 3)
    assert prep["lam"] == pytest.approx(0.1 * (3 + 1 + 5 + 3 + 1) / 5)
    assert np.allclose(np.diag(prep["H_damped"]) - np.diag(prep["H_undamped"]), prep["lam"])
    assert prep["H_undamped"][0, 1] == 0.5           # H[2, 0] moved with the permutation
    ident = oracle.prepare(H, W, damp=0.1, desc_act=False)
    assert list(ident["perm"]) == [0, 1, 2, 3, 4]


def test_teacher_forcing_accepts_itself_and_flags_a_planted_error():
    """Forcing the loop with its own outputs reports no tie and no error; a
    code moved by one level away from a tie is reported invalid."""
    rng = np.random.default_rng(9)
    d = 48
    H = _spd(d, 3, cond_spread=0.5)
    W0 = rng.standard_normal((10, d)) * 0.02
    Minv = oracle.inverse(H)
    ref = oracle.gptq_columns(W0, Minv, 4, 16)
    same = oracle.gptq_columns(W0, Minv, 4, 16, forced_codes=ref.codes,
                               forced_zeros=ref.zeros, forced_w=ref.w_at_quant,
                               forced_scales=ref.scales)
    assert same.stats["code_ties"] == 0 and same.stats["code_invalid"] == 0
    assert same.stats["zero_invalid"] == 0 and same.stats["max_dev"] == 0.0
    assert same.stats["scale_invalid"] == 0
    assert same.stats["elements"] == 10 * d
    assert np.all(same.first_tie == d)
    bad = ref.codes.copy()
    rows, cols = np.nonzero((ref.codes > 0) & (ref.codes < 15))
    row, col = int(rows[0]), int(cols[0])
    q = int(bad[row, col])
    y = ref.w_at_quant[row, col] / ref.scales[col // 16, row] + ref.zeros[col // 16, row]
    bad[row, col] = q - 1 if y >= q else q + 1   # one level away from y's side
    planted = oracle.gptq_columns(W0, Minv, 4, 16, forced_codes=bad, forced_zeros=ref.zeros)
    assert planted.stats["code_invalid"] >= 1
    assert planted.first_tie[row] == col
    # a scale off by far more than the 1e-4 tolerance does not open the code
    # windows: the planted code stays invalid, and the scale itself is flagged
    wide = ref.scales * 1.5
    planted = oracle.gptq_columns(W0, Minv, 4, 16, forced_codes=bad, forced_zeros=ref.zeros,
                                  forced_w=ref.w_at_quant, forced_scales=wide)
    assert planted.stats["code_invalid"] >= 1
    assert planted.stats["scale_invalid"] == ref.scales.size


@pytest.mark.parametrize("loop", ["eliminated", "u_rows"])
def test_teacher_forcing_flags_a_planted_scale(loop):
    """A forced scale within the 1e-4 relative tolerance passes; one group's
    scale off by 1e-3 is flagged (by both loops)."""
    rng = np.random.default_rng(21)
    d = 64
    H = _spd(d, 4, cond_spread=0.5)
    W0 = rng.standard_normal((6, d)) * 0.02

    def run(**kw):
        if loop == "eliminated":
            return oracle.gptq_columns(W0, oracle.inverse(H), 4, 16, **kw)
        return oracle.gptq_columns_u(W0, oracle.upper_factor(H), 4, 16, **kw)

    ref = run()
    close = ref.scales * (1.0 + 1e-5)
    ok = run(forced_codes=ref.codes, forced_zeros=ref.zeros, forced_w=ref.w_at_quant,
             forced_scales=close)
    assert ok.stats["scale_invalid"] == 0 and ok.stats["code_invalid"] == 0
    off = ref.scales.copy()
    off[2, 3] *= 1.0 + 1e-3
    bad = run(forced_codes=ref.codes, forced_zeros=ref.zeros, forced_w=ref.w_at_quant,
              forced_scales=off)
    assert bad.stats["scale_invalid"] == 1


@pytest.mark.parametrize("loop", ["eliminated", "u_rows"])
def test_teacher_forcing_judges_a_planted_zero_point(loop):
    """Zero points: with H diagonal there is no feedback, so one row's group
    of values -a .. b gives s = (a + b) / 15 and the real zero point
    15 a / (a + b) exactly as built.  (1) A zero point one level away from a
    real zero point far from a rounding boundary is invalid.  (2) A real zero
    point 2e-4 levels past the boundary 7.5 rounds to 8; the forced 7 is
    invalid when the other side's weights show no drift, and a legitimate
    tie when they drift by 1e-3 levels (more than the 2e-4 miss)."""
    d = 16
    H = np.eye(d) * 3.0

    def run(W0, **kw):
        if loop == "eliminated":
            return oracle.gptq_columns(W0, oracle.inverse(H), 4, d, **kw)
        return oracle.gptq_columns_u(W0, oracle.upper_factor(H), 4, d, **kw)

    # (1) a = 0.2, b = 0.8: the real zero point 3.0 sits half a level from either boundary
    w = np.linspace(-0.2, 0.8, d)[None, :]
    ref = run(w)
    zr = 15 * 0.2 / 1.0
    assert ref.zeros[0, 0] == round(zr) == 3
    planted = run(w, forced_codes=ref.codes, forced_zeros=ref.zeros + 1, forced_w=w)
    assert planted.stats["zero_invalid"] == 1 and planted.stats["zero_ties"] == 0
    assert planted.first_tie[0] == 0
    # (2) a real zero point 2e-4 levels past 7.5
    eps = 2e-4 / 15.0
    a, b = 0.5 + eps, 0.5 - eps
    w = np.linspace(-a, b, d)[None, :]
    ref = run(w)
    assert ref.zeros[0, 0] == 8
    s = ref.scales[0, 0]
    forced = np.clip(np.rint(w / s) + 7, 0, 15).astype(np.uint8)
    no_drift = run(w, forced_codes=forced, forced_zeros=ref.zeros - 1, forced_w=w)
    assert no_drift.stats["zero_invalid"] == 1
    drift = w.copy()
    drift[0, 5] += 1e-3 * s
    tie = run(w, forced_codes=forced, forced_zeros=ref.zeros - 1, forced_w=drift)
    assert tie.stats["zero_invalid"] == 0 and tie.stats["zero_ties"] == 1


@pytest.mark.parametrize("d,g", [(64, 16), (200, 32), (256, -1)])
def test_u_row_loop_equals_the_eliminated_loop(d, g):
    """Driving the column loop by the rows of U (from a library Cholesky of
    the library inverse) gives the eliminated loop's codes, scales and
    weights, and the library U equals the elimination rows."""
    rng = np.random.default_rng(d)
    H = _spd(d, 5 * d, cond_spread=0.6)
    W0 = rng.standard_normal((9, d)) * 0.02
    res = oracle.gptq_columns(W0, oracle.inverse(H), 4, g, want_U=True)
    U = oracle.upper_factor(H)
    assert np.abs(U - res.U).max() <= 1e-10 * np.abs(U).max()
    ru = oracle.gptq_columns_u(W0, U, 4, g)
    assert np.array_equal(ru.codes, res.codes)
    assert np.array_equal(ru.zeros, res.zeros)
    assert np.allclose(ru.scales, res.scales, rtol=1e-12, atol=0)
    assert np.abs(ru.w_at_quant - res.w_at_quant).max() <= 1e-10 * np.abs(W0).max()
    forced = oracle.gptq_columns_u(W0, U, 4, g, forced_codes=res.codes, forced_zeros=res.zeros,
                                   forced_w=res.w_at_quant)
    assert forced.stats["code_invalid"] == 0 and forced.stats["code_ties"] == 0


def _golden_kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = (t.strip() for t in line.split("|", 1))
        out[k] = v.split()
    return out


def test_dequant_matmul_hand_example():
    """Product with a quantized layer: hand-computed example (golden file),
    act-order permutation and two groups included."""
    g = _golden_kv("dequant_matmul_worked_example.txt")
    bits, gs = int(g["bits"][0]), int(g["group"][0])
    perm = np.array([int(v) for v in g["perm"]])
    X = np.array([[float(v) for v in g["x"]]])
    packed = np.array([[int(w, 16)] for w in g["packed"]], dtype=np.uint32)
    sc = np.array([float(v) for v in g["scales"]]).reshape(2, 2)
    ze = np.array([int(v) for v in g["zeros"]], dtype=np.int32).reshape(2, 2)
    Y = oracle.dequant_matmul(X, packed, sc, ze, perm, bits, gs, len(perm))
    assert np.array_equal(Y, np.array([[float(v) for v in g["y"]]]))
    # the packed words are the pages' layout of these codes
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8], [15, 0, 15, 0, 3, 3, 3, 3]], dtype=np.uint8)
    assert np.array_equal(oracle.pack(codes, 4), packed)
    # without the permutation the same codes meet the activations unreversed
    Y_id = oracle.dequant_matmul(X, packed, sc, ze, None, bits, gs, len(perm))
    assert Y_id[0, 1] == 1 * 16 + 2 * -14 + 3 * 16 + 4 * -14


def test_bf16_rounding_agrees_with_an_independent_conversion():
    """The oracle's bf16 rounding against torch's float32 -> bfloat16 cast on
    the CPU (round to nearest, ties to even; an implementation the oracle does
    not share): random magnitudes over 60 binades of both signs, exact ties
    (the dropped half exactly 0x8000, even and odd kept parts) and values one
    ulp either side of them."""
    import torch
    rng = np.random.default_rng(42)
    x = (rng.standard_normal(100000) * 2.0 ** rng.integers(-30, 30, 100000)).astype(np.float32)
    u = rng.integers(0x00800000, 0x7F000000, 20000, dtype=np.uint64).astype(np.uint32)
    ties = (u & 0xFFFF0000) | 0x8000
    near = np.concatenate([ties, ties + 1, ties - 1]).astype(np.uint32).view(np.float32)
    x = np.concatenate([x, near, -near])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.bf16_round(x), ref)


def test_bf16_dequantized_weights_hand_example():
    """The many-token product's 16-bit weights ("GPTQ (GPT Quantization)",
    "Limitations": weights dequantized to 16 bits before the product):
    bf16 rounding to nearest, ties to even, worked by hand: 0.3 (float32
    0.300000012) has the bf16 neighbours 0.30078125 (1.203125 x 2^-2) and
    0.298828125 and rounds up; 1 + 2^-8 lies halfway between 1 and 1 + 2^-7
    and goes to the even mantissa, 1; 1 + 3 2^-8 lies halfway between
    1 + 2^-7 and 1 + 2^-6 and goes to 1 + 2^-6.  A one-row layer with scale
    1 + 2^-8, zero point 0 and codes 1, 1 then gives X W_hat^T = 1 + 2 = 3
    for X = [1, 2], against 3 + 3 2^-8 with the exact weights."""
    got = oracle.bf16_round(np.array([0.3, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)],
                                     dtype=np.float32))
    assert list(got) == [0.30078125, 1.0, 1.015625, -1.0]
    codes = np.array([[1, 1, 0, 0, 0, 0, 0, 0]], dtype=np.uint8)
    packed = oracle.pack(codes, 4)
    X = np.array([[1.0, 2.0, 0, 0, 0, 0, 0, 0]])
    sc = np.array([[1 + 2.0 ** -8]], dtype=np.float32)
    ze = np.zeros((1, 1), dtype=np.int32)
    assert oracle.dequant_matmul(X, packed, sc, ze, None, 4, 8, 8, weights_bf16=True)[0, 0] == 3.0
    assert oracle.dequant_matmul(X, packed, sc, ze, None, 4, 8, 8)[0, 0] == 3 + 3 * 2.0 ** -8


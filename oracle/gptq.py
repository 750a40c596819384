"""Float64 reference of the GPTQ layer quantizer -- TEST INFRASTRUCTURE ONLY.

See the package docstring for who may import this module.  Citations name the
page and the section of the GPTQ pages each step restates:

* [OBQ]    "GPTQ (GPT Quantization)", "Fondation theorique : OBQ (Optimal Brain
           Quantization)" -- quantize column i, e = w_i - q_i,
           W_F <- W_F - e / (H^-1)_ii * (H^-1)_{i,F}; H = 2 X^T X.
* [ALGO]   "GPTQ (GPT Quantization)", "Algorithme complet (pseudo-code)" --
           H = 2 X^T X; H += lambda I; H^-1 through Cholesky; batches of
           columns with a lazy update of the remaining ones.
* [GROUP]  "Optimization Gptq" (AutoGPTQ guide), "Quantizacao group-wise" and
           "Trade-off de tamanho de grupo" -- own scale and zero point per group
           of consecutive weights; group size -1 means one group per row here.
* [CONFIG] "Optimization Gptq", "Quantizar seu proprio modelo" --
           BaseQuantizeConfig(bits, group_size, desc_act, damp_percent=0.01).
* [ORDER]  "GPTQ (GPT Quantization)", "Quantification avec AutoGPTQ" --
           desc_act=True quantizes in order of importance.
* [MEM]    "GPTQ" (encyclopedic article), "Desempenho e Precisao" -- 175B
           parameters at 4 bits take about 87.5 GB (0.5 byte per weight).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gptq_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "liboracle.so")
_lib_handle = None


def build_native(force: bool = False) -> str:
    """Compile the C part of the oracle (gcc, -O2, OpenMP, strict IEEE)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        os.makedirs(_BUILD, exist_ok=True)
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build_native())
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.orc_quant_params.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P, P]
        lib.orc_quant_params.restype = None
        lib.orc_quantize.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_int32, ctypes.c_int]
        lib.orc_quantize.restype = ctypes.c_int32
        lib.orc_gptq_columns.argtypes = [P, i64, i64, P, ctypes.c_int, i64, ctypes.c_int, P, P,
                                         P, P, P, P, P, P, ctypes.c_double, ctypes.c_double, P, P,
                                         P]
        lib.orc_gptq_columns.restype = ctypes.c_int
        lib.orc_gptq_columns_u.argtypes = [P, i64, i64, P, ctypes.c_int, i64, ctypes.c_int, P, P,
                                           P, P, P, P, P, ctypes.c_double, ctypes.c_double, P, P,
                                           P]
        lib.orc_gptq_columns_u.restype = ctypes.c_int
        lib.orc_eliminate.argtypes = [P, i64, i64, P]
        lib.orc_eliminate.restype = ctypes.c_int
        lib.orc_gptq_blocked.argtypes = [P, i64, i64, P, ctypes.c_int, i64, ctypes.c_int, i64, P,
                                         P, P]
        lib.orc_gptq_blocked.restype = ctypes.c_int
        lib.orc_rtn.argtypes = [P, i64, i64, ctypes.c_int, i64, ctypes.c_int, P, P, P]
        lib.orc_rtn.restype = None
        _lib_handle = lib
    return _lib_handle


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    """Any array-like (numpy, torch CPU incl. bfloat16) as contiguous float64."""
    if hasattr(a, "detach"):  # a torch tensor; bf16 -> f32 is exact
        import torch
        a = a.detach().to("cpu")
        if a.dtype == torch.bfloat16:
            a = a.to(torch.float32)
        a = a.numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def n_groups(d_col: int, group_size: int) -> int:
    """Number of groups per row: ceil(d_col / g), g = -1 meaning one group
    per row [GROUP]."""
    g = d_col if group_size == -1 else group_size
    return -(-d_col // g)


def _g(d_col: int, group_size: int) -> int:
    return d_col if group_size == -1 else int(group_size)


# --------------------------------------------------------------------------
# Stage 1: Hessian  [ALGO] step 1, [OBQ] "H = 2 X^T X"
# --------------------------------------------------------------------------
def hessian(X, chunk: int = 8192) -> np.ndarray:
    """H = 2 X^T X in float64 over all n tokens of X (n x d).

    X's values are taken exactly as given (bf16 inputs are exact in float64);
    the product is accumulated in float64 chunk by chunk of tokens."""
    n, d = X.shape
    H = np.zeros((d, d), dtype=np.float64)
    for t0 in range(0, n, chunk):
        xc = _f64(X[t0:t0 + chunk])
        H += xc.T @ xc
    return 2.0 * H


def hessian_rows(X, idx, chunk: int = 8192) -> np.ndarray:
    """Rows idx of H = 2 X^T X: H[idx, :] = 2 X[:, idx]^T X (float64)."""
    idx = np.asarray(idx)
    n, d = X.shape
    out = np.zeros((len(idx), d), dtype=np.float64)
    for t0 in range(0, n, chunk):
        xc = _f64(X[t0:t0 + chunk])
        out += xc[:, idx].T @ xc
    return 2.0 * out


# --------------------------------------------------------------------------
# Stage 2: dead columns, act-order, damping  [ALGO] "H += lambda * I",
# [CONFIG] damp_percent, [ORDER] desc_act
# --------------------------------------------------------------------------
def dead_columns(H) -> np.ndarray:
    """Columns whose Hessian diagonal is exactly zero (an input channel that is
    zero on every calibration token).  Reading: the pages are silent; such a
    column gets H_ii := 1 and its weights are set to 0."""
    return np.diag(np.asarray(H)) == 0.0


def act_order(H) -> np.ndarray:
    """desc_act permutation: perm[k] = original column quantized k-th, by
    descending diag(H) [ORDER]; ties keep the lower original index first
    (a stable sort -- the pages give no tie rule)."""
    return np.argsort(-np.diag(np.asarray(H, dtype=np.float64)), kind="stable")


def damp_lambda(H, damp: float) -> float:
    """lambda = damp * mean(diag H) [ALGO] "H += lambda * I" with the
    relative damp_percent of [CONFIG]."""
    return float(damp) * float(np.mean(np.diag(np.asarray(H, dtype=np.float64))))


def prepare(H, W, damp: float = 0.01, desc_act: bool = False) -> dict:
    """Dead-column fix -> act-order permutation -> damping.

    Returns the undamped and damped Hessians and the weights in quantization
    order, the permutation and the dead mask.  lambda is permutation
    invariant, so applying it after the permutation changes nothing."""
    Hf = np.array(H, dtype=np.float64, copy=True)
    Wf = _f64(W).copy()
    dead = dead_columns(Hf)
    idx = np.nonzero(dead)[0]
    Hf[idx, idx] = 1.0
    Wf[:, idx] = 0.0
    d = Hf.shape[0]
    perm = act_order(Hf) if desc_act else np.arange(d)
    Hu = Hf[np.ix_(perm, perm)]
    W0 = np.ascontiguousarray(Wf[:, perm])
    lam = damp_lambda(Hu, damp)
    Hd = Hu.copy()
    Hd[np.diag_indices(d)] += lam
    return dict(H_undamped=Hu, H_damped=Hd, W0=W0, perm=perm.astype(np.int64),
                dead=dead, lam=lam)


# --------------------------------------------------------------------------
# Stage 3: the inverse and its per-column elimination  [ALGO] step 2, [OBQ]
# --------------------------------------------------------------------------
def inverse(Hd) -> np.ndarray:
    """H^-1 of the damped Hessian (a library inverse, float64)."""
    return np.linalg.inv(np.asarray(Hd, dtype=np.float64))


def eliminate(Minv, steps: int | None = None):
    """Per-column Gaussian elimination of M = H^-1 [OBQ].

    Returns (M_after, U): after k steps M_after[k:, k:] equals inv(H[k:, k:])
    (upper triangle stored); U's row i is the eliminated row i divided by
    sqrt(M_ii), so U^T U = H^-1 with U upper (rows >= steps are zero)."""
    M = np.array(Minv, dtype=np.float64, copy=True, order="C")
    d = M.shape[0]
    k = d if steps is None else int(steps)
    U = np.zeros((d, d), dtype=np.float64)
    rc = _lib().orc_eliminate(_ptr(M), d, k, _ptr(U))
    if rc != 0:
        raise np.linalg.LinAlgError("non-positive pivot in the elimination")
    return M, U


# --------------------------------------------------------------------------
# The quantizer  [GROUP]
# --------------------------------------------------------------------------
def quant_params(x, bits: int, pure: bool = False):
    """(scale, zero_real, zero) of one group: asymmetric min-max over the
    group's current weights [GROUP].  Default: 0 always inside the range (so
    the integer zero point lies in [0, 2^b - 1]) and an all-zero group widened
    to [-1, 1].  pure: the group's own [min, max] (the zero point may fall
    outside [0, 2^b - 1]); a constant group, or one whose real zero point lies
    more than 2^20 levels away, falls back to the widened range.
    zero = rint(-xmin / scale), round half to even."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    s = ctypes.c_double()
    zr = ctypes.c_double()
    z = ctypes.c_int32()
    _lib().orc_quant_params(_ptr(x), x.size, bits, int(bool(pure)), ctypes.byref(s),
                            ctypes.byref(zr), ctypes.byref(z))
    return s.value, zr.value, z.value


def quantize_code(w: float, s: float, z: int, bits: int) -> int:
    """clamp(rint(w / s) + z, 0, 2^b - 1)."""
    return int(_lib().orc_quantize(float(w), float(s), int(z), int(bits)))


def dequantize(codes, scales, zeros, group_size: int) -> np.ndarray:
    """W_hat[row, k] = scale[k // g, row] * (code[row, k] - zero[k // g, row])."""
    codes = np.asarray(codes)
    r, d = codes.shape
    g = _g(d, group_size)
    gi = np.arange(d) // g
    s = np.asarray(scales, dtype=np.float64)[gi, :].T
    z = np.asarray(zeros, dtype=np.float64)[gi, :].T
    return s * (codes.astype(np.float64) - z)


def rtn(W0, bits: int, group_size: int, pure: bool = False):
    """Round-to-nearest: the same group quantizer applied to W0 with no error
    feedback (the baseline GPTQ is compared with, "GPTQ" article,
    "Desempenho e Precisao")."""
    W0 = _f64(W0)
    r, d = W0.shape
    g = _g(d, group_size)
    ng = n_groups(d, group_size)
    codes = np.zeros((r, d), dtype=np.uint8)
    scales = np.zeros((ng, r), dtype=np.float64)
    zeros = np.zeros((ng, r), dtype=np.int32)
    _lib().orc_rtn(_ptr(W0), r, d, bits, g, int(bool(pure)), _ptr(codes), _ptr(scales),
                   _ptr(zeros))
    return codes, scales, zeros


def proxy_loss(W0, Q, H) -> float:
    """tr((W0 - Q) H (W0 - Q)^T): with H = 2 X^T X this is
    2 * ||(W0 - Q) X^T||_F^2, the layer-output error GPTQ minimises."""
    D = _f64(W0) - _f64(Q)
    return float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))


# --------------------------------------------------------------------------
# Stage 4: the column loop  [OBQ], [ALGO] step 3
# --------------------------------------------------------------------------
@dataclass
class GPTQResult:
    codes: np.ndarray          # r x d uint8, quantization order
    scales: np.ndarray         # [n_groups][r] float64
    zeros: np.ndarray          # [n_groups][r] int32
    w_at_quant: np.ndarray     # r x d: column i as it was when quantized
    U: np.ndarray | None       # eliminated rows / sqrt(pivot), if requested
    stats: dict                # teacher-forcing statistics (zeros if not forced)
    first_tie: np.ndarray | None = None  # per row: first forced decision that differs (d: none)


# Relative scale deviation the teacher-forced check accepts: the tolerance the
# method's statement of parity gives for scales (1e-4 relative).
SCALE_TOL = 1e-4


def _stats(stats, max_dev) -> dict:
    return dict(code_ties=int(stats[0]), code_invalid=int(stats[1]),
                zero_ties=int(stats[2]), zero_invalid=int(stats[3]),
                elements=int(stats[4]), groups=int(stats[5]), scale_invalid=int(stats[6]),
                max_dev=max_dev.value)


def gptq_columns(W0, Hinv, bits: int, group_size: int, want_U: bool = False,
                 forced_codes=None, forced_zeros=None, forced_w=None, forced_scales=None,
                 tau: float = 0.0, stol: float = SCALE_TOL, pure: bool = False) -> GPTQResult:
    """The OBQ/GPTQ loop one column at a time with explicit elimination of
    H^-1 after every column [OBQ].

    With forced_* given (another implementation's codes, zero points and
    pre-quantization weights), each of them is checked for validity and then
    adopted, so one tie decided the other way does not desynchronise the rest
    of its row: a code is valid when it is the oracle's own rounding or a
    neighbouring level whose rounding boundary lies within
    tau + |forced_w - w| / s + |y - z| min(|forced_s - s| / s, stol) of the
    oracle's real level y = w / s + z (the other side's own deviation in the
    decision's inputs).  A forced scale further than stol (relative) from the
    oracle's counts as invalid; a zero point that differs from the oracle's
    rounding is valid when the oracle's real zero point lies within the
    group's drift of the rounding boundary.  first_tie[row] is the first
    column where a forced decision differs: before it the forced run IS the
    free-running loop."""
    W = _f64(W0).copy()
    r, d = W.shape
    g = _g(d, group_size)
    ng = n_groups(d, group_size)
    M = np.array(Hinv, dtype=np.float64, copy=True, order="C")
    codes = np.zeros((r, d), dtype=np.uint8)
    scales = np.zeros((ng, r), dtype=np.float64)
    zeros = np.zeros((ng, r), dtype=np.int32)
    U = np.zeros((d, d), dtype=np.float64) if want_U else None
    fc = None if forced_codes is None else np.ascontiguousarray(forced_codes, dtype=np.uint8)
    fz = None if forced_zeros is None else np.ascontiguousarray(forced_zeros, dtype=np.int32)
    fw = None if forced_w is None else _f64(forced_w)
    fs = None if forced_scales is None else _f64(forced_scales)
    stats = np.zeros(7, dtype=np.int64)
    first = np.zeros(r, dtype=np.int64)
    max_dev = ctypes.c_double(0.0)
    rc = _lib().orc_gptq_columns(_ptr(W), r, d, _ptr(M), bits, g, int(bool(pure)), _ptr(codes),
                                 _ptr(scales),
                                 _ptr(zeros), _ptr(U), _ptr(fc), _ptr(fz), _ptr(fw), _ptr(fs),
                                 float(tau), float(stol), _ptr(stats), ctypes.byref(max_dev),
                                 _ptr(first))
    if rc != 0:
        raise np.linalg.LinAlgError(f"oracle column loop failed ({rc})")
    return GPTQResult(codes, scales, zeros, W, U, _stats(stats, max_dev), first)


def upper_factor(Hd) -> np.ndarray:
    """U upper with U^T U = inverse(Hd), from library routines (a Cholesky of
    the library inverse).  The elimination rows of `eliminate` are this same
    matrix; the pins check the two against each other.  Used where the
    explicit elimination is too slow (d > 4096)."""
    return np.ascontiguousarray(np.linalg.cholesky(inverse(Hd)).T)


def upper_factor_flip(Hd) -> np.ndarray:
    """The same U through library routines that need one factorization:
    with J the exchange matrix and J Hd J = L L^T, U = J L^-1 J (a library
    Cholesky and a library triangular inverse, float64, working in one
    Fortran-ordered copy).  Pinned equal to upper_factor and to the
    elimination rows; used for the largest d, where an explicit inverse
    costs three times as much."""
    from scipy.linalg import lapack
    F = np.array(np.asarray(Hd, dtype=np.float64)[::-1, ::-1], order="F")  # J Hd J
    c, info = lapack.dpotrf(F, lower=1, clean=1, overwrite_a=1)
    if info != 0:
        raise np.linalg.LinAlgError(f"Cholesky failed ({info})")
    c, info = lapack.dtrtri(c, lower=1, overwrite_c=1)
    if info != 0:
        raise np.linalg.LinAlgError(f"triangular inverse failed ({info})")
    return np.ascontiguousarray(c[::-1, ::-1])  # J L^-1 J, upper triangular


def gptq_columns_u(W0, U, bits: int, group_size: int, forced_codes=None, forced_zeros=None,
                   forced_w=None, forced_scales=None, tau: float = 0.0,
                   stol: float = SCALE_TOL, pure: bool = False) -> GPTQResult:
    """The OBQ column loop driven by U's rows: W_F <- W_F - (e / U_ii) U_{i,F}
    [OBQ] with row i of the reduced inverse equal to U_ii U[i, i:].  Same
    teacher-forcing options as gptq_columns."""
    W = _f64(W0).copy()
    r, d = W.shape
    g = _g(d, group_size)
    ng = n_groups(d, group_size)
    Uc = np.ascontiguousarray(U, dtype=np.float64)
    codes = np.zeros((r, d), dtype=np.uint8)
    scales = np.zeros((ng, r), dtype=np.float64)
    zeros = np.zeros((ng, r), dtype=np.int32)
    fc = None if forced_codes is None else np.ascontiguousarray(forced_codes, dtype=np.uint8)
    fz = None if forced_zeros is None else np.ascontiguousarray(forced_zeros, dtype=np.int32)
    fw = None if forced_w is None else _f64(forced_w)
    fs = None if forced_scales is None else _f64(forced_scales)
    stats = np.zeros(7, dtype=np.int64)
    first = np.zeros(r, dtype=np.int64)
    max_dev = ctypes.c_double(0.0)
    rc = _lib().orc_gptq_columns_u(_ptr(W), r, d, _ptr(Uc), bits, g, int(bool(pure)), _ptr(codes),
                                   _ptr(scales),
                                   _ptr(zeros), _ptr(fc), _ptr(fz), _ptr(fw), _ptr(fs),
                                   float(tau), float(stol), _ptr(stats), ctypes.byref(max_dev),
                                   _ptr(first))
    if rc != 0:
        raise np.linalg.LinAlgError(f"oracle U-row loop failed ({rc})")
    return GPTQResult(codes, scales, zeros, W, None, _stats(stats, max_dev), first)


def gptq_blocked(W0, U, bits: int, group_size: int, block: int, pure: bool = False):
    """The pages' batched loop [ALGO] with B = block: in-batch OBQ feedback,
    then one lazy product W[:, i1:] -= Err U[i0:i1, i1:] per batch.  Reading
    of the garbled lazy-update line: Err_j = (w_j - q_j) / U_jj is divided
    per column before the product."""
    W = _f64(W0).copy()
    r, d = W.shape
    g = _g(d, group_size)
    ng = n_groups(d, group_size)
    Uc = np.ascontiguousarray(U, dtype=np.float64)
    codes = np.zeros((r, d), dtype=np.uint8)
    scales = np.zeros((ng, r), dtype=np.float64)
    zeros = np.zeros((ng, r), dtype=np.int32)
    rc = _lib().orc_gptq_blocked(_ptr(W), r, d, _ptr(Uc), bits, g, int(bool(pure)), int(block),
                                 _ptr(codes),
                                 _ptr(scales), _ptr(zeros))
    if rc != 0:
        raise MemoryError("oracle blocked loop failed")
    return codes, scales, zeros, W


# --------------------------------------------------------------------------
# Stage 5: packing  [MEM]: 4-bit codes, 8 per uint32
# --------------------------------------------------------------------------
def pack(codes, bits: int) -> np.ndarray:
    """Each row's codes as a little-endian bit stream: code k occupies bits
    [b*k, b*k + b) of the row's uint32 words (LSB first).  For b = 4 this is
    8 codes per word, code 8m + t in bits 4t..4t+3 of word m."""
    c = np.asarray(codes, dtype=np.uint8)
    r, d = c.shape
    words = -(-(d * bits) // 32)
    bitplanes = ((c[:, :, None] >> np.arange(bits, dtype=np.uint8)) & 1).reshape(r, d * bits)
    padded = np.zeros((r, words * 32), dtype=np.uint8)
    padded[:, :d * bits] = bitplanes
    by = np.packbits(padded, axis=1, bitorder="little")
    return by.view("<u4").reshape(r, words).astype(np.uint32)


def unpack(packed, d: int, bits: int) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype="<u4")
    r = p.shape[0]
    bitstream = np.unpackbits(p.view(np.uint8), axis=1, bitorder="little")[:, :d * bits]
    planes = bitstream.reshape(r, d, bits).astype(np.uint8)
    return (planes << np.arange(bits, dtype=np.uint8)).sum(axis=2).astype(np.uint8)


# --------------------------------------------------------------------------
# Using the quantized layer  "GPTQ (GPT Quantization)", "Limitations" (items
# 1-2): weight-only quantization, the activations stay at 16 bits and the
# integer weights are dequantized before each product
# --------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), returned
    as float64: the 16 high bits of the float32 pattern after adding
    0x7FFF plus the lowest kept bit (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32).astype(np.float64)


def dequant_matmul(X, packed, scales, zeros, perm, bits: int, group_size: int,
                   d_col: int, weights_bf16: bool = False) -> np.ndarray:
    """Y = X W_hat^T for a layer quantized by this library: X is tokens x d_col
    in the layer's original column order, the packed codes are in quantization
    order, and W_hat[:, perm[k]] = scale[k // g] * (code[:, k] - zero[k // g]).
    perm None is the identity.  float64 throughout, except with weights_bf16:
    each weight is then the 16-bit value the "Limitations" passage speaks of,
    bf16_round(float32(scale) * float32(code - zero)) (one float32 product,
    rounded to the nearest bf16)."""
    Xf = _f64(X)
    Xq = Xf if perm is None else Xf[:, np.asarray(perm)]
    if weights_bf16:
        codes = unpack(packed, d_col, bits)
        r, d = codes.shape
        g = _g(d, group_size)
        gi = np.arange(d) // g
        s = np.asarray(scales, dtype=np.float32)[gi, :].T
        z = np.asarray(zeros, dtype=np.float32)[gi, :].T
        Q = bf16_round(s * (codes.astype(np.float32) - z))
    else:
        Q = dequantize(unpack(packed, d_col, bits), scales, zeros, group_size)
    return Xq @ Q.T


# --------------------------------------------------------------------------
# The whole layer
# --------------------------------------------------------------------------
def quantize_layer(H, W, bits: int = 4, group_size: int = 128, desc_act: bool = False,
                   damp: float = 0.01, want_U: bool = False, rows=None,
                   forced_codes=None, forced_zeros=None, forced_w=None, forced_scales=None,
                   tau: float = 0.0, pure: bool = False) -> dict:
    """H (d x d, original column order) and W (r x d) -> GPTQ result.

    Steps [ALGO]: dead-column fix, act-order permutation, damping, H^-1, then
    the unbatched OBQ column loop with explicit elimination.  `rows` limits
    the column loop to a sample of rows (rows are independent given H^-1).
    Codes, scales and zeros are in quantization (permuted) order."""
    prep = prepare(H, W, damp=damp, desc_act=desc_act)
    W0 = prep["W0"] if rows is None else prep["W0"][np.asarray(rows)]
    Minv = inverse(prep["H_damped"])
    res = gptq_columns(W0, Minv, bits, group_size, want_U=want_U,
                       forced_codes=forced_codes, forced_zeros=forced_zeros,
                       forced_w=forced_w, forced_scales=forced_scales, tau=tau, pure=pure)
    Q = dequantize(res.codes, res.scales, res.zeros, group_size)
    rc, rs, rz = rtn(W0, bits, group_size, pure=pure)
    Qr = dequantize(rc, rs, rz, group_size)
    return dict(codes=res.codes, scales=res.scales, zeros=res.zeros, perm=prep["perm"],
                dead=prep["dead"], lam=prep["lam"], W0=W0, Q=Q, w_at_quant=res.w_at_quant,
                U=res.U, stats=res.stats,
                loss=proxy_loss(W0, Q, prep["H_undamped"]),
                loss_damped=proxy_loss(W0, Q, prep["H_damped"]),
                loss_rtn=proxy_loss(W0, Qr, prep["H_undamped"]),
                H_undamped=prep["H_undamped"], H_damped=prep["H_damped"])

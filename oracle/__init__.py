"""Float64 CPU oracle for GPTQ layer-wise INT-b weight quantization.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  It shares
no code with the CUDA path and never imports it.

Every function is a thin numpy wrapper over ``gptq_oracle.c`` (plain C,
float64, no blocking) and cites the passage it follows:

* ``hessian``      -- H accumulation, "GPTQ / AWQ / SqueezeLLM" sec. 一
                      (H = 2 X^T X / n; here the raw sum S = X^T X);
                      ``hessian_syrk`` the same sum through BLAS for full-size X.
* ``finalize``     -- H = 2S/n, relative damping, act-order permutation
                      (same page, sec. 一: damping, importance order).
* ``cholesky_lower``/``trtri_lower``/``hinv_upper_chol`` -- the "decomposition"
                      of H^-1 (same page, sec. 一; "INT4/INT8 量化推理" sec. 三);
                      ``u_rows`` selected rows of it from their definition.
* ``quantize_rows`` -- the column sweep with error feedback ("INT4/INT8 量化推理"
                      sec. 三 loop; "校准艺术" sec. 2.2 steps 1-5).
* ``rtn``          -- round-to-nearest group min-max ("校准艺术" sec. 2.1).
* ``pack_int4``/``unpack_int4`` -- the 66.5 B / 128-weight storage format
                      ("INT4/INT8 量化推理" sec. 一); ``pack_bits``/``unpack_bits``
                      the same layout as one bit stream per row for 2..8 bits.
* ``trace_quadratic`` -- tr(D H D^T), the layer loss of sec. 三 of that page.
* ``w4a16_matmul`` -- y = x Q^T from the packed layer (weight-only INT4 with
                      fp16 activations, "INT4/INT8 量化推理" sec. 六).
* ``channel_magnitude``/``awq_search``/``awq_then_gptq`` -- activation-aware
                      channel scaling ahead of the sweep ("GPTQ / AWQ /
                      SqueezeLLM" sec. 二; "INT4/INT8 量化推理" sec. 四).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        lib.orc_half_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_half_to_double.restype = ctypes.c_double
        lib.orc_float_to_half_rne.argtypes = [ctypes.c_float]
        lib.orc_float_to_half_rne.restype = ctypes.c_uint16
        lib.orc_hessian_accumulate.argtypes = [P, I64, I64, P]
        lib.orc_hessian_accumulate.restype = None
        lib.orc_finalize.argtypes = [P, I64, I64, ctypes.c_double, ctypes.c_int, P, P, P, P]
        lib.orc_finalize.restype = ctypes.c_int
        lib.orc_act_order_perm.argtypes = [P, I64, P]
        lib.orc_act_order_perm.restype = None
        lib.orc_cholesky_lower.argtypes = [P, I64, P]
        lib.orc_cholesky_lower.restype = ctypes.c_int
        lib.orc_trtri_lower_T.argtypes = [P, I64, P]
        lib.orc_trtri_lower_T.restype = None
        lib.orc_hinv_upper_chol.argtypes = [P, I64, P]
        lib.orc_hinv_upper_chol.restype = ctypes.c_int
        lib.orc_quantize_rows.argtypes = [P, P, I64, I64, ctypes.c_int, I64,
                                          P, P, P, P, P, P, P, P, P, P, P, P, P, P]
        lib.orc_quantize_rows.restype = None
        lib.orc_rtn.argtypes = [P, I64, I64, ctypes.c_int, I64, P, P, P, P]
        lib.orc_rtn.restype = None
        lib.orc_pack_int4.argtypes = [P, P, I64, I64, I64, P, P]
        lib.orc_pack_int4.restype = None
        lib.orc_unpack_int4.argtypes = [P, P, I64, I64, I64, P, P]
        lib.orc_unpack_int4.restype = None
        lib.orc_pack_bits.argtypes = [P, P, I64, I64, I64, ctypes.c_int, P, P]
        lib.orc_pack_bits.restype = None
        lib.orc_unpack_bits.argtypes = [P, P, I64, I64, I64, ctypes.c_int, P, P]
        lib.orc_unpack_bits.restype = None
        lib.orc_trace_quadratic.argtypes = [P, P, I64, I64]
        lib.orc_trace_quadratic.restype = ctypes.c_double
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# --------------------------------------------------------------------------
# fp16 helpers (IEEE binary16 from the format definition)
# --------------------------------------------------------------------------

def half_bits_to_float64(h: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.ascontiguousarray(h, dtype=np.uint16).ravel()
    out = np.fromiter((lib.orc_half_to_double(int(v)) for v in flat), dtype=np.float64,
                      count=flat.size)
    return out.reshape(np.shape(h))


def float32_to_half_bits(x: float) -> int:
    return int(_load().orc_float_to_half_rne(ctypes.c_float(x)))


def _as_half_bits(X) -> np.ndarray:
    X = np.asarray(X)
    if X.dtype == np.float16:
        return np.ascontiguousarray(X).view(np.uint16)
    if X.dtype == np.uint16:
        return np.ascontiguousarray(X)
    raise TypeError("X must be float16 (or its uint16 bit pattern)")


# --------------------------------------------------------------------------
# Hessian and its preparation
# --------------------------------------------------------------------------

def hessian(X, S: np.ndarray | None = None) -> np.ndarray:
    """S += X^T X for X (n x d) fp16, in float64 (fp16 values promoted exactly)."""
    Xb = _as_half_bits(X)
    n, d = Xb.shape
    if S is None:
        S = np.zeros((d, d), dtype=np.float64)
    assert S.dtype == np.float64 and S.shape == (d, d) and S.flags["C_CONTIGUOUS"]
    _load().orc_hessian_accumulate(_p(Xb), n, d, _p(S))
    return S



def hessian_syrk(X, chunk: int = 16384) -> np.ndarray:
    """S = X^T X for X (n x d) fp16 in float64 through the BLAS rank-k update
    (dsyrk) over token chunks: the same sum as ``hessian`` (every fp16 value is
    exact in float64; only the float64 summation order differs), for inputs
    where the plain loop takes minutes.  X may be a numpy array or a CPU torch
    tensor of float16.  Returns the full symmetric matrix."""
    from scipy.linalg import blas
    if hasattr(X, "numpy"):
        X = X.numpy()
    X = np.asarray(X)
    assert X.dtype == np.float16
    n, d = X.shape
    S = np.zeros((d, d), dtype=np.float64, order="F")
    for t0 in range(0, n, chunk):
        Xc = np.asfortranarray(X[t0:t0 + chunk].astype(np.float64))
        S = blas.dsyrk(1.0, Xc, beta=1.0, c=S, trans=1, lower=0, overwrite_c=1)
    S = np.ascontiguousarray(S)
    return np.triu(S) + np.triu(S, 1).T

def finalize(S: np.ndarray, n: int, damp_rel: float = 0.01, act_order: bool = False):
    """H = 2S/n; perm (stable descending argsort of diag H when act_order);
    H <- H[perm][:, perm]; lambda = damp_rel * mean(diag H); Hd = H + lambda I.

    Returns (H, Hd, perm, lam, status) with status 0, or 3 when mean(diag H) <= 0.
    """
    S = np.ascontiguousarray(S, dtype=np.float64)
    d = S.shape[0]
    H = np.empty_like(S)
    Hd = np.empty_like(S)
    perm = np.empty(d, dtype=np.int32)
    lam = ctypes.c_double(0.0)
    st = _load().orc_finalize(_p(S), int(n), d, float(damp_rel), int(bool(act_order)),
                              _p(H), _p(Hd), _p(perm), ctypes.byref(lam))
    return H, Hd, perm, float(lam.value), int(st)


def act_order_perm(diag: np.ndarray) -> np.ndarray:
    """Stable descending argsort of diag(H) (ties: lower index first)."""
    diag = np.ascontiguousarray(diag, dtype=np.float64)
    perm = np.empty(diag.shape[0], dtype=np.int32)
    _load().orc_act_order_perm(_p(diag), diag.shape[0], _p(perm))
    return perm


def cholesky_lower(A: np.ndarray):
    """Lower Cholesky factor; returns (L, info) with info = 1-based failing pivot or 0."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    L = np.empty_like(A)
    info = _load().orc_cholesky_lower(_p(A), A.shape[0], _p(L))
    return L, int(info)


def trtri_lower(L: np.ndarray) -> np.ndarray:
    """Inverse of a lower-triangular matrix (returned in normal orientation)."""
    L = np.ascontiguousarray(L, dtype=np.float64)
    LinvT = np.empty_like(L)
    _load().orc_trtri_lower_T(_p(L), L.shape[0], _p(LinvT))
    return np.ascontiguousarray(LinvT.T)


def hinv_upper_chol(Hd: np.ndarray):
    """U upper with U^T U = Hd^-1 (plain route: chol, triangular inverse,
    form the inverse, chol again, transpose).  Returns (U, info)."""
    Hd = np.ascontiguousarray(Hd, dtype=np.float64)
    U = np.empty_like(Hd)
    info = _load().orc_hinv_upper_chol(_p(Hd), Hd.shape[0], _p(U))
    return U, int(info)



def u_rows(Hd: np.ndarray, rows) -> np.ndarray:
    """Selected rows of U (upper, U^T U = Hd^-1) from their definition: row j
    of U is the first row of the inverse of the trailing sub-Hessian
    Hd[j:, j:] (the Hessian of the not-yet-quantized columns once columns
    0..j-1 are fixed) divided by the square root of its first entry ("GPTQ /
    AWQ / SqueezeLLM" sec. 一: the decomposition of H^-1 the sweep reads
    row by row).  Each row is one float64 solve with that sub-matrix (a
    library Cholesky solve as the step), so a few rows of a d = 14336 factor
    cost seconds where the whole factor costs minutes.  Returns a
    len(rows) x d array, zero left of the diagonal."""
    from scipy.linalg import cho_factor, cho_solve
    Hd = np.asarray(Hd, dtype=np.float64)
    d = Hd.shape[0]
    out = np.zeros((len(rows), d), dtype=np.float64)
    for i, j in enumerate(rows):
        j = int(j)
        e = np.zeros(d - j)
        e[0] = 1.0
        x = cho_solve(cho_factor(Hd[j:, j:], lower=False, check_finite=False), e,
                      check_finite=False)
        out[i, j:] = x / np.sqrt(x[0])
    return out

# --------------------------------------------------------------------------
# Sweep, RTN, packing
# --------------------------------------------------------------------------

def n_groups(d: int, group_size: int) -> int:
    g = d if group_size <= 0 else group_size
    return (d + g - 1) // g


def quantize_rows(W: np.ndarray, U: np.ndarray, bits: int = 4, group_size: int = 128,
                  forced_codes=None, forced_scales=None, forced_zeros=None,
                  record=False, return_wq=False):
    """Column sweep over the rows of W (sweep order) with U (d x d upper).

    Returns dict(codes uint8 m x d, scales uint16 (fp16 bits) m x G, zeros uint8
    m x G, row_loss float64 m = sum_j (e_j / U_jj)^2, s_pre float32 m x G) and,
    with ``record``, own_codes / tie_dist (the oracle's own decision and the
    distance of w/s from the nearest rounding boundary) and, per group,
    own_scales / own_zeros / zero_tie_dist (the oracle's own fp16 scale and
    zero point on this trajectory, and the distance of -mn/s from the nearest
    rounding boundary) for teacher forcing.
    """
    W = np.ascontiguousarray(W, dtype=np.float64)
    U = np.ascontiguousarray(U, dtype=np.float64)
    m, d = W.shape
    G = n_groups(d, group_size)
    out = dict(codes=np.empty((m, d), np.uint8), scales=np.empty((m, G), np.uint16),
               zeros=np.empty((m, G), np.uint8), row_loss=np.empty(m, np.float64),
               s_pre=np.empty((m, G), np.float32))
    fc = None if forced_codes is None else np.ascontiguousarray(forced_codes, dtype=np.int16)
    fs = None if forced_scales is None else np.ascontiguousarray(forced_scales, dtype=np.uint16)
    fz = None if forced_zeros is None else np.ascontiguousarray(forced_zeros, dtype=np.uint8)
    if record or fc is not None:
        out["own_codes"] = np.empty((m, d), np.uint8)
        out["tie_dist"] = np.empty((m, d), np.float32)
        out["own_scales"] = np.empty((m, G), np.uint16)
        out["own_zeros"] = np.empty((m, G), np.uint8)
        out["zero_tie_dist"] = np.empty((m, G), np.float32)
    wq = np.empty((m, d), np.float64) if return_wq else None
    _load().orc_quantize_rows(_p(W), _p(U), m, d, int(bits), int(group_size),
                              _p(out["codes"]), _p(out["scales"]), _p(out["zeros"]),
                              _p(out["row_loss"]), _p(out["s_pre"]), _p(fc), _p(fs), _p(fz),
                              _p(out.get("own_codes")), _p(out.get("tie_dist")),
                              _p(out.get("own_scales")), _p(out.get("own_zeros")),
                              _p(out.get("zero_tie_dist")), _p(wq))
    if return_wq:
        out["wq"] = wq
    return out


def quantize_rows_static(W: np.ndarray, U: np.ndarray, bits: int = 4, group_size: int = 128):
    """The column sweep with STATIC groups: every group's scale and zero point
    are taken from the rows as they are before the sweep (the original W in
    sweep order, i.e. the round-to-nearest parameters of ``rtn``) instead of
    from the corrected values at the group's first column; the codes and the
    error feedback are those of ``quantize_rows``.  The pages fix the group
    parameters only by the min-max rule ("校准艺术" sec. 2.1); taking them
    before any correction is the alternative reading to the default one."""
    p = rtn(W, bits, group_size)
    out = quantize_rows(W, U, bits, group_size, forced_scales=p["scales"],
                        forced_zeros=p["zeros"])
    out["s_pre"] = p["s_pre"]
    return out


def rtn(W: np.ndarray, bits: int = 4, group_size: int = 128):
    W = np.ascontiguousarray(W, dtype=np.float64)
    m, d = W.shape
    G = n_groups(d, group_size)
    out = dict(codes=np.empty((m, d), np.uint8), scales=np.empty((m, G), np.uint16),
               zeros=np.empty((m, G), np.uint8), s_pre=np.empty((m, G), np.float32))
    _load().orc_rtn(_p(W), m, d, int(bits), int(group_size), _p(out["codes"]),
                    _p(out["scales"]), _p(out["zeros"]), _p(out["s_pre"]))
    return out


def pack_int4(codes: np.ndarray, zeros: np.ndarray):
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    m, d = codes.shape
    G = zeros.shape[1]
    assert d % 8 == 0
    qweight = np.empty((m, d // 8), np.uint32)
    qzeros = np.empty((m, (G + 1) // 2), np.uint8)
    _load().orc_pack_int4(_p(codes), _p(zeros), m, d, G, _p(qweight), _p(qzeros))
    return qweight, qzeros


def unpack_int4(qweight: np.ndarray, qzeros: np.ndarray, d: int, G: int):
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    qzeros = np.ascontiguousarray(qzeros, dtype=np.uint8)
    m = qweight.shape[0]
    codes = np.empty((m, d), np.uint8)
    zeros = np.empty((m, G), np.uint8)
    _load().orc_unpack_int4(_p(qweight), _p(qzeros), m, d, G, _p(codes), _p(zeros))
    return codes, zeros


def pack_bits(codes: np.ndarray, zeros: np.ndarray, bits: int):
    """b-bit storage (b in 2..8): each row's codes as one little-endian bit
    stream in uint32 words (d * b / 32 per row), its zero points as a second
    stream in bytes (ceil(G b / 8) per row).  b = 4 is the INT4 layout of
    ``pack_int4`` ("INT4/INT8 量化推理" sec. 一); other widths extend it."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    zeros = np.ascontiguousarray(zeros, dtype=np.uint8)
    m, d = codes.shape
    G = zeros.shape[1]
    assert (d * bits) % 32 == 0 and 2 <= bits <= 8
    qweight = np.empty((m, d * bits // 32), np.uint32)
    qzeros = np.empty((m, (G * bits + 7) // 8), np.uint8)
    _load().orc_pack_bits(_p(codes), _p(zeros), m, d, G, int(bits), _p(qweight), _p(qzeros))
    return qweight, qzeros


def unpack_bits(qweight: np.ndarray, qzeros: np.ndarray, d: int, G: int, bits: int):
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    qzeros = np.ascontiguousarray(qzeros, dtype=np.uint8)
    m = qweight.shape[0]
    codes = np.empty((m, d), np.uint8)
    zeros = np.empty((m, G), np.uint8)
    _load().orc_unpack_bits(_p(qweight), _p(qzeros), m, d, G, int(bits), _p(codes), _p(zeros))
    return codes, zeros


def dequantize(codes: np.ndarray, scales16: np.ndarray, zeros: np.ndarray,
               group_size: int, perm: np.ndarray | None = None) -> np.ndarray:
    """Q in ORIGINAL column order: Q[:, perm[k]] = s(r, k//g) * (c[r, k] - z(r, k//g))."""
    m, d = codes.shape
    g = d if group_size <= 0 else group_size
    gi = np.arange(d) // g
    s = np.ascontiguousarray(scales16, dtype=np.uint16).view(np.float16).astype(np.float64)[:, gi]
    z = zeros.astype(np.float64)[:, gi]
    Qs = s * (codes.astype(np.float64) - z)
    if perm is None:
        return Qs
    Q = np.empty_like(Qs)
    Q[:, np.asarray(perm, dtype=np.int64)] = Qs
    return Q


def w4a16_matmul(x, qweight: np.ndarray, qzeros: np.ndarray, scales16: np.ndarray, d: int,
                 group_size: int, perm: np.ndarray | None = None) -> np.ndarray:
    """y = x Q^T straight from the packed INT4 layer, in float64: the
    weight-only-quantized product (W4A16) of "INT4/INT8 量化推理" sec. 六,
    on the storage of sec. 一 of the same page.

    x: b x d fp16 activations (original column order); qweight / qzeros /
    scales16 as gptq_pack_int4 and the sweep write them (codes in sweep
    order); Q[:, perm[k]] = s (c_k - z) as in ``dequantize``.
    """
    xb = np.asarray(x)
    if xb.dtype == np.uint16:
        xb = xb.view(np.float16)
    xb = xb.astype(np.float64)
    G = n_groups(d, group_size)
    codes, zeros = unpack_int4(qweight, qzeros, d, G)
    Q = dequantize(codes, scales16, zeros, group_size, perm)
    return xb @ Q.T


def trace_quadratic(D: np.ndarray, H: np.ndarray) -> float:
    """tr(D H D^T) in float64."""
    D = np.ascontiguousarray(D, dtype=np.float64)
    H = np.ascontiguousarray(H, dtype=np.float64)
    return float(_load().orc_trace_quadratic(_p(D), _p(H), D.shape[0], D.shape[1]))


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------

def gptq_layer(W: np.ndarray, S: np.ndarray, n: int, bits: int = 4, group_size: int = 128,
               damp_rel: float = 0.01, act_order: bool = False, record=False):
    """Whole-layer GPTQ from the raw token sum S = X^T X over n tokens.

    W is m x d (any float dtype; promoted to float64) in ORIGINAL column order.
    Returns dict with perm, H (undamped, permuted), Hd, lam, U and the sweep
    outputs (codes/scales/zeros in sweep order, row_loss).
    """
    H, Hd, perm, lam, st = finalize(S, n, damp_rel, act_order)
    if st != 0:
        raise ValueError("mean(diag H) <= 0: no damping can make H positive definite")
    U, info = hinv_upper_chol(Hd)
    if info != 0:
        raise ValueError(f"H + lambda I is not positive definite (pivot {info})")
    Wp = np.ascontiguousarray(np.asarray(W, dtype=np.float64)[:, perm])
    res = quantize_rows(Wp, U, bits, group_size, record=record)
    res.update(perm=perm, H=H, Hd=Hd, lam=lam, U=U)
    return res


def layer_loss(W: np.ndarray, Q: np.ndarray, H_orig: np.ndarray) -> float:
    """tr((W-Q) H (W-Q)^T) with H in ORIGINAL column order; times n/2 this is
    ||(W - Q) X^T||_F^2 for H = 2 X^T X / n."""
    D = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    return trace_quadratic(D, H_orig)


# --------------------------------------------------------------------------
# Activation-aware channel scaling ahead of the sweep
# --------------------------------------------------------------------------

def channel_magnitude(X) -> np.ndarray:
    """a_j = mean over tokens of |X[t, j]|: the per-input-channel activation
    magnitude AWQ scales by ("GPTQ / AWQ / SqueezeLLM" sec. 二: the mean of
    the absolute activations per channel)."""
    Xf = np.asarray(X)
    if Xf.dtype == np.uint16:
        Xf = Xf.view(np.float16)
    return np.abs(Xf.astype(np.float64)).mean(axis=0)


def awq_candidate_scales(a: np.ndarray, alpha: float) -> np.ndarray:
    """s = (a / mean(a))^alpha per input channel; a channel whose magnitude is
    0 takes the smallest positive one instead (the pages do not say; a zero
    scale would erase the channel)."""
    a = np.asarray(a, dtype=np.float64)
    pos = a[a > 0]
    floor = pos.min() if pos.size else 1.0
    a = np.where(a > 0, a, floor)
    return (a / a.mean()) ** alpha


def awq_search(W: np.ndarray, S: np.ndarray, n: int, a: np.ndarray, bits: int = 4,
               group_size: int = 128, n_grid: int = 20):
    """Choose the channel scaling by the output error, "GPTQ / AWQ /
    SqueezeLLM" sec. 二 (scale each input channel's weights up by its
    activation magnitude before quantizing, divide back afterwards; pick
    among candidate scalings the one with the smallest output error) and
    "INT4/INT8 量化推理" sec. 四 (the transform is exact before quantization).

    For alpha = k / n_grid, k = 0 .. n_grid - 1: s = awq_candidate_scales(a,
    alpha), W' = W diag(s), Q' = the group round-to-nearest of W' (the
    quantizer AWQ uses, no error feedback), D = Q' diag(s)^-1 - W, loss =
    tr(D H D^T) with H = 2 S / n (= (2/n) ||D X^T||^2).  alpha = 0 (no
    scaling) is a candidate, so the choice never loses to round-to-nearest
    on the calibration loss.  Ties go to the smaller alpha.

    Returns dict(alpha, s, losses (n_grid,), alphas (n_grid,)).
    """
    W = np.asarray(W, dtype=np.float64)
    S = np.ascontiguousarray(S, dtype=np.float64)
    H = 2.0 * S / n
    alphas = np.arange(n_grid, dtype=np.float64) / n_grid
    losses = np.empty(n_grid)
    for k, al in enumerate(alphas):
        s = awq_candidate_scales(a, al)
        Ws = np.ascontiguousarray(W * s[None, :])
        r = rtn(Ws, bits, group_size)
        Qs = dequantize(r["codes"], r["scales"], r["zeros"], group_size)
        losses[k] = layer_loss(W, Qs / s[None, :], H)
    k = int(np.argmin(losses))
    return dict(alpha=float(alphas[k]), s=awq_candidate_scales(a, alphas[k]), losses=losses,
                alphas=alphas)


def awq_then_gptq(W: np.ndarray, S: np.ndarray, n: int, a: np.ndarray, bits: int = 4,
                  group_size: int = 128, damp_rel: float = 0.01, act_order: bool = False,
                  n_grid: int = 20):
    """The combination the pages suggest ("GPTQ / AWQ / SqueezeLLM" sec. 二:
    first the AWQ scaling, then GPTQ's error compensation): with s from
    awq_search, GPTQ quantizes W' = W diag(s) against the inputs X' = X
    diag(s)^-1, i.e. S' = diag(s)^-1 S diag(s)^-1.  The dequantized layer is
    Q' diag(s)^-1; at inference the 1/s is folded into whatever produces X.

    Returns gptq_layer's dict for (W', S') plus s and alpha."""
    sr = awq_search(W, S, n, a, bits, group_size, n_grid)
    s = sr["s"]
    Wp = np.asarray(W, dtype=np.float64) * s[None, :]
    Sp = np.asarray(S, dtype=np.float64) / np.outer(s, s)
    res = gptq_layer(Wp, Sp, n, bits, group_size, damp_rel, act_order)
    res.update(s=s, alpha=sr["alpha"], awq_losses=sr["losses"])
    return res

"""CPU checks of the parity helpers themselves: the teacher-forced check must
accept the oracle's own decisions and reject a zero point or a code moved off
a rounding tie (the planted mistake is in oracle-produced data, on the CPU)."""
import numpy as np
import pytest

import oracle
from tests import parity as P


def _layer(m=64, d=512, seed=0):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((m, d)) * 0.02
    X = rng.standard_normal((4 * d, d))
    X[:, :5] *= 30.0
    H = 2.0 * X.T @ X / X.shape[0]
    H += 0.01 * np.mean(np.diag(H)) * np.eye(d)
    U, info = oracle.hinv_upper_chol(H)
    assert info == 0
    return W, U


def _as_gpu(res):
    return dict(codes=res["codes"].copy(), scales=res["scales"].copy(), zeros=res["zeros"].copy())


def test_forced_check_accepts_the_oracles_own_decisions():
    W, U = _layer()
    res = oracle.quantize_rows(W, U, 4, 128)
    rep = {}
    assert P.teacher_forced_check(W, U, _as_gpu(res), 4, 128, report=rep) == 0
    assert rep["forced_zero_ties"] == 0 and rep["forced_scale_flips"] == 0


def test_forced_check_rejects_a_zero_point_off_a_tie():
    W, U = _layer()
    res = oracle.quantize_rows(W, U, 4, 128, record=True)
    # a group whose -mn/s sits far from a rounding boundary and whose codes all stay
    # below 15: shifting its zero point and its codes by one keeps the dequantized
    # values (and so the trajectory), so only the zero-point decision is wrong
    gmax = res["codes"].reshape(W.shape[0], -1, 128).max(axis=2)
    cand = np.argwhere((res["zero_tie_dist"] > 0.2) & (res["zeros"] < 15) & (gmax < 15))
    r, g = cand[0]
    bad = _as_gpu(res)
    bad["zeros"][r, g] += 1
    bad["codes"][r, 128 * g:128 * (g + 1)] += 1
    with pytest.raises(AssertionError, match="zero points differ off a tie"):
        P.teacher_forced_check(W, U, bad, 4, 128)


def test_forced_check_rejects_a_code_off_a_tie():
    W, U = _layer()
    res = oracle.quantize_rows(W, U, 4, 128, record=True)
    cand = np.argwhere((res["tie_dist"] > 0.2) & (res["codes"] > 0) & (res["codes"] < 15))
    r, j = cand[len(cand) // 2]
    bad = _as_gpu(res)
    bad["codes"][r, j] += 1
    with pytest.raises(AssertionError, match="non-tie mismatches"):
        P.teacher_forced_check(W, U, bad, 4, 128)


def test_zero_tie_distance_is_zero_at_a_half_integer():
    # one group of 8 columns, U = I: mn = -0.75, mx = 0.75 -> s = 0.1 (fp16 0.0999755...),
    # -mn/s ~ 7.5; choose mn so that -mn/s is exactly 7.5 in fp32 with s = 2^-4
    d = 8
    w = np.zeros((1, d))
    w[0, 0] = -7.5 * 2.0 ** -4          # mn = -0.46875
    w[0, 1] = 7.5 * 2.0 ** -4           # mx - mn = 0.9375 = 15 * 2^-4 -> s = 2^-4 exactly
    res = oracle.quantize_rows(w, np.eye(d), 4, d, record=True)
    assert res["scales"][0, 0] == np.float16(2.0 ** -4).view(np.uint16)
    assert res["zero_tie_dist"][0, 0] == 0.0
    assert res["zeros"][0, 0] == 8       # rne(7.5) = 8
    assert np.array_equal(res["own_zeros"], res["zeros"])

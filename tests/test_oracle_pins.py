"""Pins for the float64 oracle: it is checked against what the pages and the
mathematics fix, never against itself.

Each test names what pins it: a hand-worked example stored under
tests/golden/ (with its citation), a closed form, an identity, an independent
algorithm (explicit sequential OBS, lazy batches), brute force, or an
exhaustive comparison with an independent IEEE implementation (numpy).
"""
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _spd_from_tokens(n, d, seed=0, outliers=0, fac=30.0):
    rng = _rng(seed)
    X = rng.standard_normal((n, d)).astype(np.float16)
    if outliers:
        ch = rng.permutation(d)[:outliers]
        X = X.astype(np.float32)
        X[:, ch] *= fac
        X = X.astype(np.float16)
    return X


# --------------------------------------------------------------------------
# IEEE binary16 conversions: exhaustive / dense comparison with numpy
# --------------------------------------------------------------------------

def test_half_decode_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_bits_to_float64(bits)
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(np.isinf(ours), np.isinf(ref))


def test_half_encode_matches_numpy_rne():
    rng = _rng(1)
    # every fp16 value, the midpoints between neighbours (ties), and random fp32s
    h = np.arange(0, 0x7c00, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    mids = (h[:-1] + h[1:]) / 2.0
    vals = np.concatenate([h, mids, np.exp(rng.uniform(-20, 11.1, 20000))]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    ours = np.array([oracle.float32_to_half_bits(float(v)) for v in vals], dtype=np.uint16)
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# Group quantizer: hand-worked examples (golden) and storage arithmetic
# --------------------------------------------------------------------------

def _read_golden(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


def test_group_quant_hand_examples():
    rows = _read_golden("group_quant_examples.txt")
    assert len(rows) == 5
    for row in rows:
        left, mid, right = [p.strip() for p in row.split("|")]
        name, bits, ws = left.split()
        w = np.array([float(v) for v in ws.split(",")])[None, :]
        sb, z = mid.split()
        codes = [int(v) for v in right.split(",")]
        out = oracle.rtn(w, bits=int(bits), group_size=w.shape[1])
        assert out["scales"][0, 0] == int(sb, 16), name
        assert out["zeros"][0, 0] == int(z), name
        assert out["codes"][0].tolist() == codes, name
        # with a diagonal U (no cross terms) the sweep is the same quantizer
        sw = oracle.quantize_rows(w, np.eye(w.shape[1]), int(bits), w.shape[1])
        assert sw["codes"][0].tolist() == codes, name


def test_storage_arithmetic_matches_page():
    rows = _read_golden("storage_arithmetic.txt")
    table = {int(r.split()[0]): (float(r.split()[1]), float(r.split()[2])) for r in rows}
    m, d = 6, 1024
    for g, (bytes_per_group, bits_per_weight) in table.items():
        G = d // g
        codes = _rng(g).integers(0, 16, (m, d), dtype=np.uint8)
        zeros = _rng(g + 1).integers(0, 16, (m, G), dtype=np.uint8)
        qweight, qzeros = oracle.pack_int4(codes, zeros)
        scales_bytes = m * G * 2
        total = qweight.nbytes + qzeros.nbytes + scales_bytes
        assert total == bytes_per_group * m * G
        assert total * 8 / (m * d) == bits_per_weight


def test_pack_hand_examples_and_roundtrip():
    for row in _read_golden("pack_examples.txt"):
        kind, vals, packed = [p.strip() for p in row.split("|")]
        v = [int(x) for x in vals.split(",")]
        if kind == "codes":
            qw, _ = oracle.pack_int4(np.array([v], np.uint8), np.zeros((1, 1), np.uint8))
            assert int(qw[0, 0]) == int(packed, 16)
        else:
            _, qz = oracle.pack_int4(np.zeros((1, 8), np.uint8), np.array([v], np.uint8))
            assert int(qz[0, 0]) == int(packed, 16)
    rng = _rng(5)
    for (m, d, G) in [(3, 256, 2), (5, 384, 3), (1, 8, 1), (7, 4096, 32)]:
        codes = rng.integers(0, 16, (m, d), dtype=np.uint8)
        zeros = rng.integers(0, 16, (m, G), dtype=np.uint8)
        qw, qz = oracle.pack_int4(codes, zeros)
        c2, z2 = oracle.unpack_int4(qw, qz, d, G)
        assert np.array_equal(c2, codes) and np.array_equal(z2, zeros)


def test_pack_bits_hand_examples_roundtrip_and_int4_layout():
    """b-bit packing: hand-worked words and bytes (tests/golden), the round
    trip at every width, the storage arithmetic, and b = 4 equal to the INT4
    layout (pinned on its own by pack_examples.txt)."""
    for row in _read_golden("pack_bits_examples.txt"):
        kind, bits, vals, packed = [p.strip() for p in row.split("|")]
        b = int(bits)
        v = [int(x) for x in vals.split(",")]
        want = [int(x, 16) for x in packed.split(",")]
        if kind == "codes":
            d = len(v)
            qw, _ = oracle.pack_bits(np.array([v], np.uint8), np.zeros((1, 1), np.uint8), b)
            assert [int(x) for x in qw[0]] == want + [0] * (qw.shape[1] - len(want))
        else:
            _, qz = oracle.pack_bits(np.zeros((1, 32), np.uint8), np.array([v], np.uint8), b)
            assert [int(x) for x in qz[0]] == want
    rng = _rng(6)
    for b in (2, 3, 4, 5, 8):
        for (m, d, G) in [(3, 256, 2), (5, 384, 3), (2, 32, 1), (4, 4096, 32)]:
            codes = rng.integers(0, 1 << b, (m, d), dtype=np.uint8)
            zeros = rng.integers(0, 1 << b, (m, G), dtype=np.uint8)
            qw, qz = oracle.pack_bits(codes, zeros, b)
            assert qw.nbytes == m * d * b // 8 and qz.shape[1] == (G * b + 7) // 8
            c2, z2 = oracle.unpack_bits(qw, qz, d, G, b)
            assert np.array_equal(c2, codes) and np.array_equal(z2, zeros)
            if b == 4:
                q4w, q4z = oracle.pack_int4(codes, zeros)
                assert np.array_equal(qw, q4w) and np.array_equal(qz, q4z)
    # storage: b bits per weight + (b + 16) bits per group of 128
    for b, total in ((3, 50.375), (4, 66.5), (8, 131.0)):
        assert (128 * b + b + 16) / 8 == total


def test_w4a16_hand_example_and_one_hot_columns():
    rows = {}
    cases = []
    for row in _read_golden("w4a16_example.txt"):
        f = [p.strip() for p in row.split("|")]
        if f[0] == "case":
            cases.append(f[1:])
        else:
            rows[f[0]] = [[int(v, 16) for v in part.split(",")] for part in f[1].split(";")]
    qw = np.array(rows["qweight"], np.uint32)
    qz = np.array(rows["qzeros"], np.uint8)
    sc = np.array(rows["scales"], np.uint16)
    xs = {"ones": np.ones(16), "ramp": np.arange(16.0)}
    for xname, pname, want in cases:
        perm = {"none": None, "reversed": np.arange(15, -1, -1, dtype=np.int32),
                "cyclic": ((np.arange(16) + 1) % 16).astype(np.int32)}[pname]
        x = xs[xname].astype(np.float16)[None, :]
        y = oracle.w4a16_matmul(x, qw, qz, sc, 16, 8, perm)
        assert y[0].tolist() == [float(v) for v in want.split(",")]
    # one-hot activations pick out columns of the dequantized layer
    rng = _rng(17)
    m, d, g = 5, 256, 64
    codes = rng.integers(0, 16, (m, d), dtype=np.uint8)
    zeros = rng.integers(0, 16, (m, d // g), dtype=np.uint8)
    sc = rng.uniform(1e-3, 1e-1, (m, d // g)).astype(np.float16).view(np.uint16)
    perm = rng.permutation(d).astype(np.int32)
    qw, qz = oracle.pack_int4(codes, zeros)
    Q = oracle.dequantize(codes, sc, zeros, g, perm)
    for j in (0, 1, 77, 255):
        e = np.zeros((1, d), np.float16)
        e[0, j] = 1
        assert np.array_equal(oracle.w4a16_matmul(e, qw, qz, sc, d, g, perm)[0], Q[:, j])


# --------------------------------------------------------------------------
# Hessian
# --------------------------------------------------------------------------

def _sylvester(k):
    H = np.array([[1.0]])
    for _ in range(k):
        H = np.block([[H, H], [H, -H]])
    return H


def test_hessian_closed_forms():
    # Hadamard rows: X^T X = n I exactly
    Had = _sylvester(4)                      # 16 x 16, entries +-1
    S = oracle.hessian(Had.astype(np.float16))
    assert np.array_equal(S, 16.0 * np.eye(16))
    # one-hot rows: S is diagonal with the counts times value^2
    rng = _rng(2)
    idx = rng.integers(0, 10, 200)
    X = np.zeros((200, 10), np.float16)
    X[np.arange(200), idx] = 0.5
    S = oracle.hessian(X)
    assert np.array_equal(S, np.diag(np.bincount(idx, minlength=10) * 0.25))
    # a tiny hand example: rows (1,2), (3,-1) -> [[10, -1], [-1, 5]]
    S = oracle.hessian(np.array([[1, 2], [3, -1]], np.float16))
    assert np.array_equal(S, np.array([[10.0, -1.0], [-1.0, 5.0]]))
    # accumulation over batches equals one pass; S symmetric PSD
    X = _spd_from_tokens(96, 12, 3, outliers=2)
    S1 = oracle.hessian(X)
    S2 = oracle.hessian(X[:40])
    oracle.hessian(X[40:], S2)
    assert np.allclose(S1, S2, rtol=0, atol=1e-9 * np.abs(S1).max())
    assert np.array_equal(S1, S1.T)
    assert np.linalg.eigvalsh(S1).min() > -1e-9 * np.abs(S1).max()



def test_hessian_syrk_closed_forms_and_plain_loop():
    """The BLAS route of S (full-size checks) against the Hadamard closed form
    and against the plain column loop on ragged chunking."""
    Had = _sylvester(5)                      # 32 x 32 entries +-1: X^T X = 32 I
    assert np.array_equal(oracle.hessian_syrk(Had.astype(np.float16), chunk=7),
                          32.0 * np.eye(32))
    X = _spd_from_tokens(1000, 40, 5, outliers=3)
    S1 = oracle.hessian(X)
    S2 = oracle.hessian_syrk(X, chunk=333)
    assert np.array_equal(S2, S2.T)
    assert np.abs(S1 - S2).max() <= 1e-13 * np.abs(S1).max()

def test_finalize_damping_and_perm():
    X = _spd_from_tokens(64, 9, 4, outliers=2)
    S = oracle.hessian(X)
    H, Hd, perm, lam, st = oracle.finalize(S, 64, 0.01, act_order=True)
    assert st == 0
    diag = 2.0 * np.diag(S) / 64
    assert np.array_equal(perm, np.argsort(-diag, kind="stable"))
    assert np.allclose(lam, 0.01 * diag.mean(), rtol=1e-15)
    assert np.allclose(H, (2.0 * S / 64)[np.ix_(perm, perm)], rtol=1e-15)
    assert np.allclose(Hd - H, lam * np.eye(9), atol=1e-15 * lam)
    # ties keep the lower index first
    S = np.diag([2.0, 5.0, 2.0, 5.0])
    _, _, perm, _, _ = oracle.finalize(S, 2, 0.01, act_order=True)
    assert perm.tolist() == [1, 3, 0, 2]
    # all-zero input: no damping can be formed
    *_, st = oracle.finalize(np.zeros((4, 4)), 10, 0.01)
    assert st == 3


# --------------------------------------------------------------------------
# Cholesky / triangular inverse / U
# --------------------------------------------------------------------------

def test_cholesky_textbook_and_failure():
    A = np.array([[4.0, 12, -16], [12, 37, -43], [-16, -43, 98]])
    L, info = oracle.cholesky_lower(A)
    assert info == 0
    assert np.array_equal(L, np.array([[2.0, 0, 0], [6, 1, 0], [-8, 5, 3]]))
    _, info = oracle.cholesky_lower(np.array([[1.0, 2], [2, 1]]))
    assert info == 2
    _, info = oracle.cholesky_lower(np.array([[0.0, 0], [0, 1]]))
    assert info == 1


def test_trtri_closed_form():
    a = 3.25
    Linv = oracle.trtri_lower(np.array([[1.0, 0], [a, 1]]))
    assert np.array_equal(Linv, np.array([[1.0, 0], [-a, 1]]))
    L = np.array([[2.0, 0, 0], [6, 1, 0], [-8, 5, 3]])
    Linv = oracle.trtri_lower(L)
    # hand inverse: rows (1/2,0,0), (-3,1,0), (19/3,-5/3,1/3)
    exp = np.array([[0.5, 0, 0], [-3, 1, 0], [19 / 3, -5 / 3, 1 / 3]])
    assert np.allclose(Linv, exp, rtol=0, atol=1e-15)


def test_upper_chol_of_inverse_2x2_closed_form():
    a, b, c = 5.0, 1.5, 2.0
    U, info = oracle.hinv_upper_chol(np.array([[a, b], [b, c]]))
    det = a * c - b * b
    exp = np.array([[np.sqrt(c / det), (-b / det) / np.sqrt(c / det)], [0.0, np.sqrt(1.0 / c)]])
    assert info == 0
    assert np.allclose(U, exp, rtol=1e-14, atol=0)


def test_upper_chol_of_inverse_properties():
    X = _spd_from_tokens(400, 48, 6, outliers=3, fac=50.0)
    S = oracle.hessian(X)
    _, Hd, _, _, _ = oracle.finalize(S, 400, 0.01)
    U, info = oracle.hinv_upper_chol(Hd)
    assert info == 0
    assert np.array_equal(U, np.triu(U)) and (np.diag(U) > 0).all()
    R = U.T @ U @ Hd - np.eye(48)
    assert np.abs(R).max() < 1e-9
    # reverse-order route: U = J chol_lower(J H J)^-1 J
    J = np.eye(48)[::-1]
    Lr, info = oracle.cholesky_lower(J @ Hd @ J)
    U2 = J @ oracle.trtri_lower(Lr) @ J
    assert info == 0
    assert np.abs(U2 - U).max() <= 1e-10 * np.abs(U).max()
    # diagonal H: U = diag(1/sqrt(h))
    h = np.array([4.0, 0.25, 9.0, 1.0])
    U, _ = oracle.hinv_upper_chol(np.diag(h))
    assert np.allclose(U, np.diag(1 / np.sqrt(h)), rtol=1e-15, atol=0)


def _kms_u(d, rho):
    """Closed form for H = KMS(rho), H_ij = rho^|i-j|: chol(H) = L with
    L[i][0] = rho^i and L[i][j] = rho^(i-j) sqrt(1 - rho^2) (j >= 1), so L^-1
    is lower bidiagonal (1, then 1/c on the diagonal and -rho/c below it,
    c = sqrt(1 - rho^2)); H is persymmetric (J H J = H), so the upper factor
    of H^-1 is U = J L^-1 J: upper bidiagonal, U_ii = 1/c except U_{d-1,d-1}
    = 1, and U_{i,i+1} = -rho/c."""
    c = np.sqrt(1.0 - rho * rho)
    U = np.zeros((d, d))
    U[np.arange(d - 1), np.arange(d - 1)] = 1.0 / c
    U[d - 1, d - 1] = 1.0
    U[np.arange(d - 1), np.arange(1, d)] = -rho / c
    return U


def test_upper_chol_of_inverse_kms_closed_form():
    """U for a Kac-Murdock-Szego matrix at d = 256 against its closed form
    (every entry, the zeros beyond the first superdiagonal included); and
    the sweep with that U against a scalar recursion in which each column's
    error reaches the next column only (U[j][j+1], row j of U, not column j)."""
    d, rho, g = 256, 0.7, 64
    i = np.arange(d)
    H = rho ** np.abs(i[:, None] - i[None, :])
    U, info = oracle.hinv_upper_chol(H)
    assert info == 0
    assert np.abs(U - _kms_u(d, rho)).max() <= 1e-12
    rng = _rng(41)
    W = 0.02 * rng.standard_normal((5, d))
    r = oracle.quantize_rows(W, U, 4, g)
    for row in range(W.shape[0]):
        w = W[row].copy()
        for j in range(d):
            if j % g == 0:                       # parameters from the values as they stand
                p = oracle.rtn(w[None, j:j + g], 4, g)
                s = float(p["scales"].view(np.float16)[0, 0])
                z = int(p["zeros"][0, 0])
            x = np.float32(w[j])
            c = int(min(max(np.rint(np.float32(x / np.float32(s))) + z, 0), 15))
            assert c == r["codes"][row, j], (row, j)
            E = (w[j] - s * (c - z)) / U[j, j]
            if j + 1 < d:
                w[j + 1] -= E * U[j, j + 1]



def test_u_rows_closed_form_and_full_factor():
    """Rows of U from the trailing sub-Hessians against the KMS closed form
    (upper bidiagonal) and against the full factor of the plain route."""
    d, rho = 200, 0.6
    i = np.arange(d)
    H = rho ** np.abs(i[:, None] - i[None, :])
    rows = [0, 1, 77, 198, 199]
    assert np.abs(oracle.u_rows(H, rows) - _kms_u(d, rho)[rows]).max() <= 1e-12
    X = _spd_from_tokens(600, 150, 6, outliers=3).astype(np.float64)
    Hd = 2.0 * X.T @ X / 600
    Hd += 0.01 * np.diag(Hd).mean() * np.eye(150)
    U, info = oracle.hinv_upper_chol(Hd)
    assert info == 0
    rows = [0, 64, 100, 149]
    assert np.abs(oracle.u_rows(Hd, rows) - U[rows]).max() <= 1e-10 * np.abs(U).max()

# --------------------------------------------------------------------------
# The sweep
# --------------------------------------------------------------------------

def test_gptq_equals_rtn_when_hessian_is_isotropic():
    # X with X^T X proportional to I (Hadamard rows): U is diagonal, so the
    # error feedback vanishes and GPTQ must reproduce RTN bit for bit.
    Had = _sylvester(7)                          # 128 x 128
    X = np.vstack([Had, Had]).astype(np.float16) # n = 256, d = 128
    S = oracle.hessian(X)
    rng = _rng(7)
    W = (0.02 * rng.standard_normal((64, 128))).astype(np.float32)
    res = oracle.gptq_layer(W, S, 256, bits=4, group_size=32)
    assert np.abs(res["U"] - np.diag(np.diag(res["U"]))).max() == 0.0
    r = oracle.rtn(W, bits=4, group_size=32)
    assert np.array_equal(res["codes"], r["codes"])
    assert np.array_equal(res["scales"], r["scales"])
    assert np.array_equal(res["zeros"], r["zeros"])
    # and any diagonal H (random positive diagonal)
    S = np.diag(rng.uniform(0.5, 30.0, 128))
    res = oracle.gptq_layer(W, S, 1, bits=3, group_size=64)
    r = oracle.rtn(W, bits=3, group_size=64)
    assert np.array_equal(res["codes"], r["codes"])


def test_static_groups_special_cases():
    """Static groups take every group's parameters from the uncorrected row:
    with a diagonal U (no feedback) they equal the dynamic ones and RTN; per
    channel (one group per row, parameterized at column 0 before any
    correction) the two readings coincide for any U; otherwise the scales are
    RTN's and the feedback still obeys the loss identity."""
    rng = _rng(23)
    m, d = 48, 128
    W = 0.02 * rng.standard_normal((m, d))
    Ud = np.diag(rng.uniform(0.2, 2.0, d))
    st = oracle.quantize_rows_static(W, Ud, 4, 32)
    dy = oracle.quantize_rows(W, Ud, 4, 32)
    r = oracle.rtn(W, 4, 32)
    for k in ("codes", "scales", "zeros"):
        assert np.array_equal(st[k], dy[k]) and np.array_equal(st[k], r[k])
    X = rng.standard_normal((400, d)).astype(np.float16)
    X[:, 5] *= 30
    S = oracle.hessian(X)
    _, Hd, _, _, _ = oracle.finalize(S, 400, 0.01, False)
    U, info = oracle.hinv_upper_chol(Hd)
    assert info == 0
    for g in (d, -1):
        st = oracle.quantize_rows_static(W, U, 4, g)
        dy = oracle.quantize_rows(W, U, 4, g)
        for k in ("codes", "scales", "zeros"):
            assert np.array_equal(st[k], dy[k])
    st = oracle.quantize_rows_static(W, U, 4, 32)
    dy = oracle.quantize_rows(W, U, 4, 32)
    assert np.array_equal(st["scales"], oracle.rtn(W, 4, 32)["scales"])
    assert not np.array_equal(st["scales"], dy["scales"])
    Q = oracle.dequantize(st["codes"], st["scales"], st["zeros"], 32)
    D = W - Q
    assert abs(st["row_loss"].sum() - oracle.trace_quadratic(D, Hd)) <= 1e-9 * st["row_loss"].sum()


def test_awq_search_pins():
    """The channel-scaling search: the alpha = 0 candidate is round-to-nearest,
    every candidate's loss equals the output error evaluated through X itself,
    the choice is the first minimizer, and the search depends on the
    activations only through a / mean(a)."""
    rng = _rng(31)
    n, m, d, g = 600, 40, 128, 32
    X = rng.standard_normal((n, d))
    X[:, [3, 50]] *= 40.0
    X = X.astype(np.float16)
    W = 0.02 * rng.standard_normal((m, d))
    S = oracle.hessian(X)
    a = oracle.channel_magnitude(X)
    r = oracle.awq_search(W, S, n, a, 4, g, n_grid=10)
    X64 = X.astype(np.float64)

    def through_x(alpha):
        sc = oracle.awq_candidate_scales(a, alpha)
        q = oracle.rtn(W * sc, 4, g)
        Q = oracle.dequantize(q["codes"], q["scales"], q["zeros"], g) / sc
        return (2.0 / n) * float(np.sum(((W - Q) @ X64.T) ** 2))

    rt = oracle.rtn(W, 4, g)
    Q0 = oracle.dequantize(rt["codes"], rt["scales"], rt["zeros"], g)
    l0 = (2.0 / n) * float(np.sum(((W - Q0) @ X64.T) ** 2))
    assert abs(r["losses"][0] - l0) <= 1e-9 * l0
    for k in (3, 7, 9):
        lk = through_x(r["alphas"][k])
        assert abs(r["losses"][k] - lk) <= 1e-9 * lk
    assert r["alpha"] == r["alphas"][int(np.argmin(r["losses"]))]
    assert r["losses"].min() <= r["losses"][0]
    # two channels with 40x activations: protecting them pays off here
    assert r["alpha"] > 0 and r["losses"].min() < r["losses"][0]
    # X -> 4 X: S -> 16 S, a -> 4 a; the scales and choice are unchanged, the
    # losses x16 (up to the summation order of the oracle's threaded trace)
    r2 = oracle.awq_search(W, 16.0 * S, n, 4.0 * a, 4, g, n_grid=10)
    assert r2["alpha"] == r["alpha"]
    assert np.allclose(r2["losses"], 16.0 * r["losses"], rtol=1e-12, atol=0)


def test_awq_then_gptq_pins():
    """GPTQ after the scaling works on W' = W diag(s) and S' = diag(s)^-1 S
    diag(s)^-1: with one candidate (alpha = 0, s = 1) it is plain GPTQ, and
    the loss of the layer mapped back, Q' diag(s)^-1, against the original
    H equals the loss in the scaled coordinates."""
    rng = _rng(37)
    n, m, d, g = 500, 24, 128, 32
    X = rng.standard_normal((n, d))
    X[:, [9]] *= 30.0
    X = X.astype(np.float16)
    W = 0.02 * rng.standard_normal((m, d))
    S = oracle.hessian(X)
    a = oracle.channel_magnitude(X)
    one = oracle.awq_then_gptq(W, S, n, a, 4, g, n_grid=1)
    ref = oracle.gptq_layer(W, S, n, 4, g)
    assert np.all(one["s"] == 1.0) and np.array_equal(one["codes"], ref["codes"])
    res = oracle.awq_then_gptq(W, S, n, a, 4, g, n_grid=10)
    s = res["s"]
    Qp = oracle.dequantize(res["codes"], res["scales"], res["zeros"], g, res["perm"])
    H = 2.0 * S / n
    l_orig = oracle.layer_loss(W, Qp / s[None, :], H)
    l_scaled = oracle.layer_loss(W * s[None, :], Qp, H / np.outer(s, s))
    assert abs(l_orig - l_scaled) <= 1e-10 * l_orig


def test_loss_closed_form_identity():
    # sum_j (e_j/U_jj)^2 = tr(D Hd D^T) = (2/n)||D X^T||^2 + lam ||D||^2, and
    # D = E U (the accumulated corrections): exact for any quantizer decisions.
    n, d, m = 300, 64, 40
    X = _spd_from_tokens(n, d, 8, outliers=3, fac=40.0)
    S = oracle.hessian(X)
    rng = _rng(9)
    W = 0.02 * rng.standard_normal((m, d))
    for bits, g in [(4, 32), (2, 64), (3, -1)]:
        res = oracle.gptq_layer(W, S, n, bits=bits, group_size=g)
        Q = oracle.dequantize(res["codes"], res["scales"], res["zeros"], g)
        D = W - Q
        lhs = res["row_loss"].sum()
        rhs1 = oracle.trace_quadratic(D, res["Hd"])
        Xf = X.astype(np.float64)
        rhs2 = 2.0 / n * np.sum((D @ Xf.T) ** 2) + res["lam"] * np.sum(D * D)
        assert abs(lhs - rhs1) <= 1e-10 * rhs1
        assert abs(lhs - rhs2) <= 1e-10 * rhs2


def _sequential_obs(w, Hd, bits, gsize):
    """Explicit sequential OBS (independent of U): at each column, the
    inverse of the remaining sub-Hessian is recomputed from scratch."""
    d = w.shape[0]
    w = w.astype(np.float64).copy()
    maxq = 2 ** bits - 1
    codes = np.zeros(d, np.uint8)
    for j in range(d):
        if j % gsize == 0:
            x = w[j:j + gsize].astype(np.float32)
            mn = min(np.float32(0), x.min())
            mx = max(np.float32(0), x.max())
            if mn == mx:
                mn, mx = np.float32(-1), np.float32(1)
            s = np.float32(np.float32(mx - mn) / np.float32(maxq)).astype(np.float16).astype(np.float32)
            z = int(np.clip(np.rint(np.float32(-mn) / s), 0, maxq))
        c = int(np.clip(np.rint(np.float32(w[j]) / s) + z, 0, maxq))
        codes[j] = c
        q = float(s) * (c - z)
        Fi = np.linalg.inv(Hd[j:, j:])       # remaining columns j..d-1
        e = w[j] - q
        w[j:] -= e / Fi[0, 0] * Fi[0, :]
        w[j] = q
    return codes


def test_u_form_equals_explicit_sequential_obs():
    n, d, m = 200, 20, 30
    X = _spd_from_tokens(n, d, 10, outliers=2, fac=20.0)
    S = oracle.hessian(X)
    rng = _rng(11)
    W = 0.02 * rng.standard_normal((m, d))
    res = oracle.gptq_layer(W, S, n, bits=3, group_size=10)
    for r in range(m):
        assert np.array_equal(res["codes"][r], _sequential_obs(W[r], res["Hd"], 3, 10)), r


def _lazy_batch(W, U, bits, gsize, B):
    """Lazy-batch form: sweep B columns with updates confined to the batch,
    then apply the batch's accumulated corrections to the later columns."""
    W = W.astype(np.float64).copy()
    m, d = W.shape
    maxq = 2 ** bits - 1
    codes = np.zeros((m, d), np.uint8)
    for b0 in range(0, d, B):
        b1 = min(d, b0 + B)
        E = np.zeros((m, b1 - b0))
        for j in range(b0, b1):
            if j % gsize == 0:
                x = W[:, j:j + gsize].astype(np.float32)
                mn = np.minimum(np.float32(0), x.min(axis=1))
                mx = np.maximum(np.float32(0), x.max(axis=1))
                eq = mn == mx
                mn = np.where(eq, np.float32(-1), mn)
                mx = np.where(eq, np.float32(1), mx)
                s = ((mx - mn) / np.float32(maxq)).astype(np.float32).astype(np.float16).astype(np.float32)
                z = np.clip(np.rint(-mn / s), 0, maxq)
            c = np.clip(np.rint(W[:, j].astype(np.float32) / s) + z, 0, maxq)
            codes[:, j] = c
            q = s.astype(np.float64) * (c - z)
            e = W[:, j] - q
            Ej = e / U[j, j]
            E[:, j - b0] = Ej
            W[:, j:b1] -= np.outer(Ej, U[j, j:b1])
        W[:, b1:] -= E @ U[b0:b1, b1:]
    return codes


def test_lazy_batch_equals_unblocked():
    n, d, m = 256, 64, 48
    X = _spd_from_tokens(n, d, 12, outliers=3, fac=30.0)
    S = oracle.hessian(X)
    rng = _rng(13)
    W = 0.02 * rng.standard_normal((m, d))
    res = oracle.gptq_layer(W, S, n, bits=4, group_size=16)
    for B in (8, 16, 32):
        assert np.array_equal(_lazy_batch(W, res["U"], 4, 16, B), res["codes"]), B


def test_hessian_scale_invariance():
    n, d, m = 256, 48, 32
    X = _spd_from_tokens(n, d, 14, outliers=2, fac=25.0)
    S = oracle.hessian(X)
    W = 0.02 * _rng(15).standard_normal((m, d))
    a = oracle.gptq_layer(W, S, n, group_size=16)
    b = oracle.gptq_layer(W, 7.25 * S, n, group_size=16)      # 2X^TX/n vs scaled
    c = oracle.gptq_layer(W, S, 2 * n, group_size=16)          # X^T X / n
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["codes"], c["codes"])
    assert np.array_equal(a["scales"], b["scales"])


def test_act_order_is_gptq_on_permuted_problem():
    n, d, m = 256, 64, 24
    X = _spd_from_tokens(n, d, 16, outliers=4, fac=40.0)
    S = oracle.hessian(X)
    W = 0.02 * _rng(17).standard_normal((m, d))
    res = oracle.gptq_layer(W, S, n, group_size=16, act_order=True)
    perm = res["perm"]
    assert np.array_equal(perm, np.argsort(-np.diag(S), kind="stable"))
    Sp = S[np.ix_(perm, perm)]
    ref = oracle.gptq_layer(W[:, perm], Sp, n, group_size=16, act_order=False)
    assert np.array_equal(res["codes"], ref["codes"])
    assert np.array_equal(res["scales"], ref["scales"])
    # dequantized weights land back in original column order
    Q = oracle.dequantize(res["codes"], res["scales"], res["zeros"], 16, perm)
    Qp = oracle.dequantize(ref["codes"], ref["scales"], ref["zeros"], 16)
    assert np.array_equal(Q[:, perm], Qp)


def _loss_of(w, q, Hd):
    dlt = w - q
    return float(dlt @ Hd @ dlt)


def test_brute_force_tiny_layers():
    # d_in <= 6, 2-bit, one group per row: the grid is fixed from the original
    # row (no update precedes column 0), so the 4^d code vectors are the whole
    # search space.  Optimum <= GPTQ always; GPTQ <= RTN in aggregate.
    rng = _rng(21)
    ratios, tot_g, tot_r = [], 0.0, 0.0
    for trial in range(40):
        d = int(rng.integers(3, 7))
        X = _spd_from_tokens(64, d, 100 + trial, outliers=1, fac=8.0)
        S = oracle.hessian(X)
        W = 0.02 * rng.standard_normal((30, d))
        res = oracle.gptq_layer(W, S, 64, bits=2, group_size=-1)
        rt = oracle.rtn(W, bits=2, group_size=-1)
        Hd = res["Hd"]
        grid = np.array(np.meshgrid(*[np.arange(4)] * d, indexing="ij")).reshape(d, -1).T
        for r in range(W.shape[0]):
            s = float(oracle.half_bits_to_float64(res["scales"][r:r + 1, 0])[0])
            z = int(res["zeros"][r, 0])
            assert res["scales"][r, 0] == rt["scales"][r, 0] and z == rt["zeros"][r, 0]
            Qall = s * (grid - z)
            Dl = W[r][None, :] - Qall
            losses = np.einsum("ki,ij,kj->k", Dl, Hd, Dl)
            lopt = losses.min()
            lg = _loss_of(W[r], s * (res["codes"][r].astype(float) - z), Hd)
            lr = _loss_of(W[r], s * (rt["codes"][r].astype(float) - z), Hd)
            assert abs(lg - res["row_loss"][r]) <= 1e-9 * max(lg, 1e-30)
            assert lopt <= lg * (1 + 1e-12)
            tot_g += lg
            tot_r += lr
            ratios.append(lg / lopt if lopt > 0 else 1.0)
    assert tot_g <= tot_r
    # the greedy gap has no bound on the pages: recorded, not asserted
    print(f"greedy gap L_GPTQ/L_opt: median {np.median(ratios):.4f} max {np.max(ratios):.4f}; "
          f"L_GPTQ/L_RTN aggregate {tot_g / tot_r:.4f}")


def test_gptq_beats_rtn_on_outlier_inputs():
    # "校准艺术" sec. 2.2: GPTQ exploits weight correlation and beats min-max at
    # low bit; a statistical check on an outlier-channel workload.
    n, d, m = 512, 128, 64
    X = _spd_from_tokens(n, d, 22, outliers=3, fac=50.0)
    S = oracle.hessian(X)
    W = 0.02 * _rng(23).standard_normal((m, d))
    res = oracle.gptq_layer(W, S, n, group_size=64)
    Qg = oracle.dequantize(res["codes"], res["scales"], res["zeros"], 64)
    rt = oracle.rtn(W, group_size=64)
    Qr = oracle.dequantize(rt["codes"], rt["scales"], rt["zeros"], 64)
    H = 2.0 * S / n
    assert oracle.layer_loss(W, Qg, H) < oracle.layer_loss(W, Qr, H)


def test_teacher_forcing_reproduces_forced_decisions():
    n, d, m = 256, 64, 16
    X = _spd_from_tokens(n, d, 24, outliers=2)
    S = oracle.hessian(X)
    W = 0.02 * _rng(25).standard_normal((m, d))
    res = oracle.gptq_layer(W, S, n, group_size=32, record=True)
    assert np.array_equal(res["own_codes"], res["codes"])
    forced = res["codes"].astype(np.int16)
    forced[3, 10] = (forced[3, 10] + 1) % 16
    f = oracle.quantize_rows(np.ascontiguousarray(W[:, res["perm"]]), res["U"], 4, 32,
                             forced_codes=forced, forced_scales=res["scales"],
                             forced_zeros=res["zeros"])
    assert f["codes"][3, 10] == forced[3, 10]
    assert np.array_equal(f["codes"][:3], res["codes"][:3])
    assert np.array_equal(f["codes"][3, :10], res["codes"][3, :10])

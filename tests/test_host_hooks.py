"""Host-side checks of two properties the CUDA kernels rely on, through the
library's test hooks (no GPU needed):

  * the tiled factorization's task order is topological: every task's
    dependencies (the tiles its sums and its final product read) have
    smaller numbers, which is what makes its claim-a-number scheduling free
    of deadlock without co-resident CTAs;
  * the sweep's division-free code decision returns exactly the IEEE
    quotient fl(x / s) (numpy's float32 division) for every positive fp16
    scale, including x within a few ulp of the half-integer multiples of s
    where a rounded code would flip.
"""
import numpy as np
import pytest

from post_weight_quantization_11_b200 import gptq as G


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


def _deps(ty, i, j):
    """Tiles a task reads, from the block recurrences of L (A = L L^T) and
    X = L^-1 (L X = I): F(j) = diagonal tile, S(i, j) = L_ij, I(i, j) = X_ij."""
    if ty == 0:                                   # L_jj from A_jj - sum_k L_jk L_jk^T
        return [(1, j, k) for k in range(j)]
    if ty == 1:                                   # L_ij = (A_ij - sum L_ik L_jk^T) L_jj^-T
        return [(1, i, k) for k in range(j)] + [(1, j, k) for k in range(j)] + [(0, j, j)]
    # X_ij = -X_ii sum_{j<=k<i} L_ik X_kj  (X_jj from the diagonal task)
    return ([(0, i, i), (0, j, j)] + [(1, i, k) for k in range(j, i)]
            + [(2, k, j) for k in range(j + 1, i)])


@pytest.mark.parametrize("d", [128, 256, 384, 640, 1152, 4096, 14336])
def test_factorization_task_order_is_topological(d):
    order = G.gptq_debug_chol_task_order(d)
    T = d // 128
    tasks = [tuple(int(v) for v in row) for row in order]
    expected = ({(0, j, j) for j in range(T)} | {(1, i, j) for i in range(T) for j in range(i)}
                | {(2, i, j) for i in range(T) for j in range(i)})
    assert len(tasks) == T * T and set(tasks) == expected
    pos = {t: n for n, t in enumerate(tasks)}
    for t, n in pos.items():
        for dep in _deps(*t):
            assert pos[dep] < n, (t, dep)


def test_task_order_rejects_bad_sizes():
    with pytest.raises(G.GptqError):
        G.gptq_debug_chol_task_order(100)


def _fp16_positive_finite():
    h = np.arange(1, 0x7C00, dtype=np.uint16)
    return h.view(np.float16).astype(np.float32)


def test_division_free_quotient_is_ieee():
    rng = np.random.default_rng(7)
    s = _fp16_positive_finite()                   # every positive finite fp16 scale
    xs, ss = [], []
    for _ in range(24):                           # near (k + 1/2) s, within 4 ulp
        k = rng.integers(-40, 40, size=s.size).astype(np.float32)
        base = ((k + np.float32(0.5)) * s).astype(np.float32)
        off = rng.integers(-4, 5, size=s.size)
        x = (base.view(np.int32) + off.astype(np.int32)).view(np.float32)
        xs.append(x); ss.append(s)
    for scale in (40.0, 1.0e6):                   # random, moderate and large quotients
        for _ in range(8):
            x = (rng.uniform(-1.0, 1.0, size=s.size) * scale * s).astype(np.float32)
            xs.append(x); ss.append(s)
    x = np.concatenate(xs); s2 = np.concatenate(ss)
    ok = np.isfinite(x)
    x, s2 = x[ok], s2[ok]
    got = G.gptq_debug_div_rn(x, s2)
    want = (x / s2).astype(np.float32)             # IEEE float32 division
    bad = got.view(np.int32) != want.view(np.int32)
    assert not bad.any(), (f"{int(bad.sum())} of {x.size} quotients differ, e.g. "
                           f"x={x[bad][0]!r} s={s2[bad][0]!r}")
    # and the decision built on it: rne of the quotient
    assert np.array_equal(np.rint(got), np.rint(want))


def test_magic_number_rounding_matches_rint_under_the_clamp():
    """The sweep's rounding on the FMA pipe: fl(fl(x + 1.5 * 2^23) - 1.5 * 2^23)
    is round-to-nearest-even for |x| <= 2^22 and, past that, gives the same
    clamped code as rint (codes in [0, maxq], maxq <= 255).  Float32 numpy
    arithmetic is IEEE round-to-nearest, as the kernel's __fadd_rn/__fsub_rn."""
    rng = np.random.default_rng(11)
    M = np.float32(12582912.0)
    parts = [np.arange(-600, 601, dtype=np.float32) * np.float32(0.5),      # every half-integer tie
             rng.uniform(-300, 300, 200000).astype(np.float32),
             rng.uniform(-2.0 ** 24, 2.0 ** 24, 200000).astype(np.float32)]
    for e in (22, 23, 24, 30):                                               # around the limits
        b = np.float32(2.0 ** e)
        near = (np.array([b, -b], np.float32).view(np.int32)[:, None] +
                np.arange(-64, 65, dtype=np.int32)[None, :]).ravel().view(np.float32)
        parts.append(near)
    parts.append(np.array([3.4e38, -3.4e38, 1e-40, -1e-40, 0.0, -0.0], np.float32))
    x = np.concatenate(parts).astype(np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        trick = ((x + M).astype(np.float32) - M).astype(np.float32)
    exact = np.rint(x)
    small = np.abs(x) <= np.float32(2.0 ** 22)
    assert np.array_equal(trick[small], exact[small])
    for maxq in (3, 15, 255):
        for z in sorted({0, 1, maxq // 2, maxq}):
            zf, mq = np.float32(z), np.float32(maxq)
            a = np.minimum(np.maximum((trick + zf).astype(np.float32), 0), mq)
            b = np.minimum(np.maximum((exact + zf).astype(np.float32), 0), mq)
            assert np.array_equal(a, b), (maxq, z)


def test_code_byte_from_float_bits():
    """An integral c in [0, 255] as a byte: the low 8 bits of fl(c + 2^23)."""
    c = np.arange(256, dtype=np.float32)
    got = (c + np.float32(8388608.0)).astype(np.float32).view(np.uint32) & 0xFF
    assert np.array_equal(got, np.arange(256, dtype=np.uint32))

"""W4A16 product on the packed INT4 layer (gptq_w4a16_gemm) against the
float64 oracle (oracle.w4a16_matmul).

Two kinds of case:
  * exact: activations are small integers and the scales powers of two, so
    every product, chunk sum and total is an fp32-representable value and
    the kernel's y must equal the oracle's bit for bit (a single wrong code,
    zero point, nibble order or permutation entry shows);
  * general: Gaussian activations with outlier channels, fp16 scales; the
    error of fp32 sums is bounded by 1e-5 of sum_j |x_j| s (c + z) (the
    chunk sums a = sum c x and z sum x are formed separately, so the scale
    of the rounding is that of c + z, not of c - z; the realized error is
    about 1e-7 of it).
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_11_b200 import gptq as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


def _layer(rng, m, d, g, act, exact):
    ng = 1 if g == -1 else d // g
    codes = rng.integers(0, 16, (m, d), dtype=np.uint8)
    zeros = rng.integers(0, 16, (m, ng), dtype=np.uint8)
    if exact:
        sc = (2.0 ** -rng.integers(4, 9, (m, ng))).astype(np.float16)
    else:
        sc = rng.uniform(1e-3, 5e-2, (m, ng)).astype(np.float16)
    perm = rng.permutation(d).astype(np.int32) if act else None
    qw, qz = oracle.pack_int4(codes, zeros)
    return codes, zeros, sc.view(np.uint16), perm, qw, qz


def _run(x, qw, sc16, qz, g, perm, tc=False):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)    # noqa: E731
    fn = G.gptq_w4a16_matmul if tc else G.gptq_w4a16_gemm
    y = fn(t(x), t(qw.view(np.int32)), t(sc16.view(np.float16)), t(qz), g,
           None if perm is None else t(perm))
    torch.cuda.synchronize()
    return y.cpu().numpy()


def _bound(x, codes, zeros, sc16, d, g, perm):
    """1e-5 of sum_j |x_j| s (c + z) in original column order"""
    gi = np.arange(d) // (d if g == -1 else g)
    s = sc16.view(np.float16).astype(np.float64)[:, gi]
    mag_sweep = s * (codes.astype(np.float64) + zeros.astype(np.float64)[:, gi])
    mag = np.empty_like(mag_sweep)
    mag[:, perm if perm is not None else np.arange(d)] = mag_sweep
    return 1e-5 * (np.abs(x.astype(np.float64)) @ mag.T)


@pytest.mark.parametrize("m,d,g,b,act", [(300, 256, 128, 1, False), (77, 4096, 128, 4, True),
                                         (33, 14336, 64, 2, False), (129, 1024, 32, 3, True),
                                         (50, 2048, -1, 1, True), (257, 4096, 32, 5, True),
                                         (64, 6144, 128, 8, False)])
def test_w4a16_exact_on_representable_values(m, d, g, b, act):
    rng = np.random.default_rng(1000 + m + d)
    codes, zeros, sc16, perm, qw, qz = _layer(rng, m, d, g, act, exact=True)
    x = rng.integers(-3, 4, (b, d)).astype(np.float16)
    y = _run(x, qw, sc16, qz, g, perm)
    ref = oracle.w4a16_matmul(x, qw, qz, sc16, d, g, perm)
    assert np.array_equal(y.astype(np.float64), ref)


@pytest.mark.parametrize("m,d,g,b,act", [(300, 256, 128, 1, False), (77, 4096, 128, 4, True),
                                         (33, 14336, 64, 2, False), (129, 6144, 256, 2, True),
                                         (50, 2048, -1, 3, False), (200, 4096, 128, 8, True),
                                         (31, 2304, 64, 6, False)])
def test_w4a16_general_within_fp32_bound(m, d, g, b, act):
    rng = np.random.default_rng(2000 + m + d)
    codes, zeros, sc16, perm, qw, qz = _layer(rng, m, d, g, act, exact=False)
    x = rng.standard_normal((b, d)).astype(np.float32)
    x[:, rng.permutation(d)[: max(1, d // 100)]] *= 40.0
    x = x.astype(np.float16)
    y = _run(x, qw, sc16, qz, g, perm)
    ref = oracle.w4a16_matmul(x, qw, qz, sc16, d, g, perm)
    # |x| (s (c + z)) in original column order
    gi = np.arange(d) // (d if g == -1 else g)
    s = sc16.view(np.float16).astype(np.float64)[:, gi]
    mag_sweep = s * (codes.astype(np.float64) + zeros.astype(np.float64)[:, gi])
    mag = np.empty_like(mag_sweep)
    mag[:, perm if perm is not None else np.arange(d)] = mag_sweep
    bound = 1e-5 * (np.abs(x.astype(np.float64)) @ mag.T)
    assert (np.abs(y.astype(np.float64) - ref) <= bound).all()


# ---- the tensor-core path (gptq_w4a16_matmul), any batch -------------------

@pytest.mark.parametrize("m,d,g,b,act", [(300, 256, 128, 1, False), (77, 4096, 128, 16, True),
                                         (130, 1024, 64, 37, False), (129, 2048, -1, 129, True),
                                         (256, 768, 256, 300, False)])
def test_w4a16_tc_exact_on_representable_values(m, d, g, b, act):
    rng = np.random.default_rng(3000 + m + d + b)
    codes, zeros, sc16, perm, qw, qz = _layer(rng, m, d, g, act, exact=True)
    x = rng.integers(-3, 4, (b, d)).astype(np.float16)
    y = _run(x, qw, sc16, qz, g, perm, tc=True)
    ref = oracle.w4a16_matmul(x, qw, qz, sc16, d, g, perm)
    assert np.array_equal(y.astype(np.float64), ref)


@pytest.mark.parametrize("m,d,g,b,act", [(14336, 4096, 128, 1, True), (4096, 14336, 128, 4, False),
                                         (4096, 4096, 128, 200, True), (11008, 4096, 64, 16, False),
                                         (4096, 11008, -1, 3, True)])
def test_w4a16_tc_full_size_within_fp32_bound(m, d, g, b, act):
    """Layers of the 7B / 8B shapes, act-order permutations on and off."""
    rng = np.random.default_rng(4000 + m + d + b)
    codes, zeros, sc16, perm, qw, qz = _layer(rng, m, d, g, act, exact=False)
    x = rng.standard_normal((b, d)).astype(np.float32)
    x[:, rng.permutation(d)[: max(1, d // 100)]] *= 40.0
    x = x.astype(np.float16)
    y = _run(x, qw, sc16, qz, g, perm, tc=True)
    ref = oracle.w4a16_matmul(x, qw, qz, sc16, d, g, perm)
    assert (np.abs(y.astype(np.float64) - ref) <= _bound(x, codes, zeros, sc16, d, g, perm)).all()


def test_w4a16_tc_of_a_gptq_layer():
    """The product of a layer the library quantized and packed (act-order),
    against the oracle's product of the same packed bytes."""
    W = (torch.randn(512, 1024) * 0.02).half().to(DEV)
    X = torch.randn(3000, 1024).half().to(DEV)
    res = G.quantize_layer_from_inputs(W, X, 4, 128, act_order=True)
    x = torch.randn(8, 1024).half().to(DEV)
    y = G.gptq_w4a16_matmul(x, res.qweight, res.scales, res.qzeros, 128, res.perm)
    torch.cuda.synchronize()
    t = lambda a: a.cpu().numpy()                                    # noqa: E731
    qw, qz, sc = t(res.qweight).view(np.uint32), t(res.qzeros), t(res.scales).view(np.uint16)
    ref = oracle.w4a16_matmul(t(x), qw, qz, sc, 1024, 128, t(res.perm))
    codes, zeros = oracle.unpack_int4(qw, qz, 1024, 8)
    assert (np.abs(t(y).astype(np.float64) - ref) <= _bound(t(x), codes, zeros, sc, 1024, 128,
                                                            t(res.perm))).all()

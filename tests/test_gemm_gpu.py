"""The stand-alone split-TF32 tensor-core GEMM (C = beta C + alpha A B^T),
which takes its products the way the factorization and the block update do,
checked directly against a float64 product.  Split-TF32 (Ootomo & Yokota 2022) keeps about fp32 accuracy: the
test bound is 2e-6 * max(1, sqrt(K / 512)) of |alpha| |A| |B|^T + |beta C| per
element (accumulation error grows like sqrt(K); a lost hi/lo term would show
as ~5e-4)."""
import numpy as np
import pytest
import torch

from post_weight_quantization_11_b200 import gptq as G

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


@pytest.mark.parametrize("M,N,K,alpha,beta,lower", [
    (128, 128, 32, 1.0, 0.0, False),
    (300, 200, 64, -1.0, 1.0, False),       # ragged M and N
    (512, 384, 1024, 0.5, -2.0, False),
    (640, 640, 128, -1.0, 1.0, True),       # lower tiles only
    (129, 4, 4096, 1.0, 0.0, False),        # long K, narrow output
    (4096, 128, 128, 1.0, 0.0, False),      # the Cholesky's panel solve shape
])
def test_gemm_nt_matches_float64(M, N, K, alpha, beta, lower):
    g = torch.Generator(device="cpu").manual_seed(M * 7 + N * 13 + K)
    A = torch.randn(M, K, generator=g, dtype=torch.float64)
    B = torch.randn(N, K, generator=g, dtype=torch.float64)
    C0 = torch.randn(M, N, generator=g, dtype=torch.float64)
    A32, B32, C32 = A.float(), B.float(), C0.float()
    C = C32.clone().to(DEV)
    G.gptq_debug_gemm_nt(A32.to(DEV), B32.to(DEV), C, alpha, beta, lower)
    torch.cuda.synchronize()
    got = C.cpu().double()
    ref = beta * C32.double() + alpha * (A32.double() @ B32.double().T)
    scale = (abs(alpha) * (A32.double().abs() @ B32.double().abs().T) + abs(beta) * C32.double().abs())
    if lower:
        mask = torch.zeros(M, N, dtype=torch.bool)
        for tm in range((M + 127) // 128):
            for tn in range(tm + 1):
                mask[tm * 128:(tm + 1) * 128, tn * 128:(tn + 1) * 128] = True
        assert torch.equal(got[~mask], C32.double()[~mask])      # untouched above
        got, ref, scale = got[mask], ref[mask], scale[mask]
    err = (got - ref).abs() / scale.clamp_min(1e-30)
    bound = 2e-6 * max(1.0, (K / 512) ** 0.5)
    assert float(err.max()) <= bound, float(err.max())
    assert G.gptq_device_status(reset=True) == 0

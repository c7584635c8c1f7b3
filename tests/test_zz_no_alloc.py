"""The allocation-free entry point gptq_prepare_hinv_static, for callers that
cannot allocate device memory (for example code running inside a CUDA graph
capture, or a plug-in whose host engine owns all device memory).  Checked
through the C ABI against gptq_prepare_hinv (the workspace version) on the
same inputs, on two calls in a row; its fixed scratch is shared by all calls
and keeps the previous call's contents, so the second call also shows that
nothing stale leaks through.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_11_b200 import gptq as G
from post_weight_quantization_11_b200 import inputs
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    return G.load_library()


def _S(n, d, seed):
    spec = inputs.LayerSpec("t", 1, d, 0.02, "fp16", n, "gauss", 5, 40.0, 40.0, False, seed)
    X = inputs.calibration_x(spec, device="cpu")
    return torch.from_numpy(oracle.hessian(X.numpy()).astype(np.float32)).to(DEV)


def _call_static(lib, S, n, act, free_mem=None):
    """One call through the C ABI; outputs are allocated (by torch) before it.
    free_mem: a list that receives the device's free bytes right before and
    right after the call (the call itself must allocate nothing)."""
    d = S.shape[0]
    perm = torch.empty(d, dtype=torch.int32, device=DEV)
    U = torch.full((d, d), float("nan"), dtype=torch.float32, device=DEV)
    info = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    if free_mem is not None:
        free_mem.append(torch.cuda.mem_get_info()[0])
    st = lib.gptq_prepare_hinv_static(ctypes.c_void_p(S.data_ptr()), d, n, 0.01, int(act),
                                      ctypes.c_void_p(perm.data_ptr()),
                                      ctypes.c_void_p(U.data_ptr()),
                                      ctypes.c_void_p(info.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, G.gptq_status_string(st)
    torch.cuda.synchronize()
    if free_mem is not None:
        free_mem.append(torch.cuda.mem_get_info()[0])
    return perm, U, info


def test_static_scratch_matches_workspace_version(lib):
    """Two calls in a row, each against the workspace version on the same S.
    The factorization is deterministic for a given input (no atomics touch
    its data), so U, perm and info must be equal bit for bit: stale scratch
    from the previous call would show.  Around every call after the first
    (which looks up the scratch's address) the device's free memory must not
    change."""
    cases = [(2048, 512, 31, True), (1536, 1024, 32, False), (2048, 512, 33, False)]
    free = []
    for k, (n, d, seed, act) in enumerate(cases):
        S = _S(n, d, seed)
        p_ref, U_ref, i_ref = G.gptq_prepare_hinv(S, n, 0.01, act)
        p_st, U_st, i_st = _call_static(lib, S, n, act, free if k > 0 else None)
        torch.cuda.synchronize()
        assert int(i_ref.item()) == 0 and int(i_st.item()) == 0
        assert torch.equal(p_ref, p_st)
        assert torch.equal(U_st, U_ref)
        # and both against the oracle's float64 U
        S64 = P.mirror_upper(P.to_np(S))
        _, Hd, _, _, st = oracle.finalize(S64, n, 0.01, act)
        U64, inf = oracle.hinv_upper_chol(Hd)
        assert P.rel_fro(P.to_np(U_st).astype(np.float64), U64) <= P.U_TOL
    assert len(free) == 4 and free[0] == free[1] and free[2] == free[3], free
    assert G.gptq_device_status(reset=True) == 0


def test_static_rejects_d_beyond_limit(lib):
    fake = ctypes.c_void_p(1 << 20)
    assert lib.gptq_prepare_hinv_static(fake, 1152, 10, 0.01, 0, fake, fake, fake, None) == 2

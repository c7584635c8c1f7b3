"""GPU parity of the activation-aware scaling pre-pass ("GPTQ / AWQ /
SqueezeLLM" sec. 二; "INT4/INT8 量化推理" sec. 四) against the oracle's
awq_search / awq_then_gptq, on the GPU's own S and channel sums (the
H-forced protocol of tests/parity.py):

  * channel sums: fp64 on both sides, per channel within 1e-12 relative;
  * losses: every candidate's tr(D H D^T) within 1e-4 relative (the GPU
    takes D H in split-TF32 with D rounded to fp32);
  * the choice: the oracle's first minimizer, or a candidate whose oracle
    loss is within 1e-5 of the minimum (a near-tie of the argmin);
  * the chosen scales within 1e-12 relative of the oracle's s(alpha);
  * GPTQ in the scaled coordinates: the tolerances of every layer test.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_11_b200 import gptq as G
from tests import parity as P
from tests.test_parity_gpu import _gauss_x, _weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


def _inputs(m=192, d=512, n=2000, seed=0):
    W = _weights(m, d, torch.float16, 300 + seed)
    X = _gauss_x(n, d, 6, 40.0, 301 + seed)
    X[:, 7] = 0                                  # a dead channel: its magnitude is 0
    return W, X


def test_channel_abs_sum_matches_oracle():
    _, X = _inputs()
    Xd = X.to(DEV)
    acc = G.gptq_channel_abs_sum(Xd[:700].contiguous())
    G.gptq_channel_abs_sum(Xd[700:].contiguous(), acc)
    torch.cuda.synchronize()
    a_gpu = P.to_np(acc) / X.shape[0]
    a_or = oracle.channel_magnitude(X.numpy())
    assert a_gpu[7] == 0.0 and a_or[7] == 0.0
    nz = a_or > 0
    assert np.all(np.abs(a_gpu[nz] - a_or[nz]) <= 1e-12 * a_or[nz])


@pytest.mark.parametrize("bits,gs,dtype", [(4, 128, torch.float16), (3, 64, torch.float32),
                                           (4, -1, torch.float16)])
def test_awq_search_matches_oracle(bits, gs, dtype):
    W, X = _inputs()
    W = W.to(dtype)
    n, d = X.shape
    Wd, Xd = W.to(DEV), X.to(DEV)
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, Xd)
    acc = G.gptq_channel_abs_sum(Xd)
    res = G.gptq_awq_search(Wd, S, n, acc, 20, bits, gs)
    torch.cuda.synchronize()
    a = P.to_np(acc) / n
    S64 = P.mirror_upper(P.to_np(S))
    ref = oracle.awq_search(W.double().numpy(), S64, n, a, bits, gs, 20)
    lg, lo = P.to_np(res.losses), ref["losses"]
    assert np.all(np.abs(lg - lo) <= 1e-4 * lo), (lg, lo)
    b = int(res.best.item())
    kmin = int(np.argmin(lo))
    assert b == kmin or lo[b] <= (1 + 1e-5) * lo[kmin], (b, kmin, lo)
    s_ref = oracle.awq_candidate_scales(a, b / 20.0)
    assert np.all(np.abs(P.to_np(res.scales) - s_ref) <= 1e-12 * s_ref)
    # the scaled outputs
    Ws = P.to_np(res.W_scaled)
    assert np.array_equal(Ws, (W.double().numpy() * s_ref[None, :]).astype(np.float32))
    Ss = P.to_np(res.S_scaled).astype(np.float64)
    want = np.triu(S64 / np.outer(s_ref, s_ref))
    assert np.all(np.abs(np.triu(Ss) - want) <= 1e-6 * np.abs(want).max())
    assert np.all(np.tril(P.to_np(res.S_scaled), -1) == 0)
    print((bits, gs), "alpha", b / 20.0, "losses", lg[[0, b]])


def test_awq_then_gptq_matches_oracle():
    """GPTQ in the scaled coordinates from the pre-pass's outputs against the
    oracle's GPTQ on (W diag(s), S') with the GPU's S' (H-forced)."""
    W, X = _inputs(m=256, d=1024, n=3000, seed=5)
    n, d = X.shape
    Wd, Xd = W.to(DEV), X.to(DEV)
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, Xd)
    acc = G.gptq_channel_abs_sum(Xd)
    r = G.gptq_awq_search(Wd, S, n, acc, 20, 4, 128)
    perm, U, info = G.gptq_prepare_hinv(r.S_scaled, n, 0.01, False)
    codes, scales, zeros, loss = G.gptq_quantize_layer(r.W_scaled, U, None, 4, 128)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    s = P.to_np(r.scales)
    Wsc = W.double().numpy() * s[None, :]
    Ssc = P.mirror_upper(P.to_np(r.S_scaled))
    ref = oracle.gptq_layer(Wsc, Ssc, n, 4, 128, 0.01, False)
    assert P.rel_fro(P.to_np(U).astype(np.float64), ref["U"]) <= P.U_TOL
    gpu = dict(codes=P.to_np(codes), scales=P.to_np(scales), zeros=P.to_np(zeros))
    P.compare_sweep(gpu, ref, 128)
    P.teacher_forced_check(np.ascontiguousarray(Wsc), ref["U"], gpu, 4, 128)
    # the layer loss in the original coordinates: Q diag(s)^-1 against W with H
    H64 = 2.0 * P.mirror_upper(P.to_np(S)) / n
    Qg = oracle.dequantize(gpu["codes"], gpu["scales"], gpu["zeros"], 128) / s[None, :]
    Qo = oracle.dequantize(ref["codes"], ref["scales"], ref["zeros"], 128) / s[None, :]
    lg = oracle.layer_loss(W.double().numpy(), Qg, H64)
    lo = oracle.layer_loss(W.double().numpy(), Qo, H64)
    assert abs(lg - lo) <= P.LOSS_REL * lo
    # the scaled GPTQ beats the scaling alone (the pre-pass's chosen RTN loss)
    assert lg < float(r.losses[int(r.best.item())].item())

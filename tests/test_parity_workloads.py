"""Full-size parity for the other layer workloads, each run in the launch
configuration bench.py uses (one Hessian call over all 262144 tokens,
prepare, sweep, pack):

  * mlp7b: 7B MLP pair, up 11008x4096 and down 4096x11008 (SiLU-gated X)
  * mlp8b_act: 8B MLP with act-order, 14336x4096 and 4096x14336
  * moe8: all eight 14336x4096 experts, each on its routed tokens (the
    coldest capped at 2048 routed tokens, so its Hessian is rank-deficient)

At these sizes the oracle computes what it can one piece at a time:
  * S: a 96-column block (outlier channels included) over all tokens;
  * perm: the oracle's stable descending argsort of the GPU's diag(S);
  * U: a size-independent backward-error property of the Cholesky factor of
    Hd^-1: U^-1 U^-T v = Hd v for random v (float64 triangular solves with the
    GPU's U), |residual| <= 1e-4 |Hd v|; plus triangular shape and U_jj > 0;
    and sampled rows of U (the first, the last 128, and seeded ones between)
    against the oracle's rows from the same Hd, each the normalized first
    row of the inverse of a trailing sub-Hessian, within the U tolerance
    (the oracle's whole float64 U at d = 4096 is compared in
    test_parity_fullsize.py; at d = 11008 / 14336 it takes minutes);
  * sweep: a seeded sample of rows through the oracle's sweep with the GPU's
    U promoted to float64 (rows are independent given U), the same code,
    scale, zero and loss tolerances as everywhere, plus the teacher-forced
    tie check;
  * packing: bit-exact on the whole layer.
"""
import numpy as np
import pytest
import scipy.linalg as sla
import torch

import oracle
from post_weight_quantization_11_b200 import gptq as G
from post_weight_quantization_11_b200 import inputs
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


def _run_layer(W, X, n, act_order):
    m, d = W.shape
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, X)
    perm, U, info = G.gptq_prepare_hinv(S, n, 0.01, act_order)
    codes, scales, zeros, loss = G.gptq_quantize_layer(W, U, perm if act_order else None, 4, 128)
    qw, qz = G.gptq_pack_int4(codes, zeros)
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0
    assert int(info.item()) == 0
    return dict(S=P.to_np(S), perm=P.to_np(perm), U=P.to_np(U), codes=P.to_np(codes),
                scales=P.to_np(scales), zeros=P.to_np(zeros), loss=P.to_np(loss),
                qw=P.to_np(qw).view(np.uint32), qz=P.to_np(qz))


def _check(spec, W, X, g, seed):
    n = X.shape[0]
    m, d = W.shape
    rng = np.random.default_rng(seed)
    # S: a column block over all tokens
    ch, _ = inputs.outlier_channels(spec)
    cols = np.unique(np.concatenate([ch[:8], rng.choice(d, 88, replace=False)]))
    Xc = X[:, torch.as_tensor(cols, device=DEV)].contiguous().cpu().numpy()
    ref = oracle.hessian(Xc)
    S64 = P.mirror_upper(g["S"])
    assert P.rel_fro(S64[np.ix_(cols, cols)], ref) <= P.S_TOL
    # perm
    diag = 2.0 * np.diag(S64) / n
    perm = oracle.act_order_perm(diag) if spec.act_order else np.arange(d, dtype=np.int32)
    assert np.array_equal(g["perm"], perm)
    # U: backward error of the factorization, U^-1 U^-T v = Hd v
    U64 = g["U"].astype(np.float64)
    assert np.all(np.tril(U64, -1) == 0) and np.all(np.diag(U64) > 0)
    lam = 0.01 * diag.mean()
    for _ in range(4):
        v = rng.standard_normal(d)
        w = np.empty(d)
        w[perm] = v                                   # H[perm][:, perm] v = (H w)[perm]
        hv = (2.0 / n) * (S64 @ w)[perm] + lam * v
        z = sla.solve_triangular(U64, sla.solve_triangular(U64, v, trans="T"), trans="N")
        assert np.linalg.norm(z - hv) <= 1e-4 * np.linalg.norm(hv)
    # U: sampled rows against the oracle's rows of the same Hd
    Hd = (2.0 / n) * S64[np.ix_(perm, perm)]
    Hd[np.arange(d), np.arange(d)] += lam
    urows = np.unique(np.concatenate([[0, 1, d // 3, (2 * d) // 3], np.arange(d - 128, d),
                                      rng.choice(d, 4, replace=False)]))
    R = oracle.u_rows(Hd, urows)
    del Hd
    u_err = P.rel_fro(U64[urows], R)
    assert u_err <= P.U_TOL, u_err
    # sweep on sampled rows with the GPU's U
    rows = np.sort(rng.choice(m, 24, replace=False))
    W64 = W[torch.as_tensor(rows, device=DEV)].double().cpu().numpy()
    Wp = np.ascontiguousarray(W64[:, perm])
    res = oracle.quantize_rows(Wp, U64, 4, 128)
    gpu = dict(codes=g["codes"][rows], scales=g["scales"][rows], zeros=g["zeros"][rows])
    st = P.compare_sweep(gpu, res, 128)
    assert abs(g["loss"][rows].sum() - res["row_loss"].sum()) <= P.LOSS_REL * res["row_loss"].sum()
    tf = {}
    P.teacher_forced_check(Wp, U64, gpu, 4, 128, report=tf)
    st.update(tf, u_rows_rel_err=u_err)
    # packing of the whole layer
    rq, rz = oracle.pack_int4(g["codes"], g["zeros"])
    assert np.array_equal(g["qw"], rq) and np.array_equal(g["qz"], rz)
    return st


@pytest.mark.parametrize("workload,layer", [("mlp7b", 0), ("mlp7b", 1), ("mlp8b_act", 0),
                                            ("mlp8b_act", 1)])
def test_dense_workload_layer(workload, layer):
    spec = inputs.WORKLOADS[workload].layers[layer]
    W = inputs.weights(spec, device=DEV)
    X = inputs.calibration_x(spec, device=DEV)
    g = _run_layer(W, X, X.shape[0], spec.act_order)
    st = _check(spec, W, X, g, 100 + layer)
    print(workload, layer, st)
    del X
    torch.cuda.empty_cache()


@pytest.fixture(scope="module")
def moe8_batched():
    """The whole MoE layer through the batched path, as bench.py runs it:
    routed rows gathered expert-major, one grouped Hessian launch, one
    factorization launch for the eight experts, the batched sweep, one pack."""
    wl = inputs.WORKLOADS["moe8"]
    spec0 = wl.layers[0]
    X = inputs.calibration_x(spec0, device=DEV)
    lists = inputs.moe_routing(X.shape[0], wl.n_experts, wl.zipf_s, wl.top_k, wl.cold_cap,
                               spec0.seed)
    W = torch.stack([inputs.weights(sp, device=DEV) for sp in wl.layers]).contiguous()
    routes = [torch.as_tensor(np.asarray(r), dtype=torch.int32, device=DEV) for r in lists]
    res = G.quantize_moe_from_inputs(W, X, routes)
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0
    assert not P.to_np(res.info).any()
    out = dict(wl=wl, X=X, lists=lists, W=W, res=res)
    yield out
    del out, X, W, res
    torch.cuda.empty_cache()


@pytest.mark.parametrize("expert", range(8))
def test_moe_expert(moe8_batched, expert):
    """Every expert of the MoE layer on its own routed tokens (the coldest
    capped at 2048, rank-deficient before damping), all eight quantized by
    the batched entry points in one pass."""
    b = moe8_batched
    wl, res = b["wl"], b["res"]
    counts = [len(x) for x in b["lists"]]
    assert sum(counts) <= 2 * b["X"].shape[0] and min(counts) == wl.cold_cap
    spec = wl.layers[expert]
    Xe = b["X"].index_select(0, torch.as_tensor(b["lists"][expert], device=DEV)).contiguous()
    e = expert
    g = dict(S=P.to_np(res.S[e]), perm=P.to_np(res.perm[e]), U=P.to_np(res.U[e]),
             codes=P.to_np(res.codes[e]), scales=P.to_np(res.scales[e]),
             zeros=P.to_np(res.zeros[e]), loss=P.to_np(res.row_loss[e]),
             qw=P.to_np(res.qweight[e]).view(np.uint32), qz=P.to_np(res.qzeros[e]))
    st = _check(spec, b["W"][e], Xe, g, 200 + e)
    print("expert", e, "tokens", counts[e], st)

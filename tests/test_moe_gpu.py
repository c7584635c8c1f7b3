"""GPU tests of the mixture-of-experts path ("INT4/INT8 量化推理" sec. 五:
every expert is calibrated on its own routed tokens): the routed-row gather,
the grouped Hessian (one launch, one S per expert, ragged segments), and
the batched preparation and quantization, each against the oracle and
against the single-layer entry points (same kernels, same inputs: equal bit
for bit).  Tolerances are those of tests/parity.py."""
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


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0, "a bounded device wait gave up"


def test_gather_rows_bit_exact():
    X = _gauss_x(3000, 384, 3, 50.0, 5)
    rng = np.random.default_rng(6)
    idx = rng.integers(0, 3000, 5000).astype(np.int32)            # repeats included
    out = G.gptq_gather_rows(X.to(DEV), torch.from_numpy(idx).to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(P.to_np(out), X.numpy().view(np.uint16)[idx])


def test_gather_rows_out_of_range_index_is_not_followed():
    X = _gauss_x(100, 128, 0, 1.0, 7).to(DEV)
    idx = torch.tensor([3, -1, 99, 100, 5], dtype=torch.int32, device=DEV)
    out = G.gptq_gather_rows(X, idx)
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0x201
    o = P.to_np(out)
    x = P.to_np(X)
    assert np.array_equal(o[[0, 2, 4]], x[[3, 99, 5]])
    assert not o[[1, 3]].any()


@pytest.mark.parametrize("d,lens", [
    (256, [0, 37, 64, 1000, 4099, 130]),     # empty, shorter than a box, ragged ends
    (384, [5000, 1, 700]),
    (128, [3] * 70),                         # more than one launch of 64 groups
])
def test_grouped_hessian_parity(d, lens):
    n = sum(lens)
    X = _gauss_x(max(n, 1), d, 3, 50.0, d + n)[:n]
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    E = len(lens)
    S = torch.zeros(E, d, d, dtype=torch.float32, device=DEV)
    counts = G.gptq_hessian_accumulate_grouped(S, X.to(DEV).contiguous(), off)
    assert counts == lens
    # a second call adds the same sums again
    G.gptq_hessian_accumulate_grouped(S, X.to(DEV).contiguous(), off)
    torch.cuda.synchronize()
    Sg = P.to_np(S)
    Xn = X.numpy()
    for e in range(E):
        ref = 2.0 * oracle.hessian(Xn[off[e]:off[e + 1]]) if lens[e] else np.zeros((d, d))
        assert np.all(np.tril(Sg[e], -1) == 0)
        if lens[e] == 0:
            assert not Sg[e].any()
            continue
        assert P.rel_fro(np.triu(Sg[e].astype(np.float64)), np.triu(ref)) <= P.S_TOL, e


def test_grouped_hessian_equals_the_dense_call_on_one_group():
    """One group takes the dense call's work split; the two differ only in
    the order of the items' fp32 atomic adds into S."""
    X = _gauss_x(4099, 512, 5, 40.0, 17).to(DEV)
    S1 = torch.zeros(1, 512, 512, dtype=torch.float32, device=DEV)
    S2 = torch.zeros(512, 512, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate_grouped(S1, X, [0, 4099])
    G.gptq_hessian_accumulate(S2, X)
    torch.cuda.synchronize()
    a, b = P.to_np(S1[0]).astype(np.float64), P.to_np(S2).astype(np.float64)
    assert P.rel_fro(a, b) <= 1e-6


def _expert_set(d=512, lens=(3000, 700, 256), seed=30):
    """Hessians of a few experts; the last one rank-deficient (fewer tokens than d)."""
    Xs = [_gauss_x(n, d, 4, 30.0, seed + i) for i, n in enumerate(lens)]
    S = torch.stack([torch.from_numpy(oracle.hessian(x.numpy()).astype(np.float32)) for x in Xs])
    return S.to(DEV).contiguous(), list(lens)


@pytest.mark.parametrize("act_order", [False, True])
def test_batched_prepare_equals_single_and_oracle(act_order):
    S, lens = _expert_set()
    E, d = S.shape[0], S.shape[1]
    perm_b, U_b, info_b = G.gptq_prepare_hinv_batched(S, lens, 0.01, act_order)
    torch.cuda.synchronize()
    assert not P.to_np(info_b).any()
    for e in range(E):
        perm_s, U_s, info_s = G.gptq_prepare_hinv(S[e].contiguous(), lens[e], 0.01, act_order)
        torch.cuda.synchronize()
        assert int(info_s.item()) == 0
        assert torch.equal(U_b[e], U_s), e
        assert torch.equal(perm_b[e], perm_s), e
        S64 = P.mirror_upper(P.to_np(S[e]))
        H, Hd, rperm, lam, st = oracle.finalize(S64, lens[e], 0.01, act_order)
        U64, inf = oracle.hinv_upper_chol(Hd)
        assert np.array_equal(P.to_np(perm_b[e]), rperm)
        assert P.rel_fro(P.to_np(U_b[e]).astype(np.float64), U64) <= P.U_TOL


def test_batched_prepare_reports_each_matrix_pivot():
    S, lens = _expert_set(d=256, lens=(900, 300))
    S = torch.cat([S, torch.zeros(1, 256, 256, device=DEV)]).contiguous()   # no PD matrix
    _, _, info = G.gptq_prepare_hinv_batched(S, lens + [50], 0.01, False)
    torch.cuda.synchronize()
    inf = P.to_np(info)
    assert inf[0] == 0 and inf[1] == 0 and inf[2] != 0


@pytest.mark.parametrize("act_order,dtype,gs,shared", [
    (False, torch.float16, 128, False),   # a workspace per layer: the layers swept together
    (True, torch.float32, 128, False),
    (False, torch.float16, 64, False),
    (False, torch.float16, 128, True),    # one shared workspace: one layer after the other
    (False, torch.float16, 256, False),   # 256-column dynamic groups: per-block launches
])
def test_batched_quantize_equals_single_and_oracle(act_order, dtype, gs, shared):
    S, lens = _expert_set(d=512, lens=(2000, 400, 1500), seed=40)
    E, d = S.shape[0], S.shape[1]
    m = 200
    W = torch.stack([_weights(m, d, dtype, 50 + e) for e in range(E)]).to(DEV).contiguous()
    perm, U, info = G.gptq_prepare_hinv_batched(S, lens, 0.01, act_order)
    codes, scales, zeros, loss = G.gptq_quantize_layer_batched(
        W, U, perm if act_order else None, 4, gs, shared_workspace=shared)
    torch.cuda.synchronize()
    for e in range(E):
        c, s, z, l = G.gptq_quantize_layer(W[e].contiguous(), U[e].contiguous(),
                                           perm[e].contiguous() if act_order else None, 4, gs)
        torch.cuda.synchronize()
        assert torch.equal(codes[e], c) and torch.equal(scales[e], s)
        assert torch.equal(zeros[e], z) and torch.equal(loss[e], l)
        # against the oracle's sweep with the same U (the H-forced protocol)
        Wp = np.ascontiguousarray(W[e].double().cpu().numpy()[:, P.to_np(perm[e])])
        U64 = P.to_np(U[e]).astype(np.float64)
        ref = oracle.quantize_rows(Wp, U64, 4, gs)
        gpu = dict(codes=P.to_np(codes[e]), scales=P.to_np(scales[e]), zeros=P.to_np(zeros[e]))
        P.compare_sweep(gpu, ref, gs)
        P.teacher_forced_check(Wp, U64, gpu, 4, gs)
    qw, qz = G.gptq_pack_int4(codes.view(E * m, d), zeros.view(E * m, -1))
    rq, rz = oracle.pack_int4(P.to_np(codes).reshape(E * m, d), P.to_np(zeros).reshape(E * m, -1))
    assert np.array_equal(P.to_np(qw).view(np.uint32), rq) and np.array_equal(P.to_np(qz), rz)


def test_moe_layer_driver_small():
    """quantize_moe_from_inputs on a small MoE: routes with repeats across
    experts, one expert with fewer tokens than d; each expert's S against
    the oracle on its routed rows, its codes against the single-layer path
    (the two S differ in the order of fp32 atomic adds, so codes may part at
    ties: the code tolerance of tests/parity.py)."""
    E, m, d, n = 4, 96, 256, 3000
    X = _gauss_x(n, d, 3, 40.0, 61).to(DEV)
    rng = np.random.default_rng(62)
    routes = [torch.from_numpy(np.sort(rng.choice(n, k, replace=False)).astype(np.int32)).to(DEV)
              for k in (2500, 900, 130, 1200)]
    W = torch.stack([_weights(m, d, torch.float16, 70 + e) for e in range(E)]).to(DEV).contiguous()
    res = G.quantize_moe_from_inputs(W, X, routes)
    torch.cuda.synchronize()
    assert not P.to_np(res.info).any()
    Xn = X.cpu().numpy()
    for e in range(E):
        r = P.to_np(routes[e])
        ref = oracle.hessian(Xn[r])
        assert P.rel_fro(np.triu(P.to_np(res.S[e]).astype(np.float64)), np.triu(ref)) <= P.S_TOL
        one = G.quantize_layer_from_inputs(W[e].contiguous(), X.index_select(0, routes[e].long()))
        torch.cuda.synchronize()
        frac = float((P.to_np(one.codes) != P.to_np(res.codes[e])).mean())
        assert frac <= P.CODE_FRAC, (e, frac)
        qw, qz = G.gptq_pack_int4(res.codes[e].contiguous(), res.zeros[e].contiguous())
        assert torch.equal(qw, res.qweight[e]) and torch.equal(qz, res.qzeros[e])

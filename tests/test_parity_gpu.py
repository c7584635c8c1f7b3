"""GPU parity: the CUDA path (through the C ABI binding) against the float64
oracle on the same seeded inputs.  Tolerances are stated in tests/parity.py."""
import numpy as np
import pytest
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


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0, "a bounded device wait gave up"


def _gauss_x(n, d, n_out, fac, seed):
    spec = inputs.LayerSpec("t", 1, d, 0.02, "fp16", n, "gauss", n_out, fac, fac, False, seed)
    return inputs.calibration_x(spec, device="cpu")


def _weights(m, d, dtype, seed, std=0.02):
    spec = inputs.LayerSpec("t", m, d, std, "fp32" if dtype == torch.float32 else "fp16", 1,
                            "gauss", 0, 1, 1, False, seed)
    return inputs.weights(spec, device="cpu")


def _gpu_layer(W, X, bits=4, group_size=128, act_order=False, damp=0.01):
    Wd, Xd = W.to(DEV), X.to(DEV)
    d = W.shape[1]
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, Xd)
    perm, U, info = G.gptq_prepare_hinv(S, X.shape[0], damp, act_order)
    codes, scales, zeros, loss = G.gptq_quantize_layer(Wd, U, perm if act_order else None,
                                                       bits, group_size)
    torch.cuda.synchronize()
    return dict(S=P.to_np(S), perm=P.to_np(perm), U=P.to_np(U), info=int(info.item()),
                codes=P.to_np(codes), scales=P.to_np(scales), zeros=P.to_np(zeros),
                row_loss=P.to_np(loss))


def _check_layer(W, X, bits=4, group_size=128, act_order=False, rows=None, code_bar="free"):
    """H-forced protocol: the oracle takes the GPU's S (promoted to fp64).
    code_bar "free": at most 1e-3 of the codes differ in the free-running
    comparison (every later code a tie flip changes counts too), and the
    scale and zero-point bars hold there too; "forced": the 1e-3 bar counts
    the codes the oracle decides differently on the GPU's own trajectory
    (the teacher-forced run), i.e. the tie flips themselves, and the scale
    and zero-point bars are those of that run -- the reading for widths
    other than 4 bits, where one tie flip moves tens to hundreds of later
    codes of its row."""
    n = X.shape[0]
    g = _gpu_layer(W, X, bits, group_size, act_order)
    assert g["info"] == 0
    S_or = oracle.hessian(X.numpy())
    S_gpu = P.mirror_upper(g["S"])
    assert P.rel_fro(S_gpu, S_or) <= P.S_TOL
    W64 = W.double().numpy()
    ref = oracle.gptq_layer(W64, S_gpu, n, bits, group_size, 0.01, act_order)
    assert np.array_equal(g["perm"], ref["perm"]) if act_order else True
    assert P.rel_fro(g["U"].astype(np.float64), ref["U"]) <= P.U_TOL
    st = P.compare_sweep(g, dict(codes=ref["codes"], scales=ref["scales"], zeros=ref["zeros"],
                                 s_pre=ref["s_pre"]), group_size,
                         code_frac=P.CODE_FRAC if code_bar == "free" else 1.0,
                         group_bars=code_bar == "free")
    H64 = 2.0 * S_gpu / n
    perm = ref["perm"]
    lg = P.layer_loss_of(W64, g["codes"], g["scales"], g["zeros"], group_size, perm, H64)
    lo = P.layer_loss_of(W64, ref["codes"], ref["scales"], ref["zeros"], group_size, perm, H64)
    assert abs(lg - lo) <= P.LOSS_REL * lo, (lg, lo)
    # the GPU's own bookkeeping: sum E_j^2 = tr(D Hd D^T)
    assert abs(g["row_loss"].sum() - ref["row_loss"].sum()) <= P.LOSS_REL * ref["row_loss"].sum()
    Wp = np.ascontiguousarray(W64[:, perm])
    n_ties = P.teacher_forced_check(Wp, ref["U"], g, bits, group_size, rows)
    if code_bar == "forced":
        n_w = g["codes"].size if rows is None else len(rows) * g["codes"].shape[1]
        assert n_ties <= P.CODE_FRAC * n_w, (n_ties, n_w)
    st.update(loss_gpu=lg, loss_oracle=lo, teacher_forced_ties=n_ties)
    return st, g, ref


# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits,gs", [(4, 128), (4, 64), (3, 32), (2, 128), (8, 64), (4, 256),
                                     (3, 384), (4, -1), (8, -1)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16])
def test_rtn_bit_exact(bits, gs, dtype):
    W = _weights(300, 768, dtype, 3)
    W[5, :] = 0                       # an all-zero row: degenerate groups
    W[7, :128] = -0.01                # one-signed group
    c, s, z = G.rtn_quantize(W.to(DEV), bits, gs)
    ref = oracle.rtn(W.double().numpy(), bits, gs)
    assert np.array_equal(P.to_np(c), ref["codes"])
    assert np.array_equal(P.to_np(s), ref["scales"])
    assert np.array_equal(P.to_np(z), ref["zeros"])


@pytest.mark.parametrize("m,d,G_", [(1, 128, 1), (300, 1024, 8), (77, 256, 3), (5, 8, 1)])
def test_pack_bit_exact(m, d, G_):
    rng = np.random.default_rng(m + d)
    codes = rng.integers(0, 16, (m, d), dtype=np.uint8)
    zeros = rng.integers(0, 16, (m, G_), dtype=np.uint8)
    qw, qz = G.gptq_pack_int4(torch.from_numpy(codes).to(DEV), torch.from_numpy(zeros).to(DEV))
    rq, rz = oracle.pack_int4(codes, zeros)
    assert np.array_equal(P.to_np(qw).view(np.uint32), rq)
    assert np.array_equal(P.to_np(qz), rz)
    c2, z2 = G.gptq_unpack_int4(qw, qz, d, G_)
    assert np.array_equal(P.to_np(c2), codes) and np.array_equal(P.to_np(z2), zeros)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("m,d,G_", [(1, 32, 1), (77, 256, 3), (300, 1024, 8), (5, 4096, 33)])
def test_pack_bits_bit_exact(bits, m, d, G_):
    """b-bit packing against the oracle's bit stream (and, at b = 4, against
    the INT4 packing), with the round trip."""
    rng = np.random.default_rng(bits * 1000 + m + d)
    codes = rng.integers(0, 1 << bits, (m, d), dtype=np.uint8)
    zeros = rng.integers(0, 1 << bits, (m, G_), dtype=np.uint8)
    qw, qz = G.gptq_pack_bits(torch.from_numpy(codes).to(DEV), torch.from_numpy(zeros).to(DEV),
                              bits)
    rq, rz = oracle.pack_bits(codes, zeros, bits)
    assert np.array_equal(P.to_np(qw).view(np.uint32), rq)
    assert np.array_equal(P.to_np(qz), rz)
    c2, z2 = G.gptq_unpack_bits(qw, qz, d, G_, bits)
    assert np.array_equal(P.to_np(c2), codes) and np.array_equal(P.to_np(z2), zeros)
    if bits == 4:
        q4w, q4z = G.gptq_pack_int4(torch.from_numpy(codes).to(DEV),
                                    torch.from_numpy(zeros).to(DEV))
        assert torch.equal(q4w, qw) and torch.equal(q4z, qz)


def test_pack_bits_of_gptq_results_at_3_and_8_bits():
    """INT3 and INT8 layers quantized by the sweep, packed, unpacked, and
    dequantized back to the sweep's own values."""
    W = _weights(128, 512, torch.float16, 5).to(DEV)
    X = _gauss_x(2000, 512, 3, 30.0, 6).to(DEV)
    for bits in (3, 8):
        res = G.quantize_layer_from_inputs(W, X, bits, 128, pack=False)
        qw, qz = G.gptq_pack_bits(res.codes, res.zeros, bits)
        torch.cuda.synchronize()
        rq, rz = oracle.pack_bits(P.to_np(res.codes), P.to_np(res.zeros), bits)
        assert np.array_equal(P.to_np(qw).view(np.uint32), rq) and np.array_equal(P.to_np(qz), rz)
        nbytes = qw.numel() * 4 + qz.numel() + res.scales.numel() * 2
        m, d, G_ = 128, 512, 4          # b bits per weight, b per zero point (bytes padded)
        assert nbytes == m * d * bits // 8 + m * ((G_ * bits + 7) // 8) + 2 * m * G_


@pytest.mark.parametrize("n,d", [(512, 256), (777, 384), (64, 128), (4099, 1024), (60001, 1152)])
def test_hessian_parity(n, d):
    X = _gauss_x(n, d, 3, 50.0, d + n)
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    S.fill_(0)
    Xd = X.to(DEV)
    # two batches accumulate into the same S
    G.gptq_hessian_accumulate(S, Xd[: n // 3])
    G.gptq_hessian_accumulate(S, Xd[n // 3:])
    G.gptq_hessian_accumulate(S, Xd[:0])  # empty batch: no-op
    Sg = P.to_np(S)
    ref = oracle.hessian(X.numpy())
    assert P.rel_fro(np.triu(Sg.astype(np.float64)), np.triu(ref)) <= P.S_TOL
    assert np.all(np.tril(Sg, -1) == 0)   # lower triangle untouched


@pytest.mark.parametrize("n,d,chunk,pinned", [(5000, 256, 1024, True), (777, 384, 4096, True),
                                              (3000, 128, 700, False)])
def test_hessian_from_host_memory(n, d, chunk, pinned):
    """The host-streamed accumulation: ragged last chunks, a batch smaller
    than one chunk, pageable memory, and a second batch through the same
    ring (its first copies wait for the first batch's last accumulation)."""
    X = _gauss_x(n, d, 3, 50.0, d + n + 1).contiguous()
    Xh = X.pin_memory() if pinned else X
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    hh = G.HostHessian(d, DEV, chunk_tokens=chunk)
    assert hh.accumulate(S, Xh) == n
    assert hh.accumulate(S, Xh[: n // 2]) == n // 2
    torch.cuda.synchronize()
    Sg = P.to_np(S)
    ref = oracle.hessian(np.concatenate([X.numpy(), X.numpy()[: n // 2]]))
    assert P.rel_fro(np.triu(Sg.astype(np.float64)), np.triu(ref)) <= P.S_TOL
    assert np.all(np.tril(Sg, -1) == 0)


def test_sharded_layer_on_one_process_matches_the_direct_path():
    """The one-layer-over-ranks driver without a process group: the same
    library calls as quantize_layer_from_inputs, on real kernels."""
    from post_weight_quantization_11_b200 import sharded
    W = _weights(300, 512, torch.float16, 21)
    X = _gauss_x(3000, 512, 3, 50.0, 22)
    Wd, Xd = W.to(DEV), X.to(DEV)
    L = sharded.ShardedLayer(300, 512, 3000, DEV)
    assert L.rows == (0, 300) and L.n_total == 3000
    L.step(Wd, Xd)
    ref = G.quantize_layer_from_inputs(Wd, Xd)
    torch.cuda.synchronize()
    assert int(L.info.item()) == 0
    S1, S2 = P.to_np(L.S).astype(np.float64), P.to_np(ref.S).astype(np.float64)
    assert P.rel_fro(np.triu(S1), np.triu(S2)) <= 1e-6
    assert float((P.to_np(L.codes) != P.to_np(ref.codes)).mean()) <= 1e-3
    qw, qz = G.gptq_pack_int4(L.codes, L.zeros)
    assert torch.equal(qw, L.qweight) and torch.equal(qz, L.qzeros)


@pytest.mark.parametrize("gs,static,act", [(32, True, False), (128, True, True), (256, True, False),
                                           (-1, True, False), (-1, False, True)])
def test_static_and_per_channel_groups(gs, static, act):
    """Static groups (parameters from the rows before the sweep) and one
    group per row, against the oracle on the GPU's S: the parameters come
    from the uncorrected weights, so scales and zero points are bit-exact;
    codes and loss as in every layer test.  d = 1024 takes the far update.
    (Dynamic groups wider than a block: test_wide_dynamic_groups.)"""
    m, d, n = 200, 1024, 2048
    W = _weights(m, d, torch.float16, 31)
    X = _gauss_x(n, d, 3, 50.0, 32)
    Wd, Xd = W.to(DEV), X.to(DEV)
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, Xd)
    perm, U, info = G.gptq_prepare_hinv(S, n, 0.01, act)
    codes, scales, zeros, _ = G.gptq_quantize_layer(Wd, U, perm if act else None, 4, gs,
                                                    static_groups=static)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    S64 = P.mirror_upper(P.to_np(S))
    _, Hd, perm_o, _, st = oracle.finalize(S64, n, 0.01, act)
    U_o, inf = oracle.hinv_upper_chol(Hd)
    assert st == 0 and inf == 0
    assert np.array_equal(P.to_np(perm), perm_o)
    W64 = W.double().numpy()
    Wp = np.ascontiguousarray(W64[:, perm_o])
    ref = (oracle.quantize_rows_static if static else oracle.quantize_rows)(Wp, U_o, 4, gs)
    sc, zr, cd = P.to_np(scales), P.to_np(zeros), P.to_np(codes)
    assert np.array_equal(sc, ref["scales"]) and np.array_equal(zr, ref["zeros"])
    assert float((cd != ref["codes"]).mean()) <= P.CODE_FRAC
    H64 = 2.0 * S64 / n
    lg = P.layer_loss_of(W64, cd, sc, zr, gs, perm_o, H64)
    lo = P.layer_loss_of(W64, ref["codes"], ref["scales"], ref["zeros"], gs, perm_o, H64)
    assert abs(lg - lo) <= P.LOSS_REL * lo, (lg, lo)


@pytest.mark.parametrize("gs,act,d", [(256, False, 1024), (256, True, 1536), (512, False, 2048),
                                      (1024, True, 2048)])
def test_wide_dynamic_groups(gs, act, d):
    """Dynamic groups wider than one 128-column block: each group's
    parameters come from the row as it stands at the group's first column,
    after every earlier column's correction (the oracle's unblocked sweep
    takes them exactly there), through the full H-forced protocol of
    _check_layer, teacher-forced tie check included."""
    W = _weights(160, d, torch.float16, 90 + gs)
    X = _gauss_x(3 * d, d, max(1, d // 100), 40.0, 91 + gs)
    st, _, _ = _check_layer(W, X, 4, gs, act)
    print((gs, act, d), st)


@pytest.mark.parametrize("act", [False, True])
def test_sharded_layer_against_the_oracle(monkeypatch, act):
    """The one-layer-over-ranks driver as three ranks would run it, on real
    kernels in one process: each emulated rank accumulates S over its token
    share (unequal shares), the all-reduce is emulated by summing the ranks'
    S, every rank prepares U and quantizes its share of the rows (an odd row
    count).  The concatenated codes, scales and zero points against the
    oracle on the summed S (H-forced protocol), packing bit-exact."""
    import torch.distributed as dist
    from post_weight_quantization_11_b200 import sharded
    world, m, d, n = 3, 301, 512, 3001
    W = _weights(m, d, torch.float16, 41 + act)
    X = _gauss_x(n, d, 4, 40.0, 42 + act)
    Wd, Xd = W.to(DEV), X.to(DEV)
    monkeypatch.setattr(dist, "all_reduce", lambda *a, **k: None)   # emulated below
    monkeypatch.setattr(sharded.ShardedLayer, "_sum_over_ranks", lambda self, v, dev: n)
    ranks = []
    for r in range(world):
        monkeypatch.setattr(sharded, "_world", lambda g, r=r: (world, r))
        t0, t1 = sharded.share(n, world, r)
        L = sharded.ShardedLayer(m, d, t1 - t0, DEV, act_order=act)
        L.hessian(Xd[t0:t1].contiguous())
        ranks.append(L)
    S_sum = sum(L.S for L in ranks)
    for L in ranks:
        L.S.copy_(S_sum)                                  # what the all-reduce leaves
        lo, hi = L.rows
        L.quantize(Wd[lo:hi].contiguous())
    torch.cuda.synchronize()
    assert all(int(L.info.item()) == 0 for L in ranks)
    g = dict(codes=np.concatenate([P.to_np(L.codes) for L in ranks]),
             scales=np.concatenate([P.to_np(L.scales) for L in ranks]),
             zeros=np.concatenate([P.to_np(L.zeros) for L in ranks]))
    S64 = P.mirror_upper(P.to_np(S_sum))
    assert P.rel_fro(S64, oracle.hessian(X.numpy())) <= P.S_TOL
    ref = oracle.gptq_layer(W.double().numpy(), S64, n, 4, 128, 0.01, act)
    assert all(np.array_equal(P.to_np(L.perm), ref["perm"]) for L in ranks)
    P.compare_sweep(g, ref, 128)
    Wp = np.ascontiguousarray(W.double().numpy()[:, ref["perm"]])
    P.teacher_forced_check(Wp, ref["U"], g, 4, 128)
    rq, rz = oracle.pack_int4(g["codes"], g["zeros"])
    qw = np.concatenate([P.to_np(L.qweight).view(np.uint32) for L in ranks])
    qz = np.concatenate([P.to_np(L.qzeros) for L in ranks])
    assert np.array_equal(qw, rq) and np.array_equal(qz, rz)


@pytest.mark.parametrize("act_order,d", [(False, 512), (True, 512), (False, 640), (True, 1152)])
def test_prepare_parity(act_order, d):
    n = 2048
    X = _gauss_x(n, d, 5, 40.0, 11)
    S = torch.from_numpy(oracle.hessian(X.numpy()).astype(np.float32)).to(DEV)
    perm, U, info = G.gptq_prepare_hinv(S, n, 0.01, act_order)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    S64 = P.mirror_upper(P.to_np(S))
    H, Hd, rperm, lam, st = oracle.finalize(S64, n, 0.01, act_order)
    U64, inf = oracle.hinv_upper_chol(Hd)
    assert np.array_equal(P.to_np(perm), rperm)
    Ug = P.to_np(U).astype(np.float64)
    assert np.all(np.tril(Ug, -1) == 0)
    assert P.rel_fro(Ug, U64) <= P.U_TOL


def test_prepare_kms_closed_form():
    """The GPU's U for H = KMS(0.7) (H_ij = 0.7^|i-j|, no damping) against
    its closed form, an upper bidiagonal matrix (every entry checked, the
    zeros included): no oracle involved."""
    d, n, rho = 512, 1000, 0.7
    i = np.arange(d)
    H = rho ** np.abs(i[:, None] - i[None, :])
    S = torch.from_numpy((n / 2.0) * H).float().to(DEV)
    perm, U, info = G.gptq_prepare_hinv(S, n, 0.0, False)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    c = np.sqrt(1.0 - rho * rho)
    ref = np.zeros((d, d))
    ref[i[:-1], i[:-1]] = 1.0 / c
    ref[d - 1, d - 1] = 1.0
    ref[i[:-1], i[1:]] = -rho / c
    Ug = P.to_np(U).astype(np.float64)
    assert np.abs(Ug - ref).max() <= 1e-5 * np.abs(ref).max()
    assert np.array_equal(P.to_np(perm), np.arange(d, dtype=np.int32))


def test_gptq_equals_rtn_when_hessian_is_isotropic():
    """X of Hadamard rows: X^T X = n I exactly (integer sums), so U is diagonal
    and the error feedback vanishes; the GPU's GPTQ must then give the GPU's
    and the oracle's round-to-nearest codes, scales and zero points bit for
    bit, with and without act-order (equal diagonal: identity order)."""
    d, reps = 256, 2
    Hd_ = np.array([[1.0]])
    while Hd_.shape[0] < d:
        Hd_ = np.block([[Hd_, Hd_], [Hd_, -Hd_]])
    X = torch.from_numpy(np.vstack([Hd_] * reps).astype(np.float16)).to(DEV)
    n = X.shape[0]
    W = _weights(96, d, torch.float16, 43).to(DEV)
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S, X)
    Sg = P.to_np(S)
    assert np.array_equal(np.triu(Sg), n * np.eye(d, dtype=np.float32))
    rc, rs, rz = G.rtn_quantize(W, 4, 128)
    ref = oracle.rtn(W.double().cpu().numpy(), 4, 128)
    assert np.array_equal(P.to_np(rc), ref["codes"])
    for act in (False, True):
        perm, U, info = G.gptq_prepare_hinv(S, n, 0.01, act)
        c, sc, z, _ = G.gptq_quantize_layer(W, U, perm if act else None, 4, 128)
        torch.cuda.synchronize()
        assert int(info.item()) == 0
        Ug = P.to_np(U)
        assert np.array_equal(Ug, np.diag(np.diag(Ug)))
        assert np.array_equal(P.to_np(perm), np.arange(d, dtype=np.int32))
        assert np.array_equal(P.to_np(c), P.to_np(rc))
        assert np.array_equal(P.to_np(sc), P.to_np(rs)) and np.array_equal(P.to_np(z), P.to_np(rz))


def test_cta_caps_keep_the_results():
    """The persistent kernels on fewer CTAs than SMs: the Hessian sums in
    another order (within fp32 rounding), the factorization's tasks do the
    same arithmetic whichever CTA runs them (U bit for bit)."""
    d, n = 1024, 4096
    X = _gauss_x(n, d, 3, 50.0, 51).to(DEV)
    S0 = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    G.gptq_hessian_accumulate(S0, X)
    _, U0, info0 = G.gptq_prepare_hinv(S0, n, 0.01, False)
    try:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, 24)
        G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, 7)
        S1 = torch.zeros_like(S0)
        G.gptq_hessian_accumulate(S1, X)
        _, U1, info1 = G.gptq_prepare_hinv(S0, n, 0.01, False)
        torch.cuda.synchronize()
    finally:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, 0)
        G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, 0)
    assert int(info0.item()) == 0 and int(info1.item()) == 0
    a, b = P.to_np(S1).astype(np.float64), P.to_np(S0).astype(np.float64)
    assert P.rel_fro(np.triu(a), np.triu(b)) <= 1e-6
    assert torch.equal(U1, U0)
    # the quantization's persistent updates on 20 CTAs: every tile's
    # arithmetic is the same whichever CTA computes it (codes bit for bit)
    W = _weights(384, d, torch.float16, 52).to(DEV)
    ref = G.gptq_quantize_layer(W, U0, None, 4, 128)
    try:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_QUANTIZE, 20)
        got = G.gptq_quantize_layer(W, U0, None, 4, 128)
        torch.cuda.synchronize()
    finally:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_QUANTIZE, 0)
    for x, y in zip(got, ref):
        assert torch.equal(x, y)


def test_prepare_reports_non_pd():
    d = 256
    S = torch.zeros(d, d, dtype=torch.float32, device=DEV)
    _, _, info = G.gptq_prepare_hinv(S, 100, 0.01, False)
    torch.cuda.synchronize()
    assert int(info.item()) != 0


def test_tiny_layer_end_to_end():
    """The tiny workload: W 256x256 fp32, X 512x256 fp16 with 3 outlier channels x50."""
    wl = inputs.WORKLOADS["tiny"]
    spec = wl.layers[0]
    W = inputs.weights(spec)
    X = inputs.calibration_x(spec)
    st, g, ref = _check_layer(W, X, 4, 128)
    # against the oracle's OWN Hessian as well (end to end)
    S_or = oracle.hessian(X.numpy())
    own = oracle.gptq_layer(W.double().numpy(), S_or, X.shape[0], 4, 128)
    H64 = 2.0 * S_or / X.shape[0]
    lg = P.layer_loss_of(W.double().numpy(), g["codes"], g["scales"], g["zeros"], 128, None, H64)
    lo = P.layer_loss_of(W.double().numpy(), own["codes"], own["scales"], own["zeros"], 128, None,
                         H64)
    assert abs(lg - lo) <= P.LOSS_REL * lo
    # GPTQ beats RTN on this outlier workload
    r = oracle.rtn(W.double().numpy(), 4, 128)
    lr = P.layer_loss_of(W.double().numpy(), r["codes"], r["scales"], r["zeros"], 128, None, H64)
    assert lg < lr
    print("tiny:", st)


@pytest.mark.parametrize("m,d,n,bits,gs,act,dtype", [
    (1, 128, 300, 4, 128, False, torch.float16),      # single row, single block
    (300, 256, 700, 4, 128, False, torch.float16),    # ragged rows and tokens
    (129, 384, 1000, 3, 64, True, torch.float32),     # act-order, 3-bit, g64
    (64, 512, 1500, 2, 32, False, torch.float16),     # 2-bit, g32
    (1000, 1024, 4096, 4, 128, False, torch.float16), # several tiles in every dimension
])
def test_layer_parity_cases(m, d, n, bits, gs, act, dtype):
    W = _weights(m, d, dtype, m + d)
    X = _gauss_x(n, d, max(1, d // 100), 30.0, n + d)
    st, _, _ = _check_layer(W, X, bits, gs, act)
    print((m, d, n, bits, gs, act), st)


def test_pack_of_gptq_result_matches_storage_format():
    wl = inputs.WORKLOADS["tiny"]
    spec = wl.layers[0]
    W, X = inputs.weights(spec).to(DEV), inputs.calibration_x(spec).to(DEV)
    res = G.quantize_layer_from_inputs(W, X, 4, 128)
    torch.cuda.synchronize()
    qw, qz = P.to_np(res.qweight).view(np.uint32), P.to_np(res.qzeros)
    rq, rz = oracle.pack_int4(P.to_np(res.codes), P.to_np(res.zeros))
    assert np.array_equal(qw, rq) and np.array_equal(qz, rz)
    m, d = W.shape
    nbytes = qw.nbytes + qz.nbytes + res.scales.numel() * 2
    assert nbytes == 66.5 * m * d / 128

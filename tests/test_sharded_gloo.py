"""The one-layer-over-N-ranks path (post_weight_quantization_11_b200.sharded)
on CPU: two gloo ranks, unequal token shares, an odd row count.

The CUDA kernels cannot run on CPU ranks, so each rank's library calls are
replaced by stand-ins built on the float64 oracle (S, U, codes rounded to the
kernels' fp32 / fp16 outputs).  What is checked is the host logic: each rank
accumulates only its tokens, S is summed over the ranks before the
preparation, n is the total token count, the rows are split without gap or
overlap, and every rank's rows come out as the same layer quantized on one
device would give them.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from post_weight_quantization_11_b200 import sharded

M, D, N = 37, 256, 300
N0 = 173                      # rank 0's tokens; rank 1 takes the other 127


class _OracleKernels:
    """Stand-ins for the library's calls on CPU tensors (test use only)."""

    @staticmethod
    def gptq_prepare_workspace_bytes(d):
        return 16

    @staticmethod
    def gptq_quantize_workspace_bytes(m, d, b):
        return 16

    @staticmethod
    def gptq_hessian_accumulate(S, X):
        S += torch.from_numpy(np.triu(oracle.hessian(X.numpy()))).float()

    @staticmethod
    def gptq_prepare_hinv(S, n, damp, act_order, perm, U, info, ws):
        s = S.double().numpy()
        s = np.triu(s) + np.triu(s, 1).T
        _, Hd, p, _, st = oracle.finalize(s, n, damp, act_order)
        assert st == 0
        u, inf = oracle.hinv_upper_chol(Hd)
        perm.copy_(torch.from_numpy(p))
        U.copy_(torch.from_numpy(u).float())
        info.fill_(inf)

    @staticmethod
    def gptq_quantize_layer(W, U, perm, bits, gs, bs, codes, scales, zeros, loss, ws):
        w = W.double().numpy()
        if perm is not None:
            w = np.ascontiguousarray(w[:, perm.numpy()])
        r = oracle.quantize_rows(w, U.double().numpy(), bits, gs)
        codes.copy_(torch.from_numpy(r["codes"]))
        scales.copy_(torch.from_numpy(r["scales"].view(np.float16)))
        zeros.copy_(torch.from_numpy(r["zeros"]))
        loss.copy_(torch.from_numpy(r["row_loss"]).float())

    @staticmethod
    def gptq_pack_int4(codes, zeros, qweight, qzeros):
        qw, qz = oracle.pack_int4(codes.numpy(), zeros.numpy())
        qweight.copy_(torch.from_numpy(qw.view(np.int32)))
        qzeros.copy_(torch.from_numpy(qz))


def _inputs():
    g = torch.Generator().manual_seed(11)
    X = torch.randn(N, D, generator=g)
    X[:, [3, 70, 200]] *= 40.0
    W = 0.02 * torch.randn(M, D, generator=g)
    return X.half(), W


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, act_order, out):
    os.environ["CUDA_VISIBLE_DEVICES"] = ""
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        sharded.G = _OracleKernels()
        X, W = _inputs()
        t0, t1 = (0, N0) if rank == 0 else (N0, N)
        L = sharded.ShardedLayer(M, D, t1 - t0, "cpu", act_order=act_order)
        lo, hi = L.rows
        L.step(W[lo:hi].contiguous(), X[t0:t1].contiguous())
        out.put((rank, L.rows, L.n_total, L.S.numpy().copy(), L.perm.numpy().copy(),
                 L.codes.numpy().copy(), L.scales.numpy().copy(), L.zeros.numpy().copy(),
                 L.qweight.numpy().copy(), L.qzeros.numpy().copy()))
    finally:
        dist.destroy_process_group()


def _expected(act_order):
    X, W = _inputs()
    f32 = lambda a: torch.from_numpy(np.triu(a)).float()          # noqa: E731
    S = f32(oracle.hessian(X[:N0].numpy())) + f32(oracle.hessian(X[N0:].numpy()))
    k = _OracleKernels
    perm = torch.empty(D, dtype=torch.int32)
    U = torch.empty(D, D)
    info = torch.zeros(1, dtype=torch.int32)
    k.gptq_prepare_hinv(S, N, 0.01, act_order, perm, U, info, None)
    w = W.double().numpy()
    if act_order:
        w = np.ascontiguousarray(w[:, perm.numpy()])
    r = oracle.quantize_rows(w, U.double().numpy(), 4, 128)
    qw, qz = oracle.pack_int4(r["codes"], r["zeros"])
    return S.numpy(), perm.numpy(), r, qw.view(np.int32), qz


def test_share_covers_rows_without_gaps():
    for total in (0, 1, 7, 37, 4096):
        for world in (1, 2, 3, 8):
            parts = [sharded.share(total, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == total
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        sharded.share(5, 2, 2)


def test_token_shares_reassemble_the_calibration_set():
    """Each rank draws only its share of the tokens; the shares are the rows
    of the one seeded calibration set (chunk boundaries inside shares too)."""
    from post_weight_quantization_11_b200 import inputs
    spec = inputs.WORKLOADS["tiny"].layers[0]
    full = inputs.calibration_x(spec, n_tokens=1000, chunk=128)
    for world in (1, 2, 3, 7):
        parts = [inputs.calibration_x(spec, n_tokens=hi - lo, chunk=128, first_token=lo)
                 for lo, hi in (sharded.share(1000, world, r) for r in range(world))]
        assert torch.equal(torch.cat(parts), full)


@pytest.mark.parametrize("act_order", [False, True])
def test_one_layer_over_two_gloo_ranks(act_order):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, act_order, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(2):
            item = q.get(timeout=240)
            res[item[0]] = item[1:]
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    S, perm, r, qw, qz = _expected(act_order)
    assert res[0][0] == (0, 19) and res[1][0] == (19, 37)
    for rank in (0, 1):
        rows, n_total, S_r, perm_r, codes, scales, zeros, qweight, qzeros = res[rank]
        lo, hi = rows
        assert n_total == N
        assert np.array_equal(S_r, S)              # the summed S, on every rank
        assert np.array_equal(perm_r, perm)
        assert np.array_equal(codes, r["codes"][lo:hi])
        assert np.array_equal(scales.view(np.uint16), r["scales"][lo:hi])
        assert np.array_equal(zeros, r["zeros"][lo:hi])
        assert np.array_equal(qweight, qw[lo:hi]) and np.array_equal(qzeros, qz[lo:hi])

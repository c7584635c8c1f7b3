"""N > 1 plumbing of bench.py on CPU: two gloo ranks (world_size 2).

Under torchrun every rank quantizes its own independent layer (weak scaling,
no collective on the data path); the only collectives are the barriers around
the timed region and the max-over-ranks reduction of the step time.  This
checks those helpers, that the ranks get distinct layers, and that the
reference arm runs on rank 0 alone.
"""
import contextlib
import io
import os
import socket
import types

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, ws: int, port: int, out):
    # CPU ranks even on a machine with a GPU: the plumbing picks gloo when no
    # device is visible (NCCL would need one GPU per rank)
    os.environ["CUDA_VISIBLE_DEVICES"] = ""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(ws))
    import bench
    import torch.distributed as dist
    from post_weight_quantization_11_b200 import inputs

    got_ws, got_rank, got_local = bench._dist_init()
    try:
        assert (got_ws, got_rank, got_local) == (ws, rank, rank)
        assert dist.get_backend() == "gloo"
        bench._barrier(ws)
        # max over ranks of a rank-dependent step time
        t = bench._max_over_ranks(10.0 + 3.5 * rank, ws)
        # every rank quantizes a different layer: the weights differ by rank
        spec = inputs.WORKLOADS["tiny"].layers[0]
        W = inputs.weights(spec, seed_offset=rank).float()
        gathered = [torch.empty_like(W) for _ in range(ws)]
        dist.all_gather(gathered, W)
        distinct = not torch.equal(gathered[0], gathered[1])
        # reference arm: rank 0 alone works and prints; the others return at once
        printed = None
        if rank != 0:
            buf = io.StringIO()
            args = types.SimpleNamespace(workload="attn7b", layer=0, tokens=0, warmup=3, steps=1)
            with contextlib.redirect_stdout(buf):
                bench.run_reference(args)
            printed = buf.getvalue()
        bench._barrier(ws)
        out.put((rank, t, distinct, printed))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(2):
            rank, t, distinct, printed = q.get(timeout=240)
            res[rank] = (t, distinct, printed)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert res[0][0] == pytest.approx(13.5) and res[1][0] == pytest.approx(13.5)
    assert res[0][1] and res[1][1]
    assert res[1][2] == ""

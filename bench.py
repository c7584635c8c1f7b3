#!/usr/bin/env python
"""GPTQ INT4-g128 layer-quantization benchmark (one JSON line on rank 0).

A step is one pass of the whole hot path over one layer whose inputs are
resident in HBM: zero S, accumulate S = X^T X over all calibration tokens,
prepare U (damp, factor, invert), sweep all columns with error feedback, and
pack to INT4.  Default workload: the 7B attention projection (W 4096 x 4096
fp16, X 262144 tokens x 4096 fp16 with 1 % outlier channels), synthetic and
seeded.  Under torchrun every rank quantizes its own independent layer (weak
scaling, no collective on the data path); value = weights of all ranks / the
max-over-ranks time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the float64 CPU oracle (the only other implementation
of this path) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np
import torch

METRIC = "GPTQ INT4-g128 weights quantized/sec per layer"
UNIT = "weights/s"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="attn7b")
    p.add_argument("--layer", type=int, default=0)
    p.add_argument("--tokens", type=int, default=0, help="override token count (0: workload's)")
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--pipeline", default="", metavar="H,P",
                   help="overlap each layer's preparation with the next layer's Hessian on two "
                        "streams, the Hessian on at most H CTAs and the factorization on at "
                        "most P (e.g. 116,32)")
    p.add_argument("--w4a16", type=int, default=0, metavar="BATCH",
                   help="time the W4A16 product of packed layers shaped like the workload's "
                        "instead of the quantization step (batch 1-4 activation rows)")
    p.add_argument("--shard", choices=["layers", "layer"], default="layers",
                   help="layers: every rank quantizes its own layer (weak scaling); layer: one "
                        "layer over all ranks, tokens and rows split, S summed by one "
                        "all-reduce (strong scaling)")
    p.add_argument("--eager", action="store_true",
                   help="launch every kernel from Python each step instead of replaying a "
                        "CUDA graph of the step")
    return p.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing
# --------------------------------------------------------------------------

def _dist_init():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------
# clocks sampler
# --------------------------------------------------------------------------

class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        """Start sampling every 25 ms and return once the first sample (taken
        before the timed region, and discarded) has arrived, so the samples
        that follow cover the timed region even when it lasts under 100 ms."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "25"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            import select
            ready, _, _ = select.select([self.proc.stdout], [], [], 3.0)
            if ready:
                self.proc.stdout.readline()
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for r in rows:
            if r["hw"] == "Active":
                reasons.add("hw_slowdown")
            if r["hwt"] == "Active":
                reasons.add("hw_thermal_slowdown")
            if r["swt"] == "Active":
                reasons.add("sw_thermal_slowdown")
            if r["pcap"] == "Active":
                reasons.add("sw_power_cap")
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# --------------------------------------------------------------------------
# workload
# --------------------------------------------------------------------------

def _workload(name, layer, tokens):
    from post_weight_quantization_11_b200 import inputs
    wl = inputs.WORKLOADS[name]
    spec = wl.layers[layer]
    n = tokens or spec.n_tokens
    return wl, spec, n


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


def _traffic_for(kernel_file: str, summary_name: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", summary_name)
    src = os.path.join(ROOT, "post_weight_quantization_11_b200", "csrc", kernel_file)
    try:
        with open(path) as f:
            rec = json.load(f)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if rec.get("source_sha") != sha:
            return None
        return rec.get("dram_bytes_per_launch_full_size")
    except Exception:
        return None


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------

class Layer:
    """Preallocated buffers and one step of the path through the C ABI."""

    def __init__(self, spec, n, dev, seed_offset=0):
        from post_weight_quantization_11_b200 import gptq as G
        from post_weight_quantization_11_b200 import inputs
        self.G = G
        self.m, self.d, self.n = spec.d_out, spec.d_in, n
        self.act_order = spec.act_order
        m, d = self.m, self.d
        self.W = inputs.weights(spec, device=dev, seed_offset=seed_offset)
        self.X = inputs.calibration_x(spec, n_tokens=n, device=dev)
        self.S = torch.zeros(d, d, dtype=torch.float32, device=dev)
        self.perm = torch.empty(d, dtype=torch.int32, device=dev)
        self.U = torch.empty(d, d, dtype=torch.float32, device=dev)
        self.info = torch.zeros(1, dtype=torch.int32, device=dev)
        self.ws_p = torch.empty(G.gptq_prepare_workspace_bytes(d), dtype=torch.uint8, device=dev)
        self.ws_q = torch.empty(G.gptq_quantize_workspace_bytes(m, d, 128), dtype=torch.uint8,
                                device=dev)
        self.codes = torch.empty(m, d, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(m, d // 128, dtype=torch.float16, device=dev)
        self.zeros = torch.empty(m, d // 128, dtype=torch.uint8, device=dev)
        self.loss = torch.empty(m, dtype=torch.float32, device=dev)
        self.qweight = torch.empty(m, d // 8, dtype=torch.int32, device=dev)
        self.qzeros = torch.empty(m, (d // 128 + 1) // 2, dtype=torch.uint8, device=dev)

    def step(self, ev=None):
        """ev: None or 5 CUDA events recorded at the phase boundaries."""
        self.S.zero_()
        if ev is not None:
            ev[0].record()
        self.G.gptq_hessian_accumulate(self.S, self.X)
        if ev is not None:
            ev[1].record()
        self.after_hessian(ev)

    def after_hessian(self, ev=None):
        """Prepare, quantize and pack once S holds the layer's sum."""
        G = self.G
        G.gptq_prepare_hinv(self.S, self.n, 0.01, self.act_order, self.perm, self.U, self.info,
                            self.ws_p)
        if ev is not None:
            ev[2].record()
        G.gptq_quantize_layer(self.W, self.U, self.perm if self.act_order else None, 4, 128, 128,
                              self.codes, self.scales, self.zeros, self.loss, self.ws_q)
        if ev is not None:
            ev[3].record()
        G.gptq_pack_int4(self.codes, self.zeros, self.qweight, self.qzeros)
        if ev is not None:
            ev[4].record()


def _cpu_baseline(spec, n, reps=1):
    """The float64 oracle, as it stands, on a bounded sample of the workload:
    S over n_s tokens, the full d x d preparation, the sweep and packing of m_s
    rows; the token and row parts are scaled linearly to the full layer (their
    cost is exactly linear in tokens and rows)."""
    import oracle
    from post_weight_quantization_11_b200 import inputs
    m, d = spec.d_out, spec.d_in
    n_s = max(8, min(n, int(2 ** 22 // d)))       # ~4M token-features
    m_s = min(m, 64)
    X = inputs.calibration_x(spec, n_tokens=n_s, device="cpu").numpy()
    W = inputs.weights(spec, device="cpu")[:m_s].double().numpy()
    t0 = time.perf_counter()
    S = oracle.hessian(X)
    t_s = time.perf_counter() - t0
    t0 = time.perf_counter()
    H, Hd, perm, lam, st = oracle.finalize(S, n_s, 0.01, spec.act_order)
    U, info = oracle.hinv_upper_chol(Hd)
    t_p = time.perf_counter() - t0
    t0 = time.perf_counter()
    r = oracle.quantize_rows(np.ascontiguousarray(W[:, perm]), U, 4, 128)
    oracle.pack_int4(r["codes"], r["zeros"])
    t_q = time.perf_counter() - t0
    total = t_s * (n / n_s) + t_p + t_q * (m / m_s)
    return dict(value=m * d / total, unit=UNIT, cores=oracle.num_threads(), kind="oracle",
                sample=f"S over {n_s} of {n} tokens (x{n / n_s:.0f}), full {d}x{d} prepare, "
                       f"sweep+pack of {m_s} of {m} rows (x{m / m_s:.0f}); "
                       f"measured {t_s + t_p + t_q:.1f} s, extrapolated layer {total:.0f} s",
                phase_s=dict(hessian=t_s * (n / n_s), prepare=t_p, quantize_pack=t_q * (m / m_s)))


def run_ours(a):
    ws, rank, local = _dist_init()
    from post_weight_quantization_11_b200 import gptq as G
    G.load_library()
    dev = torch.device("cuda", local)
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    lay = Layer(spec, n, dev, seed_offset=rank)
    m, d = lay.m, lay.d
    torch.cuda.synchronize()
    for _ in range(max(3, a.warmup)):
        lay.step()
    torch.cuda.synchronize()
    assert int(lay.info.item()) == 0, "non-positive pivot in the workload"
    c0 = G.gptq_debug_launch_count()
    lay.step()
    graph_launches = G.gptq_debug_launch_count() - c0
    torch.cuda.synchronize()

    # per-phase split (eager launches, CUDA events between the ABI calls)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(3)]
    for e in evs:
        lay.step(e)
    torch.cuda.synchronize()
    phase = {name: statistics.mean(e[k].elapsed_time(e[k + 1]) for e in evs)
             for k, name in enumerate(("hessian", "prepare", "quantize", "pack"))}

    # the timed region: the step captured once as a CUDA graph and replayed
    # (the library's calls never synchronize or allocate, so they capture)
    graph = None
    if not a.eager:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            lay.step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            lay.step()
        torch.cuda.synchronize()
        for _ in range(max(3, a.warmup)):
            graph.replay()
        torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = G.gptq_debug_launch_count()
    _barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for i in range(a.steps):
            if graph is not None:
                graph.replay()
            else:
                lay.step()
        end.record()
        torch.cuda.synchronize()
    _barrier(ws)
    launches = G.gptq_debug_launch_count() - launches0
    if graph is not None:
        launches = graph_launches * a.steps
    ms = start.elapsed_time(end) / a.steps
    ms = _max_over_ranks(ms, ws)
    assert int(lay.info.item()) == 0 and G.gptq_device_status(reset=True) == 0
    # the dominant kernel's time inside the same timed loop: one more eager
    # pass with events around the Hessian call only
    k1 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(a.steps)]
    for i in range(a.steps):
        lay.S.zero_()
        k1[i][0].record()
        G.gptq_hessian_accumulate(lay.S, lay.X)
        k1[i][1].record()
    torch.cuda.synchronize()
    k1_ms = statistics.mean(s_.elapsed_time(e_) for s_, e_ in k1)

    # end to end through the public API from pinned host memory: X streams
    # through the library's two-slot ring (each chunk's PCIe copy overlaps the
    # accumulation of the one before, and the next layer's copies overlap this
    # layer's prepare / quantize / pack); W goes in and the packed result
    # comes back with plain copies on the compute stream
    Xh = lay.X.cpu().pin_memory()
    Wh = lay.W.cpu().pin_memory()
    qwh = torch.empty_like(lay.qweight, device="cpu").pin_memory()
    qzh = torch.empty_like(lay.qzeros, device="cpu").pin_memory()
    sch = torch.empty_like(lay.scales, device="cpu").pin_memory()
    hh = G.HostHessian(d, dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize()
    e_start.record()
    hh.copy_stream.wait_stream(torch.cuda.current_stream())   # no copy starts before e_start
    for _ in range(a.e2e_steps):
        lay.S.zero_()
        hh.accumulate(lay.S, Xh)
        lay.W.copy_(Wh, non_blocking=True)
        lay.after_hessian()
        qwh.copy_(lay.qweight, non_blocking=True)
        qzh.copy_(lay.qzeros, non_blocking=True)
        sch.copy_(lay.scales, non_blocking=True)
    e_end.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e_start.elapsed_time(e_end) / a.e2e_steps, ws)
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (qwh, qzh, sch))

    peaks, src = _peaks()
    flops = float(n) * d * d                         # SYRK, upper triangle: n d^2
    achieved = flops / (k1_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    traffic = _traffic_for("hessian.cu", "hessian_syrk_attn7b.json")
    line = {
        "metric": METRIC,
        "value": ws * m * d / (ms * 1e-3),
        "unit": UNIT,
        "n_gpus": ws,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; random-init weights, Gaussian calibration inputs with "
                "outlier channels)",
        "config": {"workload": f"{spec.name} ({a.workload}): W {m}x{d} fp16, X {n}x{d} fp16, "
                               f"INT4 g128, damp 0.01, act_order={spec.act_order}",
                   "layers_per_rank": 1, "tokens": n,
                   "l2": "inputs larger than L2 (X %.2f GB re-read every step)" %
                         (n * d * 2 / 1e9)},
        "e2e": {"value": ws * m * d / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "roofline": {"bound": "tensor", "kernel": "hessian_accumulate (S += X^T X)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"bf16_tflops_sustained of {src} (fp16 = bf16 rate)",
                     "kernel_ms": k1_ms},
        "clocks": clk.summary(),
        "phase_ms": phase,
        "phase_note": "per-phase split from eager launches; the timed steps replay a CUDA graph"
                      if graph is not None else "eager launches",
        "launch_mode": "cuda_graph" if graph is not None else "eager",
        # one Hessian serves q/k/v (or up/gate) in a model: the rate of the
        # rest of the path, from the per-phase split
        "without_hessian": {
            "value": m * d / (1e-3 * (phase["prepare"] + phase["quantize"] + phase["pack"])),
            "unit": UNIT, "note": "prepare + quantize + pack of the eager per-phase split"},
    }
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = _cpu_baseline(spec, n)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# --------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# --------------------------------------------------------------------------

def run_reference(a):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    for _ in range(a.warmup):
        _cpu_baseline(spec, n)
    vals, samples = [], None
    t0 = time.perf_counter()
    for _ in range(a.steps):
        r = _cpu_baseline(spec, n)
        vals.append(r["value"])
        samples = r
    wall = time.perf_counter() - t0
    v = statistics.median(vals)
    m, d = spec.d_out, spec.d_in
    line = {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": m * d / v * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "impl": "reference",
        "config": {"workload": f"{spec.name} ({a.workload}): W {m}x{d} fp16, X {n}x{d} fp16, "
                               f"INT4 g128, damp 0.01, act_order={spec.act_order}",
                   "tokens": n},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": samples["cores"], "kind": "oracle",
                         "sample": samples["sample"]},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)


def run_ours_one_layer(a):
    """--shard layer: one layer per step over all ranks.  Rank r accumulates
    S over its share of the tokens, S is summed by one all-reduce, every rank
    prepares U from it and quantizes and packs its share of the rows."""
    ws, rank, local = _dist_init()
    from post_weight_quantization_11_b200 import gptq as G
    from post_weight_quantization_11_b200 import inputs, sharded
    G.load_library()
    dev = torch.device("cuda", local)
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    m, d = spec.d_out, spec.d_in
    t0, t1 = sharded.share(n, ws, rank)
    L = sharded.ShardedLayer(m, d, t1 - t0, dev, act_order=spec.act_order)
    lo, hi = L.rows
    W = inputs.weights(spec, device=dev)[lo:hi].contiguous()
    X = inputs.calibration_x(spec, n_tokens=t1 - t0, device=dev, first_token=t0)
    for _ in range(max(3, a.warmup)):
        L.step(W, X)
    torch.cuda.synchronize()
    assert int(L.info.item()) == 0, "non-positive pivot in the workload"

    def ev():
        return torch.cuda.Event(enable_timing=True)

    start, end = ev(), ev()
    launches0 = G.gptq_debug_launch_count()
    _barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record()
        for _ in range(a.steps):
            L.step(W, X)
        end.record()
        torch.cuda.synchronize()
    _barrier(ws)
    launches = G.gptq_debug_launch_count() - launches0
    ms = _max_over_ranks(start.elapsed_time(end) / a.steps, ws)
    assert int(L.info.item()) == 0 and G.gptq_device_status(reset=True) == 0

    # per-phase split (this rank): local Hessian, the all-reduce, the rest
    evs = [[ev() for _ in range(4)] for _ in range(3)]
    for e in evs:
        L.S.zero_()
        e[0].record()
        G.gptq_hessian_accumulate(L.S, X)
        e[1].record()
        if ws > 1:
            import torch.distributed as dist
            dist.all_reduce(L.S)
        e[2].record()
        L.quantize(W)
        e[3].record()
    torch.cuda.synchronize()
    phase = {name: statistics.mean(e[k].elapsed_time(e[k + 1]) for e in evs)
             for k, name in enumerate(("hessian_local", "all_reduce_S", "prepare_quantize_pack"))}
    k1_ms = phase["hessian_local"]

    # end to end: this rank's tokens and rows from pinned host memory
    Xh = X.cpu().pin_memory()
    Wh = W.cpu().pin_memory()
    outs = [L.qweight, L.qzeros, L.scales]
    host_outs = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
    hh = G.HostHessian(d, dev)
    e_start, e_end = ev(), ev()
    _barrier(ws)
    torch.cuda.synchronize()
    e_start.record()
    hh.copy_stream.wait_stream(torch.cuda.current_stream())
    for _ in range(a.e2e_steps):
        L.hessian_from_host(hh, Xh)
        W.copy_(Wh, non_blocking=True)
        L.quantize(W)
        for h_, t_ in zip(host_outs, outs):
            h_.copy_(t_, non_blocking=True)
    e_end.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e_start.elapsed_time(e_end) / a.e2e_steps, ws)

    peaks, src = _peaks()
    achieved = float(t1 - t0) * d * d / (k1_ms * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    line = {
        "metric": METRIC, "value": m * d / (ms * 1e-3), "unit": UNIT, "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; random-init weights, Gaussian calibration inputs with "
                "outlier channels)",
        "config": {"workload": f"{spec.name} ({a.workload}): W {m}x{d} fp16, X {n}x{d} fp16, "
                               f"INT4 g128, damp 0.01, act_order={spec.act_order}",
                   "parallelism": f"one layer over {ws} rank(s): tokens and rows split, S "
                                  f"summed by one all-reduce, U prepared on every rank",
                   "tokens_per_rank": t1 - t0, "rows_per_rank": hi - lo,
                   "l2": "inputs larger than L2" if (t1 - t0) * d * 2 > 126e6
                         else "X share smaller than L2"},
        "e2e": {"value": m * d / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": Xh.numel() * 2 + Wh.numel() * Wh.element_size(),
                "d2h_bytes_per_step": sum(h_.numel() * h_.element_size() for h_ in host_outs)},
        "gpu_launches": int(launches),
        "roofline": {"bound": "tensor", "kernel": "hessian_accumulate (this rank's tokens)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"bf16_tflops_sustained of {src} (fp16 = bf16 rate)",
                     "kernel_ms": k1_ms},
        "clocks": clk.summary(),
        "phase_ms": phase,
        "launch_mode": "eager",
    }
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = _cpu_baseline(spec, n)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_ours_pipelined(a):
    """Consecutive layers through the path with layer i's preparation on a
    second stream beside layer i+1's Hessian: the factorization is a latency
    chain that needs few SMs, the Hessian keeps the rest busy.  S, U, perm and
    info are double-buffered; every layer still runs every step, and the
    timed region covers K whole layers (whole-job throughput)."""
    ws, rank, local = _dist_init()
    from post_weight_quantization_11_b200 import gptq as G
    G.load_library()
    dev = torch.device("cuda", local)
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    h_ctas, p_ctas = (int(v) for v in a.pipeline.split(","))
    lay = Layer(spec, n, dev, seed_offset=rank)
    m, d = lay.m, lay.d
    S2 = [lay.S, torch.zeros_like(lay.S)]
    U2 = [lay.U, torch.empty_like(lay.U)]
    perm2 = [lay.perm, torch.empty_like(lay.perm)]
    info2 = [lay.info, torch.zeros_like(lay.info)]
    sH = torch.cuda.current_stream(dev)
    sP = torch.cuda.Stream(device=dev)

    def run(layers):
        evH = [torch.cuda.Event() for _ in range(layers)]
        evP = [torch.cuda.Event() for _ in range(layers)]

        def hess(i):
            S2[i % 2].zero_()
            G.gptq_hessian_accumulate(S2[i % 2], lay.X)
            evH[i].record(sH)

        def prep(i):
            sP.wait_event(evH[i])
            with torch.cuda.stream(sP):
                G.gptq_prepare_hinv(S2[i % 2], n, 0.01, lay.act_order, perm2[i % 2], U2[i % 2],
                                    info2[i % 2], lay.ws_p)
            evP[i].record(sP)

        def quant(i):
            sH.wait_event(evP[i])
            G.gptq_quantize_layer(lay.W, U2[i % 2], perm2[i % 2] if lay.act_order else None, 4,
                                  128, 128, lay.codes, lay.scales, lay.zeros, lay.loss, lay.ws_q)
            G.gptq_pack_int4(lay.codes, lay.zeros, lay.qweight, lay.qzeros)

        hess(0)
        prep(0)
        for i in range(layers):
            if i + 1 < layers:
                hess(i + 1)           # beside prep(i) on the other stream
                prep(i + 1)
            quant(i)

    G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, h_ctas)
    G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, p_ctas)
    try:
        run(max(3, a.warmup))
        torch.cuda.synchronize()
        assert int(info2[0].item()) == 0 and int(info2[1].item()) == 0
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches0 = G.gptq_debug_launch_count()
        _barrier(ws)
        torch.cuda.synchronize()
        with ClockSampler(local) as clk:
            start.record(sH)
            run(a.steps)
            end.record(sH)
            torch.cuda.synchronize()
        _barrier(ws)
        launches = G.gptq_debug_launch_count() - launches0
        ms = _max_over_ranks(start.elapsed_time(end) / a.steps, ws)
        assert G.gptq_device_status(reset=True) == 0
    finally:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, 0)
        G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, 0)
    line = {
        "metric": METRIC, "value": ws * m * d / (ms * 1e-3), "unit": UNIT, "n_gpus": ws,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded; random-init weights, Gaussian calibration inputs with "
                "outlier channels)",
        "config": {"workload": f"{spec.name} ({a.workload}): W {m}x{d} fp16, X {n}x{d} fp16, "
                               f"INT4 g128, damp 0.01, act_order={spec.act_order}",
                   "layers_per_rank": a.steps, "tokens": n,
                   "pipeline": {"hessian_ctas": h_ctas, "prepare_ctas": p_ctas,
                                "note": "layer i's preparation overlaps layer i+1's Hessian"},
                   "l2": "inputs larger than L2 (X %.2f GB re-read every layer)" %
                         (n * d * 2 / 1e9)},
        "gpu_launches": int(launches), "clocks": clk.summary(), "launch_mode": "eager",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_w4a16(a):
    """The W4A16 product y = x Q^T of packed INT4 layers (batch a.w4a16 rows
    of fp16 activations).  Enough distinct layers rotate through the timed
    loop that their packed bytes exceed L2, so every launch streams its
    weights from HBM; the roofline is HBM bytes (packed weights, scales, zero
    points, activations, outputs) per launch over its CUDA-event time."""
    ws, rank, local = _dist_init()
    from post_weight_quantization_11_b200 import gptq as G
    G.load_library()
    dev = torch.device("cuda", local)
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    m, d, b, g = spec.d_out, spec.d_in, a.w4a16, 128
    ng = d // g
    per_layer = m * d // 2 + m * ng * 2 + m * ((ng + 1) // 2)
    L = max(2, int(4 * 126e6 // per_layer) + 1)
    gen = torch.Generator(device=dev).manual_seed(5)
    layers = []
    for _ in range(L):
        qw = torch.randint(-2**31, 2**31 - 1, (m, d // 8), generator=gen, device=dev,
                           dtype=torch.int32)
        sc = (torch.rand(m, ng, generator=gen, device=dev) * 0.05 + 1e-3).half()
        qz = torch.randint(0, 256, (m, (ng + 1) // 2), generator=gen, device=dev,
                           dtype=torch.uint8)
        layers.append((qw, sc, qz))
    x = torch.randn(b, d, generator=gen, device=dev).half()
    y = torch.empty(b, m, dtype=torch.float32, device=dev)
    for i in range(max(3, a.warmup) * L):
        qw, sc, qz = layers[i % L]
        G.gptq_w4a16_gemm(x, qw, sc, qz, g, None, y)
    torch.cuda.synchronize()
    reps = max(a.steps, 1) * L
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    with ClockSampler(local) as clk:
        start.record()
        for i in range(reps):
            qw, sc, qz = layers[i % L]
            G.gptq_w4a16_gemm(x, qw, sc, qz, g, None, y)
        end.record()
        torch.cuda.synchronize()
    us = _max_over_ranks(start.elapsed_time(end) * 1e3 / reps, ws)
    peaks, src = _peaks()
    bytes_ = per_layer + b * d * 2 + b * m * 4
    gbs = bytes_ / (us * 1e-6) / 1e9
    line = {"metric": "W4A16 product weights/s", "value": ws * m * d / (us * 1e-6),
            "unit": "weights/s", "n_gpus": ws, "steps": a.steps, "warmup": a.warmup,
            "us_per_launch": us, "higher_is_better": True, "scaling": "weak", "dtype": "f32",
            "data": "synthetic packed layers", "vs_baseline": None,
            "config": {"workload": f"{spec.name} ({a.workload}) packed: W {m}x{d} INT4 g{g}, "
                                   f"batch {b}", "layers_rotated": L},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks.get("hbm_gbs"),
                         "unit": "GB/s", "frac": gbs / peaks.get("hbm_gbs"),
                         "bytes_per_launch": bytes_, "peak_source": f"hbm_gbs of {src}"},
            "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    a = _args()
    if a.impl == "reference":
        run_reference(a)
    elif a.pipeline:
        run_ours_pipelined(a)
    elif a.w4a16:
        run_w4a16(a)
    elif a.shard == "layer":
        run_ours_one_layer(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""GPTQ INT4-g128 layer-quantization benchmark (one JSON line on rank 0).

A step is one pass of the whole hot path over one layer whose inputs are
resident in HBM: zero S, accumulate S = X^T X over all calibration tokens,
prepare U (damp, factor, invert), sweep all columns with error feedback, and
pack to INT4.  The timed region runs K consecutive layers, each through
every phase, with layer i's preparation (a latency chain on 12 CTAs) on a
second stream beside the next layers' Hessians (136 CTAs); value = layers'
weights / that time.  The single-layer step, replayed as a CUDA graph with nothing
overlapped, is reported beside it (single_layer).  Default workload: the 7B attention projection (W 4096 x 4096
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
PIPE_H, PIPE_P = 136, 12      # CTA caps of the Hessian and the factorization when layers overlap
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
    p.add_argument("--no-pipelined", action="store_true",
                   help="skip the consecutive-layer measurement with overlapped preparation")
    p.add_argument("--no-configs", action="store_true",
                   help="skip the per-config summary (every workload of the pages' shapes)")
    p.add_argument("--pipeline", default="", metavar="H,P",
                   help="overlap each layer's preparation with the next layer's Hessian on two "
                        "streams, the Hessian on at most H CTAs and the factorization on at "
                        "most P (e.g. 116,32)")
    p.add_argument("--w4a16", type=int, default=0, metavar="BATCH",
                   help="time the W4A16 product of packed layers shaped like the workload's "
                        "instead of the quantization step (batch rows of activations)")
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


class MoeLayer:
    """The mixture-of-experts layer (all experts at once) through the
    batched entry points: routed rows gathered expert-major, one grouped
    Hessian launch, one factorization launch for every expert, the batched
    sweep, one pack of the stacked codes."""

    def __init__(self, wl, dev, seed_offset=0):
        from post_weight_quantization_11_b200 import gptq as G
        from post_weight_quantization_11_b200 import inputs
        self.G = G
        spec0 = wl.layers[0]
        self.E = wl.n_experts
        self.m, self.d = spec0.d_out, spec0.d_in
        self.act_order = spec0.act_order
        E, m, d = self.E, self.m, self.d
        self.W = torch.stack([inputs.weights(sp, device=dev, seed_offset=seed_offset)
                              for sp in wl.layers]).contiguous()
        self.X = inputs.calibration_x(spec0, device=dev)
        lists = inputs.moe_routing(self.X.shape[0], wl.n_experts, wl.zipf_s, wl.top_k,
                                   wl.cold_cap, spec0.seed)
        self.counts = [len(x) for x in lists]
        self.offsets = np.concatenate([[0], np.cumsum(self.counts)]).astype(np.int64)
        self.idx = torch.as_tensor(np.concatenate(lists), dtype=torch.int32, device=dev)
        self.n = int(self.offsets[-1])               # routed rows (token-expert pairs)
        self.Xr = torch.empty(self.n, d, dtype=torch.float16, device=dev)
        self.S = torch.zeros(E, d, d, dtype=torch.float32, device=dev)
        self.perm = torch.empty(E, d, dtype=torch.int32, device=dev)
        self.U = torch.empty(E, d, d, dtype=torch.float32, device=dev)
        self.info = torch.zeros(E, dtype=torch.int32, device=dev)
        self.ws_p = torch.empty(G.gptq_prepare_batched_workspace_bytes(d, E), dtype=torch.uint8,
                                device=dev)
        self.ws_q = torch.empty(E * G.gptq_quantize_workspace_bytes(m, d, 128), dtype=torch.uint8,
                                device=dev)
        self.codes = torch.empty(E, m, d, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(E, m, d // 128, dtype=torch.float16, device=dev)
        self.zeros = torch.empty(E, m, d // 128, dtype=torch.uint8, device=dev)
        self.loss = torch.empty(E, m, dtype=torch.float32, device=dev)
        self.qweight = torch.empty(E * m, d // 8, dtype=torch.int32, device=dev)
        self.qzeros = torch.empty(E * m, (d // 128 + 1) // 2, dtype=torch.uint8, device=dev)

    def step(self, ev=None):
        G = self.G
        self.S.zero_()
        if ev is not None:
            ev[0].record()
        G.gptq_gather_rows(self.X, self.idx, self.Xr)
        G.gptq_hessian_accumulate_grouped(self.S, self.Xr, self.offsets)
        if ev is not None:
            ev[1].record()
        self.after_hessian(ev)

    def after_hessian(self, ev=None):
        G = self.G
        G.gptq_prepare_hinv_batched(self.S, self.counts, 0.01, self.act_order, self.perm, self.U,
                                    self.info, self.ws_p)
        if ev is not None:
            ev[2].record()
        G.gptq_quantize_layer_batched(self.W, self.U, self.perm if self.act_order else None, 4,
                                      128, 128, self.codes, self.scales, self.zeros, self.loss,
                                      self.ws_q)
        if ev is not None:
            ev[3].record()
        G.gptq_pack_int4(self.codes.view(self.E * self.m, self.d),
                         self.zeros.view(self.E * self.m, -1), self.qweight, self.qzeros)
        if ev is not None:
            ev[4].record()


def _make_layer(workload: str, layer: int, tokens: int, dev, seed_offset=0):
    """(layer object, description dict) for a workload of inputs.WORKLOADS."""
    from post_weight_quantization_11_b200 import inputs
    wl = inputs.WORKLOADS[workload]
    if getattr(wl, "n_experts", 0):
        lay = MoeLayer(wl, dev, seed_offset)
        lay.mats, lay.tokens = lay.E, lay.counts
        desc = (f"{wl.layers[0].name} ({workload}): {lay.E} experts x W {lay.m}x{lay.d} fp16, "
                f"X {lay.X.shape[0]}x{lay.d} fp16, top-{wl.top_k} routed ({lay.n} rows, "
                f"{min(lay.counts)}..{max(lay.counts)} per expert), INT4 g128, damp 0.01, "
                f"batched")
        return lay, desc
    spec = wl.layers[layer]
    n = tokens or spec.n_tokens
    lay = Layer(spec, n, dev, seed_offset=seed_offset)
    lay.mats, lay.tokens = 1, [n]
    desc = (f"{spec.name} ({workload}): W {lay.m}x{lay.d} fp16, X {n}x{lay.d} fp16, INT4 g128, "
            f"damp 0.01, act_order={spec.act_order}")
    return lay, desc


def _update_flops(m: int, d: int, B: int = 128, outer: int = 4, near: bool = True,
                  far: bool = True) -> float:
    """Algorithmic flops of the lazy-batch feedback onto later blocks: after
    each block of B columns the rest of its outer block of outer*B columns
    (K = B, `near`), and after each outer block every column beyond it
    (K = outer*B, `far`); 2 m K N per product."""
    f = 0.0
    ob = outer * B
    for j0 in range(0, d, B):
        o0 = j0 // ob * ob
        o1 = min(d, o0 + ob)
        if near and j0 + B < o1:
            f += 2.0 * m * B * (o1 - j0 - B)
        if far and j0 + B == o1 and o1 < d:
            f += 2.0 * m * (o1 - o0) * (d - o1)
    return f


def _tf32_peak(peaks) -> float:
    """TF32 dense peak from the measured bf16 burst peak and the nominal
    TF32 : bf16 ratio (1.1 : 2.25 PFLOP/s)."""
    return float(peaks["bf16_tflops"]) * (1.1 / 2.25)


def _phase_bounds(lay, peaks) -> dict:
    """Lower bounds (ms) of each phase at the measured burst peaks: the
    Hessian at the bf16 rate (fp16 runs at it) or its HBM bytes, whichever
    is larger; the factorization's and the updates' split-TF32 tensor flops
    (three MMAs per product) at the TF32 peak; the sweep's and pack's HBM
    bytes."""
    m, d, E = lay.m, lay.d, lay.mats
    hbm = float(peaks["hbm_gbs"]) * 1e9
    bf16 = float(peaks["bf16_tflops"]) * 1e12
    tf32 = _tf32_peak(peaks) * 1e12
    ntok = float(sum(lay.tokens))
    gather = 2.0 * ntok * d * 2 if E > 1 else 0.0
    hess = max(ntok * d * d / bf16, (2.0 * ntok * d + gather) / hbm)
    fact = E * 3 * (2.0 / 3.0) * d ** 3 / tf32
    upd = E * 3 * _update_flops(m, d) / tf32
    sweep_b = E * (13.0 * m * d + 4.0 * d * d)
    pack_b = E * 1.53 * m * d
    return {"hessian": hess * 1e3, "prepare": fact * 1e3, "quantize": (upd + sweep_b / hbm) * 1e3,
            "pack": pack_b / hbm * 1e3}


def _kernel_entries(lay, peaks, times: dict, steps: int) -> dict:
    """Per-kernel roofline entries from the library's per-kind event timing
    (ms per step = summed kernel time / steps)."""
    m, d, E = lay.m, lay.d, lay.mats
    hbm = float(peaks["hbm_gbs"])
    bf16 = float(peaks["bf16_tflops"])
    tf32 = _tf32_peak(peaks)
    ntok = float(sum(lay.tokens))

    def t(kind):
        v = times.get(kind)
        return (v[0] / steps, v[1] // steps) if v else (None, 0)

    out = {}
    ms, nl = t("hessian")
    if ms:
        a = ntok * d * d / (ms * 1e-3) / 1e12
        out["hessian"] = {"bound": "tensor", "ms": ms, "launches": nl, "achieved": a,
                          "peak": bf16, "unit": "TFLOP/s", "frac": a / bf16,
                          "work": "n d^2 flops (fp16 in, fp32 accumulate)"}
    ms, nl = t("factorization")
    if ms:
        a = E * 3 * (2.0 / 3.0) * d ** 3 / (ms * 1e-3) / 1e12
        out["factorization"] = {"bound": "tensor", "ms": ms, "launches": nl, "achieved": a,
                                "peak": tf32, "unit": "TFLOP/s", "frac": a / tf32,
                                "work": "3 x (d^3/3 factor + d^3/3 inverse) split-TF32 flops "
                                        "per matrix; a latency chain of d/128 diagonal tiles"}
    un, nn = t("update_near")
    uf, nf = t("update_far")
    if un or uf:
        ms = (un or 0.0) + (uf or 0.0)
        a = E * 3 * _update_flops(m, d, near=bool(un)) / (ms * 1e-3) / 1e12
        out["update"] = {"bound": "tensor", "ms": ms, "launches": nn + nf, "achieved": a,
                         "peak": tf32, "unit": "TFLOP/s", "frac": a / tf32,
                         "near_ms": un, "far_ms": uf,
                         "work": "3 x sum of 2 m K N split-TF32 flops of the tensor-core "
                                 "updates (K = 512 beyond each outer block" +
                                 (", K = 128 inside it)" if un else
                                  "; inside an outer block the sweep kernel updates on the "
                                  "CUDA cores)")}
    ms, nl = t("sweep")
    if ms:
        b = E * (13.0 * m * d + 4.0 * d * d)
        a = b / (ms * 1e-3) / 1e9
        out["sweep"] = {"bound": "hbm", "ms": ms, "launches": nl, "achieved": a, "peak": hbm,
                        "unit": "GB/s", "frac": a / hbm,
                        "work": "W fp32 in (4 B), codes (1 B) and E split (8 B) out per weight, "
                                "U diagonal blocks in; a chain of d dependent column decisions "
                                "per row in practice" +
                                ("" if un else "; fused with the fp32 updates inside each "
                                 "512-column outer block (2 m 128 N flops per block)")}
    ms, nl = t("pack")
    if ms:
        b = E * 1.53 * m * d
        a = b / (ms * 1e-3) / 1e9
        out["pack"] = {"bound": "hbm", "ms": ms, "launches": nl, "achieved": a, "peak": hbm,
                       "unit": "GB/s", "frac": a / hbm,
                       "work": "codes in (1 B per weight), packed nibbles out (0.5 B), zero "
                               "points and their packing (0.03 B)"}
    ms, nl = t("gather")
    if ms:
        b = 2.0 * ntok * d * 2
        a = b / (ms * 1e-3) / 1e9
        out["gather"] = {"bound": "hbm", "ms": ms, "launches": nl, "achieved": a, "peak": hbm,
                         "unit": "GB/s", "frac": a / hbm, "work": "routed rows read and written"}
    for k in ("finalize", "init_work", "split_u"):
        ms, nl = t(k)
        if ms:
            out[k] = {"ms": ms, "launches": nl}
    return out


def _time_layer(lay, steps: int, warmup: int, eager: bool = False):
    """(ms per step, launches per step, graph or None): the step captured
    once as a CUDA graph and replayed between CUDA events (the library's
    calls never synchronize or allocate, so they capture)."""
    G = lay.G
    c0 = G.gptq_debug_launch_count()
    lay.step()
    per_step = G.gptq_debug_launch_count() - c0
    torch.cuda.synchronize()
    graph = None
    if not eager:
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
        for _ in range(max(3, warmup)):
            graph.replay()
        torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        if graph is not None:
            graph.replay()
        else:
            lay.step()
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps, per_step, graph


def _phase_split(lay, reps: int = 3) -> dict:
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(reps)]
    for e in evs:
        lay.step(e)
    torch.cuda.synchronize()
    return {name: statistics.mean(e[k].elapsed_time(e[k + 1]) for e in evs)
            for k, name in enumerate(("hessian", "prepare", "quantize", "pack"))}


def _kernel_times(lay, reps: int = 2) -> dict:
    G = lay.G
    G.gptq_debug_kernel_times()                  # drop older records
    G.gptq_debug_kernel_timing(True)
    try:
        for _ in range(reps):
            lay.step()
        torch.cuda.synchronize()
    finally:
        G.gptq_debug_kernel_timing(False)
    return G.gptq_debug_kernel_times()


CONFIGS = (("tiny", 0), ("attn7b", 0), ("mlp7b", 0), ("mlp7b", 1), ("mlp8b_act", 0),
           ("mlp8b_act", 1), ("moe8", 0))


def _configs_summary(dev, peaks, steps: int, warmup: int, skip=None) -> dict:
    """Every workload of the pages' shapes, each timed the way the headline
    is (graph replay, inputs resident): ms per layer, weights/s, the phase
    split and the whole-layer fraction of its roofline (the sum of the
    phase bounds at the measured peaks over the measured step)."""
    out = {}
    for wname, li in CONFIGS:
        key = f"{wname}/{li}" if wname not in ("tiny", "moe8") else wname
        if skip == (wname, li):
            continue
        lay, desc = _make_layer(wname, li, 0, dev)
        for _ in range(max(3, warmup)):
            lay.step()
        torch.cuda.synchronize()
        ok = not bool(lay.info.any().item())
        k = max(steps, 200) if wname == "tiny" else steps
        ms, launches, graph = _time_layer(lay, k, warmup)
        phase = _phase_split(lay, 2)
        bounds = _phase_bounds(lay, peaks)
        kern = _kernel_entries(lay, peaks, _kernel_times(lay, 1), 1)
        units = lay.mats * lay.m * lay.d
        out[key] = {"workload": desc, "ms_per_layer": ms, "weights_per_s": units / (ms * 1e-3),
                    "steps": k, "launches_per_step": launches, "phase_ms": phase,
                    "phase_bound_ms": bounds, "whole_layer_frac": sum(bounds.values()) / ms,
                    "kernels": {n: {kk: v[kk] for kk in ("ms", "frac") if kk in v}
                                for n, v in kern.items()},
                    "info_ok": ok}
        del graph, lay
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


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
    lay, desc = _make_layer(a.workload, a.layer, a.tokens, dev, seed_offset=rank)
    m, d, E = lay.m, lay.d, lay.mats
    units = E * m * d
    torch.cuda.synchronize()
    for _ in range(max(3, a.warmup)):
        lay.step()
    torch.cuda.synchronize()
    assert not bool(lay.info.any().item()), "non-positive pivot in the workload"

    # per-phase split (eager launches, CUDA events between the ABI calls)
    phase = _phase_split(lay, 3)

    # the timed region: the step captured once as a CUDA graph and replayed
    _barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms, graph_launches, graph = _time_layer(lay, a.steps, a.warmup, a.eager)
    _barrier(ws)
    launches = graph_launches * a.steps
    ms = _max_over_ranks(ms, ws)
    assert not bool(lay.info.any().item()) and G.gptq_device_status(reset=True) == 0
    del graph

    # every kernel's time: one eager pass with the library's per-kind event
    # timing, plus the dominant kernel alone in a loop of its own
    ktimes = _kernel_times(lay, 2)
    k1 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(a.steps)]
    for i in range(a.steps):
        lay.S.zero_()
        k1[i][0].record()
        if E > 1:
            G.gptq_hessian_accumulate_grouped(lay.S, lay.Xr, lay.offsets)
        else:
            G.gptq_hessian_accumulate(lay.S, lay.X)
        k1[i][1].record()
    torch.cuda.synchronize()
    k1_ms = statistics.mean(s_.elapsed_time(e_) for s_, e_ in k1)

    # consecutive layers (exactly K of them, one per step) with every
    # layer's preparation on a second stream, layer i quantized after layer
    # i+2's Hessian (dense layers; whole-job throughput over the layers);
    # with fewer than 3 layers there is nothing to overlap
    pipelined = None
    if E == 1 and not a.no_pipelined and a.steps >= 3:
        _barrier(ws)
        with ClockSampler(local) as clk_p:
            pms, per_layer = _pipelined_ms(lay, a.steps, a.warmup, PIPE_H, PIPE_P, not a.eager)
        _barrier(ws)
        pms = _max_over_ranks(pms, ws)
        pipelined = {"value": ws * units / (pms * 1e-3), "ms_per_layer": pms,
                     "launches": int(round(per_layer * a.steps)), "clocks": clk_p.summary(),
                     "hessian_ctas": PIPE_H, "prepare_ctas": PIPE_P}

    # end to end through the public API from pinned host memory
    e2e = _e2e(lay, a, ws, dev)

    peaks, src = _peaks()
    ntok = float(sum(lay.tokens))
    flops = ntok * d * d                         # SYRK, upper triangle: n d^2
    achieved = flops / (k1_ms * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = _traffic_for("hessian.cu", "hessian_syrk_attn7b.json") if a.workload == "attn7b" \
        else None
    bounds = _phase_bounds(lay, peaks)
    # the headline: consecutive layers with each layer's preparation beside
    # the next layer's Hessian when measured (dense layers), else the single
    # layer step replayed as a CUDA graph; the other is reported beside it
    single = {"value": ws * units / (ms * 1e-3), "ms_per_step": ms, "launch_mode": "cuda_graph",
              "gpu_launches": int(launches), "clocks": clk.summary(),
              "note": "one layer per step, the step replayed as a CUDA graph, nothing overlapped"}
    head_ms = pipelined["ms_per_layer"] if pipelined else ms
    line = {
        "metric": METRIC,
        "value": ws * units / (head_ms * 1e-3),
        "unit": UNIT,
        "n_gpus": ws,
        "steps": a.steps,
        "warmup": a.warmup,
        "ms_per_step": head_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded; random-init weights, Gaussian calibration inputs with "
                "outlier channels)",
        "config": {"workload": desc, "layers_per_rank": 1, "tokens": int(ntok),
                   "l2": "inputs larger than L2 (X %.2f GB re-read every step)" %
                         (ntok * d * 2 / 1e9)},
        "e2e": e2e,
        "gpu_launches": int(pipelined["launches"] if pipelined else launches),
        "roofline": {"bound": "tensor", "kernel": "hessian_accumulate (S += X^T X)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": f"bf16_tflops (burst) of {src}: fp16 runs at the bf16 rate; "
                                    f"the kernel is timed alone, {a.steps} launches",
                     "kernel_ms": k1_ms},
        "kernels": _kernel_entries(lay, peaks, ktimes, 2),
        "whole_layer": {"bound_ms": sum(bounds.values()), "phase_bound_ms": bounds,
                        "frac": sum(bounds.values()) / ms,
                        "note": "sum of the phase bounds at the measured burst peaks (TF32 = "
                                "bf16 x 1.1/2.25) over the measured step"},
        "clocks": pipelined["clocks"] if pipelined else clk.summary(),
        "phase_ms": phase,
        "phase_note": "per-phase split of one layer from eager launches",
        "launch_mode": (("eager" if a.eager else "cuda_graph") +
                        f", consecutive layers: every layer's preparation on a second stream, "
                        f"layer i quantized after layer i+2's Hessian (persistent grids capped "
                        f"at {PIPE_H} CTAs for the Hessian and the updates, {PIPE_P} for the "
                        f"factorization but the last two layers', which have no Hessian left "
                        f"beside them); every layer runs every phase") if pipelined else
                       ("cuda_graph" if not a.eager else "eager"),
        "single_layer": single,
        # one Hessian serves q/k/v (or up/gate) in a model: the rate of the
        # rest of the path, from the per-phase split
        "without_hessian": {
            "value": units / (1e-3 * (phase["prepare"] + phase["quantize"] + phase["pack"])),
            "unit": UNIT, "note": "prepare + quantize + pack of the eager per-phase split"},
    }
    if rank == 0 and ws == 1 and not a.no_configs:
        head = {"workload": desc, "ms_per_layer": ms, "weights_per_s": units / (ms * 1e-3),
                "steps": a.steps, "launches_per_step": graph_launches, "phase_ms": phase,
                "phase_bound_ms": bounds, "whole_layer_frac": sum(bounds.values()) / ms,
                "info_ok": True, "note": "the headline measurement above"}
        del lay
        torch.cuda.empty_cache()
        cfg = _configs_summary(dev, peaks, max(3, min(a.steps, 5)), a.warmup,
                               skip=(a.workload, a.layer))
        hk = a.workload if a.workload in ("tiny", "moe8") else f"{a.workload}/{a.layer}"
        line["configs"] = {hk: head, **cfg}
    if rank == 0 and ws == 1 and not a.no_cpu_baseline and a.workload != "moe8":
        wl, spec, n = _workload(a.workload, a.layer, a.tokens)
        line["cpu_baseline"] = _cpu_baseline(spec, n)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _e2e(lay, a, ws, dev):
    """The same step through the public API from pinned host memory: X
    (dense layers) streams through the library's two-slot ring -- each
    chunk's PCIe copy overlaps the accumulation of the one before, and the
    next layer's copies overlap this layer's prepare / quantize / pack; W
    (and for the MoE layer X) go in with plain copies on the compute stream,
    the packed result comes back inside the timed region."""
    from post_weight_quantization_11_b200 import gptq as G
    Xh = lay.X.cpu().pin_memory()
    Wh = lay.W.cpu().pin_memory()
    qwh = torch.empty_like(lay.qweight, device="cpu").pin_memory()
    qzh = torch.empty_like(lay.qzeros, device="cpu").pin_memory()
    sch = torch.empty_like(lay.scales, device="cpu").pin_memory()
    dense = lay.mats == 1
    hh = G.HostHessian(lay.d, dev) if dense else None
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize()
    e_start.record()
    if dense:
        hh.copy_stream.wait_stream(torch.cuda.current_stream())   # no copy before e_start
    for _ in range(a.e2e_steps):
        if dense:
            lay.S.zero_()
            hh.accumulate(lay.S, Xh)
            lay.W.copy_(Wh, non_blocking=True)
            lay.after_hessian()
        else:
            lay.X.copy_(Xh, non_blocking=True)
            lay.W.copy_(Wh, non_blocking=True)
            lay.step()
        qwh.copy_(lay.qweight, non_blocking=True)
        qzh.copy_(lay.qzeros, non_blocking=True)
        sch.copy_(lay.scales, non_blocking=True)
    e_end.record()
    torch.cuda.synchronize()
    e2e_ms = _max_over_ranks(e_start.elapsed_time(e_end) / a.e2e_steps, ws)
    h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (qwh, qzh, sch))
    units = lay.mats * lay.m * lay.d
    return {"value": ws * units / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h}


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


def _pipelined_ms(lay, steps: int, warmup: int, h_ctas: int, p_ctas: int,
                  graph: bool = True, lag: int = 2, uncap_tail: bool = True):
    """(ms per layer, library launches per layer) of consecutive layers with
    each layer's preparation on a second stream: the factorization is a
    latency chain that needs few SMs, the Hessian and the quantization keep
    the rest busy.  Layer i is quantized after layer i + lag's Hessian, so
    its preparation (on p_ctas CTAs, slower than on the whole GPU) has lag
    Hessians and lag - 1 quantizations to finish in; preparations follow one
    another on their stream.  S, U, perm and info rotate through lag + 1
    buffers (layer i's S is overwritten by layer i + lag + 1's Hessian,
    which runs after layer i's quantization, which waits for its
    preparation).  Every layer still runs every phase.  With `graph`, the
    schedule of `steps` layers (both streams, joined by events) is captured
    once as a CUDA graph and replayed; otherwise it is launched eagerly.  The
    persistent grids are capped at h_ctas (Hessian, updates) / p_ctas
    (factorization) CTAs meanwhile (the caps are read at capture), except
    for the preparations of the last `lag` layers: no Hessian is left to
    run beside them (the last one ends while the first of them starts), so
    they take the whole GPU rather than draining on p_ctas CTAs."""
    G = lay.G
    dev = lay.S.device
    n = lay.n
    nb = lag + 1
    S2 = [lay.S] + [torch.zeros_like(lay.S) for _ in range(lag)]
    U2 = [lay.U] + [torch.empty_like(lay.U) for _ in range(lag)]
    perm2 = [lay.perm] + [torch.empty_like(lay.perm) for _ in range(lag)]
    info2 = [lay.info] + [torch.zeros_like(lay.info) for _ in range(lag)]
    sP = torch.cuda.Stream(device=dev)

    def run(layers):
        sH = torch.cuda.current_stream(dev)
        evH = [torch.cuda.Event() for _ in range(layers)]
        evP = [torch.cuda.Event() for _ in range(layers)]

        def hess(i):
            S2[i % nb].zero_()
            G.gptq_hessian_accumulate(S2[i % nb], lay.X)
            evH[i].record(sH)

        def prep(i):
            tail = uncap_tail and i >= layers - lag   # no Hessian left to share the SMs with
            if tail:
                G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, 0)
            sP.wait_event(evH[i])
            with torch.cuda.stream(sP):
                G.gptq_prepare_hinv(S2[i % nb], n, 0.01, lay.act_order, perm2[i % nb],
                                    U2[i % nb], info2[i % nb], lay.ws_p)
            evP[i].record(sP)
            if tail:
                G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, p_ctas)

        def quant(i):
            sH.wait_event(evP[i])
            G.gptq_quantize_layer(lay.W, U2[i % nb], perm2[i % nb] if lay.act_order else None,
                                  4, 128, 128, lay.codes, lay.scales, lay.zeros, lay.loss,
                                  lay.ws_q)
            G.gptq_pack_int4(lay.codes, lay.zeros, lay.qweight, lay.qzeros)

        for i in range(min(lag, layers)):
            hess(i)
            prep(i)
        for i in range(layers):
            if i + lag < layers:
                hess(i + lag)         # beside the preparations on the other stream
                prep(i + lag)
            quant(i)

    G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, h_ctas)
    G.gptq_set_max_ctas(G.GPTQ_CTAS_QUANTIZE, h_ctas)   # the SMs the preparation leaves
    G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, p_ctas)
    g = None
    try:
        run(max(3, warmup))
        torch.cuda.synchronize()
        assert all(int(x.item()) == 0 for x in info2)
        c0 = G.gptq_debug_launch_count()
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run(steps)
            torch.cuda.synchronize()
            per_layer = (G.gptq_debug_launch_count() - c0) / steps
            for _ in range(max(1, warmup // 2)):
                g.replay()
        else:
            run(steps)
            per_layer = (G.gptq_debug_launch_count() - c0) / steps
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        if g is not None:
            g.replay()
        else:
            run(steps)
        end.record()
        torch.cuda.synchronize()
        assert all(int(x.item()) == 0 for x in info2)
        assert G.gptq_device_status(reset=True) == 0
    finally:
        G.gptq_set_max_ctas(G.GPTQ_CTAS_HESSIAN, 0)
        G.gptq_set_max_ctas(G.GPTQ_CTAS_QUANTIZE, 0)
        G.gptq_set_max_ctas(G.GPTQ_CTAS_PREPARE, 0)
    del g
    return start.elapsed_time(end) / steps, per_layer


def run_ours_pipelined(a):
    """--pipeline H,P: consecutive layers, layer i's preparation beside layer
    i+1's Hessian (see _pipelined_ms), eager launches."""
    ws, rank, local = _dist_init()
    from post_weight_quantization_11_b200 import gptq as G
    G.load_library()
    dev = torch.device("cuda", local)
    wl, spec, n = _workload(a.workload, a.layer, a.tokens)
    h_ctas, p_ctas = (int(v) for v in a.pipeline.split(","))
    lay = Layer(spec, n, dev, seed_offset=rank)
    m, d = lay.m, lay.d
    _barrier(ws)
    with ClockSampler(local) as clk:
        ms, per_layer = _pipelined_ms(lay, a.steps, a.warmup, h_ctas, p_ctas, not a.eager)
    _barrier(ws)
    launches = int(round(per_layer * a.steps))
    ms = _max_over_ranks(ms, ws)
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
        "gpu_launches": int(launches), "clocks": clk.summary(),
        "launch_mode": "eager" if a.eager else "cuda_graph",
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_w4a16(a):
    """The W4A16 product y = x Q^T of packed INT4 layers (batch a.w4a16 rows
    of fp16 activations) on the tensor cores (gptq_w4a16_matmul), and for
    batches of at most 8 also the decode product (gptq_w4a16_gemm).
    Enough distinct layers rotate through the timed loop that their packed
    bytes exceed L2, so every launch streams its weights from HBM.  The
    roofline: HBM bytes per launch (packed weights, scales, zero points,
    activations, outputs) over the launch's CUDA-event time against the
    measured copy bandwidth, and 2 m d batch flops against the fp16 (= bf16)
    tensor peak; the bound is whichever is nearer."""
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
    perm = torch.randperm(d, generator=gen, device=dev).to(torch.int32) if spec.act_order \
        else None
    wsb = torch.empty(max(1, G.gptq_w4a16_matmul_workspace_bytes(b, d)), dtype=torch.uint8,
                      device=dev)

    def tc(i):
        qw, sc, qz = layers[i % L]
        G.gptq_w4a16_matmul(x, qw, sc, qz, g, perm, y, wsb)

    def cc(i):
        qw, sc, qz = layers[i % L]
        G.gptq_w4a16_gemm(x, qw, sc, qz, g, perm, y)

    def timed(fn):
        # the launches of one pass over the L layers captured once as a CUDA
        # graph and replayed, so the time is the GPU's, not the host's issue
        # rate (a launch here is a few microseconds)
        for i in range(max(3, a.warmup) * L):
            fn(i)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(L):
                fn(i)
        for _ in range(max(1, a.warmup)):
            gr.replay()
        torch.cuda.synchronize()
        reps = max(a.steps, 1)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(reps):
            gr.replay()
        end.record()
        torch.cuda.synchronize()
        del gr
        return start.elapsed_time(end) * 1e3 / (reps * L)

    peaks, src = _peaks()
    _barrier(ws)
    with ClockSampler(local) as clk:
        us = _max_over_ranks(timed(tc), ws)
    bytes_ = per_layer + b * d * 2 + b * m * 4
    gbs = bytes_ / (us * 1e-6) / 1e9
    tfs = 2.0 * m * d * b / (us * 1e-6) / 1e12
    hbm, tens = float(peaks["hbm_gbs"]), float(peaks["bf16_tflops"])
    t_hbm, t_tc = bytes_ / (hbm * 1e9), 2.0 * m * d * b / (tens * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = ({"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
            if bound == "hbm" else
            {"bound": "tensor", "achieved": tfs, "peak": tens, "unit": "TFLOP/s",
             "frac": tfs / tens})
    roof.update({"bytes_per_launch": bytes_, "flops_per_launch": 2.0 * m * d * b,
                 "peak_source": f"hbm_gbs / bf16_tflops (burst) of {src}",
                 "other": {"GB/s": gbs, "TFLOP/s": tfs}})
    line = {"metric": "W4A16 product weights/s", "value": ws * m * d / (us * 1e-6),
            "unit": "weights/s", "n_gpus": ws, "steps": a.steps, "warmup": a.warmup,
            "us_per_launch": us, "higher_is_better": True, "scaling": "weak", "dtype": "f16",
            "data": "synthetic packed layers", "vs_baseline": None, "kernel": "gptq_w4a16_matmul",
            "config": {"workload": f"{spec.name} ({a.workload}) packed: W {m}x{d} INT4 g{g}, "
                                   f"batch {b}, act_order={spec.act_order}",
                       "layers_rotated": L},
            "roofline": roof, "clocks": clk.summary()}
    if b <= 8:
        us_cc = timed(cc)
        line["decode_gemv"] = {"kernel": "gptq_w4a16_gemm", "us_per_launch": us_cc,
                               "GB/s": bytes_ / (us_cc * 1e-6) / 1e9,
                               "frac": bytes_ / (us_cc * 1e-6) / 1e9 / hbm}
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

"""Seeded synthetic layer workloads (weights, calibration inputs, MoE routing).

This module only draws random numbers and shapes them; it contains none of the
quantization arithmetic, and both the CUDA path and the float64 oracle are fed
the same bytes from it.

The workloads stand in for the calibration setups the pages describe: about
128 calibration sequences of 2048 tokens ("大模型量化实战（上）", decision-table
notes; "GPTQ / AWQ / SqueezeLLM" sec. 一), input channels of which 0.1-1 % carry
10-100x larger activations that are stable across tokens ("INT4/INT8 量化推理"
sec. 二), and mixture-of-experts layers whose cold experts see few tokens
(same page, sec. 五).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LayerSpec:
    name: str
    d_out: int
    d_in: int
    w_std: float
    w_dtype: str            # "fp32" | "fp16"
    n_tokens: int
    x_kind: str             # "gauss" | "silu"
    n_outliers: int
    outlier_lo: float
    outlier_hi: float
    act_order: bool = False
    seed: int = 0


@dataclass(frozen=True)
class Workload:
    name: str
    layers: tuple
    n_experts: int = 0      # > 0: per-expert layers share X through a routing
    zipf_s: float = 1.2
    top_k: int = 2
    cold_cap: int = 2048
    bits: int = 4
    group_size: int = 128
    damp_rel: float = 0.01
    description: str = ""


N_TOK = 128 * 2048

WORKLOADS = {
    "tiny": Workload(
        "tiny",
        (LayerSpec("tiny", 256, 256, 0.02, "fp32", 512, "gauss", 3, 50.0, 50.0, False, 0),),
        description="W 256x256 fp32 N(0,0.02^2); X 512x256 fp16 N(0,1), 3 channels x50"),
    "attn7b": Workload(
        "attn7b",
        (LayerSpec("attn_proj", 4096, 4096, 0.02, "fp16", N_TOK, "gauss", 41, 20.0, 100.0,
                   False, 1),),
        description="7B attention projection: W 4096x4096 fp16; X 128x2048 tokens x 4096, "
                    "1% channels x U(20,100)"),
    "mlp7b": Workload(
        "mlp7b",
        (LayerSpec("up", 11008, 4096, 0.02, "fp16", N_TOK, "gauss", 41, 20.0, 100.0, False, 2),
         LayerSpec("down", 4096, 11008, 0.02, "fp16", N_TOK, "silu", 55, 20.0, 100.0, False, 2)),
        description="7B MLP pair: up 11008x4096 (X as attn7b), down 4096x11008 "
                    "(X = silu(a)*b, 0.5% channels x U(20,100))"),
    "mlp8b_act": Workload(
        "mlp8b_act",
        (LayerSpec("up", 14336, 4096, 0.015, "fp16", N_TOK, "gauss", 41, 50.0, 50.0, True, 3),
         LayerSpec("down", 4096, 14336, 0.015, "fp16", N_TOK, "gauss", 143, 50.0, 50.0, True, 3)),
        description="8B MLP with act-order: 14336x4096 and 4096x14336 N(0,0.015^2); "
                    "1% channels x50"),
    "moe8": Workload(
        "moe8",
        tuple(LayerSpec(f"expert{e}", 14336, 4096, 0.02, "fp16", N_TOK, "gauss", 0, 1.0, 1.0,
                        False, 4) for e in range(8)),
        n_experts=8,
        description="MoE: 8 experts x 14336x4096; X 262144x4096 N(0,1) top-2 Zipf(1.2) routing, "
                    "coldest expert capped at 2048 tokens"),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def weights(spec: LayerSpec, device="cpu", seed_offset: int = 0) -> torch.Tensor:
    """W (d_out x d_in) ~ N(0, w_std^2), drawn in fp32 then cast to the spec dtype."""
    g = _gen(1000 * spec.seed + 17 + seed_offset, device)
    w = torch.randn(spec.d_out, spec.d_in, generator=g, device=device, dtype=torch.float32)
    w.mul_(spec.w_std)
    return w if spec.w_dtype == "fp32" else w.to(torch.float16)


def outlier_channels(spec: LayerSpec):
    """Seeded choice of outlier channels and their fixed per-channel factors."""
    rng = np.random.default_rng(7919 * spec.seed + 3)
    ch = np.sort(rng.permutation(spec.d_in)[: spec.n_outliers]).astype(np.int64)
    fac = rng.uniform(spec.outlier_lo, spec.outlier_hi, size=spec.n_outliers)
    return ch, fac.astype(np.float32)


def calibration_x(spec: LayerSpec, n_tokens: int | None = None, device="cpu",
                  chunk: int = 16384, first_token: int = 0) -> torch.Tensor:
    """X (n x d_in) fp16, token-major. Gaussian N(0,1) or silu(a)*b with a, b
    N(0,1); then the outlier channels are multiplied by their factor (the same
    factor for every token).  Drawn chunk by chunk so that any prefix of the
    tokens is the same whatever n is asked for; first_token > 0 gives rows
    [first_token, first_token + n) of that same sequence (one rank's share)."""
    n = spec.n_tokens if n_tokens is None else int(n_tokens)
    d = spec.d_in
    ch, fac = outlier_channels(spec)
    ch_t = torch.as_tensor(ch, device=device)
    fac_t = torch.as_tensor(fac, device=device)
    out = torch.empty(n, d, dtype=torch.float16, device=device)
    t_end = first_token + n
    for k in range(first_token // chunk, (t_end + chunk - 1) // chunk):
        a0, a1 = max(first_token, k * chunk), min(t_end, (k + 1) * chunk)   # absolute rows
        g = _gen(1_000_003 * spec.seed + 101 + k, device)
        if spec.x_kind == "gauss":
            x = torch.randn(chunk, d, generator=g, device=device, dtype=torch.float32)
        elif spec.x_kind == "silu":
            a = torch.randn(chunk, d, generator=g, device=device, dtype=torch.float32)
            b = torch.randn(chunk, d, generator=g, device=device, dtype=torch.float32)
            x = torch.nn.functional.silu(a) * b
            del a, b
        else:
            raise ValueError(spec.x_kind)
        if len(ch):
            x[:, ch_t] *= fac_t
        out[a0 - first_token:a1 - first_token] = x[a0 - k * chunk:a1 - k * chunk].to(torch.float16)
        del x
    return out


def moe_routing(n_tokens: int, n_experts: int = 8, zipf_s: float = 1.2, top_k: int = 2,
                cold_cap: int = 2048, seed: int = 4):
    """Top-k routing with Zipf(s) expert popularity: the first expert of each
    token is drawn with p_e ~ 1/(e+1)^s, the next ones without replacement.
    The coldest expert's token list is truncated to its first ``cold_cap``
    tokens so that its Hessian is rank-deficient.  Returns a list of sorted
    int64 token-index arrays, one per expert."""
    rng = np.random.default_rng(seed)
    p = 1.0 / np.arange(1, n_experts + 1, dtype=np.float64) ** zipf_s
    p /= p.sum()
    chosen = np.zeros((n_tokens, top_k), dtype=np.int64)
    avail = np.broadcast_to(p, (n_tokens, n_experts)).copy()
    for k in range(top_k):
        cdf = np.cumsum(avail, axis=1)
        u = rng.random(n_tokens) * cdf[:, -1]
        e = (cdf < u[:, None]).sum(axis=1)
        e = np.minimum(e, n_experts - 1)
        chosen[:, k] = e
        avail[np.arange(n_tokens), e] = 0.0
    lists = [np.nonzero((chosen == e).any(axis=1))[0].astype(np.int64) for e in range(n_experts)]
    counts = [len(x) for x in lists]
    cold = int(np.argmin(counts))
    if cold_cap and counts[cold] > cold_cap:
        lists[cold] = lists[cold][:cold_cap]
    return lists

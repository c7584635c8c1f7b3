"""GPU-vs-oracle comparison helpers for the parity tests.

Tolerances (written here, used by every parity test):
  * S:      ||S_gpu - S_64||_F / ||S_64||_F <= 1e-5   (fp16 products are exact
            in fp32; only the fp32 accumulation order differs)
  * U:      relative Frobenius error <= 1e-4 against the oracle's float64 U
            computed from the SAME S (the GPU's, promoted)
  * codes:  bit-exact except at most 1e-3 of the weights (fp32 vs fp64 error
            feedback flips codes that sit at a rounding tie).  At 4 bits the
            bar holds for the free-running comparison, cascades included; at
            other widths it counts the tie flips themselves (the codes the
            oracle decides differently on the GPU's own trajectory), since
            one flip there moves tens to hundreds of later codes of its row;
            there the scale and zero-point bars are likewise taken on that
            trajectory (at 2 bits a group made only of earlier columns'
            cancelling corrections can differ by more than 1e-4 between fp32
            and fp64 feedback before any code differs)
  * scales: for every group of a row before that row's first code mismatch,
            the GPU's fp16 scale is the fp16 rounding of some value within
            1e-4 relative of the oracle's pre-fp16 scale
  * zero points: z = rne(-mn/s) is an integer rounding decision like the
            codes; under equal scales they are equal except at most 1e-3 of
            the groups, those differ by one step, and the teacher-forced run
            shows each such flip to be a near-tie: |frac(-mn/s) - 0.5| <= 1e-3
            on the oracle's side of the same trajectory
  * loss:   the layer loss tr(D H D^T) of the GPU's dequantized weights,
            evaluated in float64, within 1e-3 relative of the oracle's
  * teacher-forced diagnostic: with the GPU's decisions forced into the
            oracle, every code where the oracle would have decided otherwise
            is a near-tie: |frac(w/s) - 0.5| <= 1e-3; every zero point where it
            would have decided otherwise under the same fp16 scale is a
            near-tie of -mn/s; and every fp16 scale where it would have
            decided otherwise rounds a value within 1e-4 of the oracle's
            pre-fp16 scale (the oracle's value sits that close to an fp16
            rounding boundary)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

S_TOL = 1e-5
U_TOL = 1e-4
CODE_FRAC = 1e-3
SCALE_REL = 1e-4
LOSS_REL = 1e-3
TIE = 1e-3


def mirror_upper(S32: np.ndarray) -> np.ndarray:
    S = np.triu(S32.astype(np.float64))
    return S + np.triu(S, 1).T


def rel_fro(a, b) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def fp16_range(s_pre: np.ndarray, rel: float):
    lo = (s_pre.astype(np.float64) * (1 - rel)).astype(np.float32).astype(np.float16)
    hi = (s_pre.astype(np.float64) * (1 + rel)).astype(np.float32).astype(np.float16)
    return lo.astype(np.float32), hi.astype(np.float32)


def compare_sweep(gpu: dict, orc: dict, group_size: int, report: dict | None = None,
                  code_frac: float = CODE_FRAC, group_bars: bool = True):
    """gpu/orc: dicts with codes (m x d uint8), scales (m x G uint16 bits),
    zeros (m x G uint8); orc also has s_pre.  Asserts the code and scale
    tolerances and returns statistics.  code_frac: the bar on the free-running
    code mismatches (1.0 where the caller takes the bar on the teacher-forced
    run instead); group_bars False likewise leaves the scale and zero-point
    bars to the teacher-forced run (and reports the free-running deviation)."""
    cg, co = gpu["codes"], orc["codes"]
    m, d = co.shape
    mism = cg != co
    frac = float(mism.mean())
    assert frac <= code_frac, f"code mismatch fraction {frac:.2e} > {code_frac}"
    # first mismatching column per row (d if none)
    first = np.where(mism.any(axis=1), mism.argmax(axis=1), d)
    G = co.shape[1] // group_size if group_size > 0 else 1
    G = orc["scales"].shape[1]
    gstart = np.arange(G) * (d // G)
    ok_groups = gstart[None, :] <= first[:, None]          # group starts at/before first mismatch
    sg = gpu["scales"].view(np.float16).astype(np.float32)
    lo, hi = fp16_range(orc["s_pre"], SCALE_REL)
    in_range = (sg >= lo) & (sg <= hi)
    bad = ok_groups & ~in_range
    same_s = gpu["scales"] == orc["scales"]
    zdiff = ok_groups & same_s & (gpu["zeros"] != orc["zeros"])
    zstep = np.abs(gpu["zeros"].astype(np.int32) - orc["zeros"].astype(np.int32))
    dev = np.abs(sg.astype(np.float64) / orc["s_pre"].astype(np.float64) - 1.0)
    if group_bars:
        assert not bad.any(), f"{int(bad.sum())} scales outside 1e-4 of the oracle's pre-fp16 scale"
        assert zdiff.sum() <= CODE_FRAC * max(1, ok_groups.sum()) + 1, \
            f"{int(zdiff.sum())} zero points differ under equal scales"
        assert (zstep[zdiff] <= 1).all(), "a zero point differs by more than one step"
    st = dict(code_mismatch_frac=frac, rows_with_mismatch=int((first < d).sum()),
              scale_exact_frac=float(same_s[ok_groups].mean()) if ok_groups.any() else 1.0,
              free_scales_off=int(bad.sum()),
              free_max_scale_dev=float(dev[ok_groups].max()) if ok_groups.any() else 0.0)
    if report is not None:
        report.update(st)
    return st


def teacher_forced_check(Wp64: np.ndarray, U64: np.ndarray, gpu: dict, bits: int,
                         group_size: int, rows=None, report: dict | None = None):
    """Force the GPU's codes/scales/zeros into the oracle sweep; every place
    where the oracle's own decision differs must be a near-tie: codes by
    |frac(w/s) - 0.5|, zero points (under the same fp16 scale) by
    |frac(-mn/s) - 0.5|, scales by the fp16 rounding of a value within 1e-4
    of the oracle's pre-fp16 scale."""
    sl = slice(None) if rows is None else rows
    f = oracle.quantize_rows(Wp64[sl], U64, bits, group_size,
                             forced_codes=gpu["codes"][sl].astype(np.int16),
                             forced_scales=gpu["scales"][sl], forced_zeros=gpu["zeros"][sl])
    diff = f["own_codes"] != gpu["codes"][sl]
    if diff.any():
        td = f["tie_dist"][diff]
        assert (td <= TIE).all(), (f"{int((td > TIE).sum())} non-tie mismatches "
                                   f"(max tie distance {float(td.max()):.3g})")
    # the oracle's own pre-fp16 scale (on the forced trajectory) agrees with the GPU's fp16 scale
    sg = gpu["scales"][sl].view(np.float16).astype(np.float32)
    lo, hi = fp16_range(f["s_pre"], SCALE_REL)
    assert ((sg >= lo) & (sg <= hi)).all(), "scale outside range on the forced trajectory"
    s_flip = f["own_scales"] != gpu["scales"][sl]
    # zero points decided under the same fp16 scale: a flip must sit at a tie of -mn/s
    z_flip = ~s_flip & (f["own_zeros"] != gpu["zeros"][sl])
    if z_flip.any():
        zt = f["zero_tie_dist"][z_flip]
        assert (zt <= TIE).all(), (f"{int((zt > TIE).sum())} zero points differ off a tie "
                                   f"(max tie distance {float(zt.max()):.3g})")
    if report is not None:
        report.update(forced_code_ties=int(diff.sum()), forced_zero_ties=int(z_flip.sum()),
                      forced_scale_flips=int(s_flip.sum()),
                      max_zero_tie_dist=float(f["zero_tie_dist"][z_flip].max()) if z_flip.any() else 0.0)
    return int(diff.sum())


def mismatch_report(gpu: dict, orc: dict) -> dict:
    """Where the free-running comparison parts: per row the first mismatching
    column and the number of mismatches from there to the row's end (the
    cascade a legitimate tie flip starts)."""
    mism = gpu["codes"] != orc["codes"]
    rows = np.nonzero(mism.any(axis=1))[0]
    first = mism.argmax(axis=1)
    return dict(weights=int(mism.size), mismatches=int(mism.sum()), rows=int(rows.size),
                cascades=[(int(r), int(first[r]), int(mism[r].sum())) for r in rows[:20]])


def to_np(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.float16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def layer_loss_of(W64, codes, scales_bits, zeros, group_size, perm, H64) -> float:
    Q = oracle.dequantize(codes, scales_bits, zeros, group_size, perm)
    return oracle.layer_loss(W64, Q, H64)

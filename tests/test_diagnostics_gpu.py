"""GPU test of the library's per-kind kernel timing (diagnostics used by
bench.py): every kind a layer launches is timed, the times are positive,
and timing changes no result."""
import pytest
import torch

from post_weight_quantization_11_b200 import gptq as G
from tests.test_parity_gpu import _gauss_x, _weights

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_kernel_timing_covers_every_launch_kind_and_changes_nothing():
    from post_weight_quantization_11_b200 import build
    build.build()
    W = _weights(256, 1024, torch.float16, 3).to(DEV)
    X = _gauss_x(2000, 1024, 5, 30.0, 4).to(DEV)
    ref = G.quantize_layer_from_inputs(W, X)
    torch.cuda.synchronize()
    G.gptq_debug_kernel_times()
    G.gptq_debug_kernel_timing(True)
    try:
        res = G.quantize_layer_from_inputs(W, X)
        torch.cuda.synchronize()
    finally:
        G.gptq_debug_kernel_timing(False)
    t = G.gptq_debug_kernel_times()
    for kind in ("hessian", "finalize", "factorization", "init_work", "split_u", "sweep",
                 "update_far", "pack"):
        assert kind in t and t[kind][0] > 0.0 and t[kind][1] > 0, (kind, t)
    # one fused sweep launch per 512-column outer block, no separate near updates
    assert t["sweep"][1] == 1024 // 512 and "update_near" not in t, t
    assert G.gptq_debug_kernel_times() == {}          # records are consumed
    # dynamic groups of 256 start inside an outer block: a sweep launch per
    # 128-column block and a near update after every block but an outer block's last
    G.gptq_debug_kernel_timing(True)
    try:
        G.gptq_quantize_layer(W, res.U, None, 4, 256)
        torch.cuda.synchronize()
    finally:
        G.gptq_debug_kernel_timing(False)
    t2 = G.gptq_debug_kernel_times()
    assert t2["sweep"][1] == 1024 // 128 and t2["update_near"][1] == 6, t2
    # S's fp32 atomic adds run in no fixed order when the tokens are split,
    # so the two runs agree to rounding, not bit for bit
    a, b = ref.S.double(), res.S.double()
    assert float((a - b).norm() / b.norm()) <= 1e-6
    assert float((ref.codes != res.codes).float().mean()) <= 1e-3

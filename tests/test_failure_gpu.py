"""Failure detection without a GPU fault: a bounded device wait whose
condition never comes true gives up after its limit, records a device
status the host reads, and leaves the context usable (no trap, no hang).
The waits are the ones every kernel of the library uses (a completion flag
between CTAs, an mbarrier phase inside a CTA), run with a 50 ms limit."""
import time

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_11_b200 import gptq as G

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    G.load_library()


@pytest.mark.parametrize("which,code", [(0, 0x105), (1, 0x101)])
def test_stuck_wait_ends_as_a_device_status(which, code):
    assert G.gptq_device_status(reset=True) == 0
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)     # nothing ever sets it
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    G.gptq_debug_bounded_wait(flag, which, 50_000_000)
    torch.cuda.synchronize()
    assert 0.04 <= time.perf_counter() - t0 < 5.0
    assert G.gptq_device_status(reset=True) == code
    assert G.gptq_device_status(reset=True) == 0
    # the context still works: the next library call gives the oracle's result
    W = 0.02 * torch.randn(64, 256, generator=torch.Generator().manual_seed(which))
    c, s, z = G.rtn_quantize(W.to(DEV), 4, 128)
    ref = oracle.rtn(W.double().numpy(), 4, 128)
    assert np.array_equal(c.cpu().numpy(), ref["codes"])


def test_flag_already_set_passes_without_a_status():
    flag = torch.ones(1, dtype=torch.int32, device=DEV)
    G.gptq_debug_bounded_wait(flag, 0, 1_000_000_000)
    torch.cuda.synchronize()
    assert G.gptq_device_status(reset=True) == 0

"""GPU parity of the GPTQ sweep (not only round-to-nearest) on the quantizer's
degenerate inputs: an all-zero row (every group takes the [-1, 1] range), a
row that is zero in one group only, groups of one sign (the range is widened
to include 0, so the zero point sits at an end of the code range), and
8-bit codes.  The oracle takes the GPU's S (the H-forced protocol of
tests/parity.py) and every tolerance is the one written there."""
import numpy as np
import pytest
import torch

import oracle
from tests import parity as P
from tests.test_parity_gpu import _check_layer, _gauss_x, _gpu_layer, _weights


def _diagnose(W, X, bits, gs, act):
    """The teacher-forced tie check and the mismatch cascades, printed before
    _check_layer asserts the tolerances (a failure then shows whether the
    disagreements are near-ties and how far each one cascades)."""
    g = _gpu_layer(W, X, bits, gs, act)
    S_gpu = P.mirror_upper(g["S"])
    W64 = W.double().numpy()
    ref = oracle.gptq_layer(W64, S_gpu, X.shape[0], bits, gs, 0.01, act)
    Wp = np.ascontiguousarray(W64[:, ref["perm"]])
    rep = {}
    try:
        P.teacher_forced_check(Wp, ref["U"], g, bits, gs, report=rep)
        rep["forced_check"] = "passed"
    except AssertionError as e:
        rep["forced_check"] = f"FAILED: {e}"
    rep.update(P.mismatch_report(g, ref))
    print("diagnosis", (bits, gs, act), rep)

pytestmark = pytest.mark.gpu


def _degenerate_rows(W: torch.Tensor, g: int) -> torch.Tensor:
    W = W.clone()
    W[0, :] = 0                                   # all-zero row
    W[1, g:2 * g] = 0                             # one all-zero group inside a live row
    W[2, :g] = W[2, :g].abs() + 1e-3              # one-signed groups, both signs
    W[3, :g] = -(W[3, :g].abs() + 1e-3)
    W[4, :] = W[4, :].abs()                       # a whole row of one sign
    W[5, :] = -W[5, :].abs()
    W[6, ::2] = 0                                 # half the columns zero
    return W


@pytest.mark.parametrize("bits,gs,act,dtype", [
    (4, 128, False, torch.float16),
    (4, 128, True, torch.float32),
    (8, 128, False, torch.float16),
    (8, 64, True, torch.float16),
    (2, 32, False, torch.float32),
])
def test_sweep_degenerate_rows(bits, gs, act, dtype):
    m, d, n = 200, 512, 1500
    W = _degenerate_rows(_weights(m, d, dtype, 900 + bits + gs), gs)
    X = _gauss_x(n, d, 5, 40.0, 901 + bits)
    _diagnose(W, X, bits, gs, act)
    st, g, ref = _check_layer(W, X, bits, gs, act, code_bar="free" if bits == 4 else "forced")
    # the all-zero row quantizes to exact zeros: codes equal the zero points
    # and every group's scale is the [-1, 1] range's
    G_ = d // gs
    maxq = (1 << bits) - 1
    z0 = g["zeros"][0]
    assert np.array_equal(g["codes"][0].reshape(G_, gs), np.repeat(z0[:, None], gs, axis=1))
    s_pre = np.float32(2.0) / np.float32(maxq)
    assert np.all(g["scales"][0] == np.float16(s_pre).view(np.uint16))
    assert g["row_loss"][0] == 0.0
    print((bits, gs, act), st)


def test_sweep_bits8_tolerances_hold_on_outlier_inputs():
    """8-bit codes on an outlier workload at several tiles per dimension: at
    255 levels a group's range is cut fine enough that most of the error
    feedback sits below one step, the regime where fp32 and fp64 feedback
    most often part at ties."""
    W = _weights(384, 1024, torch.float16, 77)
    X = _gauss_x(3000, 1024, 10, 60.0, 78)
    _diagnose(W, X, 8, 128, False)
    st, _, _ = _check_layer(W, X, 8, 128, False, code_bar="forced")
    print("bits 8:", st)

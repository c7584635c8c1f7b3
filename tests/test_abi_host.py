"""Host-side checks of the C ABI (no GPU): the library loads, exports every
symbol include/gptq.h declares, and rejects bad arguments before launching
anything (every call below returns during validation)."""
import ctypes
import os
import re

import pytest

from post_weight_quantization_11_b200 import gptq as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "gptq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?(?:int64_t|int|size_t|uint64_t|char\s*\*|void)\s*\**\s*(\w+)\s*\(", txt,
                       flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from post_weight_quantization_11_b200 import build
    build.build()
    return G.load_library()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert len(names) >= 10
    assert sorted(names) == sorted(G.EXPORTED)
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {G.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_cta_caps(lib):
    assert lib.gptq_set_max_ctas(3, 10) == 1 and lib.gptq_set_max_ctas(-1, 10) == 1
    assert lib.gptq_set_max_ctas(2, 10) == 0 and lib.gptq_set_max_ctas(2, 0) == 0
    assert lib.gptq_set_max_ctas(0, -1) == 1
    assert lib.gptq_set_max_ctas(0, 32) == 0 and lib.gptq_set_max_ctas(1, 16) == 0
    assert lib.gptq_set_max_ctas(0, 0) == 0 and lib.gptq_set_max_ctas(1, 0) == 0


def test_status_strings_and_version(lib):
    assert G.gptq_abi_version() == 100
    for code, name in G._STATUS.items():
        assert G.gptq_status_string(code) == name
    assert G.gptq_status_string(99) == "GPTQ_ERR_UNKNOWN"
    assert G.gptq_debug_launch_count() >= 0


def test_workspace_sizes(lib):
    for d in (128, 256, 4096, 14336):
        b = G.gptq_prepare_workspace_bytes(d)
        # A and Y (d x d each) and Xc's two planes of d x 128 fp32
        assert b >= 2 * 4 * d * d + 2 * 4 * d * 128 and b % 256 == 0
    # the allocation-free entry point's fixed 16 MiB scratch covers every d
    # it accepts (d <= 1024, per include/gptq.h)
    assert G.gptq_prepare_workspace_bytes(1024) <= 16 << 20
    for m, d in ((1, 128), (300, 256), (4096, 4096), (14336, 4096)):
        b = G.gptq_quantize_workspace_bytes(m, d, 128)
        assert b >= 4 * m * d + 4 * m * 128
    assert G.gptq_quantize_workspace_bytes(64, 256, 64) == 0
    assert G.gptq_prepare_workspace_bytes(0) == 0


FAKE = ctypes.c_void_p(1 << 20)          # 16-byte aligned, never dereferenced
MIS = ctypes.c_void_p((1 << 20) + 4)     # misaligned


def test_validation_rejects_before_launch(lib):
    # The calls below pass fake device addresses and rely on the library
    # rejecting them before any launch; where a GPU is visible a call that
    # wrongly passed would launch on them, so these checks run without one.
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks with fake pointers run where no GPU is visible")
    n0 = ctypes.c_int64(0)
    # null / misaligned pointers
    assert lib.gptq_hessian_accumulate(None, FAKE, 10, 256, None, None) == 1
    assert lib.gptq_hessian_accumulate(MIS, FAKE, 10, 256, None, None) == 1
    # shapes
    assert lib.gptq_hessian_accumulate(FAKE, FAKE, 10, 200, None, None) == 2
    assert lib.gptq_hessian_accumulate(FAKE, FAKE, -1, 256, None, None) == 2
    assert lib.gptq_hessian_accumulate(FAKE, FAKE, 10, 64, None, None) == 2
    # n_tokens == 0 is a no-op that still counts nothing
    assert lib.gptq_hessian_accumulate(FAKE, FAKE, 0, 256, ctypes.byref(n0), None) == 0
    assert n0.value == 0
    # host-streamed accumulation: ring size, chunk, events
    H = lib.gptq_hessian_accumulate_host
    ring = 2 * 64 * 256 * 2
    assert H(None, FAKE, 10, 256, None, FAKE, ring, 64, None, FAKE, FAKE, FAKE) == 1
    assert H(FAKE, FAKE, 10, 256, None, MIS, ring, 64, None, FAKE, FAKE, FAKE) == 1
    assert H(FAKE, FAKE, 10, 256, None, FAKE, ring, 64, None, FAKE, None, FAKE) == 1
    assert H(FAKE, None, 10, 256, None, FAKE, ring, 64, None, FAKE, FAKE, FAKE) == 1
    assert H(FAKE, FAKE, 10, 256, None, FAKE, ring - 2, 64, None, FAKE, FAKE, FAKE) == 1
    assert H(FAKE, FAKE, 10, 200, None, FAKE, ring, 64, None, FAKE, FAKE, FAKE) == 2
    assert H(FAKE, FAKE, 10, 256, None, FAKE, ring, 0, None, FAKE, FAKE, FAKE) == 2
    assert H(FAKE, FAKE, 0, 256, ctypes.byref(n0), FAKE, ring, 64, None, FAKE, FAKE, FAKE) == 0
    assert n0.value == 0
    # failure-detection probe: argument checks
    assert lib.gptq_debug_bounded_wait(FAKE, 2, 50_000_000, None) == 1
    assert lib.gptq_debug_bounded_wait(None, 0, 50_000_000, None) == 1
    assert lib.gptq_debug_bounded_wait(FAKE, 0, 10, None) == 1
    assert lib.gptq_debug_bounded_wait(FAKE, 1, 2_000_000_000, None) == 1
    ws = G.gptq_prepare_workspace_bytes(256)
    assert lib.gptq_prepare_hinv(FAKE, 256, 0, 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 2
    assert lib.gptq_prepare_hinv(FAKE, 256, 10, 0.01, 1, None, FAKE, FAKE, FAKE, ws, None) == 1
    assert lib.gptq_prepare_hinv(FAKE, 256, 10, -1.0, 0, None, FAKE, FAKE, FAKE, ws, None) == 1
    assert lib.gptq_prepare_hinv(FAKE, 256, 10, 0.01, 0, None, FAKE, FAKE, FAKE, 16, None) == 1
    assert lib.gptq_prepare_hinv(FAKE, 300, 10, 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 2
    wq = G.gptq_quantize_workspace_bytes(64, 256, 128)
    args = lambda **k: dict(dict(W=FAKE, dt=1, m=64, d=256, U=FAKE, perm=None, bits=4, g=128,
                                 B=128, codes=FAKE, scales=FAKE, zeros=FAKE, loss=None, ws=FAKE,
                                 wsb=wq), **k)

    def q(**k):
        a = args(**k)
        return lib.gptq_quantize_layer(a["W"], a["dt"], a["m"], a["d"], a["U"], a["perm"],
                                       a["bits"], a["g"], a["B"], a["codes"], a["scales"],
                                       a["zeros"], a["loss"], a["ws"], a["wsb"], None)
    assert q(bits=5) == 4
    assert q(g=96) == 4
    assert q(B=64) == 4
    assert q(dt=7) == 1
    assert q(d=200) == 2
    assert q(m=0) == 2
    assert q(W=None) == 1
    assert q(U=MIS) == 1
    assert q(wsb=100) == 1
    assert q(g=384, d=768) == 4               # a dynamic group may not straddle an outer block
    assert q(g=256, d=512, wsb=100) == 1      # wide dynamic groups: accepted up to the ws check
    assert q(g=1024, d=2048, wsb=100) == 1
    assert q(g=-1, wsb=100) == 1              # one group per row: accepted up to the ws check

    def qs(**k):
        a = args(**k)
        return lib.gptq_quantize_layer_static(a["W"], a["dt"], a["m"], a["d"], a["U"], a["perm"],
                                              a["bits"], a["g"], a["B"], a["codes"], a["scales"],
                                              a["zeros"], a["loss"], a["ws"], a["wsb"], None)
    assert qs(g=96) == 4
    assert qs(g=384) == 4                     # must divide d_in
    assert qs(g=256, wsb=100) == 1            # accepted up to the ws check
    assert qs(bits=5) == 4 and qs(d=200) == 2 and qs(W=None) == 1
    assert lib.rtn_quantize(FAKE, 1, 64, 256, 3, 48, FAKE, FAKE, FAKE, None) == 4
    assert lib.rtn_quantize(FAKE, 1, 64, 384, 4, 256, FAKE, FAKE, FAKE, None) == 4
    assert lib.rtn_quantize(None, 1, 64, 256, 4, 128, FAKE, FAKE, FAKE, None) == 1
    W4 = lib.gptq_w4a16_gemm
    assert W4(None, 1, FAKE, FAKE, FAKE, None, 64, 256, 128, FAKE, None) == 1
    assert W4(FAKE, 1, MIS, FAKE, FAKE, None, 64, 256, 128, FAKE, None) == 1
    assert W4(FAKE, 9, FAKE, FAKE, FAKE, None, 64, 256, 128, FAKE, None) == 4
    assert W4(FAKE, 0, FAKE, FAKE, FAKE, None, 64, 256, 128, FAKE, None) == 4
    assert W4(FAKE, 1, FAKE, FAKE, FAKE, None, 64, 200, 128, FAKE, None) == 2
    assert W4(FAKE, 1, FAKE, FAKE, FAKE, None, 0, 256, 128, FAKE, None) == 2
    assert W4(FAKE, 1, FAKE, FAKE, FAKE, None, 64, 256, 48, FAKE, None) == 4
    assert W4(FAKE, 1, FAKE, FAKE, FAKE, None, 64, 384, 256, FAKE, None) == 4
    assert lib.gptq_pack_int4(FAKE, FAKE, 4, 12, 1, FAKE, FAKE, None) == 2
    assert lib.gptq_pack_int4(FAKE, FAKE, 4, 16, 0, FAKE, FAKE, None) == 2
    assert lib.gptq_unpack_int4(FAKE, FAKE, 0, 16, 1, FAKE, FAKE, None) == 2


def test_batched_entry_points_validate_before_launch(lib):
    """The grouped / batched entry points for mixture-of-experts layers
    reject bad arguments before launching (fake pointers; no GPU)."""
    import numpy as np
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks with fake pointers run where no GPU is visible")
    I64P = lambda a: ctypes.c_void_p(a.ctypes.data)
    off = np.array([0, 10, 10, 40], dtype=np.int64)
    Hg = lib.gptq_hessian_accumulate_grouped
    assert Hg(None, FAKE, 40, 256, I64P(off), 3, None, None) == 1
    assert Hg(FAKE, FAKE, 40, 256, None, 3, None, None) == 1
    assert Hg(MIS, FAKE, 40, 256, I64P(off), 3, None, None) == 1
    assert Hg(FAKE, FAKE, 40, 200, I64P(off), 3, None, None) == 2
    assert Hg(FAKE, FAKE, 41, 256, I64P(off), 3, None, None) == 2       # offsets[E] != n
    bad = np.array([0, 20, 10, 40], dtype=np.int64)                      # decreasing
    assert Hg(FAKE, FAKE, 40, 256, I64P(bad), 3, None, None) == 2
    assert Hg(FAKE, FAKE, 40, 256, I64P(off), 0, None, None) == 2
    # all groups empty: a no-op that counts nothing
    z = np.zeros(4, dtype=np.int64)
    seen = np.zeros(3, dtype=np.int64)
    assert Hg(FAKE, FAKE, 0, 256, I64P(z), 3, I64P(seen), None) == 0
    assert not seen.any()
    Gr = lib.gptq_gather_rows
    assert Gr(None, 10, 256, FAKE, 5, FAKE, None) == 1
    assert Gr(FAKE, 10, 256, FAKE, 5, MIS, None) == 1
    assert Gr(FAKE, 10, 252, FAKE, 5, FAKE, None) == 2
    assert Gr(FAKE, 10, 256, FAKE, -1, FAKE, None) == 2
    assert Gr(None, 10, 256, None, 0, None, None) == 0                   # nothing to gather
    ws = G.gptq_prepare_batched_workspace_bytes(256, 3)
    assert ws >= 3 * 2 * 4 * 256 * 256
    assert G.gptq_prepare_batched_workspace_bytes(256, 1) == G.gptq_prepare_workspace_bytes(256)
    nt = np.array([100, 50, 7], dtype=np.int64)
    Pb = lib.gptq_prepare_hinv_batched
    assert Pb(FAKE, 3, 256, None, 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 1
    assert Pb(FAKE, 3, 256, I64P(nt), 0.01, 1, None, FAKE, FAKE, FAKE, ws, None) == 1
    assert Pb(FAKE, 3, 256, I64P(nt), 0.01, 0, None, FAKE, FAKE, FAKE, ws - 1, None) == 1
    assert Pb(FAKE, 0, 256, I64P(nt), 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 2
    nt0 = np.array([100, 0, 7], dtype=np.int64)
    assert Pb(FAKE, 3, 256, I64P(nt0), 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 2
    assert Pb(FAKE, 3, 200, I64P(nt), 0.01, 0, None, FAKE, FAKE, FAKE, ws, None) == 2
    wq = G.gptq_quantize_workspace_bytes(64, 256, 128)
    Qb = lib.gptq_quantize_layer_batched
    assert Qb(FAKE, 1, 0, 64, 256, FAKE, None, 4, 128, 128, FAKE, FAKE, FAKE, None, FAKE, wq,
              None) == 2
    assert Qb(None, 1, 2, 64, 256, FAKE, None, 4, 128, 128, FAKE, FAKE, FAKE, None, FAKE, wq,
              None) == 1
    assert Qb(FAKE, 1, 2, 64, 256, FAKE, None, 4, 96, 128, FAKE, FAKE, FAKE, None, FAKE, wq,
              None) == 4
    # a layer slice that would leave the next one misaligned: 3 rows of fp16 scales
    assert Qb(FAKE, 1, 2, 3, 256, FAKE, None, 4, 128, 128, FAKE, FAKE, FAKE, None, FAKE, wq,
              None) == 2


def test_static_entry_checks_arguments_like_the_workspace_one(lib):
    """gptq_prepare_hinv_static returns the status gptq_prepare_hinv gives for
    the same bad argument, before its size limit and its scratch lookup."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks with fake pointers run where no GPU is visible")
    S = lib.gptq_prepare_hinv_static
    assert S(None, 2048, 10, 0.01, 0, None, FAKE, FAKE, None) == 1
    assert S(FAKE, 2048, 10, 0.01, 1, None, FAKE, FAKE, None) == 1
    assert S(FAKE, 2048, 10, -1.0, 0, None, FAKE, FAKE, None) == 1
    assert S(MIS, 512, 10, 0.01, 0, None, FAKE, FAKE, None) == 1
    assert S(FAKE, 300, 10, 0.01, 0, None, FAKE, FAKE, None) == 2
    assert S(FAKE, 512, 0, 0.01, 0, None, FAKE, FAKE, None) == 2
    assert S(FAKE, 2048, 10, 0.01, 0, None, FAKE, FAKE, None) == 2    # beyond the scratch


def test_pack_bits_validates_before_launch(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks with fake pointers run where no GPU is visible")
    Pk, Uk = lib.gptq_pack_bits, lib.gptq_unpack_bits
    for f in (Pk, Uk):
        assert f(None, FAKE, 4, 64, 1, 3, FAKE, FAKE, None) == 1
        assert f(FAKE, FAKE, 4, 64, 1, 9, FAKE, FAKE, None) == 4
        assert f(FAKE, FAKE, 4, 64, 1, 1, FAKE, FAKE, None) == 4
        assert f(FAKE, FAKE, 4, 48, 1, 3, FAKE, FAKE, None) == 2
        assert f(FAKE, FAKE, 0, 64, 1, 3, FAKE, FAKE, None) == 2
        assert f(FAKE, FAKE, 4, 64, 0, 3, FAKE, FAKE, None) == 2
    assert Pk(MIS, FAKE, 4, 64, 1, 3, FAKE, FAKE, None) == 1


def test_awq_entry_points_validate_before_launch(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks with fake pointers run where no GPU is visible")
    C = lib.gptq_channel_abs_sum
    assert C(FAKE, 10, 256, None, None) == 1
    assert C(MIS, 10, 256, FAKE, None) == 1
    assert C(FAKE, 10, 252, FAKE, None) == 2
    assert C(FAKE, -1, 256, FAKE, None) == 2
    assert C(None, 0, 256, FAKE, None) == 0                  # no tokens: nothing to add
    wb = lib.gptq_awq_workspace_bytes(64, 256)
    assert wb >= 4 * (256 * 256 + 2 * 64 * 256)
    A = lib.gptq_awq_search

    def aw(**k):
        a = dict(W=FAKE, dt=1, m=64, d=256, S=FAKE, n=100, acc=FAKE, grid=20, bits=4, g=128,
                 losses=FAKE, best=FAKE, scales=FAKE, Ws=None, Ss=None, ws=FAKE, wsb=wb)
        a.update(k)
        return A(a["W"], a["dt"], a["m"], a["d"], a["S"], a["n"], a["acc"], a["grid"],
                 a["bits"], a["g"], a["losses"], a["best"], a["scales"], a["Ws"], a["Ss"],
                 a["ws"], a["wsb"], None)
    assert aw(W=None) == 1 and aw(acc=None) == 1 and aw(dt=5) == 1 and aw(Ws=MIS) == 1
    assert aw(bits=5) == 4 and aw(g=48) == 4 and aw(g=96) == 4
    assert aw(d=200) == 2 and aw(m=0) == 2 and aw(n=0) == 2 and aw(grid=0) == 2
    assert aw(wsb=wb - 1) == 1

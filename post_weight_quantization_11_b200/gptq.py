"""Thin Python binding of libgptq.so (include/gptq.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
torch is used for device memory and the current stream.  The functions carry
the names of the C entry points; each checks dtypes/devices/contiguity,
allocates outputs and workspace with torch when they are not given, passes
raw pointers and sizes, and raises GptqError on a non-zero status.

There is no CPU fallback: if libgptq.so is missing or cannot be loaded, the
first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq.so")

GPTQ_DTYPE_F32 = 0
GPTQ_DTYPE_F16 = 1

_STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_SHAPE", 3: "GPTQ_ERR_NOT_PD",
           4: "GPTQ_ERR_UNSUPPORTED", 5: "GPTQ_ERR_CUDA", 6: "GPTQ_ERR_TIMEOUT"}

# every symbol include/gptq.h declares
EXPORTED = ("gptq_status_string", "gptq_abi_version", "gptq_debug_launch_count",
            "gptq_device_status", "gptq_set_max_ctas",
            "gptq_hessian_accumulate", "gptq_hessian_accumulate_host",
            "gptq_hessian_accumulate_grouped", "gptq_gather_rows",
            "gptq_prepare_workspace_bytes", "gptq_prepare_hinv", "gptq_prepare_hinv_static",
            "gptq_prepare_batched_workspace_bytes", "gptq_prepare_hinv_batched",
            "gptq_quantize_layer_batched",
            "gptq_quantize_workspace_bytes", "gptq_quantize_layer", "gptq_quantize_layer_static",
            "gptq_pack_int4", "gptq_pack_bits", "gptq_unpack_bits",
            "gptq_channel_abs_sum", "gptq_awq_workspace_bytes", "gptq_awq_search",
            "gptq_unpack_int4", "gptq_w4a16_gemm", "gptq_w4a16_matmul_workspace_bytes",
            "gptq_w4a16_matmul", "rtn_quantize", "gptq_debug_gemm_nt",
            "gptq_debug_chol_task_order", "gptq_debug_div_rn", "gptq_debug_bounded_wait",
            "gptq_debug_kernel_timing", "gptq_debug_kernel_times", "gptq_debug_kernel_kind_name")


class GptqError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)}")
        self.status = status


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libgptq.so (raises OSError when it is missing: no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libgptq.so not found at {path}; build it with "
                      f"`python -m post_weight_quantization_11_b200.build`")
    lib = ctypes.CDLL(path)
    P, I64, I32, F32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    SZ = ctypes.c_size_t
    sig = {
        "gptq_status_string": ([I32], ctypes.c_char_p),
        "gptq_abi_version": ([], I32),
        "gptq_debug_launch_count": ([], ctypes.c_uint64),
        "gptq_device_status": ([P, I32], I32),
        "gptq_set_max_ctas": ([I32, I32], I32),
        "gptq_hessian_accumulate": ([P, P, I64, I64, P, P], I32),
        "gptq_hessian_accumulate_host": ([P, P, I64, I64, P, P, SZ, I64, P, P, P, P], I32),
        "gptq_hessian_accumulate_grouped": ([P, P, I64, I64, P, I64, P, P], I32),
        "gptq_gather_rows": ([P, I64, I64, P, I64, P, P], I32),
        "gptq_prepare_workspace_bytes": ([I64], SZ),
        "gptq_prepare_batched_workspace_bytes": ([I64, I64], SZ),
        "gptq_prepare_hinv_batched": ([P, I64, I64, P, F32, I32, P, P, P, P, SZ, P], I32),
        "gptq_quantize_layer_batched": ([P, I32, I64, I64, I64, P, P, I32, I32, I32, P, P, P, P,
                                         P, SZ, P], I32),
        "gptq_prepare_hinv": ([P, I64, I64, F32, I32, P, P, P, P, SZ, P], I32),
        "gptq_prepare_hinv_static": ([P, I64, I64, F32, I32, P, P, P, P], I32),
        "gptq_quantize_workspace_bytes": ([I64, I64, I32], SZ),
        "gptq_quantize_layer": ([P, I32, I64, I64, P, P, I32, I32, I32, P, P, P, P, P, SZ, P],
                                I32),
        "gptq_quantize_layer_static": ([P, I32, I64, I64, P, P, I32, I32, I32, P, P, P, P, P, SZ,
                                        P], I32),
        "gptq_pack_int4": ([P, P, I64, I64, I64, P, P, P], I32),
        "gptq_unpack_int4": ([P, P, I64, I64, I64, P, P, P], I32),
        "gptq_pack_bits": ([P, P, I64, I64, I64, I32, P, P, P], I32),
        "gptq_channel_abs_sum": ([P, I64, I64, P, P], I32),
        "gptq_awq_workspace_bytes": ([I64, I64], SZ),
        "gptq_awq_search": ([P, I32, I64, I64, P, I64, P, I32, I32, I32, P, P, P, P, P, P, SZ, P],
                            I32),
        "gptq_unpack_bits": ([P, P, I64, I64, I64, I32, P, P, P], I32),
        "rtn_quantize": ([P, I32, I64, I64, I32, I32, P, P, P, P], I32),
        "gptq_w4a16_gemm": ([P, I64, P, P, P, P, I64, I64, I32, P, P], I32),
        "gptq_w4a16_matmul_workspace_bytes": ([I64, I64], SZ),
        "gptq_w4a16_matmul": ([P, I64, P, P, P, P, I64, I64, I32, P, P, SZ, P], I32),
        "gptq_debug_gemm_nt": ([P, I64, P, I64, P, I64, I64, I64, I64, F32, F32, I32, P], I32),
        "gptq_debug_chol_task_order": ([I64, P, I64], I64),
        "gptq_debug_div_rn": ([P, P, I64, P], I32),
        "gptq_debug_bounded_wait": ([P, I32, I64, P], I32),
        "gptq_debug_kernel_timing": ([I32], I32),
        "gptq_debug_kernel_times": ([P, P, I32], I32),
        "gptq_debug_kernel_kind_name": ([I32], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise GptqError(fn, status)


def _need(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _wdtype(W: torch.Tensor) -> int:
    if W.dtype == torch.float16:
        return GPTQ_DTYPE_F16
    if W.dtype == torch.float32:
        return GPTQ_DTYPE_F32
    raise ValueError("W must be float16 or float32")


# --------------------------------------------------------------------------
# Entry points
# --------------------------------------------------------------------------

def gptq_abi_version() -> int:
    return int(load_library().gptq_abi_version())


def gptq_debug_launch_count() -> int:
    return int(load_library().gptq_debug_launch_count())


def gptq_device_status(reset: bool = True) -> int:
    """0, or the error code a bounded device-side wait recorded (synchronous)."""
    v = ctypes.c_int32(0)
    _check("gptq_device_status", load_library().gptq_device_status(ctypes.byref(v), int(reset)))
    return int(v.value)


GPTQ_CTAS_HESSIAN, GPTQ_CTAS_PREPARE, GPTQ_CTAS_QUANTIZE = 0, 1, 2


def gptq_set_max_ctas(kind: int, max_ctas: int) -> None:
    """Cap the CTAs of the persistent Hessian (kind 0) or factorization
    (kind 1) kernels; 0 restores one per SM."""
    _check("gptq_set_max_ctas", load_library().gptq_set_max_ctas(int(kind), int(max_ctas)))


N_KERNEL_KINDS = 16


def gptq_debug_kernel_timing(enable: bool) -> None:
    """Per-kind CUDA-event timing of the library's launches (eager use only)."""
    _check("gptq_debug_kernel_timing", load_library().gptq_debug_kernel_timing(int(bool(enable))))


def gptq_debug_kernel_times() -> dict:
    """{kind: (milliseconds, timed launch sites)} since the last call (waits for the events)."""
    import numpy as np
    ms = np.zeros(N_KERNEL_KINDS, dtype=np.float64)
    sp = np.zeros(N_KERNEL_KINDS, dtype=np.int64)
    lib = load_library()
    _check("gptq_debug_kernel_times",
           lib.gptq_debug_kernel_times(ctypes.c_void_p(ms.ctypes.data),
                                       ctypes.c_void_p(sp.ctypes.data), N_KERNEL_KINDS))
    return {lib.gptq_debug_kernel_kind_name(k).decode(): (float(ms[k]), int(sp[k]))
            for k in range(N_KERNEL_KINDS) if sp[k]}


def gptq_status_string(status: int) -> str:
    return load_library().gptq_status_string(int(status)).decode()


def gptq_hessian_accumulate(S: torch.Tensor, X: torch.Tensor) -> int:
    """S (d x d fp32, upper triangle) += X^T X for X (n x d fp16). Returns n."""
    _need(S, "S", torch.float32)
    _need(X, "X", torch.float16)
    n, d = X.shape
    if S.shape != (d, d):
        raise ValueError("S must be d x d")
    _check("gptq_hessian_accumulate",
           load_library().gptq_hessian_accumulate(_ptr(S), _ptr(X), n, d, None, _stream(S)))
    return n


def gptq_gather_rows(X: torch.Tensor, idx: torch.Tensor, out=None) -> torch.Tensor:
    """out[r] = X[idx[r]] (the routed tokens' rows, e.g. expert-major)."""
    _need(X, "X", torch.float16)
    _need(idx, "idx", torch.int32)
    n, d = X.shape
    k = idx.numel()
    out = torch.empty(k, d, dtype=torch.float16, device=X.device) if out is None else out
    _need(out, "out", torch.float16)
    _check("gptq_gather_rows",
           load_library().gptq_gather_rows(_ptr(X), n, d, _ptr(idx), k, _ptr(out), _stream(X)))
    return out


def gptq_hessian_accumulate_grouped(S: torch.Tensor, X: torch.Tensor, offsets) -> list:
    """S[e] (E x d x d fp32, upper triangles) += X[o_e:o_{e+1}]^T X[o_e:o_{e+1}]
    for the row segments given by the host offsets (E + 1 non-decreasing
    ints, 0 .. n).  One launch for up to 64 segments.  Returns the
    segments' token counts."""
    import numpy as np
    _need(S, "S", torch.float32)
    _need(X, "X", torch.float16)
    n, d = X.shape
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64))
    E = off.size - 1
    if S.shape != (E, d, d):
        raise ValueError("S must be E x d x d")
    _check("gptq_hessian_accumulate_grouped",
           load_library().gptq_hessian_accumulate_grouped(
               _ptr(S), _ptr(X), n, d, ctypes.c_void_p(off.ctypes.data), E, None, _stream(S)))
    return [int(v) for v in np.diff(off)]


class HostHessian:
    """Accumulates S += X^T X for calibration batches held in HOST memory.

    Owns what gptq_hessian_accumulate_host needs across calls: a two-slot
    device ring of chunk_tokens x d fp16, a non-blocking copy stream and the
    two ordering events.  Each batch's PCIe copy overlaps the accumulation of
    the previous chunk, and the copies of the next batch overlap whatever the
    caller queues after accumulate() on the current stream, for as long as
    the two slots last.  The default chunk is 128 MiB of fp16 tokens (16384
    tokens at d = 4096, 2.4 ms of copy at 55 GB/s): two slots outlast the
    prepare / quantize / pack of a 4096 x 4096 layer.
    """

    def __init__(self, d: int, device=None, chunk_tokens: int | None = None):
        dev = torch.device("cuda" if device is None else device)
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.d = int(d)
        self.chunk = int(chunk_tokens) if chunk_tokens else max(64, (1 << 26) // self.d // 64 * 64)
        self.device = dev
        self.stage = torch.empty(2 * self.chunk * self.d, dtype=torch.float16, device=dev)
        self.copy_stream = torch.cuda.Stream(device=dev)
        self.ev_filled = torch.cuda.Event()
        self.ev_freed = torch.cuda.Event()
        # torch creates an event's CUDA handle at its first record
        self.ev_filled.record(self.copy_stream)
        self.ev_freed.record(self.copy_stream)
        self._inflight = []          # (event, host tensor) until that tensor's copies are done

    def accumulate(self, S: torch.Tensor, X_host: torch.Tensor) -> int:
        """S (d x d fp32 on the device, upper triangle) += X^T X for X_host
        (n x d fp16, CPU, contiguous; pinned for the copies to overlap).
        Asynchronous on the current stream.  The streamer keeps a reference to
        X_host until its copies have completed; do not modify it before then.
        Returns n."""
        _need(S, "S", torch.float32)
        if not isinstance(X_host, torch.Tensor) or X_host.is_cuda:
            raise ValueError("X_host must be a CPU tensor")
        if X_host.dtype != torch.float16 or not X_host.is_contiguous() or X_host.dim() != 2:
            raise ValueError("X_host must be a contiguous n x d float16 tensor")
        n, d = X_host.shape
        if d != self.d or S.shape != (d, d) or S.device != self.device:
            raise ValueError("S must be d x d on the streamer's device, X_host n x d")
        st = torch.cuda.current_stream(self.device)
        _check("gptq_hessian_accumulate_host",
               load_library().gptq_hessian_accumulate_host(
                   _ptr(S), ctypes.c_void_p(X_host.data_ptr()), n, d, None, _ptr(self.stage),
                   self.stage.numel() * 2, self.chunk, ctypes.c_void_p(st.cuda_stream),
                   ctypes.c_void_p(self.copy_stream.cuda_stream),
                   ctypes.c_void_p(self.ev_filled.cuda_event),
                   ctypes.c_void_p(self.ev_freed.cuda_event)))
        done = torch.cuda.Event()
        done.record(self.copy_stream)        # after this call's last copy
        self._inflight = [(e, t) for e, t in self._inflight if not e.query()]
        self._inflight.append((done, X_host))
        return n


def gptq_prepare_workspace_bytes(d: int) -> int:
    return int(load_library().gptq_prepare_workspace_bytes(int(d)))


def gptq_prepare_hinv(S: torch.Tensor, n_tokens: int, damp_rel: float = 0.01,
                      act_order: bool = False, perm=None, U=None, info=None, ws=None):
    """Returns (perm int32 d, U fp32 d x d, info int32[1] device)."""
    _need(S, "S", torch.float32)
    d = S.shape[0]
    dev = S.device
    perm = torch.empty(d, dtype=torch.int32, device=dev) if perm is None else perm
    U = torch.empty(d, d, dtype=torch.float32, device=dev) if U is None else U
    info = torch.zeros(1, dtype=torch.int32, device=dev) if info is None else info
    nb = gptq_prepare_workspace_bytes(d)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if ws is None else ws
    for t, nm in ((perm, "perm"), (U, "U"), (info, "info"), (ws, "ws")):
        _need(t, nm)
    _check("gptq_prepare_hinv",
           load_library().gptq_prepare_hinv(_ptr(S), d, int(n_tokens), float(damp_rel),
                                            int(bool(act_order)), _ptr(perm), _ptr(U), _ptr(info),
                                            _ptr(ws), ws.numel() * ws.element_size(), _stream(S)))
    return perm, U, info


def gptq_prepare_hinv_static(S: torch.Tensor, n_tokens: int, damp_rel: float = 0.01,
                             act_order: bool = False, perm=None, U=None, info=None):
    """gptq_prepare_hinv on the library's fixed scratch (no workspace; d <= 1024)."""
    _need(S, "S", torch.float32)
    d = S.shape[0]
    dev = S.device
    perm = torch.empty(d, dtype=torch.int32, device=dev) if perm is None else perm
    U = torch.empty(d, d, dtype=torch.float32, device=dev) if U is None else U
    info = torch.zeros(1, dtype=torch.int32, device=dev) if info is None else info
    _check("gptq_prepare_hinv_static",
           load_library().gptq_prepare_hinv_static(_ptr(S), d, int(n_tokens), float(damp_rel),
                                                   int(bool(act_order)), _ptr(perm), _ptr(U),
                                                   _ptr(info), _stream(S)))
    return perm, U, info


def gptq_prepare_batched_workspace_bytes(d: int, n_mats: int) -> int:
    return int(load_library().gptq_prepare_batched_workspace_bytes(int(d), int(n_mats)))


def gptq_prepare_hinv_batched(S: torch.Tensor, n_tokens, damp_rel: float = 0.01,
                              act_order: bool = False, perm=None, U=None, info=None, ws=None):
    """The preparation of E Hessians at once (one factorization launch).
    S: E x d x d fp32; n_tokens: E host ints.  Returns (perm E x d int32,
    U E x d x d fp32, info E int32 on the device)."""
    import numpy as np
    _need(S, "S", torch.float32)
    E, d = S.shape[0], S.shape[1]
    dev = S.device
    nt = np.ascontiguousarray(np.asarray(n_tokens, dtype=np.int64))
    if nt.size != E:
        raise ValueError("n_tokens must have one entry per matrix")
    perm = torch.empty(E, d, dtype=torch.int32, device=dev) if perm is None else perm
    U = torch.empty(E, d, d, dtype=torch.float32, device=dev) if U is None else U
    info = torch.zeros(E, dtype=torch.int32, device=dev) if info is None else info
    nb = gptq_prepare_batched_workspace_bytes(d, E)
    ws = torch.empty(nb, dtype=torch.uint8, device=dev) if ws is None else ws
    for t, nm in ((perm, "perm"), (U, "U"), (info, "info"), (ws, "ws")):
        _need(t, nm)
    _check("gptq_prepare_hinv_batched",
           load_library().gptq_prepare_hinv_batched(
               _ptr(S), E, d, ctypes.c_void_p(nt.ctypes.data), float(damp_rel),
               int(bool(act_order)), _ptr(perm), _ptr(U), _ptr(info), _ptr(ws),
               ws.numel() * ws.element_size(), _stream(S)))
    return perm, U, info


def gptq_quantize_layer_batched(W: torch.Tensor, U: torch.Tensor, perm=None, bits: int = 4,
                                group_size: int = 128, block_size: int = 128, codes=None,
                                scales=None, zeros=None, row_loss=None, ws=None,
                                shared_workspace: bool = False):
    """gptq_quantize_layer over E stacked layers (W: E x m x d, U: E x d x d,
    perm: E x d or None).  By default one workspace per layer (the layers are
    swept together); shared_workspace: one workspace, the layers one after
    the other.  Returns (codes E x m x d, scales E x m x G, zeros E x m x G,
    row_loss E x m)."""
    _need(W, "W")
    _need(U, "U", torch.float32)
    E, m, d = W.shape
    dev = W.device
    G = 1 if group_size in (-1, d) else d // group_size
    codes = torch.empty(E, m, d, dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty(E, m, G, dtype=torch.float16, device=dev) if scales is None else scales
    zeros = torch.empty(E, m, G, dtype=torch.uint8, device=dev) if zeros is None else zeros
    row_loss = torch.empty(E, m, dtype=torch.float32, device=dev) if row_loss is None else row_loss
    nb = gptq_quantize_workspace_bytes(m, d, block_size) * (1 if shared_workspace else E)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev) if ws is None else ws
    if perm is not None:
        _need(perm, "perm", torch.int32)
    _check("gptq_quantize_layer_batched",
           load_library().gptq_quantize_layer_batched(
               _ptr(W), _wdtype(W), E, m, d, _ptr(U), _ptr(perm), int(bits), int(group_size),
               int(block_size), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(row_loss), _ptr(ws),
               ws.numel() * ws.element_size(), _stream(W)))
    return codes, scales, zeros, row_loss


def gptq_quantize_workspace_bytes(d_out: int, d_in: int, block_size: int = 128) -> int:
    return int(load_library().gptq_quantize_workspace_bytes(int(d_out), int(d_in),
                                                            int(block_size)))


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, perm=None, bits: int = 4,
                        group_size: int = 128, block_size: int = 128, codes=None, scales=None,
                        zeros=None, row_loss=None, ws=None, static_groups: bool = False):
    """Returns (codes uint8 m x d, scales fp16 m x G, zeros uint8 m x G, row_loss fp32 m).
    group_size -1: one group per row.  static_groups: group parameters from
    the rows before the sweep (gptq_quantize_layer_static)."""
    _need(W, "W")
    _need(U, "U", torch.float32)
    m, d = W.shape
    dev = W.device
    G = 1 if group_size in (-1, d) else d // group_size
    codes = torch.empty(m, d, dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty(m, G, dtype=torch.float16, device=dev) if scales is None else scales
    zeros = torch.empty(m, G, dtype=torch.uint8, device=dev) if zeros is None else zeros
    row_loss = torch.empty(m, dtype=torch.float32, device=dev) if row_loss is None else row_loss
    nb = gptq_quantize_workspace_bytes(m, d, block_size)
    ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev) if ws is None else ws
    if perm is not None:
        _need(perm, "perm", torch.int32)
    name = "gptq_quantize_layer_static" if static_groups else "gptq_quantize_layer"
    _check(name, getattr(load_library(), name)(_ptr(W), _wdtype(W), m, d, _ptr(U), _ptr(perm),
                                               int(bits), int(group_size), int(block_size),
                                               _ptr(codes), _ptr(scales), _ptr(zeros),
                                               _ptr(row_loss), _ptr(ws),
                                               ws.numel() * ws.element_size(), _stream(W)))
    return codes, scales, zeros, row_loss


def gptq_pack_int4(codes: torch.Tensor, zeros: torch.Tensor, qweight=None, qzeros=None):
    _need(codes, "codes", torch.uint8)
    _need(zeros, "zeros", torch.uint8)
    m, d = codes.shape
    G = zeros.shape[1]
    dev = codes.device
    qweight = torch.empty(m, d // 8, dtype=torch.int32, device=dev) if qweight is None else qweight
    qzeros = torch.empty(m, (G + 1) // 2, dtype=torch.uint8, device=dev) if qzeros is None else qzeros
    _check("gptq_pack_int4",
           load_library().gptq_pack_int4(_ptr(codes), _ptr(zeros), m, d, G, _ptr(qweight),
                                         _ptr(qzeros), _stream(codes)))
    return qweight, qzeros


def gptq_pack_bits(codes: torch.Tensor, zeros: torch.Tensor, bits: int, qweight=None,
                   qzeros=None):
    """b-bit storage (one little-endian bit stream per row; b = 4 is the
    INT4 layout).  Returns (qweight int32 m x d b/32, qzeros uint8 m x ceil(G b/8))."""
    _need(codes, "codes", torch.uint8)
    _need(zeros, "zeros", torch.uint8)
    m, d = codes.shape
    G = zeros.shape[1]
    dev = codes.device
    if qweight is None:
        qweight = torch.empty(m, d * bits // 32, dtype=torch.int32, device=dev)
    if qzeros is None:
        qzeros = torch.empty(m, (G * bits + 7) // 8, dtype=torch.uint8, device=dev)
    _check("gptq_pack_bits",
           load_library().gptq_pack_bits(_ptr(codes), _ptr(zeros), m, d, G, int(bits),
                                         _ptr(qweight), _ptr(qzeros), _stream(codes)))
    return qweight, qzeros


def gptq_unpack_bits(qweight: torch.Tensor, qzeros: torch.Tensor, d_in: int, n_groups: int,
                     bits: int):
    _need(qweight, "qweight")
    _need(qzeros, "qzeros", torch.uint8)
    m = qweight.shape[0]
    dev = qweight.device
    codes = torch.empty(m, d_in, dtype=torch.uint8, device=dev)
    zeros = torch.empty(m, n_groups, dtype=torch.uint8, device=dev)
    _check("gptq_unpack_bits",
           load_library().gptq_unpack_bits(_ptr(qweight), _ptr(qzeros), m, d_in, n_groups,
                                           int(bits), _ptr(codes), _ptr(zeros), _stream(qweight)))
    return codes, zeros


def gptq_channel_abs_sum(X: torch.Tensor, abs_sum=None) -> torch.Tensor:
    """abs_sum (d fp64) += sum over tokens of |X| (X: n x d fp16)."""
    _need(X, "X", torch.float16)
    n, d = X.shape
    if abs_sum is None:
        abs_sum = torch.zeros(d, dtype=torch.float64, device=X.device)
    _need(abs_sum, "abs_sum", torch.float64)
    _check("gptq_channel_abs_sum",
           load_library().gptq_channel_abs_sum(_ptr(X), n, d, _ptr(abs_sum), _stream(X)))
    return abs_sum


def gptq_awq_search(W: torch.Tensor, S: torch.Tensor, n_tokens: int, abs_sum: torch.Tensor,
                    n_grid: int = 20, bits: int = 4, group_size: int = 128,
                    scaled_outputs: bool = True):
    """Activation-aware channel scaling chosen by output error.  Returns a
    LayerResult with losses (n_grid fp64), best (int), alpha, scales (d fp64)
    and, with scaled_outputs, W_scaled (m x d fp32) and S_scaled (d x d fp32)."""
    _need(W, "W")
    _need(S, "S", torch.float32)
    _need(abs_sum, "abs_sum", torch.float64)
    m, d = W.shape
    dev = W.device
    losses = torch.empty(n_grid, dtype=torch.float64, device=dev)
    best = torch.empty(1, dtype=torch.int32, device=dev)
    scales = torch.empty(d, dtype=torch.float64, device=dev)
    Ws = torch.empty(m, d, dtype=torch.float32, device=dev) if scaled_outputs else None
    Ss = torch.empty(d, d, dtype=torch.float32, device=dev) if scaled_outputs else None
    nb = int(load_library().gptq_awq_workspace_bytes(m, d))
    ws = torch.empty(nb, dtype=torch.uint8, device=dev)
    _check("gptq_awq_search",
           load_library().gptq_awq_search(_ptr(W), _wdtype(W), m, d, _ptr(S), int(n_tokens),
                                          _ptr(abs_sum), int(n_grid), int(bits), int(group_size),
                                          _ptr(losses), _ptr(best), _ptr(scales), _ptr(Ws),
                                          _ptr(Ss), _ptr(ws), nb, _stream(W)))
    return LayerResult(losses=losses, best=best, scales=scales, W_scaled=Ws, S_scaled=Ss,
                       n_grid=n_grid)


def gptq_w4a16_gemm(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                    qzeros: torch.Tensor, group_size: int = 128, perm=None, y=None):
    """y = x Q^T (batch x d_out fp32) from the packed INT4 layer; x: batch x
    d_in fp16 in original column order, batch 1..8."""
    _need(x, "x", torch.float16)
    _need(qweight, "qweight")
    _need(scales, "scales", torch.float16)
    _need(qzeros, "qzeros", torch.uint8)
    b, d = x.shape
    m = qweight.shape[0]
    y = torch.empty(b, m, dtype=torch.float32, device=x.device) if y is None else y
    _need(y, "y", torch.float32)
    if perm is not None:
        _need(perm, "perm", torch.int32)
    _check("gptq_w4a16_gemm",
           load_library().gptq_w4a16_gemm(_ptr(x), b, _ptr(qweight), _ptr(scales), _ptr(qzeros),
                                          _ptr(perm), m, d, int(group_size), _ptr(y), _stream(x)))
    return y


def gptq_w4a16_matmul_workspace_bytes(batch: int, d_in: int) -> int:
    return int(load_library().gptq_w4a16_matmul_workspace_bytes(int(batch), int(d_in)))


def gptq_w4a16_matmul(x: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                      qzeros: torch.Tensor, group_size: int = 128, perm=None, y=None, ws=None):
    """y = x Q^T (batch x d_out fp32) from the packed INT4 layer on the tensor
    cores, any batch; x: batch x d_in fp16 in original column order."""
    _need(x, "x", torch.float16)
    _need(qweight, "qweight")
    _need(scales, "scales", torch.float16)
    _need(qzeros, "qzeros", torch.uint8)
    b, d = x.shape
    m = qweight.shape[0]
    y = torch.empty(b, m, dtype=torch.float32, device=x.device) if y is None else y
    _need(y, "y", torch.float32)
    if perm is not None:
        _need(perm, "perm", torch.int32)
    nb = int(load_library().gptq_w4a16_matmul_workspace_bytes(b, d))
    ws = torch.empty(nb, dtype=torch.uint8, device=x.device) if ws is None else ws
    _check("gptq_w4a16_matmul",
           load_library().gptq_w4a16_matmul(_ptr(x), b, _ptr(qweight), _ptr(scales), _ptr(qzeros),
                                            _ptr(perm), m, d, int(group_size), _ptr(y), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(x)))
    return y


def gptq_unpack_int4(qweight: torch.Tensor, qzeros: torch.Tensor, d_in: int, n_groups: int):
    _need(qweight, "qweight")
    _need(qzeros, "qzeros", torch.uint8)
    m = qweight.shape[0]
    dev = qweight.device
    codes = torch.empty(m, d_in, dtype=torch.uint8, device=dev)
    zeros = torch.empty(m, n_groups, dtype=torch.uint8, device=dev)
    _check("gptq_unpack_int4",
           load_library().gptq_unpack_int4(_ptr(qweight), _ptr(qzeros), m, d_in, n_groups,
                                           _ptr(codes), _ptr(zeros), _stream(qweight)))
    return codes, zeros


def rtn_quantize(W: torch.Tensor, bits: int = 4, group_size: int = 128):
    _need(W, "W")
    m, d = W.shape
    dev = W.device
    G = 1 if group_size in (-1, d) else d // group_size
    codes = torch.empty(m, d, dtype=torch.uint8, device=dev)
    scales = torch.empty(m, G, dtype=torch.float16, device=dev)
    zeros = torch.empty(m, G, dtype=torch.uint8, device=dev)
    _check("rtn_quantize",
           load_library().rtn_quantize(_ptr(W), _wdtype(W), m, d, int(bits), int(group_size),
                                       _ptr(codes), _ptr(scales), _ptr(zeros), _stream(W)))
    return codes, scales, zeros


def gptq_debug_gemm_nt(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor, alpha: float = 1.0,
                       beta: float = 0.0, lower: bool = False):
    """C = beta C + alpha A B^T on the split-TF32 tensor-core GEMM (test hook)."""
    for t, nm in ((A, "A"), (B, "B"), (C, "C")):
        _need(t, nm, torch.float32)
    M, K = A.shape
    N = B.shape[0]
    _check("gptq_debug_gemm_nt",
           load_library().gptq_debug_gemm_nt(_ptr(A), A.stride(0), _ptr(B), B.stride(0), _ptr(C),
                                             C.stride(0), M, N, K, float(alpha), float(beta),
                                             int(bool(lower)), _stream(A)))
    return C


# --------------------------------------------------------------------------
# Whole layer (the four calls in order)
# --------------------------------------------------------------------------

class LayerResult:
    def __init__(self, **kw):
        self.__dict__.update(kw)


def quantize_layer_from_inputs(W: torch.Tensor, X_batches, bits: int = 4, group_size: int = 128,
                               damp_rel: float = 0.01, act_order: bool = False,
                               pack: bool = True) -> LayerResult:
    """GPTQ on one layer: accumulate S over the calibration batches, prepare U,
    sweep, and pack.  X_batches: a CUDA fp16 tensor (n x d) or an iterable of them."""
    m, d = W.shape
    S = torch.zeros(d, d, dtype=torch.float32, device=W.device)
    n = 0
    if isinstance(X_batches, torch.Tensor):
        X_batches = [X_batches]
    for X in X_batches:
        n += gptq_hessian_accumulate(S, X)
    perm, U, info = gptq_prepare_hinv(S, n, damp_rel, act_order)
    codes, scales, zeros, row_loss = gptq_quantize_layer(
        W, U, perm if act_order else None, bits, group_size)
    res = LayerResult(S=S, n=n, perm=perm, U=U, info=info, codes=codes, scales=scales,
                      zeros=zeros, row_loss=row_loss)
    if pack and bits == 4:
        res.qweight, res.qzeros = gptq_pack_int4(codes, zeros)
    return res


def quantize_moe_from_inputs(W: torch.Tensor, X: torch.Tensor, routes, bits: int = 4,
                             group_size: int = 128, damp_rel: float = 0.01,
                             act_order: bool = False, pack: bool = True) -> LayerResult:
    """GPTQ on every expert of a mixture-of-experts layer at once.
    W: E x m x d (the experts' weights); X: n x d fp16 calibration tokens;
    routes: E int32 CUDA tensors, the tokens routed to each expert.  The
    routed rows are gathered expert-major, the E Hessians accumulated in one
    launch, prepared in one factorization launch, and the layers swept and
    packed."""
    E, m, d = W.shape
    dev = W.device
    counts = [int(r.numel()) for r in routes]
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    idx = torch.cat([r.to(device=dev, dtype=torch.int32) for r in routes]).contiguous()
    Xr = gptq_gather_rows(X, idx)
    S = torch.zeros(E, d, d, dtype=torch.float32, device=dev)
    gptq_hessian_accumulate_grouped(S, Xr, offsets)
    perm, U, info = gptq_prepare_hinv_batched(S, counts, damp_rel, act_order)
    codes, scales, zeros, row_loss = gptq_quantize_layer_batched(
        W, U, perm if act_order else None, bits, group_size)
    res = LayerResult(S=S, counts=counts, perm=perm, U=U, info=info, codes=codes, scales=scales,
                      zeros=zeros, row_loss=row_loss)
    if pack and bits == 4:
        qw, qz = gptq_pack_int4(codes.view(E * m, d), zeros.view(E * m, -1))
        res.qweight, res.qzeros = qw.view(E, m, -1), qz.view(E, m, -1)
    return res


def gptq_debug_chol_task_order(d: int):
    """The factorization's tasks in claim order as an int32 array of shape
    (T*T, 3): (type, i, j), type 0 = diagonal tile, 1 = tile of L, 2 = tile
    of L^-1 (host only)."""
    import numpy as np
    T = d // 128
    out = np.zeros((max(T * T, 1), 3), dtype=np.int32)
    n = load_library().gptq_debug_chol_task_order(d, out.ctypes.data, out.size)
    if n < 0:
        raise GptqError("gptq_debug_chol_task_order", int(-n))
    return out[:n]


def gptq_debug_div_rn(x, s):
    """The quantizer's division-free quotient x / s (host only; float32 arrays)."""
    import numpy as np
    x = np.ascontiguousarray(x, dtype=np.float32)
    s = np.ascontiguousarray(s, dtype=np.float32)
    out = np.empty_like(x)
    _check("gptq_debug_div_rn",
           load_library().gptq_debug_div_rn(x.ctypes.data, s.ctypes.data, x.size, out.ctypes.data))
    return out


def gptq_debug_bounded_wait(flag: torch.Tensor | None, which: int, limit_ns: int) -> None:
    """Run a bounded wait that never succeeds (unless which == 0 and flag is
    non-zero) with the given limit; the outcome is read with
    gptq_device_status().  Asynchronous on the current stream."""
    if flag is not None:
        _need(flag, "flag", torch.int32)
    st = torch.cuda.current_stream() if flag is None else torch.cuda.current_stream(flag.device)
    _check("gptq_debug_bounded_wait",
           load_library().gptq_debug_bounded_wait(_ptr(flag), int(which), int(limit_ns),
                                                  ctypes.c_void_p(st.cuda_stream)))

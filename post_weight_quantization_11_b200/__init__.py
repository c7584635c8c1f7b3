"""B200-native (sm_100a) GPTQ layer-wise INT4 weight quantization.

The compute path is libgptq.so (C ABI in include/gptq.h, CUDA kernels in
csrc/); ``gptq`` is its thin Python binding and ``inputs`` holds the seeded
synthetic workloads.  Importing the package does not load the library; the
first call does, and raises if it is missing.
"""
from .gptq import (  # noqa: F401
    EXPORTED,
    GptqError,
    gptq_abi_version,
    gptq_hessian_accumulate,
    gptq_pack_int4,
    gptq_prepare_hinv,
    gptq_prepare_workspace_bytes,
    gptq_quantize_layer,
    gptq_quantize_workspace_bytes,
    gptq_status_string,
    gptq_unpack_int4,
    load_library,
    quantize_layer_from_inputs,
    rtn_quantize,
)

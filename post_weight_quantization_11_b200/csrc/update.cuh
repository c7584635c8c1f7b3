// Inter-block error feedback -- "INT4/INT8 量化推理" sec. 三 (W[:, j+1:] -=
// err * H_inv[j, j+1:]) applied a block at a time ("GPTQ / AWQ / SqueezeLLM"
// sec. 一, blocks):
//   W[:, j0+128:] -= E . U[j0:j0+128, j0+128:]
// First version: fp32 CUDA-core GEMM.
#pragma once

#include "common.cuh"
#include "simt_gemm.cuh"

namespace gptq {

struct UpdateWs {
    int unused;
};

inline size_t update_ws_bytes(int64_t, int64_t) { return 256; }
inline void update_ws_bind(int64_t, int64_t, char*, UpdateWs* w) { w->unused = 0; }
inline int update_prepare_u(const float*, int64_t, UpdateWs*, cudaStream_t) { return GPTQ_OK; }

inline int block_update(float* Wk, const float* E, const float* U, int64_t m, int64_t d,
                        int64_t j0, UpdateWs*, cudaStream_t st)
{
    const int64_t c0 = j0 + 128;
    GemmArgs g{};
    g.A = E; g.lda = 128;
    g.B = U + j0 * d + c0; g.ldb = d;
    g.C = Wk + c0; g.ldc = d;
    g.M = m; g.N = d - c0; g.K = 128;
    g.alpha = -1.f; g.beta = 1.f;
    return simt_gemm(g, st);
}

}  // namespace gptq

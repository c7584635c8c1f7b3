// Tiled fp32 CUDA-core GEMM used by the blocked Cholesky / triangular inverse:
//   C[i][j] = alpha * sum_k A[i][k] * opB[k][j] + beta * C[i][j]
// with opB[k][j] = B[k][j] (NN) or B[j][k] (NT).  Tile 64x64x16, 256 threads,
// 4x4 outputs per thread.  Masks: lower-only output tiles (tile row >= tile
// column) and a lower-triangular B (B[k][j] == 0 for k < j) whose zero chunks
// are skipped.  fp32 FMA throughout (the accuracy the Cholesky needs).
#pragma once

#include "common.cuh"

namespace gptq {

struct GemmArgs {
    const float* A; int64_t lda;
    const float* B; int64_t ldb;
    float* C; int64_t ldc;
    int64_t M, N, K;
    float alpha, beta;
    int b_trans;        // 1: opB[k][j] = B[j][k]
    int lower_tiles;    // 1: compute only tiles with tile_row >= tile_col
    int b_lower;        // 1: B (as opB) is lower triangular: opB[k][j] == 0 for k < j
};

int simt_gemm(const GemmArgs& g, cudaStream_t st);

}  // namespace gptq

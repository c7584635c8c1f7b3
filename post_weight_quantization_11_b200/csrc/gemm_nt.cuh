// Batched fp32 "NT" GEMM on tcgen05 tensor cores in split-TF32:
//   C_b = beta * C_b + alpha * A_b . B_b^T          (b = 0 .. batch-1)
// A_b: M x K and B_b: N x K are row-major sub-blocks (K contiguous) of two
// fp32 buffers; C_b: M x N row-major.  Each product is taken as
// A_hi B_hi + A_hi B_lo + A_lo B_hi with x = x_hi + x_lo (x_hi rounded to
// TF32, x_lo the fp32 remainder): the error-corrected TF32 scheme of Ootomo &
// Yokota (2022), fp32-level accuracy.  The split happens in shared memory, so
// the operands are plain fp32 in HBM.
//
// Sub-block b of an operand starts at (row0 + b*row_step, col0 + b*col_step)
// of its buffer.  `lower` computes only output tiles on or below the tile
// diagonal (M == N), for symmetric rank-k updates.  C may alias A when
// N <= 128 (each output tile then reads exactly its own rows of A, all of K,
// before writing them).
#pragma once

#include "common.cuh"

namespace gptq {

struct NtBuffer {
    const float* base;
    int64_t rows, cols;   // extent of the whole buffer
    int64_t ld;           // row stride in elements (multiple of 4)
};

struct NtGemm {
    NtBuffer A, B;
    float* C;
    int64_t ldc;
    int64_t a_row0, a_col0, a_row_step, a_col_step;
    int64_t b_row0, b_col0, b_row_step, b_col_step;
    int64_t c_row0, c_col0, c_row_step, c_col_step;
    int64_t M, N, K;      // K multiple of 32
    int batch;
    float alpha, beta;
    int lower;
};

int gemm_nt_tf32x3(const NtGemm& g, cudaStream_t st);

}  // namespace gptq

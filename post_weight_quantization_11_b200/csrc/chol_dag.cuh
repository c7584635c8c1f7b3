// Tiled Cholesky factorization + triangular inverse as one dependency-driven
// persistent kernel (chol_dag.cu).
#pragma once

#include "common.cuh"

namespace gptq {

// Bytes of the synchronization area chol_inv_dag needs for a batch of E
// matrices with T = d / 128 tiles per dimension (tile flags + the task
// ticket counter).
size_t chol_dag_sync_bytes(int64_t d, int64_t E = 1);

// A (d x d, row-major): on entry its lower 128x128 tiles hold the symmetric
// positive definite matrix to factor (the upper tiles are never read); on
// exit its strictly-lower tiles hold the TF32 heads of those of L
// (A = L L^T) and its upper tiles their remainders (mirrored tile), its
// diagonal tiles the remainders of Y's diagonal tiles.
// Xc (2 d x 128): on exit rows [128 j, 128 j + 128) hold the heads of
// X_jj = L_jj^-1 and rows [E d + 128 j, ..) their remainders.
// Y (d x d): on exit its upper tiles (block row j <= block column k) hold
// the heads of (L^-1)^T, its strictly-lower tiles their remainders.
// U (d x d): on exit U[i][j] = (L^-1)[d-1-i][d-1-j] (upper; zeros below).
// sync: chol_dag_sync_bytes(d) bytes of scratch (cleared here).
// info: a non-positive pivot stores its position (as the leaf reports it).
// Batches: E matrices stacked E high in A, Xc (each plane), Y, U (matrix e
// at rows [e d, e d + d)), one info word each (info[e]); one launch factors
// them all.
int chol_inv_dag(float* A, float* Xc, float* Y, float* U, void* sync, int64_t d, int64_t E,
                 int32_t* info, cudaStream_t st);

}  // namespace gptq

// Inter-block error feedback -- "INT4/INT8 量化推理" sec. 三 (W[:, j+1:] -=
// err * H_inv[j, j+1:]) applied a block at a time ("GPTQ / AWQ / SqueezeLLM"
// sec. 一, blocks):
//   W[:, j0+128:] -= E . U[j0:j0+128, j0+128:]
// on the tensor cores in split-TF32: with x = x_hi + x_lo (x_hi rounded to
// TF32, x_lo the exact fp32 remainder), E U ~ E_hi U_hi + E_hi U_lo + E_lo U_hi
// (the error-corrected TF32 product of Ootomo & Yokota, 2022), fp32 accuracy.
#pragma once

#include "common.cuh"

namespace gptq {

constexpr int UPD_OUTER = 4;                 // 128-column blocks per deferred outer block
constexpr int64_t UPD_LDE = 128 * UPD_OUTER;  // row stride of the E buffers (512)

struct UpdateWs {
    float* Uh;   // d x d, TF32-rounded U, TRANSPOSED (Uh[c][k] ~ U[k][c])
    float* Ul;   // d x d, U^T - Uh
    float* Eh;   // m x 512, TF32-rounded scaled errors of the current outer block
    float* El;   // m x 512, remainder
};

size_t update_ws_bytes(int64_t m, int64_t d);
void update_ws_bind(int64_t m, int64_t d, char* base, UpdateWs* w);
// Split U into its TF32 head and fp32 remainder, transposed (once per layer).
int update_prepare_u(const float* U, int64_t d, UpdateWs* w, cudaStream_t st);
// W[:, c_begin:c_end] -= E[:, e_col0 : e_col0+k_rows] . U[u_row0 : u_row0+k_rows, c_begin:c_end]
// with E = Eh + El, U = Uh + Ul (lo x lo dropped); k_rows a multiple of 32.
int block_update(float* Wk, const UpdateWs* w, int64_t m, int64_t d, int64_t e_col0,
                 int64_t k_rows, int64_t u_row0, int64_t c_begin, int64_t c_end, cudaStream_t st);

__device__ __forceinline__ float tf32_round(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

}  // namespace gptq

// Hessian accumulation S += X^T X (upper triangle) -- "GPTQ / AWQ /
// SqueezeLLM" sec. 一 (H from the calibration inputs).
//
// First version: CUDA-core fp32 FMA of fp16 inputs, 64x64 upper tiles,
// token range split across grid.y with fp32 atomic accumulation.
#include "common.cuh"

namespace gptq {

constexpr int HS_B = 64, HS_BK = 32;

__global__ void __launch_bounds__(256)
hessian_simt_kernel(float* __restrict__ S, const __half* __restrict__ X, int64_t n, int64_t d,
                    int64_t tokens_per_split)
{
    const int nb = (int)(d / HS_B);
    const int bi = blockIdx.x / nb, bj = blockIdx.x % nb;
    if (bi > bj) return;
    const int64_t t_begin = int64_t(blockIdx.y) * tokens_per_split;
    const int64_t t_end = min(n, t_begin + tokens_per_split);
    if (t_begin >= t_end) return;
    __shared__ __align__(16) float As[HS_BK][HS_B + 4];
    __shared__ __align__(16) float Bs[HS_BK][HS_B + 4];
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
    const int64_t i0 = int64_t(bi) * HS_B, j0 = int64_t(bj) * HS_B;
    float acc[4][4] = {};
    for (int64_t t0 = t_begin; t0 < t_end; t0 += HS_BK) {
        // 32 tokens x 64 features per operand: 256 threads x 8 halves
        int r = tid / 8, c8 = (tid % 8) * 8;
        int64_t t = t0 + r;
        __half2 va[4], vb[4];
        if (t < t_end) {
            uint4 ua = *reinterpret_cast<const uint4*>(X + t * d + i0 + c8);
            uint4 ub = *reinterpret_cast<const uint4*>(X + t * d + j0 + c8);
            memcpy(va, &ua, 16);
            memcpy(vb, &ub, 16);
        } else {
            for (int q = 0; q < 4; ++q) { va[q] = __float2half2_rn(0.f); vb[q] = va[q]; }
        }
        for (int q = 0; q < 4; ++q) {
            float2 fa = __half22float2(va[q]), fb = __half22float2(vb[q]);
            As[r][c8 + 2 * q] = fa.x; As[r][c8 + 2 * q + 1] = fa.y;
            Bs[r][c8 + 2 * q] = fb.x; Bs[r][c8 + 2 * q + 1] = fb.y;
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < HS_BK; ++k) {
            float4 a = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
            float4 b = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
            float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
        }
        __syncthreads();
    }
    for (int p = 0; p < 4; ++p) {
        int64_t gi = i0 + ty * 4 + p;
        for (int q = 0; q < 4; ++q) {
            int64_t gj = j0 + tx * 4 + q;
            if (gi <= gj) atomicAdd(S + gi * d + gj, acc[p][q]);
        }
    }
}

}  // namespace gptq

extern "C" int gptq_hessian_accumulate(float* S, const uint16_t* X, int64_t n_tokens, int64_t d,
                                       int64_t* n_seen, void* stream)
{
    using namespace gptq;
    if (!S || (!X && n_tokens > 0)) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || (X && !aligned16(X))) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0 || n_tokens < 0) return GPTQ_ERR_SHAPE;
    if (n_tokens == 0) return GPTQ_OK;
    cudaStream_t st = as_stream(stream);
    const int nb = (int)(d / HS_B);
    const int64_t tiles = int64_t(nb) * (nb + 1) / 2;
    int64_t splits = ceil_div(4 * 148, tiles);
    splits = std::max<int64_t>(1, std::min<int64_t>(splits, ceil_div(n_tokens, 1024)));
    int64_t per = ceil_div(ceil_div(n_tokens, splits), HS_BK) * HS_BK;
    splits = ceil_div(n_tokens, per);
    dim3 grid((unsigned)(nb * nb), (unsigned)splits);
    hessian_simt_kernel<<<grid, 256, 0, st>>>(S, reinterpret_cast<const __half*>(X), n_tokens, d, per);
    count_launches();
    int rc = launch_status();
    if (rc == GPTQ_OK && n_seen) *n_seen += n_tokens;
    return rc;
}

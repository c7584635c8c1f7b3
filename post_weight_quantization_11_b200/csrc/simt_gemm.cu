// Tiled fp32 CUDA-core GEMM (see simt_gemm.cuh).
#include "simt_gemm.cuh"

namespace gptq {

constexpr int SG_BM = 64, SG_BN = 64, SG_BK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(GemmArgs g)
{
    __shared__ __align__(16) float As[SG_BK][SG_BM + 4];
    __shared__ __align__(16) float Bs[SG_BK][SG_BN + 4];
    const int bm = blockIdx.y, bn = blockIdx.x;
    if (g.lower_tiles && bn > bm) return;
    const int64_t i0 = int64_t(bm) * SG_BM, j0 = int64_t(bn) * SG_BN;
    const int tid = threadIdx.x;
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;

    int64_t k_begin = 0;
    if (g.b_lower) k_begin = (j0 / SG_BK) * SG_BK;
    for (int64_t k0 = k_begin; k0 < g.K; k0 += SG_BK) {
        // A tile: 64 rows x 16 k -> As[k][i]
        {
            int r = tid / 4, c4 = (tid % 4) * 4;
            int64_t gi = i0 + r;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (gi < g.M) {
                const float* p = g.A + gi * g.lda + k0 + c4;
                if (k0 + c4 + 3 < g.K) v = *reinterpret_cast<const float4*>(p);
                else {
                    float t[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int q = 0; q < 4; ++q) if (k0 + c4 + q < g.K) t[q] = p[q];
                    v = make_float4(t[0], t[1], t[2], t[3]);
                }
            }
            As[c4 + 0][r] = v.x; As[c4 + 1][r] = v.y; As[c4 + 2][r] = v.z; As[c4 + 3][r] = v.w;
        }
        if (!g.b_trans) {
            // B[k][j]: 16 k-rows x 64 cols
            int kr = tid / 16, c4 = (tid % 16) * 4;
            int64_t gk = k0 + kr;
            float t[4] = {0.f, 0.f, 0.f, 0.f};
            if (gk < g.K) {
                const float* p = g.B + gk * g.ldb + j0 + c4;
                if (j0 + c4 + 3 < g.N) {
                    float4 v = *reinterpret_cast<const float4*>(p);
                    t[0] = v.x; t[1] = v.y; t[2] = v.z; t[3] = v.w;
                } else {
                    for (int q = 0; q < 4; ++q) if (j0 + c4 + q < g.N) t[q] = p[q];
                }
            }
            *reinterpret_cast<float4*>(&Bs[kr][c4]) = make_float4(t[0], t[1], t[2], t[3]);
        } else {
            // B[j][k]: 64 j-rows x 16 k
            int r = tid / 4, c4 = (tid % 4) * 4;
            int64_t gj = j0 + r;
            float t[4] = {0.f, 0.f, 0.f, 0.f};
            if (gj < g.N) {
                const float* p = g.B + gj * g.ldb + k0 + c4;
                if (k0 + c4 + 3 < g.K) {
                    float4 v = *reinterpret_cast<const float4*>(p);
                    t[0] = v.x; t[1] = v.y; t[2] = v.z; t[3] = v.w;
                } else {
                    for (int q = 0; q < 4; ++q) if (k0 + c4 + q < g.K) t[q] = p[q];
                }
            }
            Bs[c4 + 0][r] = t[0]; Bs[c4 + 1][r] = t[1]; Bs[c4 + 2][r] = t[2]; Bs[c4 + 3][r] = t[3];
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SG_BK; ++k) {
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
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        int64_t gi = i0 + ty * 4 + p;
        if (gi >= g.M) continue;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            int64_t gj = j0 + tx * 4 + q;
            if (gj >= g.N) continue;
            float* c = g.C + gi * g.ldc + gj;
            float v = g.alpha * acc[p][q];
            *c = (g.beta == 0.f) ? v : fmaf(g.beta, *c, v);
        }
    }
}

int simt_gemm(const GemmArgs& g, cudaStream_t st)
{
    if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
    dim3 grid((unsigned)ceil_div(g.N, SG_BN), (unsigned)ceil_div(g.M, SG_BM));
    simt_gemm_kernel<<<grid, 256, 0, st>>>(g);
    count_launches();
    return launch_status();
}

}  // namespace gptq

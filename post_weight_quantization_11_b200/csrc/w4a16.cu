// Weight-only INT4 product (W4A16) on the packed layer -- "INT4/INT8 量化推理"
// sec. 六 (weights in 4 bits, activations kept in fp16) on the storage of
// sec. 一 of the same page (fp16 scale and 4-bit zero point per group):
//
//   y[b][r] = sum_j x[b][j] Q[r][j],   Q[r][perm[k]] = s[r][k/g] (c[r][k] - z[r][k/g])
//
// for a small batch of activation rows (decode).  The weights stream from
// HBM once; every product is fp32 with exact dequantization:
//  * a code c in nibble i (0..3) of a 16-bit half of a packed word becomes
//    the fp32 value c 16^i with one AND/OR and one subtraction (the bits go
//    into the mantissa of 2^23), and the activation it meets is stored
//    pre-multiplied by 16^-i (a power of two: exact), so c x needs no
//    integer conversion;
//  * per 16-code chunk (inside one group, g >= 16) the lane forms
//    a = sum c x and adds s (a - z sum x) to its row's sum, the chunk's
//    sum x taken once per CTA.
// CTA: 8 warps x 4 rows, one K-slice of 2048 columns whose activations
// (permuted to sweep order, pre-scaled) sit in shared memory; lanes take
// 16-code chunks of the slice; the slices' partial sums meet in y by atomic
// adds (y is zeroed first).
#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

constexpr int W4_KS = 2048;                 // columns per K-slice (CTA)
constexpr int W4_WARPS = 8, W4_ROWS = 4;    // rows per warp
constexpr int W4_THREADS = W4_WARPS * 32;
constexpr int W4_CHUNK = 16;                // codes per lane step (two packed words)
constexpr unsigned W4_FULL = 0xffffffffu;

__device__ __forceinline__ float nib16(uint32_t v, int i)
{
    // c 16^i for the nibble i (0..3) of the low 16 bits of v, exactly
    return __int_as_float(0x4B000000u | (v & (0xFu << (4 * i)))) - 8388608.0f;
}

template <int B>
__global__ void __launch_bounds__(W4_THREADS)
w4a16_kernel(const __half* __restrict__ x, const uint32_t* __restrict__ qweight,
             const __half* __restrict__ scales, const uint8_t* __restrict__ qzeros,
             const int32_t* __restrict__ perm, int64_t m, int64_t d, int64_t g,
             float* __restrict__ y)
{
    __shared__ __align__(16) float xs[B][W4_KS];               // pre-scaled x, sweep order
    __shared__ float xsum[B][W4_KS / W4_CHUNK];                 // per-chunk sum of x
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t k0 = int64_t(blockIdx.y) * W4_KS;
    const int klen = (int)(d - k0 < W4_KS ? d - k0 : W4_KS);         // a multiple of 128
    const int nch = klen / W4_CHUNK;
    const int64_t row0 = int64_t(blockIdx.x) * (W4_WARPS * W4_ROWS) + warp * W4_ROWS;
    auto load = [&](int c, uint2 (&q)[W4_ROWS]) {
        const int64_t gc = k0 / W4_CHUNK + c;
#pragma unroll
        for (int r = 0; r < W4_ROWS; ++r) {
            const int64_t row = row0 + r;
            q[r] = row < m ? *reinterpret_cast<const uint2*>(qweight + row * (d / 8) + 2 * gc)
                           : make_uint2(0u, 0u);
        }
    };
    // the lane's first two chunks of weights are requested before the
    // activations are staged: their latency overlaps the staging below
    uint2 q0[W4_ROWS], q1[W4_ROWS];
    if (lane < nch) load(lane, q0);
    if (lane + 32 < nch) load(lane + 32, q1);
    for (int idx = tid; idx < B * klen; idx += W4_THREADS) {
        const int b = idx / klen, kk = idx - b * klen;
        const int64_t k = k0 + kk;
        const int64_t src = perm ? int64_t(perm[k]) : k;
        const bool in = src >= 0 && src < d;          // a bad index is not followed
        if (!in) atomicCAS(&g_device_status, 0, kErrIndex);
        xs[b][kk] = in ? ldexpf(__half2float(x[b * d + src]), -4 * (kk & 3)) : 0.f;
    }
    __syncthreads();
    for (int idx = tid; idx < B * nch; idx += W4_THREADS) {
        const int b = idx / nch, c = idx - b * nch;
        float sum = 0.f;
#pragma unroll
        for (int t = 0; t < W4_CHUNK; ++t) sum += ldexpf(xs[b][c * W4_CHUNK + t], 4 * (t & 3));
        xsum[b][c] = sum;
    }
    __syncthreads();

    const int64_t G = d / g, Gz = (G + 1) / 2;
    float acc[W4_ROWS][B];
#pragma unroll
    for (int r = 0; r < W4_ROWS; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) acc[r][b] = 0.f;

    // one chunk of 16 codes for the warp's rows, packed words already loaded
    auto chunk = [&](int c, const uint2 (&q)[W4_ROWS]) {
        const int64_t gc = k0 / W4_CHUNK + c;                   // chunk index in the row
        const int64_t gi = gc * W4_CHUNK / g;                   // its group
        float xv[B][W4_CHUNK];
#pragma unroll
        for (int b = 0; b < B; ++b)
#pragma unroll
            for (int t4 = 0; t4 < W4_CHUNK / 4; ++t4) {
                const float4 v = *reinterpret_cast<const float4*>(&xs[b][c * W4_CHUNK + 4 * t4]);
                xv[b][4 * t4] = v.x; xv[b][4 * t4 + 1] = v.y;
                xv[b][4 * t4 + 2] = v.z; xv[b][4 * t4 + 3] = v.w;
            }
#pragma unroll
        for (int r = 0; r < W4_ROWS; ++r) {
            const int64_t row = row0 + r;
            if (row >= m) continue;
            const float s = __half2float(scales[row * G + gi]);
            const uint32_t zb = qzeros[row * Gz + gi / 2];
            const float z = float((gi & 1) ? (zb >> 4) : (zb & 0xFu));
            float a[B];
#pragma unroll
            for (int b = 0; b < B; ++b) a[b] = 0.f;
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const uint32_t word = w ? q[r].y : q[r].x;
                const uint32_t hi = word >> 16;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float flo = nib16(word, i), fhi = nib16(hi, i);
#pragma unroll
                    for (int b = 0; b < B; ++b) {
                        a[b] = fmaf(flo, xv[b][8 * w + i], a[b]);
                        a[b] = fmaf(fhi, xv[b][8 * w + 4 + i], a[b]);
                    }
                }
            }
#pragma unroll
            for (int b = 0; b < B; ++b) acc[r][b] = fmaf(s, fmaf(-z, xsum[b][c], a[b]), acc[r][b]);
        }
    };
    // two chunks per step; the next step's two chunks are requested before
    // this step's are used, so each warp keeps up to 4 KB of loads in flight
    for (int c = lane; c < nch; c += 64) {
        uint2 n0[W4_ROWS], n1[W4_ROWS];
        const int cn = c + 64;
        if (cn < nch) load(cn, n0);
        if (cn + 32 < nch) load(cn + 32, n1);
        chunk(c, q0);
        if (c + 32 < nch) chunk(c + 32, q1);
#pragma unroll
        for (int r = 0; r < W4_ROWS; ++r) { q0[r] = n0[r]; q1[r] = n1[r]; }
    }
#pragma unroll
    for (int r = 0; r < W4_ROWS; ++r)
#pragma unroll
        for (int b = 0; b < B; ++b) {
            float v = acc[r][b];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(W4_FULL, v, o);
            acc[r][b] = v;
        }
    if (lane == 0) {
#pragma unroll
        for (int r = 0; r < W4_ROWS; ++r) {
            const int64_t row = row0 + r;
            if (row < m)
#pragma unroll
                for (int b = 0; b < B; ++b) atomicAdd(y + b * m + row, acc[r][b]);
        }
    }
}

}  // namespace gptq

extern "C" int gptq_w4a16_gemm(const uint16_t* x, int64_t batch, const uint32_t* qweight,
                               const uint16_t* scales, const uint8_t* qzeros,
                               const int32_t* perm, int64_t d_out, int64_t d_in, int group_size,
                               float* y, void* stream)
{
    using namespace gptq;
    if (!x || !qweight || !scales || !qzeros || !y) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(qweight) || !aligned16(scales) || !aligned16(qzeros) ||
        !aligned16(y) || (perm && !aligned16(perm)))
        return GPTQ_ERR_INVALID_ARG;
    if (batch < 1 || batch > 4) return GPTQ_ERR_UNSUPPORTED;
    if (d_in < 128 || d_in > kMaxDim || d_in % 128 != 0 || d_out < 1 || d_out > kMaxRows)
        return GPTQ_ERR_SHAPE;
    const int64_t g = (group_size == -1) ? d_in : group_size;
    if (g < 32 || g % 32 != 0 || d_in % g != 0) return GPTQ_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    KernelTimer kt(kKW4A16, st);
    if (cudaMemsetAsync(y, 0, sizeof(float) * size_t(batch) * size_t(d_out), st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const dim3 grid((unsigned)ceil_div(d_out, W4_WARPS * W4_ROWS), (unsigned)ceil_div(d_in, W4_KS));
    const __half* xh = reinterpret_cast<const __half*>(x);
    const __half* sh = reinterpret_cast<const __half*>(scales);
    switch (batch) {
        case 1: w4a16_kernel<1><<<grid, W4_THREADS, 0, st>>>(xh, qweight, sh, qzeros, perm, d_out, d_in, g, y); break;
        case 2: w4a16_kernel<2><<<grid, W4_THREADS, 0, st>>>(xh, qweight, sh, qzeros, perm, d_out, d_in, g, y); break;
        case 3: w4a16_kernel<3><<<grid, W4_THREADS, 0, st>>>(xh, qweight, sh, qzeros, perm, d_out, d_in, g, y); break;
        default: w4a16_kernel<4><<<grid, W4_THREADS, 0, st>>>(xh, qweight, sh, qzeros, perm, d_out, d_in, g, y); break;
    }
    count_launches();
    return launch_status();
}

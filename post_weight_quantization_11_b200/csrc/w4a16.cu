// Weight-only INT4 product (W4A16) on the packed layer -- "INT4/INT8 量化推理"
// sec. 六 (weights in 4 bits, activations kept in fp16) on the storage of
// sec. 一 of the same page (fp16 scale and 4-bit zero point per group):
//
//   y[b][r] = sum_j x[b][j] Q[r][j],   Q[r][perm[k]] = s[r][k/g] (c[r][k] - z[r][k/g])
//
// for a decode-sized batch (1..8 activation rows).  The weights stream from
// HBM once, and a decode product is that stream: every CTA asks for all of
// its packed bytes at once (one 1-D bulk copy per row onto one mbarrier), so
// each SM has tens of KB in flight from the start.
//  * CTA: one K-slice of 2048 columns and every gridDim.x-th tile of 32 rows
//    (persistent over row tiles: the slice's activations are gathered once,
//    the next tile's bytes are copied into the second of two buffers while
//    this one is multiplied); 8 warps = 2 row halves of 16 x 4 K-quarters;
//    the slices' partial sums meet in y by atomic adds (y is zeroed first).
//  * Products on the tensor cores, m16n8k16 mma.sync, fp16 x fp16 -> fp32
//    (exact products, fp32 sums): the 16 x 16 weight fragment of a block of
//    16 columns is two packed words per row; a word's nibble pair (j, j+4)
//    becomes the fp16 pair (1024 + c_j, 1024 + c_{j+4}) by one AND/OR, and
//    subtracting 1024 + z leaves the exact c - z.  Lane (g, t) takes pair
//    t of each word, so the fragment's columns 2t, 2t+1, 2t+8, 2t+9 are the
//    block's columns t, t+4, 8+t, 12+t: the activations are gathered into
//    that order once per CTA (through perm), batch columns past the batch
//    zero.
//  * Per group (a multiple of 32 columns) the fp32 partial of each row is
//    scaled by its fp16 scale in fp32; a warp's quarter is at most 512
//    columns, so no accumulator sums more than 512 products.
#include <atomic>

#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

constexpr int WD_KS = 2048;                   // columns per K-slice (CTA)
constexpr int WD_ROWS = 32;                   // rows per CTA
constexpr int WD_THREADS = 256;               // 8 warps: 2 row tiles x 4 K-quarters
constexpr int WD_WLD = WD_KS / 8 + 4;         // words per shared row (rows 4 banks apart)
constexpr int WD_NB = 8;                      // batch columns of the mma (n = 8)
constexpr size_t WD_WBUF = size_t(WD_ROWS) * WD_WLD * 4;   // one row tile's packed slice
constexpr size_t WD_SMEM = 2 * WD_WBUF + size_t(WD_KS) * WD_NB * 2 + 4 * WD_ROWS * WD_NB * 4 + 16;

// One 1-D bulk copy global -> shared completing on an mbarrier (no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// D (16x8 fp32) += A (16x16 fp16, row) B (16x8 fp16, col)
__device__ __forceinline__ void mma_f16_m16n8k16(float (&c)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Nibbles (j, j+4) of w as the fp16 pair (c_j - z, c_{j+4} - z), exact:
// zz = the fp16 pair (1024 + z, 1024 + z) as bits.
__device__ __forceinline__ uint32_t nib_pair(uint32_t w, int j, uint32_t zz)
{
    const uint32_t v = ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
    const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&v),
                              *reinterpret_cast<const __half2*>(&zz));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__global__ void __launch_bounds__(WD_THREADS)
w4a16_dec_kernel(const __half* __restrict__ x, int batch, const uint32_t* __restrict__ qweight,
                 const __half* __restrict__ scales, const uint8_t* __restrict__ qzeros,
                 const int32_t* __restrict__ perm, int64_t m, int64_t d, int64_t g,
                 float* __restrict__ y)
{
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t* Wb0 = reinterpret_cast<uint32_t*>(smem);      // buffer i at Wb0 + i * WD_WBUF / 4
    __half* Xs = reinterpret_cast<__half*>(smem + 2 * WD_WBUF);
    float* red = reinterpret_cast<float*>(smem + 2 * WD_WBUF + size_t(WD_KS) * WD_NB * 2);
    uint64_t* bar = reinterpret_cast<uint64_t*>(red + 4 * WD_ROWS * WD_NB);   // two
    __shared__ int abort_flag;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t k0 = int64_t(blockIdx.y) * WD_KS;
    const int klen = (int)min(int64_t(WD_KS), d - k0);     // a multiple of 128
    const int64_t wpr = d / 8;                             // packed words per row
    const int64_t ntiles = (m + WD_ROWS - 1) / WD_ROWS;
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // thread 0: the copies of row tile `tile` into buffer `buf`
    auto issue = [&](int64_t tile, int buf) {
        const int64_t r0 = tile * WD_ROWS;
        const int rows = (int)min(int64_t(WD_ROWS), m - r0);
        uint32_t* W = Wb0 + buf * (WD_WBUF / 4);
        mbar_arrive_expect_tx(&bar[buf], uint32_t(rows) * uint32_t(klen / 2));
        for (int r = 0; r < rows; ++r)
            bulk_load(W + r * WD_WLD, qweight + (r0 + r) * wpr + k0 / 8, uint32_t(klen / 2),
                      &bar[buf]);
    };
    if (tid == 0 && int64_t(blockIdx.x) < ntiles) issue(blockIdx.x, 0);
    // activations of the slice in fragment order: element (q, n, L) at
    // (q * 8 + n) * 16 + L is column 16 q + p(L) of batch row n, with
    // p(2t + e) = t + 4 e and p(8 + 2t + e) = 8 + t + 4 e (columns < 2^15:
    // 32-bit indices)
    {
        constexpr int PER = WD_KS / WD_THREADS;            // slots per thread
        int src[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + u * WD_THREADS;            // slot (q, L) of the slice
            const int L = i & 15;
            const int p = 8 * (L >> 3) + ((L & 7) >> 1) + 4 * (L & 1);
            const int col = int(k0) + (i & ~15) + p;
            src[u] = (i < klen) ? (perm ? perm[col] : col) : 0;
        }
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int i = tid + u * WD_THREADS;
            if (i >= klen) continue;
            const bool ok = src[u] >= 0 && src[u] < int(d);
            if (!ok) atomicCAS(&g_device_status, 0, kErrIndex);   // a bad index is not followed
            __half* dst = Xs + (i >> 4) * (WD_NB * 16) + (i & 15);
#pragma unroll
            for (int n = 0; n < WD_NB; ++n)
                dst[n * 16] = (n < batch && ok) ? x[n * int(d) + src[u]] : __float2half(0.f);
        }
    }
    __syncthreads();

    const int mt = warp & 1, kq = warp >> 1;               // row half, K quarter
    const int gq = lane >> 2, tq = lane & 3;
    const int qlen = klen / 4;                             // a multiple of 32
    const int kb0 = kq * qlen;
    const int ra = 16 * mt + gq, rb = ra + 8;              // rows inside the tile
    const int gi = int(g);
    const int64_t G = d / g, Gb = (G + 1) / 2;
    int it = 0;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        if (tid == 0 && tile + gridDim.x < ntiles) issue(tile + gridDim.x, buf ^ 1);
        mbar_wait(&bar[buf], uint32_t((it >> 1) & 1), kErrWaitFull, &abort_flag);
        const uint32_t* Wsm = Wb0 + buf * (WD_WBUF / 4);
        const int64_t r0 = tile * WD_ROWS;
        const int rows = (int)min(int64_t(WD_ROWS), m - r0);
        const bool va = ra < rows, vb = rb < rows;        // rows past m: stale words, no output
        float acc[4] = {0.f, 0.f, 0.f, 0.f};               // (ra, 2tq), (ra, 2tq+1), (rb, 2tq), (rb, 2tq+1)
        // the quarter in segments of one group each (a group may start before
        // the quarter or end after it): the group's scales and zero points,
        // then its blocks of 16 columns with no per-block bookkeeping
        const int kend = kb0 + qlen;
        int col = int(k0) + kb0;                           // absolute column of kb
        int grp = col / gi;
        for (int kb = kb0; kb < kend; ++grp) {
            const int seg_end = min(kend, kb + (grp + 1) * gi - col);
            uint32_t zra = 0u, zrb = 0u;
            float sa = 0.f, sb = 0.f;
            if (va) {
                zra = (qzeros[(r0 + ra) * Gb + grp / 2] >> (4 * (grp & 1))) & 0xFu;
                sa = __half2float(scales[(r0 + ra) * G + grp]);
            }
            if (vb) {
                zrb = (qzeros[(r0 + rb) * Gb + grp / 2] >> (4 * (grp & 1))) & 0xFu;
                sb = __half2float(scales[(r0 + rb) * G + grp]);
            }
            const uint32_t ha = __half_as_ushort(__float2half(1024.f + float(zra)));
            const uint32_t hb = __half_as_ushort(__float2half(1024.f + float(zrb)));
            const uint32_t za = ha | (ha << 16), zb = hb | (hb << 16);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            const uint32_t* pa = Wsm + ra * WD_WLD + kb / 8;
            const uint32_t* pb = Wsm + rb * WD_WLD + kb / 8;
            const __half* xb = Xs + ((kb >> 4) * WD_NB + gq) * 16;
#pragma unroll 4
            for (int k = kb; k < seg_end; k += 16) {
                const uint2 wa = *reinterpret_cast<const uint2*>(pa);
                const uint2 wb = *reinterpret_cast<const uint2*>(pb);
                uint32_t a[4];
                a[0] = nib_pair(wa.x, tq, za);             // row ra, columns t, t+4
                a[1] = nib_pair(wb.x, tq, zb);             // row rb
                a[2] = nib_pair(wa.y, tq, za);             // row ra, columns 8+t, 12+t
                a[3] = nib_pair(wb.y, tq, zb);
                const uint32_t b0 = *reinterpret_cast<const uint32_t*>(xb + 2 * tq);
                const uint32_t b1 = *reinterpret_cast<const uint32_t*>(xb + 8 + 2 * tq);
                mma_f16_m16n8k16(part, a, b0, b1);
                pa += 2;
                pb += 2;
                xb += WD_NB * 16;
            }
            acc[0] = fmaf(sa, part[0], acc[0]); acc[1] = fmaf(sa, part[1], acc[1]);
            acc[2] = fmaf(sb, part[2], acc[2]); acc[3] = fmaf(sb, part[3], acc[3]);
            col += seg_end - kb;
            kb = seg_end;
        }
        float* rq = red + kq * WD_ROWS * WD_NB;
        rq[ra * WD_NB + 2 * tq] = acc[0];
        rq[ra * WD_NB + 2 * tq + 1] = acc[1];
        rq[rb * WD_NB + 2 * tq] = acc[2];
        rq[rb * WD_NB + 2 * tq + 1] = acc[3];
        __syncthreads();
        const int rr = tid >> 3, cc = tid & 7;             // one output per thread
        if (rr < rows && cc < batch) {
            float v = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) v += red[k * WD_ROWS * WD_NB + rr * WD_NB + cc];
            atomicAdd(&y[int64_t(cc) * m + r0 + rr], v);
        }
        __syncthreads();                                   // red and this buffer free again
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
    if (batch < 1 || batch > WD_NB) return GPTQ_ERR_UNSUPPORTED;
    if (d_in < 128 || d_in > kMaxDim || d_in % 128 != 0 || d_out < 1 || d_out > kMaxRows)
        return GPTQ_ERR_SHAPE;
    const int64_t g = (group_size == -1) ? d_in : group_size;
    if (g < 32 || g % 32 != 0 || d_in % g != 0) return GPTQ_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    KernelTimer kt(kKW4A16, st);
    if (cudaMemsetAsync(y, 0, sizeof(float) * size_t(batch) * size_t(d_out), st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    {   // the shared-memory opt-in, once per device
        static std::atomic<bool> done[64];
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
        if (dev < 0 || dev >= 64 || !done[dev].load()) {
            if (cudaFuncSetAttribute(w4a16_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)WD_SMEM) != cudaSuccess)
                return GPTQ_ERR_CUDA;
            if (dev >= 0 && dev < 64) done[dev].store(true);
        }
    }
    // persistent over row tiles: two CTAs per SM over the slices
    const int64_t slices = ceil_div(d_in, WD_KS), tiles = ceil_div(d_out, WD_ROWS);
    const int64_t per_slice = std::max<int64_t>(1, ceil_div(2 * int64_t(device_sm_count()), slices));
    const dim3 grid((unsigned)std::min(tiles, per_slice), (unsigned)slices);
    w4a16_dec_kernel<<<grid, WD_THREADS, WD_SMEM, st>>>(
        reinterpret_cast<const __half*>(x), (int)batch, qweight,
        reinterpret_cast<const __half*>(scales), qzeros, perm, d_out, d_in, g, y);
    count_launches();
    return launch_status();
}

// Batched split-TF32 NT GEMM on tcgen05 (see gemm_nt.cuh for the contract).
//
// Persistent CTAs over (batch, 128x128 output tile) items; K in stages of 32.
//   warp 0     TMA: A and B fp32 tiles (K-major, 128-byte swizzle), 3 stages
//   warps 2-5  split each landed tile in shared memory: hi = TF32(x) in place,
//              lo = x - hi beside it; then make the writes visible to the
//              tensor core (proxy fence) and arrive on the stage's barrier
//   warp 1     per 8-wide k-step: A_hi B_hi + A_hi B_lo + A_lo B_hi into one of
//              two TMEM accumulators (2 x 128 columns)
//   warps 6-9  C = beta C + alpha D from the other accumulator
// Every mbarrier wait is bounded (tc_common.cuh).
#include "common.cuh"
#include "gemm_nt.cuh"
#include "tc_common.cuh"
#include "update.cuh"

namespace gptq {

constexpr int GN_T = 128, GN_KC = 32, GN_STAGES = 3;
constexpr int GN_TILE_BYTES = GN_T * GN_KC * 4;             // 16 KB
constexpr int GN_STAGE_BYTES = 4 * GN_TILE_BYTES;           // A hi, A lo, B hi, B lo
constexpr int GN_THREADS = 320;
constexpr int GN_SMEM = GN_STAGES * GN_STAGE_BYTES + 1024 + 512;
constexpr uint32_t GN_IDESC = make_idesc(2 /*tf32*/, GN_T, GN_T, 0, 0);

struct GnParams {
    float* C;
    int64_t ldc;
    int64_t a_row0, a_col0, a_row_step, a_col_step;
    int64_t b_row0, b_col0, b_row_step, b_col_step;
    int64_t c_row0, c_col0, c_row_step, c_col_step;
    int64_t M, N;
    int kchunks;
    int n_tm, n_tn, tiles, items;
    float alpha, beta;
    int lower;
};

__device__ __forceinline__ void gn_tile(const GnParams& p, int q, int& b, int& tm, int& tn)
{
    b = q / p.tiles;
    const int t = q - b * p.tiles;
    if (p.lower) {
        int r = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
        while ((r + 1) * (r + 2) / 2 <= t) ++r;
        while (r > 0 && r * (r + 1) / 2 > t) --r;
        tm = r;
        tn = t - r * (r + 1) / 2;
    } else {
        tm = t % p.n_tm;
        tn = t / p.n_tm;
    }
}

__global__ void __launch_bounds__(GN_THREADS, 1)
gemm_nt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const GnParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + GN_STAGES * GN_STAGE_BYTES);
    uint64_t* conv_bar = full_bar + GN_STAGES;
    uint64_t* empty_bar = conv_bar + GN_STAGES;
    uint64_t* accf_bar = empty_bar + GN_STAGES;
    uint64_t* acce_bar = accf_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < GN_STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&conv_bar[s], 128);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf_bar[a], 1); mbar_init(&acce_bar[a], 128); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = gridDim.x;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                int b, tm, tn;
                gn_tile(p, q, b, tm, tn);
                const int ya = (int)(p.a_row0 + b * p.a_row_step + int64_t(tm) * GN_T);
                const int xa = (int)(p.a_col0 + b * p.a_col_step);
                const int yb = (int)(p.b_row0 + b * p.b_row_step + int64_t(tn) * GN_T);
                const int xb = (int)(p.b_col0 + b * p.b_col_step);
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kErrWaitEmpty, abort)) { ok = false; break; }
                    uint8_t* st = smem + stage * GN_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], 2 * GN_TILE_BYTES);
                    tma_load_2d(st, &tmA, &full_bar[stage], xa + kc * GN_KC, ya);
                    tma_load_2d(st + 2 * GN_TILE_BYTES, &tmB, &full_bar[stage], xb + kc * GN_KC, yb);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == GN_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            for (int s = 0; s < GN_STAGES; ++s)
                if (armed & (1u << s)) mbar_drain(&full_bar[s], (armed_par >> s) & 1u);
        }
    } else if (warp >= 2 && warp <= 5) {
        // split converters
        const int ct = threadIdx.x - 64;
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int q = blockIdx.x; q < p.items && ok; q += P) {
            for (int kc = 0; kc < p.kchunks; ++kc) {
                if (!mbar_wait(&full_bar[stage], phase, kErrWaitFull, abort)) { ok = false; break; }
                uint8_t* st = smem + stage * GN_STAGE_BYTES;
#pragma unroll
                for (int op = 0; op < 2; ++op) {
                    float4* hi = reinterpret_cast<float4*>(st + op * 2 * GN_TILE_BYTES);
                    float4* lo = reinterpret_cast<float4*>(st + op * 2 * GN_TILE_BYTES + GN_TILE_BYTES);
#pragma unroll
                    for (int u = 0; u < GN_TILE_BYTES / 16 / 128; ++u) {
                        const int i = ct + 128 * u;
                        const float4 x = hi[i];
                        float4 h, l;
                        h.x = tf32_round(x.x); l.x = x.x - h.x;
                        h.y = tf32_round(x.y); l.y = x.y - h.y;
                        h.z = tf32_round(x.z); l.z = x.z - h.z;
                        h.w = tf32_round(x.w); l.w = x.w - h.w;
                        hi[i] = h;
                        lo[i] = l;
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&conv_bar[stage]);
                if (++stage == GN_STAGES) { stage = 0; phase ^= 1; }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, it = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P, ++it) {
                const int a = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait(&acce_bar[a], aph ^ 1, kErrWaitAccEmpty, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem + uint32_t(a * GN_T);
                uint32_t acc = 0;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&conv_bar[stage], phase, kErrWaitFull, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sAh = smem_u32(smem + stage * GN_STAGE_BYTES);
                    const uint32_t sAl = sAh + GN_TILE_BYTES;
                    const uint32_t sBh = sAh + 2 * GN_TILE_BYTES;
                    const uint32_t sBl = sAh + 3 * GN_TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < GN_KC / 8; ++kk) {
                        const uint64_t aH = smem_desc_sw128(sAh + kk * 32, 16, 1024);
                        const uint64_t aL = smem_desc_sw128(sAl + kk * 32, 16, 1024);
                        const uint64_t bH = smem_desc_sw128(sBh + kk * 32, 16, 1024);
                        const uint64_t bL = smem_desc_sw128(sBl + kk * 32, 16, 1024);
                        mma_tf32(d_tmem, aH, bH, GN_IDESC, acc);
                        mma_tf32(d_tmem, aH, bL, GN_IDESC, 1u);
                        mma_tf32(d_tmem, aL, bH, GN_IDESC, 1u);
                        acc = 1;
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == GN_STAGES) { stage = 0; phase ^= 1; }
                }
                mma_commit(&accf_bar[a]);
            }
        }
    } else {
        // epilogue warps 6-9
        const int qr = warp & 3;
        int it = 0;
        for (int q = blockIdx.x; q < p.items; q += P, ++it) {
            int b, tm, tn;
            gn_tile(p, q, b, tm, tn);
            const int a = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            if (!mbar_wait(&accf_bar[a], aph, kErrWaitAccFull, abort)) break;
            tc_fence_after();
            const int64_t r = int64_t(tm) * GN_T + qr * 32 + lane;      // row within the block
            float* Crow = p.C + (p.c_row0 + b * p.c_row_step + r) * p.ldc +
                          (p.c_col0 + b * p.c_col_step);
#pragma unroll 1
            for (int c = 0; c < GN_T / 32; ++c) {
                float v[32];
                tmem_ld32(tmem + uint32_t(a * GN_T + c * 32) + (uint32_t(qr * 32) << 16), v);
                const int64_t col0 = int64_t(tn) * GN_T + c * 32;
                if (r >= p.M || col0 >= p.N) continue;
                if (col0 + 32 <= p.N) {
                    float4* cp = reinterpret_cast<float4*>(Crow + col0);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float4 o = make_float4(p.alpha * v[4 * u], p.alpha * v[4 * u + 1],
                                               p.alpha * v[4 * u + 2], p.alpha * v[4 * u + 3]);
                        if (p.beta != 0.f) {
                            const float4 cv = cp[u];
                            o.x = fmaf(p.beta, cv.x, o.x);
                            o.y = fmaf(p.beta, cv.y, o.y);
                            o.z = fmaf(p.beta, cv.z, o.z);
                            o.w = fmaf(p.beta, cv.w, o.w);
                        }
                        cp[u] = o;
                    }
                } else {
                    for (int u = 0; u < 32 && col0 + u < p.N; ++u) {
                        float o = p.alpha * v[u];
                        if (p.beta != 0.f) o = fmaf(p.beta, Crow[col0 + u], o);
                        Crow[col0 + u] = o;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acce_bar[a]);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

int gemm_nt_tf32x3(const NtGemm& g, cudaStream_t st)
{
    if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return GPTQ_OK;
    if (g.K <= 0 || g.K % GN_KC != 0) return GPTQ_ERR_SHAPE;
    if (g.lower && g.M != g.N) return GPTQ_ERR_SHAPE;
    GnParams p{};
    p.C = g.C;
    p.ldc = g.ldc;
    p.a_row0 = g.a_row0; p.a_col0 = g.a_col0; p.a_row_step = g.a_row_step; p.a_col_step = g.a_col_step;
    p.b_row0 = g.b_row0; p.b_col0 = g.b_col0; p.b_row_step = g.b_row_step; p.b_col_step = g.b_col_step;
    p.c_row0 = g.c_row0; p.c_col0 = g.c_col0; p.c_row_step = g.c_row_step; p.c_col_step = g.c_col_step;
    p.M = g.M;
    p.N = g.N;
    p.kchunks = (int)(g.K / GN_KC);
    p.n_tm = (int)ceil_div(g.M, GN_T);
    p.n_tn = (int)ceil_div(g.N, GN_T);
    p.tiles = g.lower ? p.n_tm * (p.n_tm + 1) / 2 : p.n_tm * p.n_tn;
    p.items = p.tiles * g.batch;
    p.alpha = g.alpha;
    p.beta = g.beta;
    p.lower = g.lower;
    CUtensorMap tA, tB;
    if (encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.A.base, (uint64_t)g.A.cols,
                       (uint64_t)g.A.rows, (uint64_t)g.A.ld * 4, GN_KC, GN_T,
                       CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK ||
        encode_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.B.base, (uint64_t)g.B.cols,
                       (uint64_t)g.B.rows, (uint64_t)g.B.ld * 4, GN_KC, GN_T,
                       CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
        return GPTQ_ERR_CUDA;
    if (cudaFuncSetAttribute(gemm_nt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             GN_SMEM) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const int grid = std::min(p.items, device_sm_count());
    gemm_nt_kernel<<<grid, GN_THREADS, GN_SMEM, st>>>(tA, tB, p);
    count_launches();
    return launch_status();
}

}  // namespace gptq

// Test hook: C (M x N) = beta C + alpha A B^T for dense row-major fp32
// A (M x K, lda), B (N x K, ldb), C (ldc); K a multiple of 32.
extern "C" int gptq_debug_gemm_nt(const float* A, int64_t lda, const float* B, int64_t ldb,
                                  float* C, int64_t ldc, int64_t M, int64_t N, int64_t K,
                                  float alpha, float beta, int lower, void* stream)
{
    using namespace gptq;
    if (!A || !B || !C) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(A) || !aligned16(B) || !aligned16(C) || lda % 4 || ldb % 4 || ldc % 4)
        return GPTQ_ERR_INVALID_ARG;
    if (M < 0 || N < 0 || K < 32 || K % 32 || lda < K || ldb < K || ldc < N) return GPTQ_ERR_SHAPE;
    NtGemm g{};
    g.A = NtBuffer{A, M, K, lda};
    g.B = NtBuffer{B, N, K, ldb};
    g.C = C;
    g.ldc = ldc;
    g.M = M;
    g.N = N;
    g.K = K;
    g.batch = 1;
    g.alpha = alpha;
    g.beta = beta;
    g.lower = lower;
    return gemm_nt_tf32x3(g, as_stream(stream));
}

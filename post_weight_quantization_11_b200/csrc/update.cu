// Error-feedback update W[:, c0:c1] -= E[:, e0:e0+K] . U[u0:u0+K, c0:c1] on tcgen05
// tensor cores in split-TF32 (three kind::tf32 products, fp32 accumulation in
// TMEM); K = 128 (the rest of an outer block) or 512 (a whole outer block).
//
//  * Items are 128-row x N-column output tiles of the trailing columns
//    (N = 128), handed round-robin to one persistent CTA per SM.
//  * K in chunks of 32: E_hi, E_lo tiles (rows x 32) and U_hi^T, U_lo^T
//    tiles (N columns x 32), all K-major with 128-byte swizzle, one TMA box
//    each.  U is stored transposed because an MN-major tf32 operand would
//    need the 32-byte-atom swizzle; K-major is the plain layout for both.
//    2 stages of 96 KB (N = 256) or 3 of 64 KB (N = 128).
//  * warp 0: TMA; warp 1: per 8-wide k-step E_hi U_hi + E_hi U_lo + E_lo U_hi
//    into one of two TMEM accumulators (2 x N columns); warps 2-5: read the
//    accumulator (tcgen05.ld) and write W - D back, overlapping the next
//    tile's MMAs; each thread's row of W is read two 32-column chunks ahead,
//    the first two before the accumulator is ready.
//  * Every mbarrier wait is bounded (see tc_common.cuh).
#include "common.cuh"
#include "tc_common.cuh"
#include "update.cuh"

namespace gptq {

// Tile width N (128 is the one launched: more CTAs and a shorter MMA chain
// for the near updates, and three pipeline stages instead of two).
constexpr int UB_M = 128, UB_KC = 32;
constexpr int UB_A_BYTES = UB_M * UB_KC * 4;                  // 16 KB per E tile
constexpr int UB_THREADS = 192;
template <int N> struct UbCfg {
    static constexpr int B_BYTES = UB_KC * N * 4;               // U tile: 32 KB (N=256)
    static constexpr int STAGE_BYTES = 2 * UB_A_BYTES + 2 * B_BYTES;   // 96 KB (N=256)
    static constexpr int STAGES = N == 128 ? 3 : 2;
    static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 + 256;
    static constexpr uint32_t IDESC = make_idesc(2 /*tf32*/, UB_M, N, 0 /*A K-major*/, 0 /*B K-major*/);
    static constexpr uint32_t TMEM_COLS = 2 * N;
};

struct UpdParams {
    float* W;
    int64_t m, d, e0, u0, c0, c1;
    int kchunks;
    int n_rt, n_ct, items;
};

template <int N>
__global__ void __launch_bounds__(UB_THREADS, 1)
block_update_tc_kernel(const __grid_constant__ CUtensorMap tmEh,
                       const __grid_constant__ CUtensorMap tmEl,
                       const __grid_constant__ CUtensorMap tmUh,
                       const __grid_constant__ CUtensorMap tmUl, const UpdParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + UbCfg<N>::STAGES * UbCfg<N>::STAGE_BYTES);
    uint64_t* empty_bar = full_bar + UbCfg<N>::STAGES;
    uint64_t* accf_bar = empty_bar + UbCfg<N>::STAGES;
    uint64_t* acce_bar = accf_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < UbCfg<N>::STAGES; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf_bar[a], 1); mbar_init(&acce_bar[a], 128); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, UbCfg<N>::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = gridDim.x;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmEh); prefetch_tmap(&tmEl); prefetch_tmap(&tmUh); prefetch_tmap(&tmUl);
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                const int rt = q % p.n_rt, ct = q / p.n_rt;
                const int y_e = rt * UB_M;
                const int x_u = (int)(p.c0 + int64_t(ct) * N);
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kErrWaitEmpty, abort)) { ok = false; break; }
                    uint8_t* sEh = smem + stage * UbCfg<N>::STAGE_BYTES;
                    uint8_t* sEl = sEh + UB_A_BYTES;
                    uint8_t* sUh = sEl + UB_A_BYTES;
                    uint8_t* sUl = sUh + UbCfg<N>::B_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], UbCfg<N>::STAGE_BYTES);
                    tma_load_2d(sEh, &tmEh, &full_bar[stage], (int)(p.e0 + kc * UB_KC), y_e);
                    tma_load_2d(sEl, &tmEl, &full_bar[stage], (int)(p.e0 + kc * UB_KC), y_e);
                    const int k_u = (int)(p.u0 + kc * UB_KC);
                    tma_load_2d(sUh, &tmUh, &full_bar[stage], k_u, x_u);
                    tma_load_2d(sUl, &tmUl, &full_bar[stage], k_u, x_u);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == UbCfg<N>::STAGES) { stage = 0; phase ^= 1; }
                }
            }
            for (int s = 0; s < UbCfg<N>::STAGES; ++s)
                if (armed & (1u << s)) mbar_drain(&full_bar[s], (armed_par >> s) & 1u);
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
                const uint32_t d_tmem = tmem + uint32_t(a * N);
                uint32_t acc = 0;
                for (int kc = 0; kc < p.kchunks; ++kc) {
                    if (!mbar_wait(&full_bar[stage], phase, kErrWaitFull, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sEh = smem_u32(smem + stage * UbCfg<N>::STAGE_BYTES);
                    const uint32_t sEl = sEh + UB_A_BYTES;
                    const uint32_t sUh = sEl + UB_A_BYTES;
                    const uint32_t sUl = sUh + UbCfg<N>::B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < UB_KC / 8; ++kk) {
                        // A: K-major rows of 128 B; an 8-wide k-step is 32 B along the row
                        const uint64_t aH = smem_desc_sw128(sEh + kk * 32, 16, 1024);
                        const uint64_t aL = smem_desc_sw128(sEl + kk * 32, 16, 1024);
                        const uint64_t bH = smem_desc_sw128(sUh + kk * 32, 16, 1024);
                        const uint64_t bL = smem_desc_sw128(sUl + kk * 32, 16, 1024);
                        mma_tf32(d_tmem, aH, bH, UbCfg<N>::IDESC, acc);
                        mma_tf32(d_tmem, aH, bL, UbCfg<N>::IDESC, 1u);
                        mma_tf32(d_tmem, aL, bH, UbCfg<N>::IDESC, 1u);
                        acc = 1;
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == UbCfg<N>::STAGES) { stage = 0; phase ^= 1; }
                }
                mma_commit(&accf_bar[a]);
            }
        }
    } else {
        const int qr = warp & 3;
        int it = 0;
        for (int q = blockIdx.x; q < p.items; q += P, ++it) {
            const int rt = q % p.n_rt, ct = q / p.n_rt;
            const int a = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const int64_t i = int64_t(rt) * UB_M + qr * 32 + lane;
            const bool row_ok = i < p.m;
            float* Wrow = p.W + i * p.d;
            const int64_t col0 = p.c0 + int64_t(ct) * N;
            // W is read two 32-column chunks ahead; the first two are requested
            // before the accumulator is ready, so their latency hides behind the
            // tile's MMAs.
            constexpr int NCH = N / 32;
            float4 wbuf[2][8];
            auto load_chunk = [&](int c, float4 (&dst)[8]) {
                const int64_t col = col0 + c * 32;
                if (row_ok && col < p.c1) {
                    const float4* wp = reinterpret_cast<const float4*>(Wrow + col);
#pragma unroll
                    for (int u = 0; u < 8; ++u) dst[u] = wp[u];
                }
            };
            load_chunk(0, wbuf[0]);
            load_chunk(1, wbuf[1]);
            if (!mbar_wait(&accf_bar[a], aph, kErrWaitAccFull, abort)) break;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float v[32];
                tmem_ld32(tmem + uint32_t(a * N + c * 32) + (uint32_t(qr * 32) << 16), v);
                const int64_t col = col0 + c * 32;
                float4 (&cur)[8] = wbuf[c & 1];
                if (row_ok && col < p.c1) {
                    float4* wp = reinterpret_cast<float4*>(Wrow + col);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        float4 w4 = cur[u];
                        w4.x -= v[4 * u + 0];
                        w4.y -= v[4 * u + 1];
                        w4.z -= v[4 * u + 2];
                        w4.w -= v[4 * u + 3];
                        wp[u] = w4;
                    }
                }
                if (c + 2 < NCH) load_chunk(c + 2, cur);
            }
            tc_fence_before();
            mbar_arrive(&acce_bar[a]);
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, UbCfg<N>::TMEM_COLS);
    }
}

// hiT[c][k] = tf32(U[k][c]), loT[c][k] = U[k][c] - hiT[c][k]: 32x32 tiles
// through shared memory so both the reads and the writes are coalesced.
__global__ void __launch_bounds__(256)
split_tf32_transpose_kernel(const float* __restrict__ U, int64_t d, float* __restrict__ hiT,
                            float* __restrict__ loT)
{
    __shared__ float t[32][33];
    const int64_t r0 = int64_t(blockIdx.y) * 32, c0 = int64_t(blockIdx.x) * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
#pragma unroll
    for (int k = 0; k < 32; k += 8) t[ty + k][tx] = U[(r0 + ty + k) * d + c0 + tx];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 32; k += 8) {
        const float v = t[tx][ty + k];               // U[r0 + tx][c0 + ty + k]
        const float h = tf32_round(v);
        hiT[(c0 + ty + k) * d + r0 + tx] = h;
        loT[(c0 + ty + k) * d + r0 + tx] = v - h;
    }
}

size_t update_ws_bytes(int64_t m, int64_t d)
{
    return align_up(sizeof(float) * d * d, 1024) * 2 +
           align_up(sizeof(float) * m * UPD_LDE, 1024) * 2;
}

void update_ws_bind(int64_t m, int64_t d, char* base, UpdateWs* w)
{
    const size_t u = align_up(sizeof(float) * d * d, 1024);
    const size_t e = align_up(sizeof(float) * m * UPD_LDE, 1024);
    w->Uh = reinterpret_cast<float*>(base);
    w->Ul = reinterpret_cast<float*>(base + u);
    w->Eh = reinterpret_cast<float*>(base + 2 * u);
    w->El = reinterpret_cast<float*>(base + 2 * u + e);
}

int update_prepare_u(const float* U, int64_t d, UpdateWs* w, cudaStream_t st)
{
    const dim3 grid((unsigned)(d / 32), (unsigned)(d / 32));
    split_tf32_transpose_kernel<<<grid, 256, 0, st>>>(U, d, w->Uh, w->Ul);
    count_launches();
    return launch_status();
}

int block_update(float* Wk, const UpdateWs* w, int64_t m, int64_t d, int64_t e_col0,
                 int64_t k_rows, int64_t u_row0, int64_t c_begin, int64_t c_end, cudaStream_t st)
{
    if (c_end <= c_begin) return GPTQ_OK;
    if (k_rows <= 0 || k_rows % UB_KC != 0 || e_col0 + k_rows > UPD_LDE) return GPTQ_ERR_SHAPE;
    UpdParams p{};
    p.W = Wk;
    p.m = m;
    p.d = d;
    p.e0 = e_col0;
    p.u0 = u_row0;
    p.c0 = c_begin;
    p.c1 = c_end;
    p.kchunks = (int)(k_rows / UB_KC);
    p.n_rt = (int)ceil_div(m, UB_M);
    const int64_t cols = c_end - c_begin;
    CUtensorMap tEh, tEl, tUh, tUl;
    if (encode_tmap_2d(&tEh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->Eh, UPD_LDE, (uint64_t)m,
                       UPD_LDE * 4, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK ||
        encode_tmap_2d(&tEl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->El, UPD_LDE, (uint64_t)m,
                       UPD_LDE * 4, 32, 128, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
        return GPTQ_ERR_CUDA;
    auto launch = [&](auto kern, int n, int smem) -> int {
        p.n_ct = (int)ceil_div(cols, int64_t(n));
        p.items = p.n_rt * p.n_ct;
        if (encode_tmap_2d(&tUh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->Uh, (uint64_t)d, (uint64_t)d,
                           (uint64_t)d * 4, 32, n, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK ||
            encode_tmap_2d(&tUl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, w->Ul, (uint64_t)d, (uint64_t)d,
                           (uint64_t)d * 4, 32, n, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
            return GPTQ_ERR_CUDA;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        const int grid = std::min(p.items, persistent_ctas(kCtaQuantize));
        kern<<<grid, UB_THREADS, smem, st>>>(tEh, tEl, tUh, tUl, p);
        return GPTQ_OK;
    };
    // 128-wide tiles for near and far updates alike: three 64 KB stages hide
    // the operand latency better than two of 96 KB (measured faster for the
    // far updates too, despite reading E twice as often per output column)
    const int rc = launch(block_update_tc_kernel<128>, 128, UbCfg<128>::SMEM);
    if (rc != GPTQ_OK) return rc;
    count_launches();
    return launch_status();
}

}  // namespace gptq

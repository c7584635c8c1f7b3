// Hessian accumulation S += X^T X (upper triangle) -- "GPTQ / AWQ /
// SqueezeLLM" sec. 一 (H from the calibration inputs).
//
// sm_100a design: 5th-generation tensor cores, fp16 x fp16 -> fp32.
//  * Output tiles of 128 (rows i) x 256 (columns j) covering the upper
//    triangle; the work items are (token split, tile) pairs handed out
//    round-robin to one persistent CTA per SM.  Items of one round share the
//    same token window, so concurrently running CTAs re-read X from L2.
//  * X is token-major (n x d), so both operands of S = X^T X are "MN-major":
//    a TMA box of 64 features x 64 tokens (128-byte swizzle) is exactly one
//    canonical MN-major atom column; A = X[t, i0:i0+128] (2 boxes) and
//    B = X[t, j0:j0+256] (4 boxes) per 64-token stage, 4 stages.
//  * warp 0 issues TMA, warp 1 issues tcgen05.mma (M=128, N=256, K=16).
//  * Accuracy: the tensor core's fp32 accumulator loses low-order bits on
//    every accumulate (measured: about 1.5e-3 relative after 262144 tokens in
//    one accumulator).  So a TMEM accumulator only ever sums one chunk of 512
//    tokens (32 MMAs); eight epilogue warps (warps 2-9, two per TMEM lane
//    quarter, 128 columns each) fold every chunk into fp32 registers with
//    round-to-nearest adds while the MMAs fill the other of two TMEM
//    accumulators, and add the item's sum into S with vector atomics.
//  * Segments: one launch can accumulate several independent sums, one per
//    segment of consecutive rows of X, each into its own S (S_e at
//    S + e d^2): the per-expert Hessians of a mixture-of-experts layer from
//    the experts' routed tokens ("INT4/INT8 量化推理" sec. 五: every expert
//    needs its own calibration statistics).  Work items are (segment, token
//    split, tile), segment-major, so the CTAs of one round still share a
//    token window.  A box that runs past its segment's end is cut in shared
//    memory: the MMA-issuing thread zeroes its rows beyond the end before
//    the MMAs read it (the rows there belong to the next segment).
//  * Every mbarrier wait is bounded (see tc_common.cuh).
#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

constexpr int HB_M = 128, HB_N = 256, HB_K = 64, HB_STAGES = 4;
constexpr int HB_A_BYTES = HB_M * HB_K * 2;                 // 16 KB
constexpr int HB_B_BYTES = HB_N * HB_K * 2;                 // 32 KB
constexpr int HB_STAGE_BYTES = HB_A_BYTES + HB_B_BYTES;     // 48 KB
constexpr int HB_THREADS = 320;
constexpr int HB_EPI_THREADS = 256;
constexpr int HB_CHUNK = 512;                                // tokens per TMEM accumulation
constexpr int HB_SMEM = HB_STAGES * HB_STAGE_BYTES + 1024 + 256;
constexpr uint32_t HB_IDESC = make_idesc(0 /*f16*/, HB_M, HB_N, 1 /*A MN-major*/, 1 /*B MN*/);
constexpr uint32_t HB_TMEM_COLS = 512;

constexpr int HB_MAX_SEG = 64;

struct SyrkParams {
    float* S;         // segment e accumulates into S + e d^2
    int64_t d;
    int nbi;          // row blocks of 128
    int tiles;        // upper-triangle tiles
    int items;        // all segments' items
    int nseg;
    int item0[HB_MAX_SEG + 1];      // first item of each segment
    int64_t row0[HB_MAX_SEG];       // first row of X of each segment
    int64_t row1[HB_MAX_SEG];       // end row (exclusive)
    int64_t per[HB_MAX_SEG];        // tokens per split (multiple of 64)
};

struct HbItem {
    int seg, bi, bj;
    int64_t t0, t1;   // rows of X [t0, t1)
};

__device__ __forceinline__ HbItem hb_item(const SyrkParams& p, int q);

// Tiles are enumerated column-block-major: column block bj (256 wide) holds
// row blocks bi = 0 .. 2 bj + 1 (the last one possibly truncated to nbi).
__device__ __forceinline__ void tile_coords(int t, int& bi, int& bj)
{
    int b = (int)((sqrtf(4.f * (float)t + 1.f) - 1.f) * 0.5f);
    while ((b + 1) * (b + 2) <= t) ++b;
    while (b > 0 && b * (b + 1) > t) --b;
    bj = b;
    bi = t - b * (b + 1);
}

__device__ __forceinline__ HbItem hb_item(const SyrkParams& p, int q)
{
    int e = 0;
    while (e + 1 < p.nseg && p.item0[e + 1] <= q) ++e;
    const int local = q - p.item0[e];
    const int s = local / p.tiles, t = local - s * p.tiles;
    HbItem it;
    it.seg = e;
    tile_coords(t, it.bi, it.bj);
    it.t0 = p.row0[e] + int64_t(s) * p.per[e];
    it.t1 = min(p.row1[e], it.t0 + p.per[e]);
    return it;
}

__global__ void __launch_bounds__(HB_THREADS, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap tmX, const SyrkParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + HB_STAGES * HB_STAGE_BYTES);
    uint64_t* empty_bar = full_bar + HB_STAGES;
    uint64_t* accf_bar = empty_bar + HB_STAGES;
    uint64_t* acce_bar = accf_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < HB_STAGES; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf_bar[a], 1); mbar_init(&acce_bar[a], HB_EPI_THREADS); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, HB_TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = gridDim.x;

    if (warp == 0) {
        if (lane == 0) {
            prefetch_tmap(&tmX);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_par = 0;   // per-stage: armed at least once / last parity
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                const HbItem it = hb_item(p, q);
                const int bi = it.bi, bj = it.bj;
                for (int64_t k = it.t0; k < it.t1; k += HB_K) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1, kErrWaitEmpty, abort)) { ok = false; break; }
                    uint8_t* sa = smem + stage * HB_STAGE_BYTES;
                    uint8_t* sb = sa + HB_A_BYTES;
                    mbar_arrive_expect_tx(&full_bar[stage], HB_STAGE_BYTES);
                    tma_load_2d(sa, &tmX, &full_bar[stage], bi * HB_M, (int)k);
                    tma_load_2d(sa + 8192, &tmX, &full_bar[stage], bi * HB_M + 64, (int)k);
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        tma_load_2d(sb + h * 8192, &tmX, &full_bar[stage], bj * HB_N + 64 * h, (int)k);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == HB_STAGES) { stage = 0; phase ^= 1; }
                }
            }
            // every copy this thread issued has landed before the CTA exits
            for (int s = 0; s < HB_STAGES; ++s)
                if (armed & (1u << s)) mbar_drain(&full_bar[s], (armed_par >> s) & 1u);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0, ch = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                const HbItem it = hb_item(p, q);
                for (int64_t c0 = it.t0; c0 < it.t1 && ok; c0 += HB_CHUNK, ++ch) {
                    const int64_t c1 = min(it.t1, c0 + HB_CHUNK);
                    const int a = ch & 1;
                    const uint32_t aph = (ch >> 1) & 1;
                    if (!mbar_wait(&acce_bar[a], aph ^ 1, kErrWaitAccEmpty, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + uint32_t(a * HB_N);
                    uint32_t acc = 0;
                    for (int64_t k = c0; k < c1; k += HB_K) {
                        if (!mbar_wait(&full_bar[stage], phase, kErrWaitFull, abort)) { ok = false; break; }
                        const int64_t valid = it.t1 - k;
                        if (valid < HB_K) {
                            // the box runs past its segment: zero its rows beyond the end
                            // (each 8 KB box holds 64 token rows of 128 bytes; the swizzle
                            // permutes 16-byte chunks inside a row only).  Only a segment's
                            // last box takes this path.
                            uint8_t* base = smem + stage * HB_STAGE_BYTES;
                            for (int box = 0; box < 6; ++box)
                                for (int64_t o = valid * 128; o < 8192; o += 16)
                                    *reinterpret_cast<uint4*>(base + box * 8192 + o) =
                                        make_uint4(0u, 0u, 0u, 0u);
                            fence_proxy_async_smem();
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(smem + stage * HB_STAGE_BYTES);
                        const uint32_t sb = sa + HB_A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < HB_K / 16; ++kk) {
                            const uint64_t da = smem_desc_sw128(sa + kk * 2048, 8192, 1024);
                            const uint64_t db = smem_desc_sw128(sb + kk * 2048, 8192, 1024);
                            mma_f16(d_tmem, da, db, HB_IDESC, acc);
                            acc = 1;
                        }
                        mma_commit(&empty_bar[stage]);
                        if (++stage == HB_STAGES) { stage = 0; phase ^= 1; }
                    }
                    mma_commit(&accf_bar[a]);
                }
            }
        }
    } else {
        const int ew = warp - 2;                 // 0..7
        const int qr = warp & 3;                 // TMEM lane quarter of this warp
        const int half = ew >> 2;                // columns [128*half, 128*half + 128)
        int ch = 0;
        bool ok = true;
        for (int q = blockIdx.x; q < p.items && ok; q += P) {
            const HbItem it = hb_item(p, q);
            const int bi = it.bi, bj = it.bj;
            float sum[128];
#pragma unroll
            for (int u = 0; u < 128; ++u) sum[u] = 0.f;
            for (int64_t c0 = it.t0; c0 < it.t1; c0 += HB_CHUNK, ++ch) {
                const int a = ch & 1;
                const uint32_t aph = (ch >> 1) & 1;
                if (!mbar_wait(&accf_bar[a], aph, kErrWaitAccFull, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t base = tmem + uint32_t(a * HB_N + half * 128) + (uint32_t(qr * 32) << 16);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float v[32];
                    tmem_ld32(base + uint32_t(c * 32), v);
#pragma unroll
                    for (int u = 0; u < 32; ++u) sum[c * 32 + u] = __fadd_rn(sum[c * 32 + u], v[u]);
                }
                tc_fence_before();
                mbar_arrive(&acce_bar[a]);
            }
            if (!ok) break;
            const int64_t i = int64_t(bi) * HB_M + qr * 32 + lane;
            float* Srow = p.S + int64_t(it.seg) * p.d * p.d + i * p.d;
            const int64_t jb = int64_t(bj) * HB_N + half * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int64_t j0 = jb + c * 32;
                if (j0 >= p.d || j0 + 31 < i) continue;
#pragma unroll
                for (int u = 0; u < 32; u += 4) {
                    const int64_t j = j0 + u;
                    const float* v = sum + c * 32 + u;
                    if (j >= i) {
                        atomicAdd(reinterpret_cast<float4*>(Srow + j),
                                  make_float4(v[0], v[1], v[2], v[3]));
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (j + e >= i) atomicAdd(Srow + j + e, v[e]);
                    }
                }
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, HB_TMEM_COLS);
    }
}

}  // namespace gptq

namespace gptq {

// Launch the accumulation of nseg (<= HB_MAX_SEG) segments [row0[e], row1[e])
// of the rows of X (n_rows x d) into S + e d^2.  Empty segments get no items.
static int hessian_launch(float* S, const uint16_t* X, int64_t n_rows, int64_t d, int nseg,
                          const int64_t* row0, const int64_t* row1, cudaStream_t st)
{
    SyrkParams p{};
    p.S = S;
    p.d = d;
    p.nseg = nseg;
    p.nbi = (int)(d / HB_M);
    const int nbj = (int)ceil_div(d, HB_N);
    p.tiles = (nbj - 1) * nbj + std::min(2 * nbj, p.nbi);
    const int P = persistent_ctas(kCtaHessian);
    if (nseg == 1) {
        // smallest token split count whose round-robin over P CTAs is >= 90 % busy
        const int64_t n = row1[0] - row0[0];
        const int64_t ksteps = ceil_div(n, HB_K);
        int64_t best_s = 1;
        double best_eff = 0.0;
        for (int64_t s = 1; s <= std::min<int64_t>(ksteps, 64); ++s) {
            const int64_t items = p.tiles * s;
            const double eff = double(items) / double(ceil_div(items, P) * P);
            if (eff > best_eff + 1e-9) { best_eff = eff; best_s = s; }
            if (eff >= 0.9) { best_s = s; break; }
        }
        p.per[0] = ceil_div(ksteps, best_s) * HB_K;
    } else {
        // one split length for every segment (a multiple of the 512-token
        // accumulation chunk), chosen by a round model: rounds of P items,
        // each as long as its longest item plus the item's flush into S
        // (about 300 tokens' worth of MMA time)
        int64_t nmax = 0;
        for (int e = 0; e < nseg; ++e) nmax = std::max(nmax, row1[e] - row0[e]);
        int64_t best_per = ceil_div(std::max<int64_t>(nmax, 1), HB_CHUNK) * HB_CHUNK;
        double best_cost = 1e300;
        for (int64_t sp = 1; sp <= 256; ++sp) {          // the longest segment in sp splits
            const int64_t per = ceil_div(ceil_div(std::max<int64_t>(nmax, 1), sp), HB_CHUNK) *
                                HB_CHUNK;
            int64_t items = 0;
            for (int e = 0; e < nseg; ++e) items += p.tiles * ceil_div(row1[e] - row0[e], per);
            const double cost = double(ceil_div(items, P)) * double(per + 300);
            if (cost < best_cost - 1e-9) { best_cost = cost; best_per = per; }
        }
        for (int e = 0; e < nseg; ++e) p.per[e] = best_per;
    }
    int64_t items = 0;
    for (int e = 0; e < nseg; ++e) {
        p.item0[e] = (int)items;
        p.row0[e] = row0[e];
        p.row1[e] = row1[e];
        const int64_t n = row1[e] - row0[e];
        if (n > 0) items += p.tiles * ceil_div(n, p.per[e]);
    }
    p.item0[nseg] = (int)items;
    p.items = (int)items;
    if (items == 0) return GPTQ_OK;
    if (items > (int64_t(1) << 30)) return GPTQ_ERR_SHAPE;

    CUtensorMap tm;
    if (encode_tmap_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X, (uint64_t)d, (uint64_t)n_rows,
                       (uint64_t)d * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
        return GPTQ_ERR_CUDA;
    if (cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             HB_SMEM) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const int grid = (int)std::min<int64_t>(items, P);
    KernelTimer kt(kKHessian, st);
    hessian_tc_kernel<<<grid, HB_THREADS, HB_SMEM, st>>>(tm, p);
    count_launches();
    return launch_status();
}

}  // namespace gptq

extern "C" int gptq_hessian_accumulate(float* S, const uint16_t* X, int64_t n_tokens, int64_t d,
                                       int64_t* n_seen, void* stream)
{
    using namespace gptq;
    if (!S || (!X && n_tokens > 0)) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || (X && !aligned16(X))) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0 || n_tokens < 0 || n_tokens > (int64_t(1) << 31))
        return GPTQ_ERR_SHAPE;
    if (n_tokens == 0) return GPTQ_OK;
    const int64_t r0 = 0, r1 = n_tokens;
    const int rc = hessian_launch(S, X, n_tokens, d, 1, &r0, &r1, as_stream(stream));
    if (rc == GPTQ_OK && n_seen) *n_seen += n_tokens;
    return rc;
}

extern "C" int gptq_hessian_accumulate_grouped(float* S, const uint16_t* X, int64_t n_rows,
                                               int64_t d, const int64_t* offsets,
                                               int64_t n_groups, int64_t* n_seen, void* stream)
{
    using namespace gptq;
    if (!S || !offsets || (!X && n_rows > 0)) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || (X && !aligned16(X))) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0 || n_rows < 0 || n_rows > (int64_t(1) << 31) ||
        n_groups < 1 || n_groups > (int64_t(1) << 20))
        return GPTQ_ERR_SHAPE;
    if (offsets[0] != 0 || offsets[n_groups] != n_rows) return GPTQ_ERR_SHAPE;
    for (int64_t e = 0; e < n_groups; ++e)
        if (offsets[e + 1] < offsets[e]) return GPTQ_ERR_SHAPE;
    if (n_rows == 0) return GPTQ_OK;
    cudaStream_t st = as_stream(stream);
    for (int64_t e0 = 0; e0 < n_groups; e0 += HB_MAX_SEG) {
        const int nseg = (int)std::min<int64_t>(HB_MAX_SEG, n_groups - e0);
        const int rc = hessian_launch(S + e0 * d * d, X, n_rows, d, nseg, offsets + e0,
                                      offsets + e0 + 1, st);
        if (rc != GPTQ_OK) return rc;
    }
    if (n_seen)
        for (int64_t e = 0; e < n_groups; ++e) n_seen[e] += offsets[e + 1] - offsets[e];
    return GPTQ_OK;
}

// Weight-only INT4 product (W4A16) on the tensor cores -- "INT4/INT8 量化推理"
// sec. 六 (weights in 4 bits, activations in fp16) on the storage of sec. 一
// of the same page:
//
//   y[b][r] = sum_j x[b][j] Q[r][j],  Q[r][perm[k]] = s[r][k/g] (c[r][k] - z[r][k/g])
//
// for any batch of activation rows.  The weights stream from HBM once, as
// packed nibbles, and become tensor-core operands in shared memory:
//  * warp 0 loads the packed words by TMA (128 rows x 64 codes = 4 KB per
//    stage, sixteen stages deep), warp 1 the activations (N x 64 fp16, 128-byte
//    swizzle; columns in sweep order, gathered first when perm is given);
//  * the dequantization warps (one or two threads per weight row) turn every
//    packed word into one 16-byte chunk of exact fp16 values c - z: one mask
//    and OR per pair of nibbles puts nibbles k and k + 4 into the mantissas
//    of two 1024.0 halves, one subtraction of 1024 + z leaves c - z (small
//    integers, exact); the chunk is stored where the 128-byte swizzle of a
//    K-major operand puts it.  Its columns are therefore in the order
//    (0, 4, 1, 5, 2, 6, 3, 7) of the word; the activations are gathered into
//    the same order first (with the act-order permutation, when given), and
//    the product does not depend on the order of K;
//  * warp 2 issues tcgen05.mma kind::f16 (M = 128 weight rows, N = the batch
//    tile, K = 16), accumulating one scale chunk (a group, at most 512
//    columns) per TMEM accumulator, two accumulators in turn;
//  * four epilogue warps fold each chunk's accumulator into fp32 registers
//    with the group's fp16 scale, then write y (atomically when K is split).
// Two shapes: batch tiles up to 32 columns with eight dequantization warps
// (decode: the dequantization sets the pace), and up to 128 columns with four
// (the epilogue's 128 accumulators per thread need the registers).
// Products (c - z) x are exact in fp32; sums are fp32 (each TMEM chunk
// accumulates at most 512 products).  Every mbarrier wait is bounded.
#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

constexpr int WQ_M = 128, WQ_K = 64, WQ_NBIG = 128;
constexpr int WQ_CH = 512;                                   // max K per accumulation chunk
constexpr int WQ_A_BYTES = WQ_M * WQ_K * 2;                  // 16 KB
constexpr int WQ_Q_BYTES = WQ_M * WQ_K / 2;                  // 4 KB
constexpr int WQ_EPI_WARPS = 4;

// The decode shape (batch tile <= 32) has a small activation tile, so it
// keeps 8 operand stages (the MMAs' commits come back late relative to the
// short dequantization of a stage); the large shape keeps 4 of 32 KB.
template <int NMAX> struct WqCfg {
    static constexpr int DEQ_WARPS = NMAX <= 32 ? 8 : 4;
    static constexpr int WORDS = 8 / (DEQ_WARPS / 4);          // packed words per thread and stage
    static constexpr int THREADS = 32 * (3 + DEQ_WARPS + WQ_EPI_WARPS);
    static constexpr uint32_t TMEM_COLS = 2 * NMAX < 32 ? 32 : 2 * NMAX;
    static constexpr int STAGES = NMAX <= 32 ? 8 : 4;
    static constexpr int QSTAGES = NMAX <= 32 ? 8 : 16;
    static constexpr int B_BYTES = NMAX * WQ_K * 2;            // 4 KB or 16 KB
    static constexpr int SMEM = STAGES * (WQ_A_BYTES + B_BYTES) + QSTAGES * WQ_Q_BYTES + 1024 + 512;
};

struct WqParams {
    float* y;
    const __half* scales;
    const uint8_t* qzeros;
    int64_t m, d, gsz, batch;
    int ntile;          // batch columns per tile (multiple of 16, <= 128)
    int n_rt, n_nt;     // row tiles, batch tiles
    int ksplit;         // K splits per (row tile, batch tile)
    int chunk;          // columns per accumulation chunk (multiple of 64)
    int chunks_per_split;
    int items;
    int atomic;         // ksplit > 1: y += (zeroed first)
};

struct WqItem { int rt, nt, c0, c1; };     // chunk range [c0, c1)

__device__ __forceinline__ WqItem wq_item(const WqParams& p, int q)
{
    WqItem it;
    const int per = p.n_rt * p.n_nt;
    const int ks = q / per, rem = q - ks * per;
    it.nt = rem / p.n_rt;
    it.rt = rem - it.nt * p.n_rt;
    const int nch = (int)(p.d / p.chunk);
    it.c0 = ks * p.chunks_per_split;
    it.c1 = min(nch, it.c0 + p.chunks_per_split);
    return it;
}

// Nibbles j and j + 4 of w (j = 0..3) as the fp16 pair (1024 + c_j, 1024 + c_{j+4})
__device__ __forceinline__ uint32_t wq_pair_bits(uint32_t w, int j)
{
    return ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
}

template <int NMAX>
__global__ void __launch_bounds__(WqCfg<NMAX>::THREADS, 1)
w4a16_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmX,
                const WqParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr int WQ_STAGES = WqCfg<NMAX>::STAGES, WQ_QSTAGES = WqCfg<NMAX>::QSTAGES;
    constexpr int WQ_B_BYTES = WqCfg<NMAX>::B_BYTES;
    uint8_t* sA = smem;                                          // stages x 16 KB
    uint8_t* sB = sA + WQ_STAGES * WQ_A_BYTES;                   // stages x (4 or 16 KB)
    uint8_t* sQ = sB + WQ_STAGES * WQ_B_BYTES;                   // qstages x 4 KB
    uint64_t* qfull = reinterpret_cast<uint64_t*>(sQ + WQ_QSTAGES * WQ_Q_BYTES);
    uint64_t* qempty = qfull + WQ_QSTAGES;
    uint64_t* afull = qempty + WQ_QSTAGES;
    uint64_t* aempty = afull + WQ_STAGES;
    uint64_t* accf = aempty + WQ_STAGES;
    uint64_t* acce = accf + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < WQ_QSTAGES; ++s) { mbar_init(&qfull[s], 1); mbar_init(&qempty[s], WqCfg<NMAX>::DEQ_WARPS); }
        for (int s = 0; s < WQ_STAGES; ++s) { mbar_init(&afull[s], WqCfg<NMAX>::DEQ_WARPS + 1); mbar_init(&aempty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf[a], 1); mbar_init(&acce[a], WQ_EPI_WARPS); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 2) tmem_alloc(tmem_slot, WqCfg<NMAX>::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int P = gridDim.x;
    const int spc = p.chunk / WQ_K;                          // stages per chunk
    const int64_t G = p.d / p.gsz, Gz = (G + 1) / 2;

    if (warp == 0 || warp == 1) {
        // producers: warp 0 the packed words, warp 1 the activations
        if (lane == 0) {
            const bool packed = warp == 0;
            const int NS = packed ? WQ_QSTAGES : WQ_STAGES;
            uint64_t* full = packed ? qfull : afull;
            uint64_t* empty = packed ? qempty : aempty;
            const uint32_t bytes = packed ? (uint32_t)WQ_Q_BYTES : uint32_t(p.ntile) * WQ_K * 2;
            const CUtensorMap* map = packed ? &tmQ : &tmX;
            prefetch_tmap(map);
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                const WqItem it = wq_item(p, q);
                for (int s = it.c0 * spc; s < it.c1 * spc; ++s) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, kErrWaitEmpty, abort)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], bytes);
                    if (packed)
                        tma_load_2d(sQ + stage * WQ_Q_BYTES, map, &full[stage], s * (WQ_K / 8),
                                    it.rt * WQ_M);
                    else
                        tma_load_2d(sB + stage * WQ_B_BYTES, map, &full[stage], s * WQ_K,
                                    it.nt * p.ntile);
                    armed |= 1u << stage;
                    armed_par = (armed_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == NS) { stage = 0; phase ^= 1; }
                }
            }
            for (int s = 0; s < NS; ++s)
                if (armed & (1u << s)) mbar_drain(&full[s], (armed_par >> s) & 1u);
        }
    } else if (warp == 2) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc(0 /*f16*/, WQ_M, p.ntile, 0, 0);
            int stage = 0, ch = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int q = blockIdx.x; q < p.items && ok; q += P) {
                const WqItem it = wq_item(p, q);
                for (int c = it.c0; c < it.c1 && ok; ++c, ++ch) {
                    const int a = ch & 1;
                    const uint32_t aph = (ch >> 1) & 1;
                    if (!mbar_wait(&acce[a], aph ^ 1, kErrWaitAccEmpty, abort)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + uint32_t(a * NMAX);
                    uint32_t acc = 0;
                    for (int s = 0; s < spc; ++s) {
                        if (!mbar_wait(&afull[stage], phase, kErrWaitFull, abort)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t a_s = smem_u32(sA + stage * WQ_A_BYTES);
                        const uint32_t b_s = smem_u32(sB + stage * WQ_B_BYTES);
#pragma unroll
                        for (int kk = 0; kk < WQ_K / 16; ++kk) {
                            const uint64_t da = smem_desc_sw128(a_s + kk * 32, 16, 1024);
                            const uint64_t db = smem_desc_sw128(b_s + kk * 32, 16, 1024);
                            mma_f16(d_tmem, da, db, idesc, acc);
                            acc = 1;
                        }
                        mma_commit(&aempty[stage]);
                        if (++stage == WQ_STAGES) { stage = 0; phase ^= 1; }
                    }
                    mma_commit(&accf[a]);
                }
            }
        }
    } else if (warp < 3 + WqCfg<NMAX>::DEQ_WARPS) {
        // dequantization: thread (h, r) = weight row r of the tile, words
        // h W .. h W + W - 1 of the row's 8 packed words of a stage -> the
        // same 16-byte chunks of its 128-byte row
        constexpr int W = WqCfg<NMAX>::WORDS;
        const int t = threadIdx.x - 96;
        const int r = t & (WQ_M - 1), h = t >> 7;
        int qs = 0, as = 0;
        uint32_t qph = 0, aph = 0;
        bool ok = true;
        for (int q = blockIdx.x; q < p.items && ok; q += P) {
            const WqItem it = wq_item(p, q);
            const int64_t row = int64_t(it.rt) * WQ_M + r;
            const bool live = row < p.m;
            // zero points: the item's first group now, every next group one
            // group ahead (its load overlaps the current group's stages)
            const int64_t s_begin = int64_t(it.c0) * spc, s_end = int64_t(it.c1) * spc;
            int64_t gi_cur = (s_begin * WQ_K) / p.gsz;
            const int64_t gi_last = ((s_end - 1) * WQ_K) / p.gsz;
            uint32_t zb_cur = live ? uint32_t(p.qzeros[row * Gz + gi_cur / 2]) : 0u;
            uint32_t zb_next = (live && gi_cur < gi_last) ? uint32_t(p.qzeros[row * Gz + (gi_cur + 1) / 2]) : 0u;
            for (int64_t s = s_begin; s < s_end; ++s) {
                const int64_t gi = (s * WQ_K) / p.gsz;
                if (gi != gi_cur) {
                    gi_cur = gi;
                    zb_cur = zb_next;
                    zb_next = (live && gi_cur < gi_last) ? uint32_t(p.qzeros[row * Gz + (gi_cur + 1) / 2]) : 0u;
                }
                if (!mbar_wait(&qfull[qs], qph, kErrWaitFull, abort)) { ok = false; break; }
                uint32_t words[W];
                {
                    const uint4* src = reinterpret_cast<const uint4*>(sQ + qs * WQ_Q_BYTES + r * 32 + h * W * 4);
#pragma unroll
                    for (int v = 0; v < W / 4; ++v) {
                        const uint4 q4 = src[v];
                        words[4 * v] = q4.x; words[4 * v + 1] = q4.y;
                        words[4 * v + 2] = q4.z; words[4 * v + 3] = q4.w;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&qempty[qs]);
                if (++qs == WQ_QSTAGES) { qs = 0; qph ^= 1; }
                const uint32_t z = (gi_cur & 1) ? (zb_cur >> 4) : (zb_cur & 0xFu);
                const uint32_t zbits = 0x64006400u | (z << 16) | z;
                const __half2 zz = *reinterpret_cast<const __half2*>(&zbits);
                if (!mbar_wait(&aempty[as], aph ^ 1, kErrWaitEmpty, abort)) { ok = false; break; }
                uint8_t* arow = sA + as * WQ_A_BYTES + r * 128;
#pragma unroll
                for (int i = 0; i < W; ++i) {
                    uint32_t o[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const uint32_t bits = wq_pair_bits(words[i], j);
                        const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&bits), zz);
                        o[j] = *reinterpret_cast<const uint32_t*>(&v);
                    }
                    const int chunk = h * W + i;
                    *reinterpret_cast<uint4*>(arow + ((chunk ^ (r & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&afull[as]);
                if (++as == WQ_STAGES) { as = 0; aph ^= 1; }
            }
        }
    } else {
        // epilogue: TMEM lane quarter of the warp, one weight row per thread
        const int qr = warp & 3;
        const int r = qr * 32 + lane;
        int ch = 0;
        bool ok = true;
        float sum[NMAX];
        for (int q = blockIdx.x; q < p.items && ok; q += P) {
            const WqItem it = wq_item(p, q);
            const int64_t row = int64_t(it.rt) * WQ_M + r;
            const bool live = row < p.m;
#pragma unroll
            for (int u = 0; u < NMAX; ++u) sum[u] = 0.f;
            for (int c = it.c0; c < it.c1; ++c, ++ch) {
                const int a = ch & 1;
                const uint32_t aph = (ch >> 1) & 1;
                // the chunk's scale is requested before the wait, which hides its latency
                const int64_t gi = (int64_t(c) * p.chunk) / p.gsz;
                const float sc = live ? __half2float(p.scales[row * G + gi]) : 0.f;
                if (!mbar_wait(&accf[a], aph, kErrWaitAccFull, abort)) { ok = false; break; }
                tc_fence_after();
                const uint32_t base = tmem + uint32_t(a * NMAX) + (uint32_t(qr * 32) << 16);
#pragma unroll
                for (int cb = 0; cb < (NMAX + 31) / 32; ++cb) {
                    if (cb * 32 < p.ntile) {
                        float v[32];
                        tmem_ld32(base + uint32_t(cb * 32), v);
#pragma unroll
                        for (int u = 0; u < 32; ++u)
                            if (cb * 32 + u < NMAX) sum[cb * 32 + u] = fmaf(sc, v[u], sum[cb * 32 + u]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[a]);
            }
            if (!ok || !live) continue;
            const int64_t b0 = int64_t(it.nt) * p.ntile;
#pragma unroll
            for (int u = 0; u < NMAX; ++u) {
                const int64_t b = b0 + u;
                if (u < p.ntile && b < p.batch) {
                    if (p.atomic) atomicAdd(p.y + b * p.m + row, sum[u]);
                    else p.y[b * p.m + row] = sum[u];
                }
            }
        }
    }
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, WqCfg<NMAX>::TMEM_COLS);
    }
}

// The activations in the order the A operand holds the columns: position
// 8q + i of a row is column 8q + sigma(i) of the codes (sweep order), with
// sigma = (0, 4, 1, 5, 2, 6, 3, 7) the order the dequantization writes a
// packed word's nibbles in; through perm (act-order) when given:
//   xp[b][8q + i] = x[b][perm[8q + sigma(i)]]
__global__ void gather_cols_kernel(const __half* __restrict__ x, const int32_t* __restrict__ perm,
                                   int64_t batch, int64_t d, __half* __restrict__ xp)
{
    const int64_t total = batch * d;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = i / d, k = i - b * d;
        const int e = int(k & 7);
        const int64_t ks = (k & ~int64_t(7)) + ((e & 1) ? 4 + (e >> 1) : (e >> 1));
        const int32_t pk = perm ? perm[ks] : int32_t(ks);
        if (pk >= 0 && pk < d) {
            xp[i] = x[b * d + pk];
        } else {                                   // not followed: zero and record
            xp[i] = __ushort_as_half(0);
            atomicCAS(&g_device_status, 0, kErrIndex);
        }
    }
}

}  // namespace gptq

extern "C" size_t gptq_w4a16_matmul_workspace_bytes(int64_t batch, int64_t d_in)
{
    if (batch <= 0 || d_in <= 0) return 0;
    return gptq::align_up(size_t(batch) * size_t(d_in) * 2, 1024);    // the reordered activations
}

extern "C" int gptq_w4a16_matmul(const uint16_t* x, int64_t batch, const uint32_t* qweight,
                                 const uint16_t* scales, const uint8_t* qzeros,
                                 const int32_t* perm, int64_t d_out, int64_t d_in, int group_size,
                                 float* y, void* ws, size_t ws_bytes, void* stream)
{
    using namespace gptq;
    if (!x || !qweight || !scales || !qzeros || !y || !ws) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(qweight) || !aligned16(y) || !aligned16(ws) ||
        (perm && !aligned16(perm)) || (reinterpret_cast<uintptr_t>(scales) & 1u))
        return GPTQ_ERR_INVALID_ARG;
    if (batch < 1 || batch > (int64_t(1) << 24)) return GPTQ_ERR_SHAPE;
    if (d_in < 128 || d_in > kMaxDim || d_in % 128 != 0 || d_out < 1 || d_out > kMaxRows)
        return GPTQ_ERR_SHAPE;
    if (ws_bytes < gptq_w4a16_matmul_workspace_bytes(batch, d_in)) return GPTQ_ERR_INVALID_ARG;
    const int64_t gsz = (group_size == -1) ? d_in : group_size;
    if (gsz < 64 || gsz % 64 != 0 || d_in % gsz != 0) return GPTQ_ERR_UNSUPPORTED;
    cudaStream_t st = as_stream(stream);
    KernelTimer kt(kKW4A16, st);
    __half* xp = reinterpret_cast<__half*>(ws);
    {
        const int64_t total = batch * d_in;
        gather_cols_kernel<<<(unsigned)std::min<int64_t>(ceil_div(total, 256),
                                                         int64_t(device_sm_count()) * 16),
                             256, 0, st>>>(reinterpret_cast<const __half*>(x), perm, batch, d_in,
                                           xp);
        count_launches();
    }
    const bool small = ceil_div(batch, 16) * 16 <= 32;          // the decode shape
    WqParams p{};
    p.y = y;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.qzeros = qzeros;
    p.m = d_out;
    p.d = d_in;
    p.gsz = gsz;
    p.batch = batch;
    p.ntile = (int)std::min<int64_t>(small ? 32 : WQ_NBIG, ceil_div(batch, 16) * 16);
    p.n_rt = (int)ceil_div(d_out, WQ_M);
    p.n_nt = (int)ceil_div(batch, p.ntile);
    // accumulation chunk: the largest multiple of 64 columns, at most 512,
    // that divides the group (a chunk never spans two groups)
    p.chunk = WQ_K;
    for (int64_t c = WQ_K; c <= std::min<int64_t>(gsz, WQ_CH); c += WQ_K)
        if (gsz % c == 0) p.chunk = (int)c;
    const int nch = (int)(d_in / p.chunk);
    const int sms = device_sm_count();
    const int64_t tiles = int64_t(p.n_rt) * p.n_nt;
    // split K (in whole chunks) when the tiles alone leave SMs idle: the
    // split count that minimizes rounds x chunks per item, i.e. the longest
    // CTA's share, among 1 .. nch (fewer splits on ties: fewer atomics)
    int ks = 1;
    if (tiles < 2 * sms) {
        double best = 1e300;
        for (int k = 1; k <= nch; ++k) {
            const int64_t cps = ceil_div(nch, k);
            const int64_t kk = ceil_div(nch, cps);
            const double cost = double(ceil_div(tiles * kk, sms)) * double(cps + 1);
            if (cost < best - 1e-9) { best = cost; ks = (int)kk; }
        }
    }
    p.chunks_per_split = (int)ceil_div(nch, ks);
    p.ksplit = (int)ceil_div(nch, p.chunks_per_split);
    p.items = (int)(tiles * p.ksplit);
    p.atomic = p.ksplit > 1;
    if (p.atomic &&
        cudaMemsetAsync(y, 0, sizeof(float) * size_t(batch) * size_t(d_out), st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    CUtensorMap tq, tx;
    if (encode_tmap_2d(&tq, CU_TENSOR_MAP_DATA_TYPE_UINT32, qweight, (uint64_t)(d_in / 8),
                       (uint64_t)d_out, (uint64_t)(d_in / 8) * 4, WQ_K / 8, WQ_M,
                       CU_TENSOR_MAP_SWIZZLE_NONE) != GPTQ_OK ||
        encode_tmap_2d(&tx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xp, (uint64_t)d_in, (uint64_t)batch,
                       (uint64_t)d_in * 2, WQ_K, (uint32_t)p.ntile,
                       CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
        return GPTQ_ERR_CUDA;
    const int grid = std::min(p.items, sms);
    auto run = [&](auto kern, int threads, int smem) -> int {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
            return GPTQ_ERR_CUDA;
        kern<<<grid, threads, smem, st>>>(tq, tx, p);
        count_launches();
        return launch_status();
    };
    return small ? run(w4a16_tc_kernel<32>, WqCfg<32>::THREADS, WqCfg<32>::SMEM)
                 : run(w4a16_tc_kernel<WQ_NBIG>, WqCfg<WQ_NBIG>::THREADS, WqCfg<WQ_NBIG>::SMEM);
}

// Cholesky factorization and triangular inverse of the damped Hessian as one
// persistent, dependency-driven kernel -- "GPTQ / AWQ / SqueezeLLM" sec. 一
// (decomposition of H^-1) and sec. 三 of "INT4/INT8 量化推理" (rows of H^-1
// carry the error).
//
// The matrix is cut into 128x128 tiles, T = d / 128 per dimension.  Each
// tile of L and of X = L^-1 is one task, left-looking:
//   F(j)    diagonal:  B = A_jj - sum_{k<j} L_jk L_jk^T, then the one-CTA leaf
//                      factors B = L_jj L_jj^T and inverts it (X_jj)
//   S(i,j)  i > j:     L_ij = (A_ij - sum_{k<j} L_ik L_jk^T) X_jj^T
//   I(i,j)  i > j:     X_ij = -X_ii sum_{j<=k<i} L_ik X_kj
// Every sum runs on the tensor cores (split-TF32: A_hi B_hi + A_hi B_lo +
// A_lo B_hi, fp32 accumulation in TMEM), one 128-deep product at a time,
// folded into fp32 registers after each product.  The I tasks accumulate
// the transpose, sum_k (X_kj)^T L_ik^T, so that every operand is read
// K-major: they read Y = X^T, which they also write.
//
// Operands are stored split by the task that writes them, so a consumer's
// TMA brings both parts and no thread touches them on the way to the MMA:
// the tile holds the head hi = rna_tf32(x) in place of x and the remainder
// x - hi sits in a tile nothing else uses -- the mirrored tile (c, r) for a
// tile (r, c) off the diagonal of A (L and the S tasks' partial sums) and of
// Y (X^T and the I tasks' partial sums), A's diagonal tile (j, j) (free once
// F(j) has read it) for Y_jj, and a second d x 128 plane of Xc for X_jj.
// The heads and remainders are the values a split in shared memory would
// give, so the products are unchanged; U is written from the fp32 results.
//
// Scheduling: tasks are numbered in an order in which every dependency of
// a task has a smaller number, and each CTA claims the next number from an
// atomic counter.  A CTA waits (bounded) only for tasks with smaller
// numbers, which CTAs that already run hold, so the smallest unfinished task
// can always proceed: no co-residency of the CTAs is needed.  Completion
// flags are released at GPU scope after the task's stores; a consumer
// acquires them and issues a proxy fence before its TMA loads read the data.
//
// Order of the numbers, phase p = 0 .. T-1 (the critical chain
// F(p) -> S(p+1,p) -> F(p+1) is claimed early):
//   phase 0:  F(0), S(1,0), F(1), S(2,0) .. S(T-1,0)
//   phase p:  S(p+1,p), F(p+1), S(p+2,p) .. S(T-1,p), I(p,p-1) .. I(p,0)
//   phase T-1: I(T-1,T-2) .. I(T-1,0)
//
// Batches: one launch can factor E independent matrices of the same size
// (the per-expert Hessians of a mixture-of-experts layer), stacked E high
// in A, Xc, Y and U.  Task number t is local task t / E of matrix t % E, so
// every matrix's tasks keep their topological order and the chains of all
// E matrices advance side by side on the SMs.
//
// CTA roles (320 threads): warp 0 TMA producer (also waits for the
// dependencies; four boxes per 32-wide K chunk: both parts of both
// operands), warp 1 MMA issuer, warps 2-9 fold each product's TMEM
// accumulator into registers (row m, 64 columns per thread) while the MMAs
// fill the other accumulator, then write the task's results, split, through
// shared memory.  The leaf runs on all 320 threads
// (warp 0 as its panel warp, warps 1-9 as its update warps).
#include "chol_dag.cuh"
#include "leaf.cuh"
#include "tc_common.cuh"
#include "update.cuh"

namespace gptq {

constexpr int CD_T = 128, CD_KC = 32, CD_STAGES = 3;
constexpr int CD_TILE_BYTES = CD_T * CD_KC * 4;             // 16 KB
constexpr int CD_STAGE_BYTES = 4 * CD_TILE_BYTES;           // A hi, A lo, B hi, B lo
constexpr int CD_PIPE_BYTES = CD_STAGES * CD_STAGE_BYTES;   // 192 KB
constexpr int CD_THREADS = 320;
constexpr int CD_SMEM = CD_PIPE_BYTES + 1024 + 256;
constexpr uint32_t CD_IDESC = make_idesc(2 /*tf32*/, CD_T, CD_T, 0, 0);
static_assert(LSMEM <= (size_t)CD_PIPE_BYTES, "the leaf reuses the pipeline's shared memory");

enum : int { kTaskF = 0, kTaskS = 1, kTaskI = 2 };
enum : int { kMapA = 0, kMapX = 1, kMapY = 2 };

struct CdParams {
    float* A;
    float* Xc;
    float* Xl;       // remainders of Xc (a second plane, E d x 128)
    float* Y;
    float* U;
    int* flagL;      // T x T: L_ij is final (for i == j: X_jj is in Xc)
    int* flagY;      // T x T: Y_jk (k >= j) is final
    int* ticket;
    int* gabort;     // set by a CTA that gave up: the others stop waiting
    int32_t* info;
    int64_t d;
    int T, total;
    int E;           // matrices in the batch (pointers above are matrix 0's)
    int roff;        // first row of this matrix in the stacked tensor maps
};

// The view of matrix e of a batch: its arrays, flags and info word, and the
// row offset of its tiles in the stacked tensor maps.
__device__ __forceinline__ CdParams cd_matrix(const CdParams& p, int e)
{
    CdParams q = p;
    const int64_t dd = p.d * p.d, TT = int64_t(p.T) * p.T;
    q.A = p.A + e * dd;
    q.Xc = p.Xc + e * p.d * 128;
    q.Xl = p.Xl + e * p.d * 128;
    q.Y = p.Y + e * dd;
    q.U = p.U + e * dd;
    q.flagL = p.flagL + e * 2 * TT;
    q.flagY = q.flagL + TT;
    q.info = p.info + e;
    q.roff = (int)(int64_t(e) * p.d);
    return q;
}

struct CdProduct {
    int ma, ra, ca;      // A operand (heads): tensor map, first row, first column
    int mb, rb, cb;      // B operand (heads)
    const int* f1;       // flags to acquire first (nullptr: none)
    const int* f2;
    int mal, ral, cal;   // where the A operand's remainders are
    int mbl, rbl, cbl;   // where the B operand's remainders are
};

// The tile holding the remainders of the operand tile at (map, tile row r,
// tile column c) of matrix 0 (see the top of this file): mirrored off the diagonal, A's
// diagonal tile for Y's diagonal, the second plane for Xc (rows E d further).
__device__ __forceinline__ void cd_lo_tile(const CdParams& p, int map, int r, int c, int& lmap,
                                           int& lr, int& lc)
{
    if (map == kMapX) { lmap = kMapX; lr = r + p.E * (int)p.d; lc = c; return; }
    const int tr = r / CD_T, tc = c / CD_T;
    lmap = (map == kMapY && tr == tc) ? kMapA : map;
    lr = tc * CD_T;
    lc = tr * CD_T;
}

// Task number -> (type, i, j); see the order above.  Host and device (the
// library's task-order test hook calls it on the host).
__host__ __device__ __forceinline__ void cd_decode(int t, int T, int& type, int& i, int& j)
{
    if (T == 1) { type = kTaskF; i = j = 0; return; }
    if (t < T + 1) {
        if (t == 0) { type = kTaskF; i = j = 0; }
        else if (t == 1) { type = kTaskS; i = 1; j = 0; }
        else if (t == 2) { type = kTaskF; i = j = 1; }
        else { type = kTaskS; i = t - 1; j = 0; }
        return;
    }
    const int r = t - (T + 1);
    const int p = 1 + r / T, u = r % T;
    if (p == T - 1) { type = kTaskI; i = p; j = p - 1 - u; return; }
    if (u == 0) { type = kTaskS; i = p + 1; j = p; }
    else if (u == 1) { type = kTaskF; i = j = p + 1; }
    else if (u < T - p) { type = kTaskS; i = p + u; j = p; }
    else { type = kTaskI; i = p; j = p - 1 - (u - (T - p)); }
}

// q-th product of a task's pass (pass 1: the sum; pass 2: the final product).
__device__ __forceinline__ CdProduct cd_product(const CdParams& p, int type, int i, int j,
                                                int pass, int q)
{
    const int T = p.T;
    CdProduct r;
    if (pass == 1) {
        if (type == kTaskI) {               // (X_kj)^T L_ik^T: A = Y_jk, B = L_ik
            const int k = j + q;
            r = CdProduct{kMapY, j * CD_T, k * CD_T, kMapA, i * CD_T, k * CD_T,
                          &p.flagY[j * T + k],
                          &p.flagL[i * T + k]};
        } else {                            // L_ik L_jk^T
            const int k = q;
            r = CdProduct{kMapA, i * CD_T, k * CD_T, kMapA, j * CD_T, k * CD_T,
                          &p.flagL[i * T + k], &p.flagL[j * T + k]};
        }
    } else if (type == kTaskS) {            // (A_ij - sum) X_jj^T
        r = CdProduct{kMapA, i * CD_T, j * CD_T, kMapX, j * CD_T, 0, nullptr,
                      &p.flagL[j * T + j]};
    } else {                                // X_ii (sum^T)^T
        r = CdProduct{kMapX, i * CD_T, 0, kMapY, j * CD_T, i * CD_T, &p.flagL[i * T + i],
                      nullptr};
    }
    cd_lo_tile(p, r.ma, r.ra, r.ca, r.mal, r.ral, r.cal);
    cd_lo_tile(p, r.mb, r.rb, r.cb, r.mbl, r.rbl, r.cbl);
    r.ra += p.roff;
    r.rb += p.roff;
    r.ral += p.roff;
    r.rbl += p.roff;
    return r;
}

// Tile copies from the shared staging tile sb (128 x LDA floats) to global
// memory, one warp per row (or column) so that every store is coalesced.

// dst[127 - r][127 - c] = sb[r][c]  (a tile of U from a tile of X)
__device__ __forceinline__ void cd_tile_out_reversed(const float* sb, float* dst, int64_t ld,
                                                     int warp, int lane)
{
    for (int r = warp; r < CD_T; r += CD_THREADS / 32) {
        const float4 v = *reinterpret_cast<const float4*>(sb + r * LDA + 4 * lane);
        *reinterpret_cast<float4*>(dst + (CD_T - 1 - r) * ld + CD_T - 4 - 4 * lane) =
            make_float4(v.w, v.z, v.y, v.x);
    }
}

// TF32 head (round to nearest) and fp32 remainder of x: the operand split
__device__ __forceinline__ void cd_split(float x, float& hi, float& lo)
{
    hi = tf32_round(x);
    lo = x - hi;
}

// dh[r][c] = head of sb[r][c], dl[r][c] = its remainder
__device__ __forceinline__ void cd_tile_out_split(const float* sb, float* dh, float* dl,
                                                  int64_t ld, int warp, int lane)
{
    for (int r = warp; r < CD_T; r += CD_THREADS / 32) {
        const float4 v = *reinterpret_cast<const float4*>(sb + r * LDA + 4 * lane);
        float4 h, l;
        cd_split(v.x, h.x, l.x);
        cd_split(v.y, h.y, l.y);
        cd_split(v.z, h.z, l.z);
        cd_split(v.w, h.w, l.w);
        *reinterpret_cast<float4*>(dh + r * ld + 4 * lane) = h;
        *reinterpret_cast<float4*>(dl + r * ld + 4 * lane) = l;
    }
}

// dh[c][r] = head of sb[r][c], dl[c][r] = its remainder (lanes along r:
// coalesced stores, 4-way bank conflicts on the reads)
__device__ __forceinline__ void cd_tile_out_transposed_split(const float* sb, float* dh, float* dl,
                                                             int64_t ld, int warp, int lane)
{
    for (int c = warp; c < CD_T; c += CD_THREADS / 32)
#pragma unroll
        for (int q = 0; q < CD_T / 32; ++q) {
            float h, l;
            cd_split(sb[(32 * q + lane) * LDA + c], h, l);
            dh[c * ld + 32 * q + lane] = h;
            dl[c * ld + 32 * q + lane] = l;
        }
}

__device__ __forceinline__ void cd_tile_zero(float* dst, int64_t ld, int warp, int lane)
{
    for (int r = warp; r < CD_T; r += CD_THREADS / 32)
        *reinterpret_cast<float4*>(dst + r * ld + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
}

__global__ void __launch_bounds__(CD_THREADS, 1)
chol_dag_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                const __grid_constant__ CUtensorMap tmY, const CdParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + CD_PIPE_BYTES);
    uint64_t* empty_bar = full_bar + CD_STAGES;
    uint64_t* accf_bar = empty_bar + CD_STAGES;
    uint64_t* acce_bar = accf_bar + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + 2);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* s_task = abort + 1;
    float* la = reinterpret_cast<float*>(smem);          // leaf: block, then L
    float* lx = la + PN * LDA;                           // leaf: X = L^-1
    float* lt = lx + PN * LDA;                           // leaf: temporary

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t d = p.d;
    const int T = p.T;
    CdParams q = p;                 // the matrix of the current task (see cd_matrix)
    if (tid == 0) {
        for (int s = 0; s < CD_STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&accf_bar[a], 1); mbar_init(&acce_bar[a], 256); }
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // pipeline state of each role, carried across tasks
    int pr_stage = 0, mm_stage = 0;
    uint32_t pr_phase = 0, mm_phase = 0;
    uint32_t armed = 0, armed_par = 0;
    int mm_it = 0, ep_it = 0;
    // warps 2-9: tile row m = qrow*32 + lane (TMEM lane quarter of the warp),
    // columns [64 half, 64 half + 64)
    const int qrow = warp & 3, half = (warp - 2) >> 2;
    const int m = qrow * 32 + lane;
    float acc[CD_T / 2];

    // one pass of n products through the pipeline; warps 2-9 call epi(v, cc)
    // with accumulator columns 64 half + 32 cc .. + 31 of each product, in order
    auto run_pass = [&](int type, int ti, int tj, int pass, int n, auto&& epi) {
        if (warp == 0) {
            if (lane == 0) {
                for (int qi = 0; qi < n; ++qi) {
                    const CdProduct pr = cd_product(q, type, ti, tj, pass, qi);
                    if (pr.f1 && !cd_wait_flag(pr.f1, abort, p.gabort)) break;
                    if (pr.f2 && !cd_wait_flag(pr.f2, abort, p.gabort)) break;
                    fence_proxy_async_global();
                    const CUtensorMap* ma = pr.ma == kMapA ? &tmA : pr.ma == kMapX ? &tmX : &tmY;
                    const CUtensorMap* mb = pr.mb == kMapA ? &tmA : pr.mb == kMapX ? &tmX : &tmY;
                    const CUtensorMap* mal = pr.mal == kMapA ? &tmA : pr.mal == kMapX ? &tmX : &tmY;
                    const CUtensorMap* mbl = pr.mbl == kMapA ? &tmA : pr.mbl == kMapX ? &tmX : &tmY;
                    bool ok = true;
                    for (int kc = 0; kc < CD_T / CD_KC; ++kc) {
                        if (!mbar_wait(&empty_bar[pr_stage], pr_phase ^ 1, kErrWaitEmpty, abort)) {
                            ok = false;
                            break;
                        }
                        uint8_t* st = smem + pr_stage * CD_STAGE_BYTES;
                        mbar_arrive_expect_tx(&full_bar[pr_stage], 4 * CD_TILE_BYTES);
                        tma_load_2d(st, ma, &full_bar[pr_stage], pr.ca + kc * CD_KC, pr.ra);
                        tma_load_2d(st + CD_TILE_BYTES, mal, &full_bar[pr_stage],
                                    pr.cal + kc * CD_KC, pr.ral);
                        tma_load_2d(st + 2 * CD_TILE_BYTES, mb, &full_bar[pr_stage],
                                    pr.cb + kc * CD_KC, pr.rb);
                        tma_load_2d(st + 3 * CD_TILE_BYTES, mbl, &full_bar[pr_stage],
                                    pr.cbl + kc * CD_KC, pr.rbl);
                        armed |= 1u << pr_stage;
                        armed_par = (armed_par & ~(1u << pr_stage)) | (pr_phase << pr_stage);
                        if (++pr_stage == CD_STAGES) { pr_stage = 0; pr_phase ^= 1; }
                    }
                    if (!ok) break;
                }
            }
        } else if (warp == 1) {
            if (lane == 0) {
                bool ok = true;
                for (int qi = 0; qi < n && ok; ++qi, ++mm_it) {
                    const int a = mm_it & 1;
                    const uint32_t aph = (mm_it >> 1) & 1;
                    if (!mbar_wait(&acce_bar[a], aph ^ 1, kErrWaitAccEmpty, abort)) break;
                    tc_fence_after();
                    const uint32_t d_tmem = tmem + uint32_t(a * CD_T);
                    uint32_t accum = 0;
                    for (int kc = 0; kc < CD_T / CD_KC; ++kc) {
                        if (!mbar_wait(&full_bar[mm_stage], mm_phase, kErrWaitFull, abort)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sAh = smem_u32(smem + mm_stage * CD_STAGE_BYTES);
                        const uint32_t sAl = sAh + CD_TILE_BYTES;
                        const uint32_t sBh = sAh + 2 * CD_TILE_BYTES;
                        const uint32_t sBl = sAh + 3 * CD_TILE_BYTES;
#pragma unroll
                        for (int kk = 0; kk < CD_KC / 8; ++kk) {
                            const uint64_t aH = smem_desc_sw128(sAh + kk * 32, 16, 1024);
                            const uint64_t aL = smem_desc_sw128(sAl + kk * 32, 16, 1024);
                            const uint64_t bH = smem_desc_sw128(sBh + kk * 32, 16, 1024);
                            const uint64_t bL = smem_desc_sw128(sBl + kk * 32, 16, 1024);
                            mma_tf32(d_tmem, aH, bH, CD_IDESC, accum);
                            mma_tf32(d_tmem, aH, bL, CD_IDESC, 1u);
                            mma_tf32(d_tmem, aL, bH, CD_IDESC, 1u);
                            accum = 1;
                        }
                        mma_commit(&empty_bar[mm_stage]);
                        if (++mm_stage == CD_STAGES) { mm_stage = 0; mm_phase ^= 1; }
                    }
                    if (ok) mma_commit(&accf_bar[a]);
                }
            }
        } else {
            // warps 2-9: fold each product as its accumulator fills (the MMAs
            // of the next product run into the other accumulator meanwhile)
            for (int qi = 0; qi < n; ++qi) {
                const int a = ep_it & 1;
                const uint32_t aph = (ep_it >> 1) & 1;
                ++ep_it;
                if (!mbar_wait(&accf_bar[a], aph, kErrWaitAccFull, abort)) break;
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float v[32];
                    tmem_ld32(tmem + uint32_t(a * CD_T + (2 * half + cc) * 32) +
                                  (uint32_t(qrow * 32) << 16), v);
                    epi(v, cc);
                }
                tc_fence_before();
                mbar_arrive(&acce_bar[a]);
            }
        }
    };

    for (;;) {
        if (tid == 0) {
            int t = p.total;
            if (*abort) atomicExch(p.gabort, 1);
            else if (!*reinterpret_cast<const volatile int*>(p.gabort)) t = atomicAdd(p.ticket, 1);
            *s_task = t;
        }
        __syncthreads();
        const int t = *s_task;
        if (t >= p.total) break;
        q = cd_matrix(p, t % p.E);
        int type, ti, tj;
        cd_decode(t / p.E, T, type, ti, tj);
        const int n1 = (type == kTaskI) ? ti - tj : tj;
        const int64_t r0 = int64_t(ti) * CD_T, c0 = int64_t(tj) * CD_T;

        const int cb = 64 * half;                          // first column of this thread
        float* sb = la;                                    // staging tile (pipeline memory)
        auto stage_acc = [&]() {                           // acc rows -> sb
            if (warp >= 2) {
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    *reinterpret_cast<float4*>(sb + m * LDA + cb + 4 * u) =
                        make_float4(acc[4 * u], acc[4 * u + 1], acc[4 * u + 2], acc[4 * u + 3]);
            }
        };
        auto release = [&](int* f) {                       // after the task's stores
            fence_proxy_async_global();
            fence_proxy_async_smem();                      // the pipeline reuses sb
            __syncthreads();
            if (tid == 0 && !*abort) {
                __threadfence();
                st_release_gpu(f, 1);
            }
        };

        // ---- pass 1: acc = A_ij - sum (F, S) or the sum's transpose (I), row m
        if (type == kTaskI) {
#pragma unroll
            for (int u = 0; u < CD_T / 2; ++u) acc[u] = 0.f;
        } else if (warp >= 2) {
            const float4* src = reinterpret_cast<const float4*>(q.A + (r0 + m) * d + c0 + cb);
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const float4 x = src[u];
                acc[4 * u] = x.x; acc[4 * u + 1] = x.y; acc[4 * u + 2] = x.z; acc[4 * u + 3] = x.w;
            }
        }
        if (type == kTaskS)           // the mirrored tile of U is zero
            cd_tile_zero(q.U + (d - CD_T - c0) * d + (d - CD_T - r0), d, warp, lane);
        const float sgn = (type == kTaskI) ? 1.f : -1.f;
        run_pass(type, ti, tj, 1, n1, [&](const float (&v)[32], int cc) {
#pragma unroll
            for (int u = 0; u < 32; ++u) acc[cc * 32 + u] = fmaf(sgn, v[u], acc[cc * 32 + u]);
        });

        if (type == kTaskF) {
            // leaf on B = A_jj - sum, X zeroed
            if (warp >= 2) {
                stage_acc();
#pragma unroll
                for (int u = 0; u < 16; ++u)
                    *reinterpret_cast<float4*>(lx + m * LDA + cb + 4 * u) =
                        make_float4(0.f, 0.f, 0.f, 0.f);
            }
            __syncthreads();
            leaf_factor_invert<CD_THREADS>(la, lx, lt, tid, q.info, d - c0, abort);
            // X_jj first: the S tasks of column j wait only for it
            for (int idx = tid * 4; idx < CD_T * CD_T; idx += CD_THREADS * 4) {
                const int r = idx / CD_T, c = idx % CD_T;
                const float4 v = *reinterpret_cast<const float4*>(lx + r * LDA + c);
                float4 h, l;
                cd_split(v.x, h.x, l.x);
                cd_split(v.y, h.y, l.y);
                cd_split(v.z, h.z, l.z);
                cd_split(v.w, h.w, l.w);
                *reinterpret_cast<float4*>(q.Xc + (c0 + r) * CD_T + c) = h;
                *reinterpret_cast<float4*>(q.Xl + (c0 + r) * CD_T + c) = l;
            }
            fence_proxy_async_global();
            __syncthreads();
            if (tid == 0 && !*abort) {
                __threadfence();
                st_release_gpu(&q.flagL[tj * T + tj], 1);
            }
            // then Y_jj = X_jj^T (remainders into A's diagonal tile, which
            // nothing reads any more) and the diagonal tile of U
            cd_tile_out_transposed_split(lx, q.Y + c0 * d + c0, q.A + c0 * d + c0, d, warp, lane);
            cd_tile_out_reversed(lx, q.U + (d - CD_T - c0) * d + (d - CD_T - c0), d, warp, lane);
            release(&q.flagY[tj * T + tj]);
        } else if (type == kTaskS) {
            {   // A_ij - sum back into A, split (remainders in the mirrored
                // tile): the final product reads it
                stage_acc();
                __syncthreads();
                cd_tile_out_split(sb, q.A + r0 * d + c0, q.A + c0 * d + r0, d, warp, lane);
                fence_proxy_async_global();
                fence_proxy_async_smem();
                __syncthreads();
            }
            // L_ij = (A_ij - sum) X_jj^T into A
            run_pass(type, ti, tj, 2, 1, [&](const float (&v)[32], int cc) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4*>(sb + m * LDA + cb + cc * 32 + 4 * u) =
                        make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
            });
            __syncthreads();
            cd_tile_out_split(sb, q.A + r0 * d + c0, q.A + c0 * d + r0, d, warp, lane);
            release(&q.flagL[ti * T + tj]);
        } else {
            // the sum's transpose into the Y_ji tile: the final product reads it
            stage_acc();
            __syncthreads();
            cd_tile_out_split(sb, q.Y + c0 * d + r0, q.Y + r0 * d + c0, d, warp, lane);
            fence_proxy_async_global();
            fence_proxy_async_smem();
            __syncthreads();
            // X_ij = -X_ii sum: Y_ji = X_ij^T, U gets X_ij reversed
            run_pass(type, ti, tj, 2, 1, [&](const float (&v)[32], int cc) {
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    *reinterpret_cast<float4*>(sb + m * LDA + cb + cc * 32 + 4 * u) =
                        make_float4(-v[4 * u], -v[4 * u + 1], -v[4 * u + 2], -v[4 * u + 3]);
            });
            __syncthreads();
            cd_tile_out_transposed_split(sb, q.Y + c0 * d + r0, q.Y + r0 * d + c0, d, warp, lane);
            cd_tile_out_reversed(sb, q.U + (d - CD_T - r0) * d + (d - CD_T - c0), d, warp, lane);
            release(&q.flagY[tj * T + ti]);
        }
    }

    if (warp == 0 && lane == 0)
        for (int s = 0; s < CD_STAGES; ++s)
            if (armed & (1u << s)) mbar_drain(&full_bar[s], (armed_par >> s) & 1u);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

size_t chol_dag_sync_bytes(int64_t d, int64_t E)
{
    const int64_t T = d / CD_T;
    return sizeof(int) * size_t(2 * T * T * E + 32);
}

int chol_inv_dag(float* A, float* Xc, float* Y, float* U, void* sync, int64_t d, int64_t E,
                 int32_t* info, cudaStream_t st)
{
    if (d < CD_T || d % CD_T) return GPTQ_ERR_SHAPE;
    const int T = (int)(d / CD_T);
    // 2 E d: the rows of Xc's two planes, int32 TMA coordinates
    if (E < 1 || 2 * E * d > (int64_t(1) << 31) - 1 || E * T * T > (int64_t(1) << 30))
        return GPTQ_ERR_SHAPE;
    CdParams p{};
    p.A = A; p.Xc = Xc; p.Y = Y; p.U = U;
    p.Xl = Xc + E * d * CD_T;          // the remainder plane
    int* s = reinterpret_cast<int*>(sync);
    p.flagL = s;
    p.flagY = s + size_t(T) * T;
    p.ticket = s + size_t(2) * T * T * E;
    p.gabort = p.ticket + 1;
    p.info = info;
    p.d = d;
    p.T = T;
    p.E = (int)E;
    p.total = (int)(E * T * T);
    p.roff = 0;
    if (cudaMemsetAsync(sync, 0, chol_dag_sync_bytes(d, E), st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    CUtensorMap tA, tX, tY;
    const uint64_t rows = uint64_t(E) * uint64_t(d);
    if (encode_tmap_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, A, (uint64_t)d, rows,
                       (uint64_t)d * 4, CD_KC, CD_T, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK ||
        encode_tmap_2d(&tX, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Xc, (uint64_t)CD_T, 2 * rows,
                       (uint64_t)CD_T * 4, CD_KC, CD_T, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK ||
        encode_tmap_2d(&tY, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y, (uint64_t)d, rows,
                       (uint64_t)d * 4, CD_KC, CD_T, CU_TENSOR_MAP_SWIZZLE_128B) != GPTQ_OK)
        return GPTQ_ERR_CUDA;
    if (cudaFuncSetAttribute(chol_dag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             CD_SMEM) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    const int grid = std::min(p.total, persistent_ctas(kCtaPrepare));
    chol_dag_kernel<<<grid, CD_THREADS, CD_SMEM, st>>>(tA, tX, tY, p);
    count_launches();
    return launch_status();
}

}  // namespace gptq

// Test hook: the factorization's tasks in claim order (host only).
extern "C" int64_t gptq_debug_chol_task_order(int64_t d, int32_t* out, int64_t cap)
{
    using namespace gptq;
    if (d < CD_T || d % CD_T || d > kMaxDim) return -GPTQ_ERR_SHAPE;
    const int T = (int)(d / CD_T);
    const int64_t total = int64_t(T) * T;
    if (!out || cap < 3 * total) return -GPTQ_ERR_INVALID_ARG;
    for (int t = 0; t < (int)total; ++t) {
        int type, i, j;
        cd_decode(t, T, type, i, j);
        out[3 * t] = type;
        out[3 * t + 1] = i;
        out[3 * t + 2] = j;
    }
    return total;
}

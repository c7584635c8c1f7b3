// 128x128 leaf of the blocked Cholesky factorization, on one CTA, in shared
// memory -- "GPTQ / AWQ / SqueezeLLM" sec. 一 (decomposition of H^-1).
//
#pragma once

#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

constexpr int PN = 128;            // leaf width
constexpr int PW = 8;              // panel width of the leaf's factorization
// leaf_factor_invert: factor the symmetric block held in `a` (lower triangle
// read) into L (lower, in `a`) and write X = L^-1 into `xs` (which the caller
// zeroed): an 8-column right-looking factorization pipelined between a panel
// warp and update warps (below), then X from the 8x8 diagonal inverses by
// four doubling levels, X_BC = -X_C (B X_A), as small GEMMs in shared memory.
constexpr int LDA = PN + 4;                  // row stride of the shared 128x128 blocks
constexpr int LDT = 68;                      // row stride of the doubling temporary
constexpr int LPC_BYTES = 2 * (PW / 4) * PN * 16;   // compact panel copies, two step parities
constexpr int LTB_BYTES = 64 * LDT * 4;      // tb: doubling temporary, or panel copies + mbarriers
static_assert(LPC_BYTES + 64 <= LTB_BYTES, "panel copies and barriers fit in tb");
constexpr size_t LSMEM = sizeof(float) * 2 * PN * LDA + LTB_BYTES;

__device__ __forceinline__ void tri_index(int t, int& r, int& c)
{
    const float x = 8.f * (float)t + 1.f;                 // estimate, corrected below
    int u = (int)((x * rsqrtf(x) - 1.f) * 0.5f);
    while ((u + 1) * (u + 2) / 2 <= t) ++u;
    while (u > 0 && u * (u + 1) / 2 > t) --u;
    r = u;
    c = t - u * (u + 1) / 2;
}

// C (4x4 tile at rows i0.., cols j0..) = sum over k in [kb, ke) of P[i][k] Q[k][j]
// with P, Q in shared memory (row strides ldp, ldq; k range a multiple of 4).
__device__ __forceinline__ void tile_gemm4(const float* P, int ldp, const float* Q, int ldq,
                                           int i0, int j0, int kb, int ke, float (&acc)[4][4])
{
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k = kb; k < ke; k += 4) {
        float4 pr[4], qr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pr[i] = *reinterpret_cast<const float4*>(P + (i0 + i) * ldp + k);
#pragma unroll
        for (int q = 0; q < 4; ++q) qr[q] = *reinterpret_cast<const float4*>(Q + (k + q) * ldq + j0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float pv[4] = {pr[i].x, pr[i].y, pr[i].z, pr[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc[i][0] = fmaf(pv[q], qr[q].x, acc[i][0]);
                acc[i][1] = fmaf(pv[q], qr[q].y, acc[i][1]);
                acc[i][2] = fmaf(pv[q], qr[q].z, acc[i][2]);
                acc[i][3] = fmaf(pv[q], qr[q].w, acc[i][3]);
            }
        }
    }
}

// Shared memory: a (128 x LDA), xs (128 x LDA), tb (64 x LDT), 16-byte aligned.
// A non-positive pivot at column c of the block stores piv0 - c into *info
// (first one wins) and the factorization continues with NaN.  NT = threads of
// the CTA; every thread must call (the function contains __syncthreads).
// Slot of row r in the compact copy of a panel: rows 4 apart (the rows one
// warp's tiles read together) fall into distinct 16-byte slots of a 128-byte
// line, so the float4 loads below take the minimum number of wavefronts.
__device__ __forceinline__ int panel_slot(int r) { return r ^ ((r >> 3) & 7); }

// a[r0..r0+3][q0..q0+3] -= L[r0..r0+3][c0..c0+3] L[q0..q0+3][c0..c0+3]^T, with
// the panel's L rows read from its compact copy pc
__device__ __forceinline__ void rank4_tile(float* __restrict__ a, const float4* __restrict__ pc,
                                           int r0, int q0)
{
    float4 lr[4], lc[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lr[i] = pc[panel_slot(r0 + i)];
        lc[i] = pc[panel_slot(q0 + i)];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 cur = *reinterpret_cast<const float4*>(a + (r0 + i) * LDA + q0);
        float cv[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float t2 = cv[j];
            t2 = fmaf(-lr[i].x, lc[j].x, t2);
            t2 = fmaf(-lr[i].y, lc[j].y, t2);
            t2 = fmaf(-lr[i].z, lc[j].z, t2);
            t2 = fmaf(-lr[i].w, lc[j].w, t2);
            cv[j] = t2;
        }
        *reinterpret_cast<float4*>(a + (r0 + i) * LDA + q0) = make_float4(cv[0], cv[1], cv[2], cv[3]);
    }
}

// Shared memory: a (128 x LDA), xs (128 x LDA), tb (LTB_BYTES), 16-byte
// aligned.  A non-positive pivot at column c of the block stores piv0 - c
// into *info (first one wins) and the factorization continues with NaN.
// NT = threads of the CTA (a multiple of 32, at least 64); every thread must
// call (the function uses __syncthreads).  `abort` is the CTA's abort flag of
// the bounded waits (tc_common.cuh): a wait that gives up records
// kErrWaitLeaf and every role leaves early; the block is then garbage.
//
// Factorization, 8 columns per step c0, software-pipelined across two roles:
//   warp 0 (panel):   factor and invert the 8x8 pivot block in registers,
//                     solve the 8 panel entries of every row below (into a,
//                     and into two compact 4-column copies in tb,
//                     double-buffered by step parity) and publish;
//   warps 1.. (update): after the publish, first apply the panel's rank-8
//                     update to the next panel's 8 columns and signal that
//                     the panel warp may go on, then apply it to the rest of
//                     the trailing triangle (columns >= c0 + 16, which the
//                     panel warp neither reads nor writes in its next step).
// Eight columns per step halve the number of steps, hence of hand-offs,
// against a 4-column panel; the panel warp's solve does twice the work.
// The hand-offs are mbarriers alternating by step parity: pub[parity]
// completes when the panel warp has published step c0 and every update warp
// has finished the trailing update of step c0 - 8 (which orders the updates
// of consecutive steps), nxt[parity] when every update warp has updated the
// next panel's columns.  The next use of a barrier always follows a wait that
// saw its previous phase complete.
template <int NT>
__device__ __forceinline__ void leaf_factor_invert(float* __restrict__ a, float* __restrict__ xs,
                                                   float* __restrict__ tb, int tid,
                                                   int32_t* __restrict__ info, int64_t piv0,
                                                   volatile int* abort)
{
    static_assert(NT % 32 == 0 && NT >= 64, "one panel warp and at least one update warp");
    constexpr int NU = NT - 32;
    const int warp = tid >> 5, lane = tid & 31;
    float4* const pcb = reinterpret_cast<float4*>(tb);     // 2 x 128 compact panel copies
    uint64_t* const pub = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(tb) + LPC_BYTES);
    uint64_t* const nxt = pub + 2;
    if (tid == 0) {
        mbar_init(&pub[0], 1 + NU / 32);
        mbar_init(&pub[1], 1 + NU / 32);
        mbar_init(&nxt[0], NU / 32);
        mbar_init(&nxt[1], NU / 32);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        for (int c0 = 0; c0 < PN; c0 += PW) {
            const int st = c0 / PW;
            if (c0 > 0 && !mbar_wait(&nxt[(st - 1) & 1], ((st - 1) >> 1) & 1, kErrWaitLeaf, abort))
                break;
            // 8x8 diagonal block: Cholesky factor g and its inverse h, in registers
            float g[PW][PW], h[PW][PW];
#pragma unroll
            for (int i = 0; i < PW; ++i)
#pragma unroll
                for (int j = 0; j < PW; ++j) g[i][j] = (j <= i) ? a[(c0 + i) * LDA + c0 + j] : 0.f;
            float rd[PW];
#pragma unroll
            for (int j = 0; j < PW; ++j) {
                const float djj = g[j][j];
                const bool bad = !(djj > 0.f);
                if (bad && lane == 0 && info)
                    atomicCAS(reinterpret_cast<int*>(info), 0, (int)(piv0 - (c0 + j)));
                // 1/sqrt(d) from the hardware estimate plus one Newton step (~1 ulp)
                float y = rsqrtf(djj);
                y = y * fmaf(-0.5f * djj * y, y, 1.5f);
                if (bad) y = __int_as_float(0x7fc00000);
                rd[j] = y;
                g[j][j] = djj * y;
#pragma unroll
                for (int i = j + 1; i < PW; ++i) g[i][j] *= rd[j];
#pragma unroll
                for (int i = j + 1; i < PW; ++i)
#pragma unroll
                    for (int k = j + 1; k <= i; ++k) g[i][k] = fmaf(-g[i][j], g[k][j], g[i][k]);
            }
#pragma unroll
            for (int c = 0; c < PW; ++c) {                // forward substitution, column c
#pragma unroll
                for (int r = 0; r < PW; ++r) {
                    if (r < c) { h[r][c] = 0.f; continue; }
                    float t = (r == c) ? 1.f : 0.f;
#pragma unroll
                    for (int k = c; k < r; ++k) t = fmaf(-g[r][k], h[k][c], t);
                    h[r][c] = t * rd[r];
                }
            }
            __syncwarp();                                  // every lane has read the pivot block
            if (lane < PW) {
#pragma unroll
                for (int i = 0; i < PW; ++i)
                    if (lane == i) {
                        *reinterpret_cast<float4*>(a + (c0 + i) * LDA + c0) =
                            make_float4(g[i][0], g[i][1], g[i][2], g[i][3]);
                        *reinterpret_cast<float4*>(a + (c0 + i) * LDA + c0 + 4) =
                            make_float4(g[i][4], g[i][5], g[i][6], g[i][7]);
                        *reinterpret_cast<float4*>(xs + (c0 + i) * LDA + c0) =
                            make_float4(h[i][0], h[i][1], h[i][2], h[i][3]);
                        *reinterpret_cast<float4*>(xs + (c0 + i) * LDA + c0 + 4) =
                            make_float4(h[i][4], h[i][5], h[i][6], h[i][7]);
                    }
            }
            // panel rows below: L[r][c0..c0+7] = A[r][c0..c0+7] h^T, into a and
            // into the compact copies (columns 0-3 in pc[0..], 4-7 in pc[PN..])
            float4* pc = pcb + (st & 1) * 2 * PN;
            for (int r = c0 + PW + lane; r < PN; r += 32) {
                const float4 v0 = *reinterpret_cast<const float4*>(a + r * LDA + c0);
                const float4 v1 = *reinterpret_cast<const float4*>(a + r * LDA + c0 + 4);
                const float av[PW] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
                float o[PW];
#pragma unroll
                for (int c = 0; c < PW; ++c) {
                    float t = 0.f;
#pragma unroll
                    for (int k = 0; k <= c; ++k) t = fmaf(av[k], h[c][k], t);
                    o[c] = t;
                }
                const float4 l0 = make_float4(o[0], o[1], o[2], o[3]);
                const float4 l1 = make_float4(o[4], o[5], o[6], o[7]);
                *reinterpret_cast<float4*>(a + r * LDA + c0) = l0;
                *reinterpret_cast<float4*>(a + r * LDA + c0 + 4) = l1;
                pc[panel_slot(r)] = l0;
                pc[PN + panel_slot(r)] = l1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pub[st & 1]);      // panel published
        }
    } else {
        const int ut = tid - 32;
        if (lane == 0) mbar_arrive(&pub[0]);              // nothing before step 0
        for (int c0 = 0; c0 < PN; c0 += PW) {
            const int st = c0 / PW;
            if (!mbar_wait(&pub[st & 1], (st >> 1) & 1, kErrWaitLeaf, abort)) break;
            const int nt = (PN - c0 - PW) / 4;             // 4-row tiles below the panel
            const float4* pc = pcb + (st & 1) * 2 * PN;
            // the next panel's 8 columns (two tile columns), lower part only
            for (int t = ut; t < 2 * nt; t += NU) {
                const int ti = t >> 1, tj = t & 1;
                if (ti < tj) continue;                     // wholly above the diagonal
                rank4_tile(a, pc, c0 + PW + 4 * ti, c0 + PW + 4 * tj);
                rank4_tile(a, pc + PN, c0 + PW + 4 * ti, c0 + PW + 4 * tj);
            }
            __syncwarp();
            if (c0 + PW < PN && lane == 0) mbar_arrive(&nxt[st & 1]);   // next panel's columns
            const int n2 = max(nt - PW / 4, 0);            // tile columns >= c0 + 16
            const int tiles = n2 * (n2 + 1) / 2;
            for (int t = ut; t < tiles; t += NU) {
                int ti, tj;
                tri_index(t, ti, tj);
                rank4_tile(a, pc, c0 + 2 * PW + 4 * ti, c0 + 2 * PW + 4 * tj);
                rank4_tile(a, pc + PN, c0 + 2 * PW + 4 * ti, c0 + 2 * PW + 4 * tj);
            }
            __syncwarp();
            if (c0 + PW < PN && lane == 0) mbar_arrive(&pub[(st + 1) & 1]);   // next step
        }
    }
    __syncthreads();
    if (tid == 0) {                     // tb becomes the doubling temporary
#pragma unroll
        for (int b = 0; b < 4; ++b) mbar_inval(&pub[b]);
    }
    __syncthreads();

    // X from the 8x8 diagonal inverses by doubling: s = 8, 16, 32, 64
    for (int s = PW; s < PN; s *= 2) {
        const int pairs = PN / (2 * s);
        const int ts = s / 4, tpp = ts * ts;               // 4x4 tiles per pair
        // T = B X_A, B = L[o+s+i][o+k], X_A = X[o+k][o+j] (zero for k < j)
        for (int t = tid; t < pairs * tpp; t += NT) {
            const int pr = t / tpp, tt = t % tpp;
            const int o = pr * 2 * s;
            const int i0 = (tt / ts) * 4, j0 = (tt % ts) * 4;
            float acc[4][4];
            tile_gemm4(a + (o + s) * LDA + o, LDA, xs + o * LDA + o, LDA, i0, j0, j0, s, acc);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(tb + (pr * s + i0 + i) * LDT + j0) =
                    make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
        }
        __syncthreads();
        // X_BC = -X_C T, X_C = X[o+s+i][o+s+k] (zero for k > i)
        for (int t = tid; t < pairs * tpp; t += NT) {
            const int pr = t / tpp, tt = t % tpp;
            const int o = pr * 2 * s;
            const int i0 = (tt / ts) * 4, j0 = (tt % ts) * 4;
            float acc[4][4];
            tile_gemm4(xs + (o + s) * LDA + o + s, LDA, tb + pr * s * LDT, LDT, i0, j0, 0, i0 + 4,
                       acc);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(xs + (o + s + i0 + i) * LDA + o + j0) =
                    make_float4(-acc[i][0], -acc[i][1], -acc[i][2], -acc[i][3]);
        }
        __syncthreads();
    }

}

}  // namespace gptq

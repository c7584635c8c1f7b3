// Inverse-Hessian preparation -- "GPTQ / AWQ / SqueezeLLM" sec. 一
// (H = 2 X^T X / n, damping, importance order, decomposition of H^-1).
//
// U = upper Cholesky factor of Hd^-1 is taken by the reverse-order route:
// with J the exchange matrix, A = J Hd J = L L^T (lower Cholesky), and
// U = J L^-1 J is upper with U^T U = Hd^-1 (uniqueness of the Cholesky
// factor): one factorization and one triangular inverse.
//
// Steps (all on the device):
//   1. keys + lambda: diag(S), lambda = damp * mean(2 S_ii / n)
//   2. perm: stable descending rank of S_ii (act-order) or identity
//   3. A[i][j] = Hd[d-1-i][d-1-j], Hd = (2/n) S[perm][:, perm] + lambda I
//   4. blocked right-looking Cholesky of A with 128-wide panels:
//        leaf:  one CTA factors the 128x128 diagonal block and inverts it
//               (L_kk, X_kk = L_kk^-1, Y_kk = X_kk^T): 4-column steps with a
//               rank-4 trailing update, then the inverse from the 4x4
//               diagonal inverses by doubling
//        TRSM:  A[below, k] <- A[below, k] X_kk^T       (tensor-core GEMM)
//        SYRK:  A[below, below] -= L21 L21^T, lower tiles (tensor-core GEMM)
//   5. X = L^-1 by recursive doubling: for blocks [[A,0],[B,C]] (A of size s,
//      C of size c <= s),  T^T = Y_A B^T,  X_BC = -X_C T,  Y_BC = X_BC^T;
//      all full pairs of one level in one batched GEMM, ceil(log2(d/128))
//      levels
//   6. U[i][j] = X[d-1-i][d-1-j] (upper), 0 below the diagonal
// The GEMMs are split-TF32 on tcgen05 (gemm_nt.cu), fp32-level accuracy.
#include "common.cuh"
#include "gemm_nt.cuh"

namespace gptq {

constexpr int PN = 128;            // panel / leaf width

struct PrepWs {
    float* A;      // d x d working matrix, then L in its lower triangle
    float* X;      // d x d, L^-1 (lower)
    float* Y;      // d x d, L^-T (upper)
    float* T;      // d x (d/2) temporary of the inverse's levels
    float* keys;   // d
    float* lam;    // 1
};

static size_t prep_layout(int64_t d, char* base, PrepWs* w)
{
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 1024); return o; };
    const int64_t h = std::max<int64_t>(d / 2, 128);
    size_t oA = take(sizeof(float) * d * d);
    size_t oX = take(sizeof(float) * d * d);
    size_t oY = take(sizeof(float) * d * d);
    size_t oT = take(sizeof(float) * d * h);
    size_t oK = take(sizeof(float) * d);
    size_t oL = take(sizeof(float) * 4);
    if (w && base) {
        w->A = reinterpret_cast<float*>(base + oA);
        w->X = reinterpret_cast<float*>(base + oX);
        w->Y = reinterpret_cast<float*>(base + oY);
        w->T = reinterpret_cast<float*>(base + oT);
        w->keys = reinterpret_cast<float*>(base + oK);
        w->lam = reinterpret_cast<float*>(base + oL);
    }
    return off;
}

__global__ void diag_lambda_kernel(const float* __restrict__ S, int64_t d, int64_t n,
                                   float damp, float* __restrict__ keys, float* __restrict__ lam,
                                   int32_t* __restrict__ info)
{
    __shared__ double red[32];
    double acc = 0.0;
    const double scale = 2.0 / double(n);
    for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
        float s = S[i * d + i];
        keys[i] = s;
        acc += scale * double(s);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
        lam[0] = float(double(damp) * (t / double(d)));
        if (info) *info = 0;
    }
}

// perm[rank(i)] = i with rank = #{j : key_j > key_i or (key_j == key_i and j < i)}
__global__ void rank_perm_kernel(const float* __restrict__ keys, int64_t d, int act_order,
                                 int32_t* __restrict__ perm)
{
    __shared__ float kc[2048];
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (!act_order) {
        if (i < d) perm[i] = (int32_t)i;
        return;
    }
    const float ki = (i < d) ? keys[i] : 0.f;
    int64_t rank = 0;
    for (int64_t c0 = 0; c0 < d; c0 += 2048) {
        __syncthreads();
        for (int t = threadIdx.x; t < 2048; t += blockDim.x)
            kc[t] = (c0 + t < d) ? keys[c0 + t] : 0.f;
        __syncthreads();
        const int64_t lim = (d - c0 < 2048) ? (d - c0) : 2048;
        for (int t = 0; t < lim; ++t) {
            float kj = kc[t];
            int64_t j = c0 + t;
            rank += (kj > ki) || (kj == ki && j < i);
        }
    }
    if (i < d) perm[rank] = (int32_t)i;
}

__global__ void build_reversed_kernel(const float* __restrict__ S, const int32_t* __restrict__ perm,
                                      const float* __restrict__ lam, int64_t d, float scale,
                                      float* __restrict__ A)
{
    const int64_t i = blockIdx.y;
    const int64_t a = d - 1 - i;
    const int32_t pa = perm[a];
    const float l = lam[0];
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < d;
         j += int64_t(gridDim.x) * blockDim.x) {
        const int64_t b = d - 1 - j;
        const int32_t pb = perm[b];
        const int64_t r = min(pa, pb), c = max(pa, pb);
        float v = scale * S[r * d + c];
        if (a == b) v += l;
        A[i * d + j] = v;
    }
}

// Leaf: factor the 128x128 diagonal block at (k0, k0) of A and invert it
// (L_kk into A, X_kk = L_kk^-1 into X, X_kk^T into Y), one CTA of 8 warps,
// every thread busy at every step:
//   * 4 columns per step: every thread factors and inverts the 4x4 diagonal
//     block itself (10 shared-memory reads, no broadcast), one thread per row
//     solves the 4 panel entries of its row, then a rank-4 update of the
//     trailing lower triangle in 4x4 tiles -- two barriers per 4 columns;
//   * X is assembled from the 4x4 diagonal inverses by five doubling levels,
//     X_BC = -X_C (B X_A), as small GEMMs in shared memory.
constexpr int LDA = PN + 4;                  // row stride of the shared 128x128 blocks
constexpr int LDT = 68;                      // row stride of the doubling temporary
constexpr int LTHREADS = 256;
constexpr size_t LSMEM = sizeof(float) * (2 * PN * LDA + 64 * LDT);

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

__global__ void __launch_bounds__(LTHREADS, 1)
leaf_potrf_inv_kernel(float* __restrict__ A, float* __restrict__ X, float* __restrict__ Y,
                      int64_t d, int64_t k0, int32_t* __restrict__ info)
{
    extern __shared__ __align__(16) float lsm[];
    float* a = lsm;                    // 128 x LDA: the block, then L (lower)
    float* xs = a + PN * LDA;          // 128 x LDA: X = L^-1 (lower)
    float* tb = xs + PN * LDA;         // 64 x LDT temporary
    const int tid = threadIdx.x;

    for (int idx = tid * 4; idx < PN * PN; idx += LTHREADS * 4) {
        const int r = idx / PN, c = idx % PN;
        *reinterpret_cast<float4*>(a + r * LDA + c) =
            *reinterpret_cast<const float4*>(A + (k0 + r) * d + k0 + c);
        *reinterpret_cast<float4*>(xs + r * LDA + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();

    for (int c0 = 0; c0 < PN; c0 += 4) {
        // 4x4 diagonal block: Cholesky factor g and its inverse h, in registers
        float g[4][4], h[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) g[i][j] = (j <= i) ? a[(c0 + i) * LDA + c0 + j] : 0.f;
        float rd[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float djj = g[j][j];
            const bool bad = !(djj > 0.f);
            if (bad && tid == 0 && info)
                atomicCAS(reinterpret_cast<int*>(info), 0, (int)(d - (k0 + c0 + j)));
            // 1/sqrt(d) from the hardware estimate plus one Newton step (~1 ulp)
            float y = rsqrtf(djj);
            y = y * fmaf(-0.5f * djj * y, y, 1.5f);
            if (bad) y = __int_as_float(0x7fc00000);
            rd[j] = y;
            g[j][j] = djj * y;
#pragma unroll
            for (int i = j + 1; i < 4; ++i) g[i][j] *= rd[j];
#pragma unroll
            for (int i = j + 1; i < 4; ++i)
#pragma unroll
                for (int k = j + 1; k <= i; ++k) g[i][k] = fmaf(-g[i][j], g[k][j], g[i][k]);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {                 // forward substitution, column c
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                if (r < c) { h[r][c] = 0.f; continue; }
                float t = (r == c) ? 1.f : 0.f;
#pragma unroll
                for (int k = c; k < r; ++k) t = fmaf(-g[r][k], h[k][c], t);
                h[r][c] = t * rd[r];
            }
        }
        // panel rows below: L[r][c0..c0+3] = A[r][c0..c0+3] h^T, one row per thread
        const int rows = PN - c0 - 4;
        if (tid < rows) {
            const int r = c0 + 4 + tid;
            const float4 v = *reinterpret_cast<const float4*>(a + r * LDA + c0);
            const float av[4] = {v.x, v.y, v.z, v.w};
            float o[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float t = 0.f;
#pragma unroll
                for (int k = 0; k <= c; ++k) t = fmaf(av[k], h[c][k], t);
                o[c] = t;
            }
            *reinterpret_cast<float4*>(a + r * LDA + c0) = make_float4(o[0], o[1], o[2], o[3]);
        }
        if (tid == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                *reinterpret_cast<float4*>(a + (c0 + i) * LDA + c0) =
                    make_float4(g[i][0], g[i][1], g[i][2], g[i][3]);
                *reinterpret_cast<float4*>(xs + (c0 + i) * LDA + c0) =
                    make_float4(h[i][0], h[i][1], h[i][2], h[i][3]);
            }
        }
        __syncthreads();
        // rank-4 update of the trailing lower triangle [c0+4, 128)
        const int nt = rows / 4, tiles = nt * (nt + 1) / 2;
        for (int t = tid; t < tiles; t += LTHREADS) {
            int ti, tj;
            tri_index(t, ti, tj);
            const int r0 = c0 + 4 + 4 * ti, q0 = c0 + 4 + 4 * tj;
            float4 lr[4], lc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                lr[i] = *reinterpret_cast<const float4*>(a + (r0 + i) * LDA + c0);
                lc[i] = *reinterpret_cast<const float4*>(a + (q0 + i) * LDA + c0);
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
                *reinterpret_cast<float4*>(a + (r0 + i) * LDA + q0) =
                    make_float4(cv[0], cv[1], cv[2], cv[3]);
            }
        }
        __syncthreads();
    }

    // X from the 4x4 diagonal inverses by doubling: s = 4, 8, ..., 64
    for (int s = 4; s < PN; s *= 2) {
        const int pairs = PN / (2 * s);
        const int ts = s / 4, tpp = ts * ts;               // 4x4 tiles per pair
        // T = B X_A, B = L[o+s+i][o+k], X_A = X[o+k][o+j] (zero for k < j)
        for (int t = tid; t < pairs * tpp; t += LTHREADS) {
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
        for (int t = tid; t < pairs * tpp; t += LTHREADS) {
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

    // write L (lower, zeros above within the block), X and Y = X^T
    for (int idx = tid * 4; idx < PN * PN; idx += LTHREADS * 4) {
        const int r = idx / PN, c = idx % PN;
        float4 lv = *reinterpret_cast<const float4*>(a + r * LDA + c);
        if (c + 0 > r) lv.x = 0.f;
        if (c + 1 > r) lv.y = 0.f;
        if (c + 2 > r) lv.z = 0.f;
        if (c + 3 > r) lv.w = 0.f;
        *reinterpret_cast<float4*>(A + (k0 + r) * d + k0 + c) = lv;
        *reinterpret_cast<float4*>(X + (k0 + r) * d + k0 + c) =
            *reinterpret_cast<const float4*>(xs + r * LDA + c);
        // Y row r holds column r of X: X[c..c+3][r]
        *reinterpret_cast<float4*>(Y + (k0 + r) * d + k0 + c) =
            make_float4(xs[(c + 0) * LDA + r], xs[(c + 1) * LDA + r], xs[(c + 2) * LDA + r],
                        xs[(c + 3) * LDA + r]);
    }
}

// Y[o : o+s, o+s : o+s+c] = X[o+s : o+s+c, o : o+s]^T for every node
// o = o0 + 2 s b (grid.x = s/32 column tiles of X_BC, grid.y = c/32 row tiles).
__global__ void __launch_bounds__(256)
transpose_nodes_kernel(const float* __restrict__ X, float* __restrict__ Y, int64_t d, int64_t s,
                       int64_t o0)
{
    __shared__ float t[32][33];
    const int64_t o = o0 + 2 * s * blockIdx.z;
    const int64_t r0 = int64_t(blockIdx.y) * 32, c0 = int64_t(blockIdx.x) * 32;   // within X_BC
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
#pragma unroll
    for (int k = 0; k < 32; k += 8) t[ty + k][tx] = X[(o + s + r0 + ty + k) * d + o + c0 + tx];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 32; k += 8) Y[(o + c0 + ty + k) * d + o + s + r0 + tx] = t[tx][ty + k];
}

__global__ void write_u_kernel(const float* __restrict__ X, int64_t d, float* __restrict__ U)
{
    const int64_t i = blockIdx.y;
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < d;
         j += int64_t(gridDim.x) * blockDim.x)
        U[i * d + j] = (j >= i) ? X[(d - 1 - i) * d + (d - 1 - j)] : 0.f;
}

}  // namespace gptq

extern "C" size_t gptq_prepare_workspace_bytes(int64_t d)
{
    if (d <= 0) return 0;
    return gptq::prep_layout(d, nullptr, nullptr);
}

extern "C" int gptq_prepare_hinv(const float* S, int64_t d, int64_t n_tokens, float damp_rel,
                                 int act_order, int32_t* perm, float* U, int32_t* info,
                                 void* ws, size_t ws_bytes, void* stream)
{
    using namespace gptq;
    if (!S || !U || !info || !ws) return GPTQ_ERR_INVALID_ARG;
    if (act_order && !perm) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || !aligned16(U) || !aligned16(ws) || (perm && !aligned16(perm)))
        return GPTQ_ERR_INVALID_ARG;
    if (!(damp_rel >= 0.f)) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0) return GPTQ_ERR_SHAPE;
    if (n_tokens <= 0) return GPTQ_ERR_SHAPE;
    if (ws_bytes < gptq_prepare_workspace_bytes(d)) return GPTQ_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    PrepWs w;
    prep_layout(d, reinterpret_cast<char*>(ws), &w);
    int32_t* p = perm ? perm : reinterpret_cast<int32_t*>(w.T);  // identity scratch
    diag_lambda_kernel<<<1, 1024, 0, st>>>(S, d, n_tokens, damp_rel, w.keys, w.lam, info);
    count_launches();
    rank_perm_kernel<<<(unsigned)ceil_div(d, 256), 256, 0, st>>>(w.keys, d, act_order, p);
    count_launches();
    {
        dim3 grid((unsigned)std::min<int64_t>(ceil_div(d, 256), 16), (unsigned)d);
        build_reversed_kernel<<<grid, 256, 0, st>>>(S, p, w.lam, d, 2.0f / float(n_tokens), w.A);
        count_launches();
    }
    if (cudaMemsetAsync(w.X, 0, sizeof(float) * d * d, st) != cudaSuccess ||
        cudaMemsetAsync(w.Y, 0, sizeof(float) * d * d, st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
    if (cudaFuncSetAttribute(leaf_potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)LSMEM) != cudaSuccess)
        return GPTQ_ERR_CUDA;

    const NtBuffer bufA{w.A, d, d, d}, bufX{w.X, d, d, d}, bufY{w.Y, d, d, d};
    const int64_t h = std::max<int64_t>(d / 2, 128);
    const NtBuffer bufT{w.T, d, h, h};
    const int64_t nblk = d / PN;
    for (int64_t k = 0; k < nblk; ++k) {
        const int64_t k0 = k * PN;
        leaf_potrf_inv_kernel<<<1, LTHREADS, LSMEM, st>>>(w.A, w.X, w.Y, d, k0, info);
        count_launches();
        const int64_t R = d - k0 - PN;
        if (R <= 0) continue;
        NtGemm t{};                               // TRSM: A21 <- A21 X_kk^T
        t.A = bufA; t.a_row0 = k0 + PN; t.a_col0 = k0;
        t.B = bufX; t.b_row0 = k0; t.b_col0 = k0;
        t.C = w.A; t.ldc = d; t.c_row0 = k0 + PN; t.c_col0 = k0;
        t.M = R; t.N = PN; t.K = PN; t.batch = 1; t.alpha = 1.f; t.beta = 0.f;
        if (gemm_nt_tf32x3(t, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
        NtGemm s{};                               // SYRK: A22 -= L21 L21^T (lower tiles)
        s.A = bufA; s.a_row0 = k0 + PN; s.a_col0 = k0;
        s.B = bufA; s.b_row0 = k0 + PN; s.b_col0 = k0;
        s.C = w.A; s.ldc = d; s.c_row0 = k0 + PN; s.c_col0 = k0 + PN;
        s.M = R; s.N = R; s.K = PN; s.batch = 1; s.alpha = -1.f; s.beta = 1.f; s.lower = 1;
        if (gemm_nt_tf32x3(s, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
    }
    // X = L^-1 by recursive doubling over block pairs.  Level sz merges the
    // inverted blocks [o, o+sz) and [o+sz, o+sz+c) for o = 2 sz b; when d/128 is
    // not a power of two the last pair has a shorter second block (c < sz).
    auto merge = [&](int64_t o0, int64_t sz, int64_t c, int nodes) -> int {
        NtGemm g1{};                              // T^T_b (sz x c) = Y_A B^T
        g1.A = bufY; g1.a_row0 = o0; g1.a_col0 = o0; g1.a_row_step = 2 * sz; g1.a_col_step = 2 * sz;
        g1.B = bufA; g1.b_row0 = o0 + sz; g1.b_col0 = o0; g1.b_row_step = 2 * sz;
        g1.b_col_step = 2 * sz;
        g1.C = w.T; g1.ldc = h; g1.c_row0 = 0; g1.c_col0 = 0; g1.c_row_step = sz; g1.c_col_step = 0;
        g1.M = sz; g1.N = c; g1.K = sz; g1.batch = nodes; g1.alpha = 1.f; g1.beta = 0.f;
        if (gemm_nt_tf32x3(g1, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
        NtGemm g2{};                              // X_BC (c x sz) = -X_C T, T = (T^T)^T
        g2.A = bufX; g2.a_row0 = o0 + sz; g2.a_col0 = o0 + sz; g2.a_row_step = 2 * sz;
        g2.a_col_step = 2 * sz;
        g2.B = bufT; g2.b_row0 = 0; g2.b_col0 = 0; g2.b_row_step = sz; g2.b_col_step = 0;
        g2.C = w.X; g2.ldc = d; g2.c_row0 = o0 + sz; g2.c_col0 = o0; g2.c_row_step = 2 * sz;
        g2.c_col_step = 2 * sz;
        g2.M = c; g2.N = sz; g2.K = c; g2.batch = nodes; g2.alpha = -1.f; g2.beta = 0.f;
        if (gemm_nt_tf32x3(g2, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
        if (!(o0 == 0 && nodes == 1 && sz + c == d)) {   // Y is read by later levels only
            dim3 grid((unsigned)(sz / 32), (unsigned)(c / 32), (unsigned)nodes);
            transpose_nodes_kernel<<<grid, 256, 0, st>>>(w.X, w.Y, d, sz, o0);
            count_launches();
        }
        return GPTQ_OK;
    };
    for (int64_t sz = PN; sz < d; sz *= 2) {
        const int full = (int)(d / (2 * sz));
        if (full > 0 && merge(0, sz, sz, full) != GPTQ_OK) return GPTQ_ERR_CUDA;
        const int64_t o = int64_t(full) * 2 * sz;
        if (o + sz < d && merge(o, sz, d - o - sz, 1) != GPTQ_OK) return GPTQ_ERR_CUDA;
    }
    {
        dim3 grid((unsigned)std::min<int64_t>(ceil_div(d, 256), 16), (unsigned)d);
        write_u_kernel<<<grid, 256, 0, st>>>(w.X, d, U);
        count_launches();
    }
    return launch_status();
}

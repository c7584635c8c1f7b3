// Inverse-Hessian preparation -- "GPTQ / AWQ / SqueezeLLM" sec. 一
// (H = 2 X^T X / n, damping, importance order, decomposition of H^-1).
//
// U = upper Cholesky factor of Hd^-1 is taken by the reverse-order route:
// with J the exchange matrix, A = J Hd J = L L^T (lower Cholesky), and
// U = J L^-1 J is upper with U^T U = Hd^-1 (uniqueness of the Cholesky
// factor).  One factorization and one triangular inverse instead of
// factor / invert / factor.
//
// Steps (all on the device):
//   1. keys + lambda: diag(S), lambda = damp * mean(2 S_ii / n)
//   2. perm: stable descending rank of S_ii (act-order) or identity
//   3. A[i][j] = Hd[d-1-i][d-1-j], Hd = (2/n) S[perm][:, perm] + lambda I
//   4. blocked right-looking Cholesky of A (64-wide panels): panel factor and
//      its inverse in one CTA, TRSM and trailing SYRK as fp32 GEMMs
//   5. blocked triangular inverse X = L^-1 by block rows
//   6. U[i][j] = X[d-1-i][d-1-j] (upper), 0 below the diagonal
#include "common.cuh"
#include "simt_gemm.cuh"

namespace gptq {

constexpr int PN = 64;   // panel width

struct PrepWs {
    float* A;      // d x d working matrix, then L in its lower triangle
    float* X;      // d x d, L^-1
    float* T;      // PN x d temporary
    float* keys;   // d
    float* lam;    // 1
};

static size_t prep_layout(int64_t d, char* base, PrepWs* w)
{
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 256); return o; };
    size_t oA = take(sizeof(float) * d * d);
    size_t oX = take(sizeof(float) * d * d);
    size_t oT = take(sizeof(float) * PN * d);
    size_t oK = take(sizeof(float) * d);
    size_t oL = take(sizeof(float) * 4);
    if (w && base) {
        w->A = reinterpret_cast<float*>(base + oA);
        w->X = reinterpret_cast<float*>(base + oX);
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

// Factor the PN x PN diagonal block k of A (lower), record the first
// non-positive pivot, write L_kk back to A and L_kk^-1 into X's diagonal block.
__global__ void __launch_bounds__(256)
potrf_panel_kernel(float* __restrict__ A, float* __restrict__ X, int64_t d, int64_t k0,
                   int32_t* __restrict__ info)
{
    __shared__ float a[PN][PN + 1];
    __shared__ float x[PN][PN + 1];
    const int tid = threadIdx.x;
    for (int idx = tid; idx < PN * PN; idx += blockDim.x) {
        int r = idx / PN, c = idx % PN;
        a[r][c] = (c <= r) ? A[(k0 + r) * d + k0 + c] : 0.f;
    }
    for (int j = 0; j < PN; ++j) {
        __syncthreads();
        const float piv = a[j][j];
        const bool bad = !(piv > 0.f);
        const float sq = bad ? __int_as_float(0x7fc00000) : sqrtf(piv);
        if (tid == 0 && bad && info)
            atomicCAS(reinterpret_cast<int*>(info), 0, (int)(d - (k0 + j)));
        __syncthreads();
        if (tid == 0) a[j][j] = sq;
        for (int r = j + 1 + tid; r < PN; r += blockDim.x) a[r][j] = a[r][j] / sq;
        __syncthreads();
        const int cnt = PN - 1 - j;
        for (int idx = tid; idx < cnt * cnt; idx += blockDim.x) {
            int r = j + 1 + idx / cnt, c = j + 1 + idx % cnt;
            if (c <= r) a[r][c] = fmaf(-a[r][j], a[c][j], a[r][c]);
        }
    }
    __syncthreads();
    // inverse of the lower-triangular block, one column per thread
    if (tid < PN) {
        const int c = tid;
        for (int r = 0; r < PN; ++r) x[r][c] = 0.f;
        x[c][c] = 1.f / a[c][c];
        for (int r = c + 1; r < PN; ++r) {
            float t = 0.f;
            for (int k = c; k < r; ++k) t = fmaf(a[r][k], x[k][c], t);
            x[r][c] = -t / a[r][r];
        }
    }
    __syncthreads();
    for (int idx = tid; idx < PN * PN; idx += blockDim.x) {
        int r = idx / PN, c = idx % PN;
        if (c <= r) A[(k0 + r) * d + k0 + c] = a[r][c];
        X[(k0 + r) * d + k0 + c] = x[r][c];
    }
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
    if (cudaMemsetAsync(w.X, 0, sizeof(float) * d * d, st) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (launch_status() != GPTQ_OK) return GPTQ_ERR_CUDA;
    const int64_t nblk = d / PN;
    for (int64_t k = 0; k < nblk; ++k) {
        const int64_t k0 = k * PN;
        potrf_panel_kernel<<<1, 256, 0, st>>>(w.A, w.X, d, k0, info);
        count_launches();
        const int64_t R = d - k0 - PN;
        if (R > 0) {
            GemmArgs t{};
            t.A = w.A + (k0 + PN) * d + k0; t.lda = d;
            t.B = w.X + k0 * d + k0; t.ldb = d; t.b_trans = 1;
            t.C = w.A + (k0 + PN) * d + k0; t.ldc = d;
            t.M = R; t.N = PN; t.K = PN; t.alpha = 1.f; t.beta = 0.f;
            if (simt_gemm(t, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
            GemmArgs s{};
            s.A = w.A + (k0 + PN) * d + k0; s.lda = d;
            s.B = w.A + (k0 + PN) * d + k0; s.ldb = d; s.b_trans = 1;
            s.C = w.A + (k0 + PN) * d + (k0 + PN); s.ldc = d;
            s.M = R; s.N = R; s.K = PN; s.alpha = -1.f; s.beta = 1.f; s.lower_tiles = 1;
            if (simt_gemm(s, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
        }
    }
    for (int64_t i = 1; i < nblk; ++i) {
        const int64_t i0 = i * PN;
        GemmArgs t{};
        t.A = w.A + i0 * d; t.lda = d;          // L[i-block, 0:i0]
        t.B = w.X; t.ldb = d; t.b_lower = 1;    // X[0:i0, 0:i0]
        t.C = w.T; t.ldc = d;
        t.M = PN; t.N = i0; t.K = i0; t.alpha = 1.f; t.beta = 0.f;
        if (simt_gemm(t, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
        GemmArgs x{};
        x.A = w.X + i0 * d + i0; x.lda = d;     // L_ii^-1
        x.B = w.T; x.ldb = d;
        x.C = w.X + i0 * d; x.ldc = d;
        x.M = PN; x.N = i0; x.K = PN; x.alpha = -1.f; x.beta = 0.f;
        if (simt_gemm(x, st) != GPTQ_OK) return GPTQ_ERR_CUDA;
    }
    {
        dim3 grid((unsigned)std::min<int64_t>(ceil_div(d, 256), 16), (unsigned)d);
        write_u_kernel<<<grid, 256, 0, st>>>(w.X, d, U);
        count_launches();
    }
    return launch_status();
}

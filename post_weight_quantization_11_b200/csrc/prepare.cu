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
//   3. A[i][j] = Hd[d-1-i][d-1-j], Hd = (2/n) S[perm][:, perm] + lambda I,
//      for the lower 128x128 tiles (the only ones the factorization reads)
//   4. L (A = L L^T) and X = L^-1 by 128x128 tiles in one dependency-driven
//      persistent kernel (chol_dag.cu): a one-CTA leaf factors and inverts
//      each diagonal tile, the off-diagonal tiles of L and X are split-TF32
//      tensor-core products; U is written by the same kernel as
//      U[i][j] = X[d-1-i][d-1-j] (upper), 0 below the diagonal
#include "common.cuh"
#include "chol_dag.cuh"

namespace gptq {

constexpr int TW = 128;            // tile width of the factorization

struct PrepWs {
    float* A;      // d x d reversed damped H (lower tiles), then L
    float* Y;      // d x d, (L^-1)^T in the upper tiles
    float* Xc;     // 2 d x 128, the diagonal tiles of L^-1 (TF32 heads, then remainders)
    void* sync;    // dependency flags of the factorization
    float* keys;   // d
    float* lam;    // 1
    int32_t* pid;  // d, identity permutation when the caller passes none
};

// Workspace of a batch of E matrices (E = 1: one layer); matrix e's parts at
// e d^2 (A, Y), e d 128 (each of Xc's two planes), e d (keys, pid) and 4 e
// (lam).
static size_t prep_layout(int64_t d, int64_t E, char* base, PrepWs* w)
{
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 1024); return o; };
    size_t oA = take(sizeof(float) * d * d * E);
    size_t oY = take(sizeof(float) * d * d * E);
    size_t oX = take(sizeof(float) * d * TW * E * 2);
    size_t oS = take(chol_dag_sync_bytes(d, E));
    size_t oK = take(sizeof(float) * d * E);
    size_t oL = take(sizeof(float) * 4 * E);
    size_t oP = take(sizeof(int32_t) * d * E);
    if (w && base) {
        w->A = reinterpret_cast<float*>(base + oA);
        w->Y = reinterpret_cast<float*>(base + oY);
        w->Xc = reinterpret_cast<float*>(base + oX);
        w->sync = base + oS;
        w->keys = reinterpret_cast<float*>(base + oK);
        w->lam = reinterpret_cast<float*>(base + oL);
        w->pid = reinterpret_cast<int32_t*>(base + oP);
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

// A[i][j] = Hd[d-1-i][d-1-j] for the lower tiles only (j < 128 (i/128 + 1)):
// the factorization reads nothing else.  Inside a diagonal tile the entries
// above the diagonal are set to 0.  For j <= i (b >= a) the source is S's
// upper triangle read along row a (coalesced for the identity permutation).
__global__ void build_reversed_kernel(const float* __restrict__ S, const int32_t* __restrict__ perm,
                                      const float* __restrict__ lam, int64_t d, float scale,
                                      float* __restrict__ A)
{
    const int64_t i = blockIdx.y;
    const int64_t a = d - 1 - i;
    const int32_t pa = perm[a];
    const float l = lam[0];
    const int64_t jend = (i / 128 + 1) * 128;
    for (int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; j < jend;
         j += int64_t(gridDim.x) * blockDim.x) {
        float v = 0.f;
        if (j <= i) {
            const int64_t b = d - 1 - j;
            const int32_t pb = perm[b];
            const int64_t r = min(pa, pb), c = max(pa, pb);
            v = scale * S[r * d + c];
            if (a == b) v += l;
        }
        A[i * d + j] = v;
    }
}

// Argument checks shared by every preparation entry point (before any launch).
int prepare_check_args(const float* S, int64_t d, float damp_rel, int act_order,
                       const int32_t* perm, const float* U, const int32_t* info)
{
    if (!S || !U || !info) return GPTQ_ERR_INVALID_ARG;
    if (act_order && !perm) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || !aligned16(U) || (perm && !aligned16(perm)))
        return GPTQ_ERR_INVALID_ARG;
    if (!(damp_rel >= 0.f)) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0) return GPTQ_ERR_SHAPE;
    return GPTQ_OK;
}

// The finalize steps of matrix e: lambda, perm, the reversed damped Hessian.
static int prepare_finalize(const float* S, int64_t d, int64_t n_tokens, float damp_rel,
                            int act_order, int32_t* perm, int32_t* info, const PrepWs& w,
                            int64_t e, cudaStream_t st)
{
    const float* Se = S + e * d * d;
    float* keys = w.keys + e * d;
    float* lam = w.lam + 4 * e;
    int32_t* p = perm ? perm + e * d : w.pid + e * d;
    KernelTimer kt(kKFinalize, st);
    diag_lambda_kernel<<<1, 1024, 0, st>>>(Se, d, n_tokens, damp_rel, keys, lam, info + e);
    count_launches();
    rank_perm_kernel<<<(unsigned)ceil_div(d, 256), 256, 0, st>>>(keys, d, act_order, p);
    count_launches();
    // one CTA per row: rows hold 128 .. d entries of the lower tiles
    build_reversed_kernel<<<dim3(1, (unsigned)d), 256, 0, st>>>(Se, p, lam, d,
                                                                2.0f / float(n_tokens),
                                                                w.A + e * d * d);
    count_launches();
    return launch_status();
}

}  // namespace gptq

extern "C" size_t gptq_prepare_workspace_bytes(int64_t d)
{
    if (d <= 0) return 0;
    return gptq::prep_layout(d, 1, nullptr, nullptr);
}

extern "C" size_t gptq_prepare_batched_workspace_bytes(int64_t d, int64_t n_mats)
{
    if (d <= 0 || n_mats <= 0) return 0;
    return gptq::prep_layout(d, n_mats, nullptr, nullptr);
}

extern "C" int gptq_prepare_hinv(const float* S, int64_t d, int64_t n_tokens, float damp_rel,
                                 int act_order, int32_t* perm, float* U, int32_t* info,
                                 void* ws, size_t ws_bytes, void* stream)
{
    using namespace gptq;
    int rc = prepare_check_args(S, d, damp_rel, act_order, perm, U, info);
    if (rc != GPTQ_OK) return rc;
    if (!ws || !aligned16(ws)) return GPTQ_ERR_INVALID_ARG;
    if (n_tokens <= 0) return GPTQ_ERR_SHAPE;
    if (ws_bytes < gptq_prepare_workspace_bytes(d)) return GPTQ_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    PrepWs w;
    prep_layout(d, 1, reinterpret_cast<char*>(ws), &w);
    rc = prepare_finalize(S, d, n_tokens, damp_rel, act_order, perm, info, w, 0, st);
    if (rc != GPTQ_OK) return rc;
    {
        KernelTimer kt(kKFactor, st);
        if (chol_inv_dag(w.A, w.Xc, w.Y, U, w.sync, d, 1, info, st) != GPTQ_OK)
            return GPTQ_ERR_CUDA;
    }
    return launch_status();
}

extern "C" int gptq_prepare_hinv_batched(const float* S, int64_t n_mats, int64_t d,
                                         const int64_t* n_tokens, float damp_rel, int act_order,
                                         int32_t* perm, float* U, int32_t* info, void* ws,
                                         size_t ws_bytes, void* stream)
{
    using namespace gptq;
    int rc = prepare_check_args(S, d, damp_rel, act_order, perm, U, info);
    if (rc != GPTQ_OK) return rc;
    if (!n_tokens || !ws || !aligned16(ws)) return GPTQ_ERR_INVALID_ARG;
    if (n_mats < 1 || n_mats > 4096 || 2 * n_mats * d > (int64_t(1) << 31) - 1)
        return GPTQ_ERR_SHAPE;
    for (int64_t e = 0; e < n_mats; ++e)
        if (n_tokens[e] <= 0) return GPTQ_ERR_SHAPE;
    if (ws_bytes < gptq_prepare_batched_workspace_bytes(d, n_mats)) return GPTQ_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    PrepWs w;
    prep_layout(d, n_mats, reinterpret_cast<char*>(ws), &w);
    for (int64_t e = 0; e < n_mats; ++e) {
        rc = prepare_finalize(S, d, n_tokens[e], damp_rel, act_order, perm, info, w, e, st);
        if (rc != GPTQ_OK) return rc;
    }
    {
        KernelTimer kt(kKFactor, st);
        if (chol_inv_dag(w.A, w.Xc, w.Y, U, w.sync, d, n_mats, info, st) != GPTQ_OK)
            return GPTQ_ERR_CUDA;
    }
    return launch_status();
}

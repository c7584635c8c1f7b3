// Activation-aware channel scaling ahead of GPTQ -- "GPTQ / AWQ /
// SqueezeLLM" sec. 二 (scale each input channel's weights by its activation
// magnitude before quantizing, divide back afterwards, and choose among
// candidate scalings the one with the smallest output error; then GPTQ) and
// "INT4/INT8 量化推理" sec. 四 (the transform is exact before quantization).
//
//   a_j     = mean_t |X[t][j]|  (channel_abs_sum accumulates the sum in fp64)
//   s(α)_j  = (a'_j / mean a')^α, a' = a with zeros raised to the smallest
//             positive magnitude, α = k / n_grid, k = 0 .. n_grid - 1
//   W'      = W diag(s);  Q' = group round-to-nearest of W' (no feedback)
//   D       = Q' diag(s)^-1 - W;  loss(α) = tr(D H D^T), H = 2 S / n
//   α*      = the first minimizer; outputs s(α*), W diag(s), S' =
//             diag(s)^-1 S diag(s)^-1 for the GPTQ that follows.
//
// Precision: the scales and W s are formed in fp64 and W' rounded once to
// fp32, so the round-to-nearest decisions see the same fp32 values a float64
// reference computing W s would round; D is formed in fp64 and rounded to
// fp32 for the product D H, taken on the tensor cores in split-TF32 (the
// library's NT GEMM, fp32-level accuracy); the row dot products D . (D H)
// are summed in fp64.
#include "common.cuh"
#include "gemm_nt.cuh"
#include "quant_common.cuh"

namespace gptq {

constexpr int AW_THREADS = 256;

// acc[j] += sum_t |X[t][j]| in fp64.  Thread = 8 consecutive columns (one
// 16-byte vector) over a strided range of tokens; one fp64 atomic per
// column and thread at the end.
__global__ void __launch_bounds__(AW_THREADS)
channel_abs_sum_kernel(const uint4* __restrict__ X, int64_t n, int64_t vpr,
                       double* __restrict__ acc)
{
    const int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (v >= vpr) return;
    double s[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int64_t t = blockIdx.y; t < n; t += gridDim.y) {
        const uint4 q = X[t * vpr + v];
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const __half2 p = *reinterpret_cast<const __half2*>(&w[h]);
            const float2 f = __half22float2(p);
            s[2 * h] += double(fabsf(f.x));
            s[2 * h + 1] += double(fabsf(f.y));
        }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) atomicAdd(acc + 8 * v + c, s[c]);
}

// r_j = a'_j / mean(a') from the sums (a_j = acc_j / n; zeros raised to the
// smallest positive magnitude, or every a' = 1 when all are zero).  One CTA.
__global__ void __launch_bounds__(1024)
awq_ratio_kernel(const double* __restrict__ acc, int64_t d, int64_t n, double* __restrict__ r)
{
    __shared__ double red[32];
    __shared__ double bc;
    const int tid = threadIdx.x;
    double mn = 1e308;
    for (int64_t j = tid; j < d; j += blockDim.x) {
        const double a = acc[j] / double(n);
        if (a > 0.0) mn = fmin(mn, a);
    }
    for (int o = 16; o > 0; o >>= 1) mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    if ((tid & 31) == 0) red[tid >> 5] = mn;
    __syncthreads();
    if (tid == 0) {
        double m = 1e308;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmin(m, red[w]);
        bc = (m < 1e308) ? m : -1.0;                 // -1: no positive magnitude at all
    }
    __syncthreads();
    const double floor_a = bc;
    double sum = 0.0;
    for (int64_t j = tid; j < d; j += blockDim.x) {
        const double a = acc[j] / double(n);
        const double ap = floor_a < 0.0 ? 1.0 : (a > 0.0 ? a : floor_a);
        r[j] = ap;
        sum += ap;
    }
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    __syncthreads();
    if ((tid & 31) == 0) red[tid >> 5] = sum;
    __syncthreads();
    if (tid == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
        bc = t / double(d);
    }
    __syncthreads();
    const double mean = bc;
    for (int64_t j = tid; j < d; j += blockDim.x) r[j] = r[j] / mean;
}

// s_j = r_j^alpha (alpha = k / n_grid; alpha = 0 gives exactly 1)
__global__ void awq_scales_kernel(const double* __restrict__ r, int64_t d, int k, int n_grid,
                                  double* __restrict__ s)
{
    const int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= d) return;
    const double alpha = double(k) / double(n_grid);
    s[j] = (k == 0) ? 1.0 : pow(r[j], alpha);
}

// One warp per (row, group): W' = fp32(W s), the group's min/max (range
// including 0), its parameters and codes as the quantizer everywhere else,
// and D = fp32(s_g (c - z) / s_j - W) formed in fp64.
template <typename T>
__global__ void __launch_bounds__(AW_THREADS)
awq_rtn_diff_kernel(const T* __restrict__ W, int64_t m, int64_t d, int64_t gsz,
                    const double* __restrict__ s, float maxqf, float* __restrict__ D)
{
    const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t G = d / gsz;
    if (wid >= m * G) return;               // whole warp exits together
    const int64_t row = wid / G, c0 = (wid - row * G) * gsz;
    const T* w = W + row * d + c0;
    float mn = 0.f, mx = 0.f;
    for (int64_t c = lane; c < gsz; c += 32) {
        const float x = float(double(float(w[c])) * s[c0 + c]);
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    const GroupQ gq = group_params(mn, mx, maxqf);
    for (int64_t c = lane; c < gsz; c += 32) {
        const double wd = double(float(w[c]));
        const double sj = s[c0 + c];
        const float x = float(wd * sj);
        const float code = quant_code(x, gq, maxqf);
        const double q = double(gq.s) * double(code - gq.z);      // exact
        D[row * d + c0 + c] = float(q / sj - wd);
    }
}

// loss += sum_{r,j} D[r][j] T[r][j] in fp64 (T = D H); grid-stride, one
// fp64 atomic per warp.
__global__ void __launch_bounds__(AW_THREADS)
rowdot_kernel(const float4* __restrict__ D, const float4* __restrict__ T, int64_t n4,
              double* __restrict__ loss)
{
    double acc = 0.0;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += int64_t(gridDim.x) * blockDim.x) {
        const float4 a = D[i], b = T[i];
        acc += double(a.x) * double(b.x) + double(a.y) * double(b.y) +
               double(a.z) * double(b.z) + double(a.w) * double(b.w);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) atomicAdd(loss, acc);
}

// H = (2 / n) S mirrored from its upper triangle (full matrix, fp32)
__global__ void mirror_scaled_kernel(const float* __restrict__ S, int64_t d, float scale,
                                     float* __restrict__ H)
{
    const int64_t total = d * d;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = i / d, c = i - r * d;
        H[i] = scale * (r <= c ? S[r * d + c] : S[c * d + r]);
    }
}

// best = the first minimizer of the losses; s_out = its scales
__global__ void awq_pick_kernel(const double* __restrict__ losses, int n_grid,
                                int32_t* __restrict__ best)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int b = 0;
    for (int k = 1; k < n_grid; ++k)
        if (losses[k] < losses[b]) b = k;
    *best = b;
}

__global__ void awq_chosen_scales_kernel(const double* __restrict__ r, int64_t d,
                                         const int32_t* __restrict__ best, int n_grid,
                                         double* __restrict__ s)
{
    const int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= d) return;
    const int k = *best;
    s[j] = (k == 0) ? 1.0 : pow(r[j], double(k) / double(n_grid));
}

// W_out = fp32(W s) and S_out = fp32(S_ij / (s_i s_j)) (upper triangle)
template <typename T>
__global__ void awq_apply_w_kernel(const T* __restrict__ W, int64_t m, int64_t d,
                                   const double* __restrict__ s, float* __restrict__ Wo)
{
    const int64_t total = m * d;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x)
        Wo[i] = float(double(float(W[i])) * s[i % d]);
}

__global__ void awq_apply_s_kernel(const float* __restrict__ S, int64_t d,
                                   const double* __restrict__ s, float* __restrict__ So)
{
    const int64_t total = d * d;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t r = i / d, c = i - r * d;
        So[i] = (r <= c) ? float(double(S[i]) / (s[r] * s[c])) : 0.f;
    }
}

struct AwqWs {
    float* H;       // d x d
    float* D;       // m x d
    float* T;       // m x d
    double* r;      // d
    double* s;      // d
};

static size_t awq_layout(int64_t m, int64_t d, char* base, AwqWs* w)
{
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off = align_up(off + bytes, 1024); return o; };
    size_t oH = take(sizeof(float) * d * d);
    size_t oD = take(sizeof(float) * m * d);
    size_t oT = take(sizeof(float) * m * d);
    size_t oR = take(sizeof(double) * d);
    size_t oS = take(sizeof(double) * d);
    if (w && base) {
        w->H = reinterpret_cast<float*>(base + oH);
        w->D = reinterpret_cast<float*>(base + oD);
        w->T = reinterpret_cast<float*>(base + oT);
        w->r = reinterpret_cast<double*>(base + oR);
        w->s = reinterpret_cast<double*>(base + oS);
    }
    return off;
}

static unsigned aw_grid(int64_t n, int threads)
{
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(n, threads),
                                                            int64_t(device_sm_count()) * 16));
}

}  // namespace gptq

extern "C" int gptq_channel_abs_sum(const uint16_t* X, int64_t n_tokens, int64_t d,
                                    double* abs_sum, void* stream)
{
    using namespace gptq;
    if (!abs_sum || (!X && n_tokens > 0)) return GPTQ_ERR_INVALID_ARG;
    if ((X && !aligned16(X)) || (reinterpret_cast<uintptr_t>(abs_sum) & 7u))
        return GPTQ_ERR_INVALID_ARG;
    if (d < 8 || d % 8 != 0 || d > kMaxDim || n_tokens < 0) return GPTQ_ERR_SHAPE;
    if (n_tokens == 0) return GPTQ_OK;
    const int64_t vpr = d / 8;
    const unsigned gx = (unsigned)ceil_div(vpr, AW_THREADS);
    const unsigned gy = (unsigned)std::max<int64_t>(
        1, std::min<int64_t>(n_tokens, int64_t(device_sm_count()) * 8 / gx));
    cudaStream_t st = as_stream(stream);
    KernelTimer kt(kKAwq, st);
    channel_abs_sum_kernel<<<dim3(gx, gy), AW_THREADS, 0, st>>>(reinterpret_cast<const uint4*>(X),
                                                                n_tokens, vpr, abs_sum);
    count_launches();
    return launch_status();
}

extern "C" size_t gptq_awq_workspace_bytes(int64_t d_out, int64_t d_in)
{
    if (d_out <= 0 || d_in <= 0) return 0;
    return gptq::awq_layout(d_out, d_in, nullptr, nullptr);
}

extern "C" int gptq_awq_search(const void* W, int w_dtype, int64_t d_out, int64_t d_in,
                               const float* S, int64_t n_tokens, const double* abs_sum,
                               int n_grid, int bits, int group_size, double* losses,
                               int32_t* best, double* scales, float* W_scaled, float* S_scaled,
                               void* ws, size_t ws_bytes, void* stream)
{
    using namespace gptq;
    if (!W || !S || !abs_sum || !losses || !best || !scales || !ws) return GPTQ_ERR_INVALID_ARG;
    if (w_dtype != GPTQ_DTYPE_F16 && w_dtype != GPTQ_DTYPE_F32) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(S) || !aligned16(ws) || (W_scaled && !aligned16(W_scaled)) ||
        (S_scaled && !aligned16(S_scaled)) || (reinterpret_cast<uintptr_t>(abs_sum) & 7u) ||
        (reinterpret_cast<uintptr_t>(losses) & 7u) || (reinterpret_cast<uintptr_t>(scales) & 7u) ||
        (reinterpret_cast<uintptr_t>(best) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    if (!(bits == 2 || bits == 3 || bits == 4 || bits == 8)) return GPTQ_ERR_UNSUPPORTED;
    if (d_in < 128 || d_in > kMaxDim || d_in % 128 != 0 || d_out < 1 || d_out > kMaxRows)
        return GPTQ_ERR_SHAPE;
    const int64_t gsz = (group_size == -1) ? d_in : group_size;
    if (gsz < 32 || gsz % 32 != 0 || d_in % gsz != 0) return GPTQ_ERR_UNSUPPORTED;
    if (n_tokens <= 0 || n_grid < 1 || n_grid > 1000) return GPTQ_ERR_SHAPE;
    if (ws_bytes < gptq_awq_workspace_bytes(d_out, d_in)) return GPTQ_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    AwqWs w;
    awq_layout(d_out, d_in, reinterpret_cast<char*>(ws), &w);
    const int64_t m = d_out, d = d_in;
    const float maxqf = float((1 << bits) - 1);
    KernelTimer kt(kKAwq, st);
    if (cudaMemsetAsync(losses, 0, sizeof(double) * size_t(n_grid), st) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    mirror_scaled_kernel<<<aw_grid(d * d, 256), 256, 0, st>>>(S, d, 2.0f / float(n_tokens), w.H);
    awq_ratio_kernel<<<1, 1024, 0, st>>>(abs_sum, d, n_tokens, w.r);
    count_launches(2);
    NtGemm g{};
    g.A = NtBuffer{w.D, m, d, d};
    g.B = NtBuffer{w.H, d, d, d};
    g.C = w.T;
    g.ldc = d;
    g.M = m;
    g.N = d;
    g.K = d;
    g.batch = 1;
    g.alpha = 1.f;
    g.beta = 0.f;
    const int64_t warps = m * (d / gsz);
    for (int k = 0; k < n_grid; ++k) {
        awq_scales_kernel<<<(unsigned)ceil_div(d, 256), 256, 0, st>>>(w.r, d, k, n_grid, w.s);
        if (w_dtype == GPTQ_DTYPE_F16)
            awq_rtn_diff_kernel<__half><<<(unsigned)ceil_div(warps * 32, AW_THREADS), AW_THREADS,
                                          0, st>>>(reinterpret_cast<const __half*>(W), m, d, gsz,
                                                   w.s, maxqf, w.D);
        else
            awq_rtn_diff_kernel<float><<<(unsigned)ceil_div(warps * 32, AW_THREADS), AW_THREADS,
                                         0, st>>>(reinterpret_cast<const float*>(W), m, d, gsz,
                                                  w.s, maxqf, w.D);
        count_launches(2);
        const int rc = gemm_nt_tf32x3(g, st);               // T = D H^T = D H
        if (rc != GPTQ_OK) return rc;
        rowdot_kernel<<<aw_grid(m * d / 4, AW_THREADS), AW_THREADS, 0, st>>>(
            reinterpret_cast<const float4*>(w.D), reinterpret_cast<const float4*>(w.T), m * d / 4,
            losses + k);
        count_launches();
    }
    awq_pick_kernel<<<1, 32, 0, st>>>(losses, n_grid, best);
    awq_chosen_scales_kernel<<<(unsigned)ceil_div(d, 256), 256, 0, st>>>(w.r, d, best, n_grid,
                                                                        scales);
    count_launches(2);
    if (W_scaled) {
        if (w_dtype == GPTQ_DTYPE_F16)
            awq_apply_w_kernel<__half><<<aw_grid(m * d, 256), 256, 0, st>>>(
                reinterpret_cast<const __half*>(W), m, d, scales, W_scaled);
        else
            awq_apply_w_kernel<float><<<aw_grid(m * d, 256), 256, 0, st>>>(
                reinterpret_cast<const float*>(W), m, d, scales, W_scaled);
        count_launches();
    }
    if (S_scaled) {
        awq_apply_s_kernel<<<aw_grid(d * d, 256), 256, 0, st>>>(S, d, scales, S_scaled);
        count_launches();
    }
    return launch_status();
}

// Routed-row gather for the per-expert Hessians of a mixture-of-experts
// layer -- "INT4/INT8 量化推理" sec. 五 (each expert is calibrated on the
// tokens routed to it; cold experts see few of them).
//
//   out[r][:] = X[idx[r]][:]      for 0 <= r < n_idx
//
// The expert-major concatenation of the routed tokens' rows is the input of
// gptq_hessian_accumulate_grouped.  HBM-bound copy: 16-byte vectors, each
// CTA walks whole rows (a row of d fp16 is d / 8 vectors), grid a multiple of
// the SM count.  An index outside [0, n_rows) is not followed: its row is
// written as zeros and the library's device status records 0x201.
#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ X, int64_t n_rows, int64_t vpr,
                   const int32_t* __restrict__ idx, int64_t n_idx, uint4* __restrict__ out)
{
    for (int64_t r = blockIdx.x; r < n_idx; r += gridDim.x) {
        const int64_t src = idx[r];
        uint4* dst = out + r * vpr;
        if (src < 0 || src >= n_rows) {
            for (int64_t v = threadIdx.x; v < vpr; v += blockDim.x) dst[v] = make_uint4(0, 0, 0, 0);
            if (threadIdx.x == 0) atomicCAS(&g_device_status, 0, kErrIndex);
            continue;
        }
        const uint4* s = X + src * vpr;
        for (int64_t v = threadIdx.x; v < vpr; v += blockDim.x) dst[v] = __ldg(s + v);
    }
}

}  // namespace gptq

extern "C" int gptq_gather_rows(const uint16_t* X, int64_t n_rows, int64_t d, const int32_t* idx,
                                int64_t n_idx, uint16_t* out, void* stream)
{
    using namespace gptq;
    if (n_idx < 0 || n_rows < 0) return GPTQ_ERR_SHAPE;
    if (n_idx == 0) return GPTQ_OK;
    if (!X || !idx || !out) return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(out) || (reinterpret_cast<uintptr_t>(idx) & 3u))
        return GPTQ_ERR_INVALID_ARG;
    if (d < 8 || d % 8 != 0 || d > kMaxDim) return GPTQ_ERR_SHAPE;
    const unsigned grid = (unsigned)std::min<int64_t>(n_idx, int64_t(device_sm_count()) * 16);
    KernelTimer kt(kKGather, as_stream(stream));
    gather_rows_kernel<<<grid, 256, 0, as_stream(stream)>>>(
        reinterpret_cast<const uint4*>(X), n_rows, d / 8, idx, n_idx, reinterpret_cast<uint4*>(out));
    count_launches();
    return launch_status();
}

// Hessian accumulation with the calibration batch streamed from host memory:
// a two-slot device ring, copies on one stream, tensor-core accumulation
// (gptq_hessian_accumulate) on the other, ordered by two events.
#include "common.cuh"

extern "C" int gptq_hessian_accumulate_host(float* S, const uint16_t* X_host, int64_t n_tokens,
                                            int64_t d, int64_t* n_seen, uint16_t* stage,
                                            size_t stage_bytes, int64_t chunk_tokens,
                                            void* stream, void* copy_stream, void* ev_filled,
                                            void* ev_freed)
{
    using namespace gptq;
    if (!S || !stage || !ev_filled || !ev_freed || (!X_host && n_tokens > 0))
        return GPTQ_ERR_INVALID_ARG;
    if (!aligned16(S) || !aligned16(stage)) return GPTQ_ERR_INVALID_ARG;
    if (d < 128 || d > kMaxDim || d % 128 != 0 || n_tokens < 0 || n_tokens > (int64_t(1) << 31))
        return GPTQ_ERR_SHAPE;
    if (chunk_tokens < 1 || chunk_tokens > (int64_t(1) << 31)) return GPTQ_ERR_SHAPE;
    const size_t slot = size_t(chunk_tokens) * size_t(d);          // elements per slot
    if (stage_bytes / sizeof(uint16_t) / 2 < slot) return GPTQ_ERR_INVALID_ARG;
    if (n_tokens == 0) return GPTQ_OK;

    cudaStream_t st = as_stream(stream), cs = as_stream(copy_stream);
    cudaEvent_t filled = reinterpret_cast<cudaEvent_t>(ev_filled);
    cudaEvent_t freed = reinterpret_cast<cudaEvent_t>(ev_freed);
    const int64_t chunks = ceil_div(n_tokens, chunk_tokens);
    auto rows_of = [&](int64_t k) { return std::min(chunk_tokens, n_tokens - k * chunk_tokens); };
    auto slot_of = [&](int64_t k) { return stage + size_t(k & 1) * slot; };

    // copy chunk k into its slot once the accumulation that last read the
    // slot is done (the latest record of ev_freed is at least that late)
    auto copy = [&](int64_t k) {
        if (cudaStreamWaitEvent(cs, freed, 0) != cudaSuccess) return false;
        const size_t bytes = size_t(rows_of(k)) * size_t(d) * sizeof(uint16_t);
        if (cudaMemcpyAsync(slot_of(k), X_host + size_t(k) * slot, bytes, cudaMemcpyHostToDevice,
                            cs) != cudaSuccess)
            return false;
        return cudaEventRecord(filled, cs) == cudaSuccess;
    };

    if (!copy(0)) return GPTQ_ERR_CUDA;
    for (int64_t k = 0; k < chunks; ++k) {
        // take chunk k's copy before the next record of ev_filled replaces it
        if (cudaStreamWaitEvent(st, filled, 0) != cudaSuccess) return GPTQ_ERR_CUDA;
        // chunk k + 1 goes into the slot that chunk k - 1 used: ev_freed's
        // latest record is still chunk k - 1's accumulation here
        if (k + 1 < chunks && !copy(k + 1)) return GPTQ_ERR_CUDA;
        const int rc = gptq_hessian_accumulate(S, slot_of(k), rows_of(k), d, nullptr, stream);
        if (rc != GPTQ_OK) return rc;
        if (cudaEventRecord(freed, st) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    if (n_seen) *n_seen += n_tokens;
    return GPTQ_OK;
}

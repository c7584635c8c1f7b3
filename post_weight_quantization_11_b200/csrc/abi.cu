// Library-wide C entry points: status names, ABI version, launch counter.
#include <atomic>

#include "common.cuh"

namespace gptq {

static std::atomic<unsigned long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

}  // namespace gptq

extern "C" const char* gptq_status_string(int status)
{
    switch (status) {
        case GPTQ_OK: return "GPTQ_OK";
        case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
        case GPTQ_ERR_SHAPE: return "GPTQ_ERR_SHAPE";
        case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
        case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
        case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
        case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
        default: return "GPTQ_ERR_UNKNOWN";
    }
}

extern "C" int gptq_abi_version(void) { return GPTQ_ABI_VERSION; }

extern "C" uint64_t gptq_debug_launch_count(void) { return gptq::g_launches.load(); }

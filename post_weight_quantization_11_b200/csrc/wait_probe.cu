// Test hook for the library's failure detection: the two bounded waits every
// kernel uses (a completion flag between CTAs, an mbarrier phase inside a
// CTA) run against a condition that never comes true, with a short limit,
// so a test can check that a stuck dependency ends as a device status while
// the context stays usable.
#include "tc_common.cuh"

namespace gptq {

__device__ int g_probe_no_abort = 0;     // the grid-wide abort word the flag wait polls

__global__ void wait_probe_kernel(const int* flag, int which, unsigned long long limit_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x != 0) return;
    abort = 0;
    if (which == 0) {
        cd_wait_flag(flag, &abort, &g_probe_no_abort, limit_ns);
    } else {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait(&bar, 0, kErrWaitFull, &abort, limit_ns);   // nobody arrives
    }
}

}  // namespace gptq

extern "C" int gptq_debug_bounded_wait(const int32_t* flag, int which, int64_t limit_ns,
                                       void* stream)
{
    using namespace gptq;
    if (which != 0 && which != 1) return GPTQ_ERR_INVALID_ARG;
    if (which == 0 && (!flag || (reinterpret_cast<uintptr_t>(flag) & 3u))) return GPTQ_ERR_INVALID_ARG;
    if (limit_ns < 1000000 || limit_ns > 1000000000) return GPTQ_ERR_INVALID_ARG;
    wait_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(flag, which,
                                                      (unsigned long long)limit_ns);
    count_launches();
    return launch_status();
}

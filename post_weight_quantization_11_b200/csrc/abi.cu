// Library-wide C entry points: status names, ABI version, launch counter,
// per-kind kernel timing (diagnostics).
#include <atomic>
#include <mutex>
#include <vector>

#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace gptq {

__device__ int g_device_status = 0;

int encode_tmap_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swz)
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p)
            return GPTQ_ERR_CUDA;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GPTQ_OK : GPTQ_ERR_CUDA;
}

static std::atomic<unsigned long long> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

int device_sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n > 0) return n;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

// ---- per-kind kernel timing (diagnostics) --------------------------------

static std::atomic<int> g_timing{0};
static std::mutex g_timing_mu;
struct TimedSpan { int kind; cudaEvent_t a, b; };
static std::vector<TimedSpan> g_spans;

KernelTimer::KernelTimer(int kind, cudaStream_t st) : kind_(kind), st_(st)
{
    if (!g_timing.load(std::memory_order_relaxed)) return;
    if (cudaEventCreate(&ev0_) != cudaSuccess) { ev0_ = nullptr; return; }
    if (cudaEventRecord(ev0_, st_) != cudaSuccess) { cudaEventDestroy(ev0_); ev0_ = nullptr; }
}

KernelTimer::~KernelTimer()
{
    if (!ev0_) return;
    cudaEvent_t ev1 = nullptr;
    if (cudaEventCreate(&ev1) != cudaSuccess || cudaEventRecord(ev1, st_) != cudaSuccess) {
        if (ev1) cudaEventDestroy(ev1);
        cudaEventDestroy(ev0_);
        return;
    }
    std::lock_guard<std::mutex> lock(g_timing_mu);
    g_spans.push_back(TimedSpan{kind_, ev0_, ev1});
}

static std::atomic<int> g_cta_cap[kCtaKinds];

int persistent_ctas(int kind)
{
    const int sms = device_sm_count();
    const int cap = (kind >= 0 && kind < kCtaKinds) ? g_cta_cap[kind].load() : 0;
    return cap > 0 ? std::min(cap, sms) : sms;
}

}  // namespace gptq

extern "C" int gptq_set_max_ctas(int kind, int max_ctas)
{
    if (kind < 0 || kind >= gptq::kCtaKinds || max_ctas < 0) return GPTQ_ERR_INVALID_ARG;
    gptq::g_cta_cap[kind].store(max_ctas);
    return GPTQ_OK;
}

extern "C" int gptq_debug_kernel_timing(int enable)
{
    gptq::g_timing.store(enable ? 1 : 0);
    return GPTQ_OK;
}

extern "C" int gptq_debug_kernel_times(double* ms, int64_t* spans, int n_kinds)
{
    using namespace gptq;
    if (!ms || !spans || n_kinds < kKKinds) return GPTQ_ERR_INVALID_ARG;
    for (int k = 0; k < n_kinds; ++k) { ms[k] = 0.0; spans[k] = 0; }
    std::vector<TimedSpan> take;
    {
        std::lock_guard<std::mutex> lock(g_timing_mu);
        take.swap(g_spans);
    }
    int rc = GPTQ_OK;
    for (const TimedSpan& t : take) {
        float v = 0.f;
        if (cudaEventSynchronize(t.b) != cudaSuccess ||
            cudaEventElapsedTime(&v, t.a, t.b) != cudaSuccess)
            rc = GPTQ_ERR_CUDA;
        else if (t.kind >= 0 && t.kind < n_kinds) {
            ms[t.kind] += double(v);
            spans[t.kind] += 1;
        }
        cudaEventDestroy(t.a);
        cudaEventDestroy(t.b);
    }
    return rc;
}

extern "C" const char* gptq_debug_kernel_kind_name(int kind)
{
    static const char* names[gptq::kKKinds] = {
        "hessian", "gather", "finalize", "factorization", "init_work", "split_u",
        "static_params", "sweep", "update_near", "update_far", "pack", "unpack", "rtn",
        "w4a16", "probe", "awq"};
    return (kind >= 0 && kind < gptq::kKKinds) ? names[kind] : "unknown";
}

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

extern "C" int gptq_device_status(int32_t* status_out, int reset)
{
    if (!status_out) return GPTQ_ERR_INVALID_ARG;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, gptq::g_device_status, sizeof(int)) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    *status_out = v;
    if (reset && v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(gptq::g_device_status, &zero, sizeof(int)) != cudaSuccess)
            return GPTQ_ERR_CUDA;
    }
    return GPTQ_OK;
}

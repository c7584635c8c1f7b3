// Library-wide C entry points: status names, ABI version, launch counter.
#include <atomic>

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

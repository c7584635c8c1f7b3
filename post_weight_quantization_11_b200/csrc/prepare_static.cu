// gptq_prepare_hinv_static: the inverse-Hessian preparation for callers that
// cannot allocate device memory -- for example code that runs while a stream
// is being captured into a CUDA graph (cudaMalloc is not allowed under a
// global-mode capture), or a plug-in inside an engine that owns the whole
// device memory pool and forbids other allocations.  Such a caller cannot
// provide the scratch buffer gptq_prepare_hinv asks for, so this entry point
// uses a fixed scratch array that lives in the library itself.
//
// The scratch is a file-scope __device__ array of kStaticScratchBytes
// (16 MiB): every GPU that loads the library holds it until the process
// exits.  Host code cannot use the array's name as a device address, so the
// first call on each device (with that device current) looks the address up
// with cudaGetSymbolAddress and caches it; make that first call before any
// stream capture starts.  All calls share the one array and it keeps the
// previous call's contents (the preparation overwrites or clears everything
// it reads), so calls that overlap on the GPU -- two streams at once -- race
// and must be serialized by the caller.
#include <mutex>

#include "common.cuh"

namespace gptq {

int prepare_check_args(const float* S, int64_t d, float damp_rel, int act_order,
                       const int32_t* perm, const float* U, const int32_t* info);

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int64_t kStaticMaxDim = 1024;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_prepare_scratch[kStaticScratchBytes];

static void* g_scratch_ptr[kMaxDevices] = {};
static std::mutex g_scratch_mu;

// Device address of g_prepare_scratch on the current device (looked up once).
static void* static_scratch(int* status)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = GPTQ_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_prepare_scratch) != cudaSuccess || !p) {
            *status = GPTQ_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev] = p;
    }
    *status = GPTQ_OK;
    return g_scratch_ptr[dev];
}

}  // namespace gptq

extern "C" int gptq_prepare_hinv_static(const float* S, int64_t d, int64_t n_tokens,
                                        float damp_rel, int act_order, int32_t* perm, float* U,
                                        int32_t* info, void* stream)
{
    using namespace gptq;
    // the argument checks of gptq_prepare_hinv first, so both entry points
    // return the same status for the same bad argument
    int rc = prepare_check_args(S, d, damp_rel, act_order, perm, U, info);
    if (rc != GPTQ_OK) return rc;
    if (n_tokens <= 0) return GPTQ_ERR_SHAPE;
    if (d > kStaticMaxDim) return GPTQ_ERR_SHAPE;               // beyond the fixed scratch
    const size_t need = gptq_prepare_workspace_bytes(d);
    if (need > kStaticScratchBytes) return GPTQ_ERR_SHAPE;
    int status = GPTQ_OK;
    void* ws = static_scratch(&status);
    if (status != GPTQ_OK) return status;
    return gptq_prepare_hinv(S, d, n_tokens, damp_rel, act_order, perm, U, info, ws,
                             kStaticScratchBytes, stream);
}

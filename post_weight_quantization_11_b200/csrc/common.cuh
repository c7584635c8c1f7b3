// Shared host/device helpers of libgptq (sm_100a).  No quantization
// arithmetic lives here.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <algorithm>
#include <cstring>

#include "../../include/gptq.h"

#define GPTQ_ABI_VERSION 100

namespace gptq {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Process-wide count of kernel launches issued by the library (diagnostics).
void count_launches(int n = 1);

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of SMs of the current device (cached per device after the first query).
int device_sm_count();

// Persistent-grid caps set by gptq_set_max_ctas (0: none): the CTAs a
// persistent kernel of that kind launches are min(SMs, cap).
enum CtaKind : int { kCtaHessian = 0, kCtaPrepare = 1, kCtaQuantize = 2, kCtaKinds = 3 };
int persistent_ctas(int kind);

// Diagnostics (gptq_debug_kernel_timing): kinds of the library's launches.
enum KernelKind : int {
    kKHessian = 0, kKGather, kKFinalize, kKFactor, kKInitWork, kKSplitU, kKStaticParams,
    kKSweep, kKUpdateNear, kKUpdateFar, kKPack, kKUnpack, kKRtn, kKW4A16, kKProbe, kKAwq,
    kKKinds
};

// While timing is enabled, the launches issued in this object's lifetime are
// bracketed by two CUDA events on `st` and their time is added to `kind`.
// Otherwise it does nothing.  For eager use (not under stream capture).
class KernelTimer {
public:
    KernelTimer(int kind, cudaStream_t st);
    ~KernelTimer();
    KernelTimer(const KernelTimer&) = delete;
    KernelTimer& operator=(const KernelTimer&) = delete;
private:
    int kind_;
    cudaStream_t st_;
    cudaEvent_t ev0_ = nullptr;
};

// Supported problem limits (validated at the ABI).
constexpr int64_t kMaxDim = 32768;
constexpr int64_t kMaxRows = int64_t(1) << 24;

}  // namespace gptq

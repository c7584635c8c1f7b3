// Group quantizer shared by the GPTQ sweep and the round-to-nearest baseline:
// asymmetric min-max over a group ("大模型量化的“校准”艺术" sec. 2.1) with an
// fp16 scale and a b-bit zero point per group ("INT4/INT8 量化推理" sec. 一).
// Every decision is an IEEE fp32 operation (correctly rounded division,
// round-half-to-even), so equal fp32 inputs give equal codes on any IEEE
// implementation.
#pragma once

#include "common.cuh"

namespace gptq {

struct GroupQ {
    float s;      // fp16 scale as fp32 (exact)
    float z;      // zero point as an integral fp32
    __half h;     // fp16 scale
};

// mn <= 0 <= mx already hold (the range includes 0).
__device__ __forceinline__ GroupQ group_params(float mn, float mx, float maxqf)
{
    if (mn == mx) { mn = -1.f; mx = 1.f; }             // all-zero group
    const float s_pre = __fdiv_rn(__fsub_rn(mx, mn), maxqf);
    __half h = __float2half_rn(s_pre);
    unsigned short hb = __half_as_ushort(h);
    if ((hb & 0x7fffu) == 0) hb = 0x0001u;               // smallest positive fp16
    if ((hb & 0x7fffu) >= 0x7c00u) hb = 0x7bffu;         // largest finite fp16
    h = __ushort_as_half(hb);
    GroupQ g;
    g.h = h;
    g.s = __half2float(h);
    float zf = rintf(__fdiv_rn(-mn, g.s));
    g.z = fminf(fmaxf(zf, 0.f), maxqf);
    return g;
}

// code = clamp(rne(x / s) + z, 0, maxq) as an integral fp32
__device__ __forceinline__ float quant_code(float x, const GroupQ& g, float maxqf)
{
    float c = __fadd_rn(rintf(__fdiv_rn(x, g.s)), g.z);
    return fminf(fmaxf(c, 0.f), maxqf);
}

}  // namespace gptq

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
    float r;      // fl(1 / s), for quant_code_fast
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
    g.r = __frcp_rn(g.s);
    return g;
}

// code = clamp(rne(x / s) + z, 0, maxq) as an integral fp32
__device__ __forceinline__ float quant_code(float x, const GroupQ& g, float maxqf)
{
    float c = __fadd_rn(rintf(__fdiv_rn(x, g.s)), g.z);
    return fminf(fmaxf(c, 0.f), maxqf);
}

// The same value as quant_code, without a division: with r = RN(1/s) and a
// quotient q within one ulp of x/s, RN(q + RN(x - q s) r) is the correctly
// rounded quotient RN(x/s) (Markstein's theorem for division with a
// correctly rounded reciprocal; x - q s is exact in one FMA).  x r alone can
// be 1.5 ulp off, so the correction is applied twice: the first brings q
// within one ulp, the second rounds it correctly.  No overflow or underflow
// can occur: s is a finite fp16 value >= 2^-24.
__host__ __device__ __forceinline__ float div_rn_recip(float x, float s, float r)
{
    float q = x * r;
    q = fmaf(fmaf(-q, s, x), r, q);
    return fmaf(fmaf(-q, s, x), r, q);
}

// Round-to-nearest-even to an integer on the FMA pipe (rintf issues on the
// slower conversion unit): adding and removing 1.5 * 2^23 leaves the sum
// with a unit last place, so the first add rounds x to an integer, ties to
// even.  Exact for |x| <= 2^22; beyond that the result stays within 2 of x,
// which the clamp of every caller (codes in [0, maxq], maxq <= 255) maps to
// the same code as the exact rounding.
__device__ __forceinline__ float rne_for_clamp(float x)
{
    constexpr float kMagic = 12582912.f;   // 1.5 * 2^23
    return __fsub_rn(__fadd_rn(x, kMagic), kMagic);
}

// The integral value of c in [0, 255] as a byte, without a conversion
// instruction: c + 2^23 holds c in its low mantissa bits.
__device__ __forceinline__ uint32_t code_byte(float c)
{
    return __float_as_uint(__fadd_rn(c, 8388608.f)) & 0xffu;
}

__device__ __forceinline__ float quant_code_fast(float x, const GroupQ& g, float maxqf)
{
    const float c = __fadd_rn(rne_for_clamp(div_rn_recip(x, g.s, g.r)), g.z);
    return fminf(fmaxf(c, 0.f), maxqf);
}

}  // namespace gptq

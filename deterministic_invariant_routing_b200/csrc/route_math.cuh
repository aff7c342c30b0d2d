// The FP32 routing contract's device arithmetic, shared by the routing kernel (route.cu)
// and the router GEMM's fused routing epilogue (tc_gemm.cu): exp_rl and the ordered
// selection key. ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1: router
// softmax and top-k are validated for precision and stability first; tie-breaking is part
// of the routing record.)
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace {

// exp_rl: Cody & Waite additive range reduction (x = n ln2 + r, ln2 split in a 12-bit
// head whose products with n are exact and an fp32 tail), then the degree-7 Taylor
// polynomial of e^r by Horner with fused multiply-adds, scaled by 2^n built from the
// exponent field. Specials: NaN -> NaN, x < -87 -> +0, x > 88 -> +inf.
__device__ __forceinline__ float exp_rl(float x)
{
    // ln 2 rounded to the nearest multiple of 2^-12 (12 significant bits: n * head is
    // exact for |n| <= 127), and the fp32 rounding of the remainder.
    const double kLn2 = 0.693147180559945309417232121458;
    const float kHead = __double2float_rn(rint(kLn2 * 4096.0) / 4096.0);
    const float kTail = __double2float_rn(kLn2 - (double)kHead);
    const float kLog2e = __double2float_rn(1.442695040888963407359924681002);
    if (isnan(x)) return x;
    if (x < -87.0f) return 0.0f;
    if (x > 88.0f) return __int_as_float(0x7f800000);
    const float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kHead, x);
    r = __fmaf_rn(-n, kTail, r);
    // Taylor coefficients 1/k!, k = 7 .. 0, each rounded once to fp32
    float p = __double2float_rn(1.0 / 5040.0);
    p = __fmaf_rn(p, r, __double2float_rn(1.0 / 720.0));
    p = __fmaf_rn(p, r, __double2float_rn(1.0 / 120.0));
    p = __fmaf_rn(p, r, __double2float_rn(1.0 / 24.0));
    p = __fmaf_rn(p, r, __double2float_rn(1.0 / 6.0));
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const float two_n = __int_as_float((__float2int_rn(n) + 127) << 23);
    return __fmul_rn(p, two_n);
}

// order-preserving 32-bit image of a choice: -0 == +0, NaN below every number
__device__ __forceinline__ uint32_t order_bits(float c)
{
    if (isnan(c)) return 0u;
    if (c == 0.0f) c = 0.0f;
    const uint32_t u = __float_as_uint(c);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace
}  // namespace moe

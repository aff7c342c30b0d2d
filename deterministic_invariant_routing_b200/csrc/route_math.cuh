// The FP32 routing contract's device arithmetic, shared by the routing kernel (route.cu)
// and the router statistics (stats.cu): exp_rl, the sqrtsoftplus score (SpecForge PR
// #1003 names it beside sigmoid; its fp32 steps are this contract's) and the ordered
// selection key. ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1: router
// softmax and top-k are validated for precision and stability first; tie-breaking is part
// of the routing record.)
#pragma once

#include "moe_internal.cuh"

namespace moe {
namespace {

// The constants of the contract's exp_rl and ln_rl, fixed at compile time: ln 2 rounded to
// the nearest multiple of 2^-12 (12 significant bits, 2839 / 4096: n * head is exact for
// |n| <= 127), the fp32 rounding of the remainder, fp32(log2 e), fp32(sqrt 2), and the
// series coefficients 1/k! and 1/(2k+1), each the fp32 rounding (a constant-expression
// cast rounds to nearest) of its double value.
constexpr double kLn2d = 0.693147180559945309417232121458;
constexpr float kLn2Head = (float)(2839.0 / 4096.0);
constexpr float kLn2Tail = (float)(kLn2d - 2839.0 / 4096.0);
constexpr float kLog2e = (float)1.442695040888963407359924681002;
constexpr float kSqrt2 = (float)1.414213562373095048801688724;
static_assert(2839.0 / 4096.0 - kLn2d < 1.0 / 8192.0 && kLn2d - 2839.0 / 4096.0 < 1.0 / 8192.0,
              "2839/4096 is ln 2 to the nearest 2^-12");

// exp_rl: Cody & Waite additive range reduction (x = n ln2 + r, ln2 split in a 12-bit
// head whose products with n are exact and an fp32 tail), then the degree-7 Taylor
// polynomial of e^r by Horner with fused multiply-adds, scaled by 2^n built from the
// exponent field. Specials: NaN -> NaN, x < -87 -> +0, x > 88 -> +inf.
__device__ __forceinline__ float exp_rl(float x)
{
    if (isnan(x)) return x;
    if (x < -87.0f) return 0.0f;
    if (x > 88.0f) return __int_as_float(0x7f800000);
    const float n = rintf(__fmul_rn(x, kLog2e));
    float r = __fmaf_rn(-n, kLn2Head, x);
    r = __fmaf_rn(-n, kLn2Tail, r);
    // Taylor coefficients 1/k!, k = 7 .. 0, each rounded once to fp32
    float p = (float)(1.0 / 5040.0);
    p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
    p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    const float two_n = __int_as_float((__float2int_rn(n) + 127) << 23);
    return __fmul_rn(p, two_n);
}

// ln_rl, for v >= 1 finite: v = m 2^k from the bits (m in [1, 2), halved with k + 1 when
// above sqrt 2), ln m = 2 atanh(z) with z = (m - 1) / (m + 1) as the odd series through
// z^9 (coefficients 1/3, 1/5, 1/7, 1/9 rounded once, Horner with fused multiply-adds),
// then k ln 2 added with the two-part ln 2 of exp_rl.
__device__ __forceinline__ float ln_rl(float v)
{
    const uint32_t b = __float_as_uint(v);
    int k = (int)(b >> 23) - 127;
    float m = __uint_as_float((b & 0x7fffffu) | 0x3f800000u);
    if (m > kSqrt2) {
        m = __fmul_rn(m, 0.5f);
        k += 1;
    }
    const float f = __fsub_rn(m, 1.0f);  // exact (Sterbenz)
    const float z = __fdiv_rn(f, __fadd_rn(2.0f, f));
    const float w = __fmul_rn(z, z);
    float q = __fmaf_rn(w, (float)(1.0 / 9.0), (float)(1.0 / 7.0));
    q = __fmaf_rn(w, q, (float)(1.0 / 5.0));
    q = __fmaf_rn(w, q, (float)(1.0 / 3.0));
    const float lnm = __fmaf_rn(__fmul_rn(2.0f, __fmul_rn(z, w)), q, __fmul_rn(2.0f, z));
    const float kf = __int2float_rn(k);
    return __fmaf_rn(kf, kLn2Head, __fmaf_rn(kf, kLn2Tail, lnm));
}

// log1p_rl, u >= 0: Goldberg's formula u * ln(1 + u) / ((1 + u) - 1), u itself when
// 1 + u rounds to 1 (the subtraction is exact)
__device__ __forceinline__ float log1p_rl(float u)
{
    const float v = __fadd_rn(1.0f, u);
    if (v == 1.0f) return u;
    return __fdiv_rn(__fmul_rn(u, ln_rl(v)), __fsub_rn(v, 1.0f));
}

// the sqrtsoftplus score: sqrt(softplus(l)), softplus(l) = l above 20, else
// log1p_rl(exp_rl(l)); IEEE square root
__device__ __forceinline__ float sqrtsoftplus_rl(float l)
{
    return __fsqrt_rn(l > 20.0f ? l : log1p_rl(exp_rl(l)));
}

// the score of one logit for the elementwise score functions (sigmoid, sqrtsoftplus)
__device__ __forceinline__ float elementwise_score(float l, int score_fn)
{
    if (score_fn == MOE_SIGMOID) return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_rl(-l)));
    return sqrtsoftplus_rl(l);
}

// The contract scores of one token's logits row, one warp: lane L holds experts L, L+32, ...
// (s[i] for expert L + 32 i; slots past E hold values that are never used). softmax: max
// by comparisons and a butterfly, e = exp_rl(l - m), the 32-lane tree sum (each lane's
// experts in increasing order, then butterfly levels 16 .. 1), s = e / S; sigmoid and
// sqrtsoftplus elementwise.
// lane L's logits of one row (experts L, L+32, ...; 0 past E)
template <int NE>
__device__ __forceinline__ void load_row(const float* __restrict__ row, int E, int lane,
                                         float (&s)[NE])
{
#pragma unroll
    for (int i = 0; i < NE; ++i) {
        const int e = lane + 32 * i;
        s[i] = (e < E) ? row[e] : 0.0f;
    }
}

// the scores of a row already loaded by load_row, in place
template <int NE>
__device__ __forceinline__ void contract_scores_of(int E, int score_fn, int lane,
                                                   float (&s)[NE])
{
    if (score_fn != MOE_SOFTMAX) {
#pragma unroll
        for (int i = 0; i < NE; ++i) s[i] = elementwise_score(s[i], score_fn);
        return;
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < NE; ++i)
        if (lane + 32 * i < E && s[i] > m) m = s[i];
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, m, off);
        if (o > m) m = o;
    }
    float part = 0.0f;
#pragma unroll
    for (int i = 0; i < NE; ++i) {
        if (lane + 32 * i < E) {
            s[i] = exp_rl(__fsub_rn(s[i], m));
            part = __fadd_rn(part, s[i]);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        part = __fadd_rn(part, __shfl_xor_sync(0xffffffffu, part, off));
#pragma unroll
    for (int i = 0; i < NE; ++i) s[i] = __fdiv_rn(s[i], part);
}

template <int NE>
__device__ __forceinline__ void contract_scores(const float* __restrict__ row, int E,
                                                int score_fn, int lane, float (&s)[NE])
{
    load_row<NE>(row, E, lane, s);
    contract_scores_of<NE>(E, score_fn, lane, s);
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

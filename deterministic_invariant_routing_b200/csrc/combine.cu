// Weighted combine: the MoE block's final floating-point reduction.
//
// "DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 3 ("Final Reduction Is
// The Core Drift Point"): the order, dtype and downcast point of the combine are the
// contract. "From Expert Reduction to Behavioral Divergence" (arXiv 2607.28097, Abstract):
// different orders of the expert sum are observably different, so one order is fixed:
// rank order 0..K-1, each product w_j * y rounded to fp32, sequential fp32 adds, the
// shared expert added last, one bf16 round-to-nearest-even at the end. No FMA, no atomics;
// every output element is produced by exactly one thread.
//
// Memory-bound: each thread owns VPT consecutive 16-byte vectors (8 columns each) of a
// token, issues its VPT * K row loads first, then reduces each column in rank order and
// writes VPT 128-bit vectors.
#include <cuda_bf16.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// bf16 round-to-nearest-even of two floats packed low/high; a NaN keeps its sign and
// payload's top bits and is made quiet (the contract's single downcast). Without a NaN the
// hardware conversion gives the same bits as the integer rounding below (round to nearest
// even, overflow to infinity, subnormals kept) in one instruction per pair.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    auto cvt = [](float f) -> uint32_t {
        const uint32_t u = __float_as_uint(f);
        if ((u & 0x7fffffffu) > 0x7f800000u) return (u >> 16) | 0x40u;
        return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
    };
    if (isnan(a) || isnan(b)) return cvt(a) | (cvt(b) << 16);
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
    return r;
}

// VPT consecutive 16-byte vectors of one token per thread: the token's K row indices and
// weights are loaded once for all of them (as 16-byte vectors when K is a multiple of 4 and
// the arrays are 16-byte aligned), and VPT * K row loads are in flight before the first
// product. Each output element is still one thread's rank-order sum.
template <int KMAX, int VPT>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ dest_row,
                                                      const uint4* __restrict__ y_shared,
                                                      const uint8_t* __restrict__ mask, int T,
                                                      int K, int vec_per_row, int vec_idx,
                                                      uint4* __restrict__ out)
{
    pdl_wait();
    const int groups_per_row = vec_per_row / VPT;
    const int64_t total = (int64_t)T * groups_per_row;
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < total;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = gi / groups_per_row;
        const int v0 = (int)(gi - t * groups_per_row) * VPT;
        const int64_t idx0 = t * vec_per_row + v0;
        if (mask != nullptr && mask[t] == 0) {
#pragma unroll
            for (int u = 0; u < VPT; ++u) out[idx0 + u] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        float wj[KMAX];
        int32_t dr[KMAX];
        if (KMAX % 4 == 0 && vec_idx) {  // K == KMAX, 16-byte aligned rows of K values
#pragma unroll
            for (int j = 0; j < KMAX; j += 4) {
                const int4 d4 = *reinterpret_cast<const int4*>(dest_row + t * KMAX + j);
                const float4 w4 = *reinterpret_cast<const float4*>(w + t * KMAX + j);
                dr[j] = d4.x;
                dr[j + 1] = d4.y;
                dr[j + 2] = d4.z;
                dr[j + 3] = d4.w;
                wj[j] = w4.x;
                wj[j + 1] = w4.y;
                wj[j + 2] = w4.z;
                wj[j + 3] = w4.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                dr[j] = (j < K) ? dest_row[t * K + j] : -1;
                wj[j] = (j < K) ? w[t * K + j] : 0.0f;
            }
        }
        uint4 rows[KMAX][VPT];
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
#pragma unroll
            for (int u = 0; u < VPT; ++u)
                rows[j][u] = (j < K && dr[j] >= 0) ? y[(int64_t)dr[j] * vec_per_row + v0 + u]
                                                    : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < VPT; ++u) {
            float acc[8];
            bool first = true;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                if (j < K && dr[j] >= 0) {
                    const uint32_t q[4] = {rows[j][u].x, rows[j][u].y, rows[j][u].z,
                                           rows[j][u].w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const float p0 = __fmul_rn(wj[j], bf16_lo(q[c]));
                        const float p1 = __fmul_rn(wj[j], bf16_hi(q[c]));
                        acc[2 * c] = first ? p0 : __fadd_rn(acc[2 * c], p0);
                        acc[2 * c + 1] = first ? p1 : __fadd_rn(acc[2 * c + 1], p1);
                    }
                    first = false;
                }
            }
            if (first) {
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
            }
            if (y_shared != nullptr) {
                const uint4 sv = y_shared[idx0 + u];
                const uint32_t q[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    acc[2 * c] = __fadd_rn(acc[2 * c], bf16_lo(q[c]));
                    acc[2 * c + 1] = __fadd_rn(acc[2 * c + 1], bf16_hi(q[c]));
                }
            }
            out[idx0 + u] = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                                       pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
        }
    }
}

// vectors per thread: 4 for top-1 layers, 2 up to top-8 (measured: 105.5 against
// 109.9 us on the 30B-A3B layer at T = 16384, 29.3 / 26.7 against 35.7 us for top-1 at
// T = 8192; 4 at top-8 holds too many rows in registers and halves the speed), 1 above
template <int KMAX>
constexpr int combine_vpt()
{
    return KMAX == 1 ? 4 : (KMAX <= 8 ? 2 : 1);
}

template <int KMAX>
cudaError_t launch_k(const moe_cfg& c, const uint16_t* y, const float* w, const int32_t* dr,
                     const uint16_t* ys, const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    constexpr int VPT = combine_vpt<KMAX>();
    const int vec = c.H / 8;  // a multiple of 16 (H % 128 == 0), so of VPT
    const int64_t total = (int64_t)c.T * (vec / VPT);
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = resident_blocks((const void*)combine_kernel<KMAX, VPT>, 256, 0);
    if (blocks > cap) blocks = cap;
    const int vec_idx = (c.K == KMAX && KMAX % 4 == 0 &&
                         (reinterpret_cast<uintptr_t>(dr) & 15u) == 0 &&
                         (reinterpret_cast<uintptr_t>(w) & 15u) == 0)
                            ? 1
                            : 0;
    return launch_pdl(combine_kernel<KMAX, VPT>, dim3((unsigned)blocks), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(y), w, dr, reinterpret_cast<const uint4*>(ys),
                      mask, c.T, c.K, vec, vec_idx, reinterpret_cast<uint4*>(out));
}

// Order-invariant variant ("From Expert Reduction to Behavioral Divergence", arXiv
// 2607.28097, Abstract: scheme C's result does not depend on the order of the expert
// terms). Per output element the terms -- w_j * y_j formed exactly in double, and the
// shared expert's y -- are summed in double in a canonical order (ascending magnitude, the
// negative of equal magnitudes first) and rounded once to fp32 then to bf16, so the result
// is a function of the multiset of terms.
//
// Two routes to the same bits. Every term has at most 32 significant bits (24 x 8), so when
// the valid nonzero terms' exponents lie within 16 of each other every partial sum of up to
// 17 of them fits in double's 53 bits exactly: any order gives the exact sum, and the terms
// are added as they come. Otherwise (or with an infinite / NaN term) they are sorted by the
// 64-bit key (|x| bits << 1) | (x is not negative) -- ascending magnitude, -x before +x --
// with an odd-even transposition network on integers, and added in that order.
__device__ __forceinline__ uint64_t canon_key(double x)
{
    const uint64_t b = (uint64_t)__double_as_longlong(x);
    return ((b & 0x7fffffffffffffffull) << 1) | ((b >> 63) ^ 1ull);
}

__device__ __forceinline__ double from_key(uint64_t k)
{
    return __longlong_as_double((long long)((k >> 1) | ((~k & 1ull) << 63)));
}

template <int KMAX>
__global__ void __launch_bounds__(256) combine_invariant_kernel(
    const uint4* __restrict__ y, const float* __restrict__ w, const int32_t* __restrict__ dest_row,
    const uint4* __restrict__ y_shared, const uint8_t* __restrict__ mask, int T, int K,
    int vec_per_row, uint4* __restrict__ out)
{
    pdl_wait();
    constexpr int N = KMAX + 1;
    const int64_t total = (int64_t)T * vec_per_row;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = idx / vec_per_row;
        const int v = (int)(idx - t * vec_per_row);
        if (mask != nullptr && mask[t] == 0) {
            out[idx] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        uint4 rows[N];
        float wj[N];
        bool ok[N];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            const int32_t r = (j < K) ? dest_row[t * K + j] : -1;
            ok[j] = r >= 0;
            wj[j] = ok[j] ? w[t * K + j] : 0.0f;
            rows[j] = ok[j] ? y[(int64_t)r * vec_per_row + v] : make_uint4(0u, 0u, 0u, 0u);
        }
        ok[KMAX] = y_shared != nullptr;
        wj[KMAX] = 1.0f;
        rows[KMAX] = ok[KMAX] ? y_shared[idx] : make_uint4(0u, 0u, 0u, 0u);
        int n_valid = 0;
#pragma unroll
        for (int j = 0; j < N; ++j) n_valid += ok[j] ? 1 : 0;
        uint32_t packed[4];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            double term[N];
            int emax = -1, emin = 4096;
            bool special = false;
#pragma unroll
            for (int j = 0; j < N; ++j) {
                const uint32_t q = (c >> 1) == 0 ? rows[j].x
                                 : (c >> 1) == 1 ? rows[j].y
                                 : (c >> 1) == 2 ? rows[j].z : rows[j].w;
                const float yv = (c & 1) ? bf16_hi(q) : bf16_lo(q);
                term[j] = ok[j] ? __dmul_rn((double)wj[j], (double)yv) : 0.0;  // exact
                const uint64_t b = (uint64_t)__double_as_longlong(term[j]);
                const int e = (int)((b >> 52) & 0x7ffu);
                if (ok[j] && e == 0x7ff) special = true;
                if (ok[j] && (b << 1) != 0) {
                    emax = e > emax ? e : emax;
                    emin = e < emin ? e : emin;
                }
            }
            double sum = 0.0;
            if (!special && emax - emin <= 16) {
#pragma unroll
                for (int j = 0; j < N; ++j)
                    if (ok[j]) sum = __dadd_rn(sum, term[j]);
            } else {
                uint64_t key[N];
#pragma unroll
                for (int j = 0; j < N; ++j) key[j] = ok[j] ? canon_key(term[j]) : ~0ull;
#pragma unroll
                for (int pass = 0; pass < N; ++pass) {
#pragma unroll
                    for (int i = pass & 1; i + 1 < N; i += 2) {
                        const uint64_t lo = key[i] < key[i + 1] ? key[i] : key[i + 1];
                        const uint64_t hi = key[i] < key[i + 1] ? key[i + 1] : key[i];
                        key[i] = lo;
                        key[i + 1] = hi;
                    }
                }
#pragma unroll
                for (int j = 0; j < N; ++j)
                    if (j < n_valid) sum = __dadd_rn(sum, from_key(key[j]));
            }
            const float f = __double2float_rn(sum);
            if (c & 1) packed[c >> 1] |= pack_bf16(0.0f, f) & 0xffff0000u;
            else packed[c >> 1] = pack_bf16(f, 0.0f) & 0xffffu;
        }
        out[idx] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    }
}

template <int KMAX>
cudaError_t launch_inv(const moe_cfg& c, const uint16_t* y, const float* w, const int32_t* dr,
                       const uint16_t* ys, const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    const int vec = c.H / 8;
    const int64_t total = (int64_t)c.T * vec;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    return launch_pdl(combine_invariant_kernel<KMAX>, dim3((unsigned)blocks), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(y), w, dr, reinterpret_cast<const uint4*>(ys),
                      mask, c.T, c.K, vec, reinterpret_cast<uint4*>(out));
}

}  // namespace

cudaError_t launch_combine(const moe_cfg& c, const uint16_t* y, const float* w,
                           const int32_t* dest_row, const uint16_t* y_shared,
                           const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    if (c.T == 0) return cudaSuccess;
    if (c.K <= 1) return launch_k<1>(c, y, w, dest_row, y_shared, mask, out, st);
    if (c.K <= 2) return launch_k<2>(c, y, w, dest_row, y_shared, mask, out, st);
    if (c.K <= 4) return launch_k<4>(c, y, w, dest_row, y_shared, mask, out, st);
    if (c.K <= 8) return launch_k<8>(c, y, w, dest_row, y_shared, mask, out, st);
    return launch_k<16>(c, y, w, dest_row, y_shared, mask, out, st);
}

cudaError_t launch_combine_invariant(const moe_cfg& c, const uint16_t* y, const float* w,
                                     const int32_t* dest_row, const uint16_t* y_shared,
                                     const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    if (c.T == 0) return cudaSuccess;
    if (c.K <= 2) return launch_inv<2>(c, y, w, dest_row, y_shared, mask, out, st);
    if (c.K <= 4) return launch_inv<4>(c, y, w, dest_row, y_shared, mask, out, st);
    if (c.K <= 8) return launch_inv<8>(c, y, w, dest_row, y_shared, mask, out, st);
    return launch_inv<16>(c, y, w, dest_row, y_shared, mask, out, st);
}

}  // namespace moe

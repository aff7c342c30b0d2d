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
// Memory-bound: each thread owns 8 consecutive columns (one 16-byte vector) of a token,
// issues the K row loads first (K independent 128-bit loads in flight), then reduces in
// rank order and writes one 128-bit vector.
#include <cuda_bf16.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// bf16 round-to-nearest-even of two floats packed low/high; a NaN keeps its sign and
// payload's top bits and is made quiet (the contract's single downcast)
__device__ __forceinline__ uint32_t pack_bf16(float a, float b)
{
    auto cvt = [](float f) -> uint32_t {
        const uint32_t u = __float_as_uint(f);
        if ((u & 0x7fffffffu) > 0x7f800000u) return (u >> 16) | 0x40u;
        return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
    };
    return cvt(a) | (cvt(b) << 16);
}

template <int KMAX>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y,
                                                      const float* __restrict__ w,
                                                      const int32_t* __restrict__ dest_row,
                                                      const uint4* __restrict__ y_shared,
                                                      const uint8_t* __restrict__ mask, int T,
                                                      int K, int vec_per_row,
                                                      uint4* __restrict__ out)
{
    const int64_t total = (int64_t)T * vec_per_row;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = idx / vec_per_row;
        const int v = (int)(idx - t * vec_per_row);
        if (mask != nullptr && mask[t] == 0) {
            out[idx] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        uint4 rows[KMAX];
        float wj[KMAX];
        int32_t dr[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K) {
                dr[j] = dest_row[t * K + j];
                wj[j] = w[t * K + j];
                rows[j] = (dr[j] >= 0) ? y[(int64_t)dr[j] * vec_per_row + v]
                                       : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        float acc[8];
        bool first = true;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < K && dr[j] >= 0) {
                const uint32_t q[4] = {rows[j].x, rows[j].y, rows[j].z, rows[j].w};
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
            const uint4 s = y_shared[idx];
            const uint32_t q[4] = {s.x, s.y, s.z, s.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                acc[2 * c] = __fadd_rn(acc[2 * c], bf16_lo(q[c]));
                acc[2 * c + 1] = __fadd_rn(acc[2 * c + 1], bf16_hi(q[c]));
            }
        }
        out[idx] = make_uint4(pack_bf16(acc[0], acc[1]), pack_bf16(acc[2], acc[3]),
                              pack_bf16(acc[4], acc[5]), pack_bf16(acc[6], acc[7]));
    }
}

template <int KMAX>
cudaError_t launch_k(const moe_cfg& c, const uint16_t* y, const float* w, const int32_t* dr,
                     const uint16_t* ys, const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    const int vec = c.H / 8;
    const int64_t total = (int64_t)c.T * vec;
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = (int64_t)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    combine_kernel<KMAX><<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const uint4*>(y), w, dr, reinterpret_cast<const uint4*>(ys), mask,
        c.T, c.K, vec, reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
}

// Order-invariant variant ("From Expert Reduction to Behavioral Divergence", arXiv
// 2607.28097, Abstract: scheme C's result does not depend on the order of the expert
// terms). Per output element the terms -- w_j * y_j formed exactly in double, and the
// shared expert's y -- are put in a canonical order (ascending magnitude, the negative of
// equal magnitudes first) by an odd-even transposition network, summed in double, and
// rounded once to fp32 then to bf16. The result is a function of the multiset of terms.
__device__ __forceinline__ bool canon_after(double a, bool va, double b, bool vb)
{
    // should slot a (valid va) come after slot b? invalid slots go last
    if (!va) return vb;
    if (!vb) return false;
    const double fa = fabs(a), fb = fabs(b);
    return fa != fb ? fa > fb : a > b;
}

template <int KMAX>
__global__ void __launch_bounds__(256) combine_invariant_kernel(
    const uint4* __restrict__ y, const float* __restrict__ w, const int32_t* __restrict__ dest_row,
    const uint4* __restrict__ y_shared, const uint8_t* __restrict__ mask, int T, int K,
    int vec_per_row, uint4* __restrict__ out)
{
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
        uint32_t packed[4];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            double term[N];
            bool val[N];
#pragma unroll
            for (int j = 0; j < N; ++j) {
                const uint32_t q = (c >> 1) == 0 ? rows[j].x
                                 : (c >> 1) == 1 ? rows[j].y
                                 : (c >> 1) == 2 ? rows[j].z : rows[j].w;
                const float yv = (c & 1) ? bf16_hi(q) : bf16_lo(q);
                term[j] = __dmul_rn((double)wj[j], (double)yv);  // exact
                val[j] = ok[j];
            }
#pragma unroll
            for (int pass = 0; pass < N; ++pass) {
#pragma unroll
                for (int i = pass & 1; i + 1 < N; i += 2) {
                    if (canon_after(term[i], val[i], term[i + 1], val[i + 1])) {
                        const double td = term[i];
                        term[i] = term[i + 1];
                        term[i + 1] = td;
                        const bool tv = val[i];
                        val[i] = val[i + 1];
                        val[i + 1] = tv;
                    }
                }
            }
            double sum = 0.0;
#pragma unroll
            for (int j = 0; j < N; ++j)
                if (val[j]) sum = __dadd_rn(sum, term[j]);
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
    combine_invariant_kernel<KMAX><<<(unsigned)blocks, 256, 0, st>>>(
        reinterpret_cast<const uint4*>(y), w, dr, reinterpret_cast<const uint4*>(ys), mask,
        c.T, c.K, vec, reinterpret_cast<uint4*>(out));
    return cudaGetLastError();
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

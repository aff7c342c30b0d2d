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
    const bool narrow = total <= 0xffffffffll;  // 32-bit division of the group index
    for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < total;
         gi += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = narrow ? (int64_t)((uint32_t)gi / (uint32_t)groups_per_row)
                                 : gi / groups_per_row;
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
// Two routes to the same bits.
// - Every term has at most 32 significant bits (24 x 8), so when the nonzero terms'
//   exponents lie within 16 of each other every partial sum of up to 17 of them fits in
//   double's 53 bits exactly: any order gives the exact sum. Each thread accumulates its
//   columns this way, by fused multiply-adds (exact product, exact sum), with the bf16 value
//   widened exactly to double (building the double from the bf16 bits with integer
//   operations was 8-10 % slower: the integer pipe is the busy one). The spread is bounded
//   from the exponent fields: the weights' spread (once per token) plus the column's y
//   spread, a product's exponent being the sum of its factors' or one more, so a bound of
//   15 keeps the products within 16. The y fields are tracked two columns at a time (16x2
//   max / min), and the vector is tested as a whole before any column is.
// - Any other column (a wider bound, a zero or subnormal y under a nonzero weight, an
//   infinite or NaN y, a subnormal, infinite or NaN weight) is written with a placeholder
//   and queued in the warp's part of shared memory. When the queue fills, and once at the
//   end, the warp's lanes take one queued column each and sum it by the definition: the
//   terms sorted by the 64-bit key (|x| bits << 1) | (x is not negative) -- ascending
//   magnitude, -x before +x -- with an odd-even transposition network on integers, added
//   in that order, and the column's two bytes rewritten. Queued columns are rare in
//   practice (0.3-0.8 % of the columns of Gaussian outputs under top-8 weights), and taking
//   them out of line keeps a warp from running the sort for one lane's sake.
__device__ __forceinline__ uint64_t canon_key(double x)
{
    const uint64_t b = (uint64_t)__double_as_longlong(x);
    return ((b & 0x7fffffffffffffffull) << 1) | ((b >> 63) ^ 1ull);
}

__device__ __forceinline__ double from_key(uint64_t k)
{
    return __longlong_as_double((long long)((k >> 1) | ((~k & 1ull) << 63)));
}

// per-halfword unsigned max / min of two words (the 16x2 SIMD forms)
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t min_u16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// bf16 bits of one output column: the canonical-order double sum of its terms, rounded to
// fp32 then to bf16
template <int KMAX>
__device__ __forceinline__ uint16_t canonical_column(const uint16_t* __restrict__ y,
                                                     const float* __restrict__ w,
                                                     const int32_t* __restrict__ dest_row,
                                                     const uint16_t* __restrict__ y_shared,
                                                     int64_t t, int64_t col, int K, int H)
{
    constexpr int N = KMAX + 1;
    uint64_t key[N];
    int n_valid = 0;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        const int32_t r = (j < K) ? dest_row[t * K + j] : -1;
        key[j] = ~0ull;
        if (r >= 0) {
            const double yv = (double)__uint_as_float((uint32_t)y[(int64_t)r * H + col] << 16);
            key[j] = canon_key(__dmul_rn((double)w[t * K + j], yv));  // exact product
            ++n_valid;
        }
    }
    key[KMAX] = ~0ull;
    if (y_shared != nullptr) {
        key[KMAX] = canon_key((double)__uint_as_float((uint32_t)y_shared[t * H + col] << 16));
        ++n_valid;
    }
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
    double sum = 0.0;
#pragma unroll
    for (int j = 0; j < N; ++j)
        if (j < n_valid) sum = __dadd_rn(sum, from_key(key[j]));
    return (uint16_t)(pack_bf16(__double2float_rn(sum), 0.0f) & 0xffffu);
}

constexpr int kInvThreads = 256;
constexpr int kInvWarpQueue = 640;  // queued columns a warp holds (> one round of two vectors a lane)

// the warp's queued columns, one per lane, then an empty queue
template <int KMAX>
__device__ __forceinline__ void drain_queue(const unsigned long long* queue, int* q_count,
                                            const uint16_t* __restrict__ y,
                                            const float* __restrict__ w,
                                            const int32_t* __restrict__ dest_row,
                                            const uint16_t* __restrict__ y_shared, int K, int H,
                                            uint16_t* __restrict__ out)
{
    const int n = *q_count;
    for (int i = (int)(threadIdx.x & 31); i < n; i += 32) {
        const unsigned long long e = queue[i];  // token << 20 | column
        const int64_t t = (int64_t)(e >> 20);
        const int64_t col = (int64_t)(e & 0xfffffu);
        out[t * H + col] = canonical_column<KMAX>(y, w, dest_row, y_shared, t, col, K, H);
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) *q_count = 0;
    __syncwarp();
}

// VPT consecutive vectors of one token per thread (the token's terms prepared once for all)
template <int KMAX, int VPT>
__global__ void __launch_bounds__(kInvThreads, (KMAX <= 8 ? 4 - VPT : 1)) combine_invariant_kernel(
    const uint4* __restrict__ y, const float* __restrict__ w, const int32_t* __restrict__ dest_row,
    const uint4* __restrict__ y_shared, const uint8_t* __restrict__ mask, int T, int K,
    int vec_per_row, uint4* __restrict__ out)
{
    pdl_wait();
    constexpr int N = KMAX + 1;
    __shared__ unsigned long long queues[kInvThreads / 32][kInvWarpQueue];
    __shared__ int q_counts[kInvThreads / 32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    unsigned long long* queue = queues[wid];
    int* q_count = &q_counts[wid];
    if (lane == 0) *q_count = 0;
    __syncwarp();
    const int H = vec_per_row * 8;
    const int groups_per_row = vec_per_row / VPT;
    const int64_t total = (int64_t)T * groups_per_row;
    const bool narrow = total <= 0xffffffffll;  // 32-bit division of the group index
    // warp-uniform trip count: every lane reaches the warp's barriers of every round
    for (int64_t base = ((int64_t)blockIdx.x * (kInvThreads / 32) + wid) * 32; base < total;
         base += (int64_t)gridDim.x * kInvThreads) {
        const int64_t gi = base + lane;
        if (gi < total) {
            const int64_t t = narrow ? (int64_t)((uint32_t)gi / (uint32_t)groups_per_row)
                                     : gi / groups_per_row;
            const int v0 = (int)(gi - t * groups_per_row) * VPT;
            const int64_t idx0 = t * vec_per_row + v0;
            if (mask != nullptr && mask[t] == 0) {
#pragma unroll
                for (int u = 0; u < VPT; ++u) out[idx0 + u] = make_uint4(0u, 0u, 0u, 0u);
            } else {
                uint4 rows[VPT][N];
                double wd[N];  // the weights, exactly (0 for a missing term)
                uint32_t livem = 0u;  // terms with a nonzero weight
                int ew_max = 0, ew_min = 255;
                bool w_ok = true;  // no present weight is subnormal, infinite or NaN
#pragma unroll
                for (int j = 0; j < KMAX; ++j) {
                    const int32_t r = (j < K) ? dest_row[t * K + j] : -1;
                    const float wv = r >= 0 ? w[t * K + j] : 0.0f;
#pragma unroll
                    for (int u = 0; u < VPT; ++u)
                        rows[u][j] = r >= 0 ? y[(int64_t)r * vec_per_row + v0 + u]
                                            : make_uint4(0u, 0u, 0u, 0u);
                    wd[j] = (double)wv;
                    const uint32_t wa = __float_as_uint(wv) & 0x7fffffffu;
                    const int ew = (int)(wa >> 23);
                    if (wa != 0u) {
                        livem |= 1u << j;
                        ew_max = ew > ew_max ? ew : ew_max;
                        ew_min = ew < ew_min ? ew : ew_min;
                        if (wa < 0x00800000u || wa >= 0x7f800000u) w_ok = false;
                    }
                }
                if (y_shared != nullptr) {
#pragma unroll
                    for (int u = 0; u < VPT; ++u) rows[u][KMAX] = y_shared[idx0 + u];
                    wd[KMAX] = 1.0;
                    livem |= 1u << KMAX;
                    ew_max = 127 > ew_max ? 127 : ew_max;
                    ew_min = 127 < ew_min ? 127 : ew_min;
                } else {
#pragma unroll
                    for (int u = 0; u < VPT; ++u) rows[u][KMAX] = make_uint4(0u, 0u, 0u, 0u);
                    wd[KMAX] = 0.0;
                }
                const int w_spread = ew_max >= ew_min ? ew_max - ew_min : 0;
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    // column pairs: column 2p is the low half of word p of each row, 2p + 1
                    // the high half; |y| bits are tracked per half, two columns per instruction
                    float f[8];
                    uint32_t a_max2[4], a_min2[4];  // per half: largest |y| bits of any term,
                                                    // smallest under a nonzero weight
#pragma unroll
                    for (int pw = 0; pw < 4; ++pw) {
                        double s0 = 0.0, s1 = 0.0;
                        uint32_t amx = 0u, amn = 0x7fff7fffu;
#pragma unroll
                        for (int j = 0; j < N; ++j) {
                            const uint32_t q = pw == 0 ? rows[u][j].x
                                             : pw == 1 ? rows[u][j].y
                                             : pw == 2 ? rows[u][j].z : rows[u][j].w;
                            const uint32_t a2 = q & 0x7fff7fffu;
                            amx = max_u16x2(amx, a2);
                            amn = min_u16x2(amn, ((livem >> j) & 1u) ? a2 : 0x7fff7fffu);
                            // each bf16 as its fp32 value, widened exactly to double (the
                            // conversion leaves the busier integer pipe alone)
                            s0 = __fma_rn(wd[j], (double)__uint_as_float(q << 16), s0);
                            s1 = __fma_rn(wd[j], (double)__uint_as_float(q & 0xffff0000u), s1);
                        }
                        a_max2[pw] = amx;
                        a_min2[pw] = amn;
                        f[2 * pw] = __double2float_rn(s0);
                        f[2 * pw + 1] = __double2float_rn(s1);
                    }
                    out[idx0 + u] = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]),
                                               pack_bf16(f[4], f[5]), pack_bf16(f[6], f[7]));
                    // the whole vector first (per half: exponent spread + 256, no borrow
                    // between halves); per column only when some column fails
                    uint32_t mx = 0u, mn = 0x7fff7fffu, sp = 0u;
#pragma unroll
                    for (int pw = 0; pw < 4; ++pw) {
                        mx = max_u16x2(mx, a_max2[pw]);
                        mn = min_u16x2(mn, a_min2[pw]);
                        sp = max_u16x2(sp, ((a_max2[pw] >> 7) & 0x00ff00ffu) + 0x01000100u -
                                               ((a_min2[pw] >> 7) & 0x00ff00ffu));
                    }
                    const uint32_t mx1 = max(mx & 0xffffu, mx >> 16);
                    const uint32_t mn1 = min(mn & 0xffffu, mn >> 16);
                    const int sp1 = (int)max(sp & 0xffffu, sp >> 16) - 256;
                    if (!w_ok || mx1 >= 0x7f80u || mn1 < 0x80u || w_spread + sp1 > 15) {
                        uint32_t slow = 0u;  // columns for the queue
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const uint32_t a_max = (a_max2[c >> 1] >> (16 * (c & 1))) & 0xffffu;
                            const uint32_t a_min = (a_min2[c >> 1] >> (16 * (c & 1))) & 0xffffu;
                            const int y_spread = (int)(a_max >> 7) - (int)(a_min >> 7);
                            if (!w_ok || a_max >= 0x7f80u || a_min < 0x80u ||
                                w_spread + y_spread > 15)
                                slow |= 1u << c;
                        }
                        int k = atomicAdd(q_count, __popc(slow));
                        for (int c = 0; c < 8; ++c)
                            if ((slow >> c) & 1u)
                                queue[k++] = ((unsigned long long)t << 20) |
                                             (unsigned)((v0 + u) * 8 + c);
                    }
                }
            }
        }
        __syncwarp();
        const int queued = *q_count;
        __syncwarp();  // every lane has read the count before the next round adds to it
        // a round adds at most 32 * VPT * 8 columns: drain before the queue could overflow
        if (queued > kInvWarpQueue - 32 * VPT * 8)
            drain_queue<KMAX>(queue, q_count, reinterpret_cast<const uint16_t*>(y), w, dest_row,
                              reinterpret_cast<const uint16_t*>(y_shared), K, H,
                              reinterpret_cast<uint16_t*>(out));
    }
    drain_queue<KMAX>(queue, q_count, reinterpret_cast<const uint16_t*>(y), w, dest_row,
                      reinterpret_cast<const uint16_t*>(y_shared), K, H,
                      reinterpret_cast<uint16_t*>(out));
}

// vectors per thread of the order-invariant combine: 2 for up to two terms (measured: 70.8
// against 81.1 us for top-1 at T = 8192, H = 4096), 1 above (two vectors of 7 or 9 rows
// lower the occupancy more than they save: 311 against 275 us for top-8 at T = 16384)
template <int KMAX>
constexpr int inv_vpt()
{
    return KMAX <= 2 ? 2 : 1;
}

template <int KMAX>
cudaError_t launch_inv(const moe_cfg& c, const uint16_t* y, const float* w, const int32_t* dr,
                       const uint16_t* ys, const uint8_t* mask, uint16_t* out, cudaStream_t st)
{
    constexpr int VPT = inv_vpt<KMAX>();
    const int vec = c.H / 8;  // a multiple of 16, so of VPT
    const int64_t total = (int64_t)c.T * (vec / VPT);
    int64_t blocks = (total + kInvThreads - 1) / kInvThreads;
    const int64_t cap = resident_blocks((const void*)combine_invariant_kernel<KMAX, VPT>,
                                        kInvThreads, 0);
    if (blocks > cap) blocks = cap;
    return launch_pdl(combine_invariant_kernel<KMAX, VPT>, dim3((unsigned)blocks),
                      dim3(kInvThreads), 0, st, reinterpret_cast<const uint4*>(y), w, dr,
                      reinterpret_cast<const uint4*>(ys), mask, c.T, c.K, vec,
                      reinterpret_cast<uint4*>(out));
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

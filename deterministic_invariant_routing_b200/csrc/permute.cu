// Dispatch kernels: a stable counting sort of the T*K (token, rank) assignments by
// expert, and the row gather x_perm[r] = x[perm_token[r]].
//
// "DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 2: the dispatch boundary
// is the token-to-expert map plus the valid token counts. The sort is stable in the flat
// assignment index a = t*K + j, so the row of every assignment is unique and does not
// depend on how the work is split over blocks and warps.
//
// Three launches: per-block expert histograms -> one-block scan (expert offsets and each
// block's base row per expert) -> placement (per-warp ranks from __match_any_sync in
// assignment order). All integer, no floating point, no order-dependent atomics (the
// only atomics are shared-memory histogram increments, whose sum is order-free).
#include "moe_internal.cuh"

namespace moe {

// Fixed scratch of moe_permute_noalloc: the per-block expert histograms live in this
// file-scope device array instead of a caller workspace. Every GPU that loads the
// library holds it (1 MiB) until the process exits; all calls share it, and calls that
// overlap on the GPU race on it.
static __device__ __align__(256) int32_t g_permute_scratch[kPermuteFixedScratchInts];

namespace {

constexpr int kWarps = 8;                // warps per block
constexpr int kPerWarp = 256;            // assignments per warp (8 rounds of 32)
constexpr int kChunk = kWarps * kPerWarp;  // assignments per block

__device__ __forceinline__ int expert_of(const int32_t* ids, int64_t a, int64_t A, int E)
{
    if (a >= A) return -1;
    const int e = ids[a];
    return (e >= 0 && e < E) ? e : -1;
}

// counts[b][e] = routed assignments of expert e in block b's chunk
__global__ void __launch_bounds__(kWarps * 32) hist_kernel(const int32_t* __restrict__ ids,
                                                           int64_t A, int E,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* status)
{
    pdl_wait();
    extern __shared__ int32_t sh[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kChunk;
    int bad = 0;
    // all of this thread's ids are loaded before any is counted (independent loads in flight)
    constexpr int kPer = kChunk / (kWarps * 32);
    int ev[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int64_t a = base + threadIdx.x + (int64_t)q * blockDim.x;
        ev[q] = a < A ? ids[a] : -1;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int e = ev[q];
        if (e >= 0 && e < E) atomicAdd(&sh[e], 1);
        else if (e >= E) ++bad;
    }
    status_add(status, MOE_ST_BAD_EXPERT_ID, bad);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) counts[(int64_t)blockIdx.x * E + e] = sh[e];
}

// offsets[e] = exclusive scan of the expert totals; counts[b][e] becomes block b's first
// row for expert e. One block of 1024 threads, thread e owns expert e (E <= 1024).
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ counts, int nblocks,
                                                    int E, int32_t* __restrict__ offsets)
{
    pdl_wait();
    __shared__ int32_t warp_tot[32];
    const int e = threadIdx.x;
    int32_t total = 0;
    // eight blocks' counts loaded at a time (independent loads in flight)
    if (e < E) {
        int b = 0;
        for (; b + 8 <= nblocks; b += 8) {
            int32_t c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) c[q] = counts[(int64_t)(b + q) * E + e];
#pragma unroll
            for (int q = 0; q < 8; ++q) total += c[q];
        }
        for (; b < nblocks; ++b) total += counts[(int64_t)b * E + e];
    }
    // block-wide exclusive scan of total over e
    const int lane = e & 31, wid = e >> 5;
    int32_t incl = total;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int32_t v = warp_tot[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int32_t o = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += o;
        }
        warp_tot[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    const int32_t excl = incl - total + (wid > 0 ? warp_tot[wid - 1] : 0);
    if (e < E) {
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + total;
        int32_t run = excl;
        int b = 0;
        for (; b + 8 <= nblocks; b += 8) {
            int32_t c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) c[q] = counts[(int64_t)(b + q) * E + e];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                counts[(int64_t)(b + q) * E + e] = run;
                run += c[q];
            }
        }
        for (; b < nblocks; ++b) {
            const int32_t c = counts[(int64_t)b * E + e];
            counts[(int64_t)b * E + e] = run;
            run += c;
        }
    }
}

// dest_row[a] and perm_token[row]: block b handles assignments [b*kChunk, (b+1)*kChunk),
// warp w the kPerWarp consecutive ones starting at w*kPerWarp, in rounds of 32 in
// increasing a.
__global__ void __launch_bounds__(kWarps * 32) place_kernel(const int32_t* __restrict__ ids,
                                                            int64_t A, int K, int E,
                                                            const int32_t* __restrict__ block_base,
                                                            int32_t* __restrict__ dest_row,
                                                            int32_t* __restrict__ perm_token)
{
    pdl_wait();
    extern __shared__ int32_t wbase[];  // [kWarps][E]
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) wbase[i] = 0;
    __syncthreads();
    const int64_t wstart = (int64_t)blockIdx.x * kChunk + (int64_t)wid * kPerWarp;
    // this lane's expert of every round, loaded once up front (independent loads in flight)
    constexpr int kRounds = kPerWarp / 32;
    int ev[kRounds];
#pragma unroll
    for (int q = 0; q < kRounds; ++q) ev[q] = expert_of(ids, wstart + 32 * q + lane, A, E);
    // pass 1: per-warp counts
#pragma unroll
    for (int q = 0; q < kRounds; ++q)
        if (ev[q] >= 0) atomicAdd(&wbase[wid * E + ev[q]], 1);
    __syncthreads();
    // per expert: scan over warps, seeded with the block's base row
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int32_t run = block_base[(int64_t)blockIdx.x * E + e];
        for (int w2 = 0; w2 < kWarps; ++w2) {
            const int32_t c = wbase[w2 * E + e];
            wbase[w2 * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    // pass 2: ranks within each round of 32 from the peer masks, rounds in order
    const unsigned lt_mask = (1u << lane) - 1u;
    int32_t* my = wbase + wid * E;
#pragma unroll
    for (int q = 0; q < kRounds; ++q) {
        const int64_t a = wstart + 32 * q + lane;
        const int e = ev[q];
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        int32_t row = -1;
        if (e >= 0) row = my[e] + __popc(peers & lt_mask);
        __syncwarp();
        if (e >= 0 && (peers & lt_mask) == 0) my[e] += __popc(peers);
        __syncwarp();
        if (a < A) {
            dest_row[a] = row;
            if (row >= 0) perm_token[row] = (int32_t)(a / K);
        }
    }
}

// x_perm[dest_row[t, j], :] = x[t, :] for every routed (t, j): one warp per token, which
// reads the token's row once (8 vectors of 16 B per lane in flight) and writes its K
// copies -- token-major, so each row of x leaves DRAM once.
__global__ void __launch_bounds__(256) gather_kernel(const uint4* __restrict__ x,
                                                     const int32_t* __restrict__ dest_row, int T,
                                                     int K, int vec_per_row,
                                                     uint4* __restrict__ x_perm)
{
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int64_t wpb = blockDim.x >> 5;
    for (int64_t t = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); t < T;
         t += (int64_t)gridDim.x * wpb) {
        const int32_t my_dest = lane < K ? dest_row[t * K + lane] : -1;
        const uint4* src = x + t * vec_per_row;
        for (int v0 = lane; v0 < vec_per_row; v0 += 32 * 8) {
            uint4 buf[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (v0 + 32 * u < vec_per_row) buf[u] = src[v0 + 32 * u];
            for (int j = 0; j < K; ++j) {
                const int32_t d = __shfl_sync(0xffffffffu, my_dest, j);
                if (d < 0) continue;
                uint4* dst = x_perm + (int64_t)d * vec_per_row;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (v0 + 32 * u < vec_per_row) dst[v0 + 32 * u] = buf[u];
            }
        }
    }
}

}  // namespace

size_t permute_ws_bytes(const moe_cfg& c)
{
    const int64_t A = (int64_t)c.T * c.K;
    const int64_t nb = (A + kChunk - 1) / kChunk;
    return (size_t)(nb > 0 ? nb : 1) * (size_t)c.E * sizeof(int32_t);
}

cudaError_t launch_permute(const moe_cfg& c, const int32_t* ids, int32_t* offsets,
                           int32_t* perm_token, int32_t* dest_row, int32_t* status, void* ws,
                           cudaStream_t st)
{
    const int64_t A = (int64_t)c.T * c.K;
    const int nb = (int)((A + kChunk - 1) / kChunk);
    int32_t* counts = static_cast<int32_t*>(ws);
    if (nb > 0) {
        if (const cudaError_t e = launch_pdl(hist_kernel, dim3(nb), dim3(kWarps * 32),
                                             c.E * sizeof(int32_t), st, ids, A, c.E, counts,
                                             status); e != cudaSuccess) return e;
    }
    if (const cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, st, counts, nb, c.E,
                                         offsets); e != cudaSuccess) return e;
    if (nb > 0) {
        const size_t smem = (size_t)kWarps * c.E * sizeof(int32_t);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(place_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
        }
        if (const cudaError_t e = launch_pdl(place_kernel, dim3(nb), dim3(kWarps * 32), smem, st,
                                             ids, A, c.K, c.E, counts, dest_row,
                                             perm_token); e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t permute_fixed_scratch(int32_t** out)
{
    // In host code g_permute_scratch is only a stand-in symbol, not a device address. The
    // runtime is asked for the address on every call, with the caller's device current: a
    // host-side lookup that allocates nothing, and that stays right when a device reset or
    // a new primary context has moved the module since the previous call (a cached address
    // would then point at freed memory).
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_permute_scratch);
    if (e != cudaSuccess) return e;
    *out = static_cast<int32_t*>(p);
    return cudaSuccess;
}

cudaError_t launch_gather_rows(const moe_cfg& c, const uint16_t* x, const int32_t* dest_row,
                               uint16_t* x_perm, cudaStream_t st)
{
    if (c.T == 0) return cudaSuccess;
    const int vec = c.H / 8;
    int64_t blocks = ((int64_t)c.T + 7) / 8;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    return launch_pdl(gather_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(x), dest_row, c.T, c.K, vec,
                      reinterpret_cast<uint4*>(x_perm));
}

}  // namespace moe

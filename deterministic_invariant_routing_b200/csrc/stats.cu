// Router statistics of one routed batch (SpecForge PR #1003, the load-balance commit): the
// tokens per expert, the mean L1-normalised score per expert and the Switch-style
// load-balance value  aux = E * sum_e load_e * mean_prob_e  over the kept tokens (K when
// balanced), where load_e = tokens_per_expert_e / N and p_{t,e} = s_{t,e} / sum_e' s_{t,e'}
// with s the unbiased scores of the routing contract (softmax, sigmoid or sqrtsoftplus).
//
// Deterministic without float atomics: block b owns 64 consecutive tokens, warp w of it 8
// of them (32 and 4 above 128 experts), summed in token order into per-lane registers (lane
// L holds experts L, L+32, ...); the 8 warp partials are added in warp order, then the block
// partials by the finishing kernel in a fixed order (contiguous slices of blocks in block
// order, then the slices in order), and aux is a fixed tree over the experts. The result
// depends on T and E (a batch statistic), never on scheduling.
#include "route_math.cuh"

namespace moe {
namespace {

// tokens per warp: 8 up to 128 experts (their rows are loaded ahead, so a warp has enough
// loads in flight), 4 above (more warps; measured 36.6 -> 26.2 us at 256 experts, T = 8192,
// and slower at 128 experts: 25.1 -> 28.9 us at T = 16384)
__host__ __device__ constexpr int tok_per_warp(int ne) { return ne <= 4 ? 8 : 4; }
constexpr int kWarps = 8;

template <int NE>
__global__ void __launch_bounds__(kWarps * 32) prob_sum_kernel(const float* __restrict__ logits,
                                                               const uint8_t* __restrict__ mask,
                                                               int T, int E, int score_fn,
                                                               float* __restrict__ partial,
                                                               int32_t* __restrict__ kept)
{
    pdl_wait();
    extern __shared__ float wsum[];  // [kWarps][E]
    __shared__ int32_t wkept[kWarps];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    float acc[NE];
#pragma unroll
    for (int i = 0; i < NE; ++i) acc[i] = 0.0f;
    int n_kept = 0;
    constexpr int kTokPerWarp = tok_per_warp(NE);
    const int64_t t0 = (int64_t)blockIdx.x * (kWarps * kTokPerWarp) + (int64_t)wid * kTokPerWarp;
    // up to 128 experts the warp's rows are loaded before the first is scored (independent
    // loads in flight); the tokens are still added in order
    constexpr int kPre = NE <= 4 ? kTokPerWarp : 1;
    float pre[kPre][NE];
    if constexpr (kPre > 1) {
#pragma unroll
        for (int r = 0; r < kPre; ++r) {
            const int64_t t = t0 + r;
            const bool live = t < T && (mask == nullptr || mask[t] != 0);
            if (live) load_row<NE>(logits + t * E, E, lane, pre[r]);
        }
    }
#pragma unroll
    for (int r = 0; r < kTokPerWarp; ++r) {
        const int64_t t = t0 + r;
        if (t >= T) break;
        if (mask != nullptr && mask[t] == 0) continue;
        ++n_kept;
        float s[NE];
        if constexpr (kPre > 1) {
#pragma unroll
            for (int i = 0; i < NE; ++i) s[i] = pre[r][i];
        } else {
            load_row<NE>(logits + t * E, E, lane, s);
        }
        contract_scores_of<NE>(E, score_fn, lane, s);
        // L1 normalisation over the experts with the same 32-lane tree
        float l1 = 0.0f;
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (lane + 32 * i < E) l1 = __fadd_rn(l1, s[i]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            l1 = __fadd_rn(l1, __shfl_xor_sync(0xffffffffu, l1, off));
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (lane + 32 * i < E) acc[i] = __fadd_rn(acc[i], __fdiv_rn(s[i], l1));
    }
#pragma unroll
    for (int i = 0; i < NE; ++i) {
        const int e = lane + 32 * i;
        if (e < E) wsum[wid * E + e] = acc[i];
    }
    if (lane == 0) wkept[wid] = n_kept;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float v = wsum[e];
        for (int w = 1; w < kWarps; ++w) v = __fadd_rn(v, wsum[w * E + e]);
        partial[(int64_t)blockIdx.x * E + e] = v;
    }
    if (threadIdx.x == 0) {
        int k = 0;
        for (int w = 0; w < kWarps; ++w) k += wkept[w];
        kept[blockIdx.x] = k;
    }
}

// One block of 1024 threads. The block partials of expert e are summed in S contiguous
// slices of blocks (S = the largest power of two <= 8 with S * E <= 1024; thread
// s * E + e sums slice s in block order), then the S slice sums in slice order by thread e;
// the kept-token count is an integer sum.
__global__ void __launch_bounds__(1024) stats_finish_kernel(const float* __restrict__ partial,
                                                            const int32_t* __restrict__ kept,
                                                            int nblocks, int E,
                                                            const int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ counts,
                                                            float* __restrict__ mean_prob,
                                                            float* __restrict__ aux)
{
    pdl_wait();
    __shared__ float wsum[32];
    __shared__ float slice_sum[1024];
    __shared__ unsigned long long n_kept;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    if (tid == 0) n_kept = 0ull;
    __syncthreads();
    {
        unsigned long long k = 0ull;
        for (int b = tid; b < nblocks; b += blockDim.x) k += (unsigned long long)kept[b];
        if (k != 0ull) atomicAdd(&n_kept, k);
    }
    int S = 1;
    while (S < 8 && 2 * S * E <= (int)blockDim.x) S *= 2;
    const int per = (nblocks + S - 1) / S;
    if (tid < S * E) {
        const int e = tid % E, sl = tid / E;
        const int b0 = sl * per, b1 = min(nblocks, b0 + per);
        float v = 0.0f;
        int b = b0;
        // eight blocks' values loaded at a time (independent loads in flight), added in order
        for (; b + 8 <= b1; b += 8) {
            float pv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) pv[q] = partial[(int64_t)(b + q) * E + e];
#pragma unroll
            for (int q = 0; q < 8; ++q) v = __fadd_rn(v, pv[q]);
        }
        for (; b < b1; ++b) v = __fadd_rn(v, partial[(int64_t)b * E + e]);
        slice_sum[tid] = v;
    }
    __syncthreads();
    const int64_t n = (int64_t)n_kept;
    const int e = tid;
    float term = 0.0f;
    if (e < E) {
        float v = slice_sum[e];
        for (int sl = 1; sl < S; ++sl) v = __fadd_rn(v, slice_sum[sl * E + e]);
        const int32_t c = offsets[e + 1] - offsets[e];
        counts[e] = c;
        const float nf = (float)n;
        const float mp = n > 0 ? __fdiv_rn(v, nf) : 0.0f;
        mean_prob[e] = mp;
        term = n > 0 ? __fmul_rn(__fdiv_rn((float)c, nf), mp) : 0.0f;
    }
    // fixed tree over the experts: warp butterfly, then the 32 warp sums in order
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
        term = __fadd_rn(term, __shfl_xor_sync(0xffffffffu, term, off));
    if (lane == 0) wsum[wid] = term;
    __syncthreads();
    if (e == 0) {
        float s = 0.0f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s = __fadd_rn(s, wsum[w]);
        *aux = __fmul_rn((float)E, s);
    }
}

template <int NE>
cudaError_t launch_ne(const moe_cfg& c, const float* logits, const uint8_t* mask, float* partial,
                      int32_t* kept, int nb, cudaStream_t st)
{
    const size_t smem = (size_t)kWarps * c.E * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(prob_sum_kernel<NE>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(prob_sum_kernel<NE>, dim3(nb), dim3(kWarps * 32), smem, st, logits, mask, c.T,
                      c.E, c.score_fn, partial, kept);
}

}  // namespace

size_t stats_ws_bytes(const moe_cfg& c)
{
    const int tpb = kWarps * tok_per_warp((c.E + 31) / 32);
    const int64_t nb = ((int64_t)c.T + tpb - 1) / tpb;
    const int64_t n = nb > 0 ? nb : 1;
    return (size_t)n * c.E * sizeof(float) + (size_t)n * sizeof(int32_t) + 256;
}

cudaError_t launch_router_stats(const moe_cfg& c, const float* logits, const uint8_t* mask,
                                const int32_t* offsets, int32_t* counts, float* mean_prob,
                                float* aux, void* ws, cudaStream_t st)
{
    const int tpb = kWarps * tok_per_warp((c.E + 31) / 32);
    const int nb = (int)(((int64_t)c.T + tpb - 1) / tpb);
    float* partial = static_cast<float*>(ws);
    int32_t* kept = reinterpret_cast<int32_t*>(
        static_cast<char*>(ws) + (size_t)(nb > 0 ? nb : 1) * c.E * sizeof(float));
    cudaError_t err = cudaSuccess;
    if (nb > 0) {
        const int ne = (c.E + 31) / 32;
        if (ne <= 1) err = launch_ne<1>(c, logits, mask, partial, kept, nb, st);
        else if (ne <= 2) err = launch_ne<2>(c, logits, mask, partial, kept, nb, st);
        else if (ne <= 4) err = launch_ne<4>(c, logits, mask, partial, kept, nb, st);
        else if (ne <= 8) err = launch_ne<8>(c, logits, mask, partial, kept, nb, st);
        else if (ne <= 16) err = launch_ne<16>(c, logits, mask, partial, kept, nb, st);
        else err = launch_ne<32>(c, logits, mask, partial, kept, nb, st);
        if (err != cudaSuccess) return err;
    }
    return launch_pdl(stats_finish_kernel, dim3(1), dim3(1024), 0, st, partial, kept, nb, c.E,
                      offsets, counts, mean_prob, aux);
}

}  // namespace moe

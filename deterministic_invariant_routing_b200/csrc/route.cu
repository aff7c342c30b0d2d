// Routing kernel: scores, selection and weights of each token, one warp per token.
//
// Follows the routing contract of "DSV4 Flash MoE Train-Inference Consistency Roadmap"
// (Problem 1: logits -> top-k ids and weights with a fixed tie rule and expert bias) and
// SpecForge PR #1003 (the selection bias moves the picks, the weights come from the
// unbiased scores; norm_topk_prob renormalisation; route_scale for the DeepSeek seam).
//
// FP32 contract, bit-exact by construction: every add, multiply and divide is an
// explicit round-to-nearest intrinsic (no contraction); the exponential is exp_rl;
// the softmax denominator is the 32-lane tree (lane L sums experts L, L+32, ... in
// increasing order, then butterfly levels 16, 8, 4, 2, 1); the selection compares
// 64-bit keys (ordered choice bits, then inverted id), so ties go to the lower id.
//
// Group-limited selection (n_group > 1, the DeepSeek family's override of the selection
// named in SpecForge PR #1003): the warp stages the token's choice values in shared
// memory, lane g scans group g in expert order for its two best keys and scores the group
// by their fp32 sum, topk_group warp arg-max rounds over the group keys pick the kept
// groups, and the experts of the other groups get key 0 before the K selection rounds.
#include "route_math.cuh"

namespace moe {
namespace {

__device__ __forceinline__ unsigned long long select_key(float c, int id)
{
    return ((unsigned long long)order_bits(c) << 32) |
           (unsigned long long)(0xffffffffu - (uint32_t)id);
}

// warp arg-max of 64-bit keys as two 32-bit reductions: the highest choice bits, then,
// among the lanes holding them, the highest inverted id; returns the id
__device__ __forceinline__ int warp_argmax_id(unsigned long long k)
{
    const uint32_t hi = (uint32_t)(k >> 32), lo = (uint32_t)k;
    const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
    const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
    return (int)(0xffffffffu - mlo);
}

// descending sort of a lane's keys: the optimal 5-exchange network for 4, odd-even
// transposition otherwise (the order of equal keys cannot matter: keys are distinct)
template <int NE, typename Key>
__device__ __forceinline__ void sort_desc(Key (&key)[NE])
{
    auto cx = [&](int a, int b) {
        const Key ka = key[a], kb = key[b];
        const bool swap = ka < kb;
        key[a] = swap ? kb : ka;
        key[b] = swap ? ka : kb;
    };
    if constexpr (NE == 4) {
        cx(0, 1);
        cx(2, 3);
        cx(0, 2);
        cx(1, 3);
        cx(1, 2);
    } else {
#pragma unroll
        for (int pass = 0; pass < NE; ++pass) {
#pragma unroll
            for (int i = pass & 1; i + 1 < NE; i += 2) cx(i, i + 1);
        }
    }
}

// Selection of the K best keys of a warp whose lanes hold NE keys each, sorted descending
// in every lane: K rounds of a warp arg-max over the lanes' heads, the winner dropping its
// head. Lane j (j < K) returns the key of round j; for 32-bit keys *boundary receives the
// best key left over.
template <int NE, int KT, typename Key>
__device__ __forceinline__ Key select_rounds(Key (&key)[NE], int K, int lane, Key* boundary)
{
    Key mine = 0;
#pragma unroll
    for (int j = 0; j < (KT > 0 ? KT : K); ++j) {
        Key m;
        if constexpr (sizeof(Key) == 8) {
            const uint32_t hi = (uint32_t)(key[0] >> 32), lo = (uint32_t)key[0];
            const uint32_t mhi = __reduce_max_sync(0xffffffffu, hi);
            const uint32_t mlo = __reduce_max_sync(0xffffffffu, hi == mhi ? lo : 0u);
            m = ((Key)mhi << 32) | mlo;
        } else {
            m = __reduce_max_sync(0xffffffffu, key[0]);
        }
        if (key[0] == m) {
#pragma unroll
            for (int i = 0; i + 1 < NE; ++i) key[i] = key[i + 1];
            key[NE - 1] = 0;
        }
        if (lane == j) mine = m;
    }
    if constexpr (sizeof(Key) == 4)
        if (boundary != nullptr) *boundary = __reduce_max_sync(0xffffffffu, key[0]);
    return mine;
}

// NE = experts held per lane (E <= 32 * NE); KT = K when fixed at compile time, else 0.
//
// Selection. The exact key of expert e is the 64-bit (ordered choice bits, inverted id).
// The common path selects on 32-bit keys that keep the top 32 - B choice bits and put the
// inverted id in the low B bits (2^B > 32 NE, so every real key is nonzero): one reduction
// per round instead of two, and half the data to sort and shift. Cutting choice bits keeps
// the order of any two keys whose kept bits differ; the cut selection equals the exact one
// when the kept bits of the picks in rank order, followed by the best key left over, are
// strictly decreasing -- then each pick beats everything after it on the kept bits alone.
// A token where two neighbours of that sequence share their kept bits (near-ties, equal
// scores, NaN rows) is selected again on the exact 64-bit keys. Both paths give the same ids.
template <int NE, int KT>
__global__ void __launch_bounds__(256, (NE <= 4 ? 6 : 1)) route_kernel(const float* __restrict__ logits, int T, int E,
                                                    int K, const float* __restrict__ sel_bias,
                                                    const uint8_t* __restrict__ mask, int score_fn,
                                                    int renorm, float route_scale,
                                                    int n_group, int topk_group,
                                                    int32_t* __restrict__ ids,
                                                    float* __restrict__ w, int32_t* status)
{
    constexpr int kIdBits = NE <= 1 ? 6 : NE <= 2 ? 7 : NE <= 4 ? 8 : NE <= 8 ? 9 : NE <= 16 ? 10 : 11;
    constexpr uint32_t kIdMask = (1u << kIdBits) - 1u;  // > every id (ids < 32 NE)
    static_assert((1 << kIdBits) > 32 * NE, "cut keys need room for every id");
    pdl_wait();
    if (KT > 0) K = KT;
    extern __shared__ float choice_smem[];  // [warps][E], group-limited selection only
    const int lane = threadIdx.x & 31;
    float* cw = choice_smem + (threadIdx.x >> 5) * E;
    const int warps_per_block = blockDim.x >> 5;
    int nan_tokens = 0, zero_den = 0;
    for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < T;
         t += gridDim.x * warps_per_block) {
        if (mask != nullptr && mask[t] == 0) {
            if (lane < K) {
                ids[(int64_t)t * K + lane] = -1;
                w[(int64_t)t * K + lane] = 0.0f;
            }
            continue;
        }
        float s[NE];
        contract_scores<NE>(logits + (int64_t)t * E, E, score_fn, lane, s);
        // choice values (empty slots are never keyed) and the cut keys
        auto choice = [&](int i) -> float {
            const int e = lane + 32 * i;
            return sel_bias != nullptr ? __fadd_rn(s[i], sel_bias[e]) : s[i];
        };
        uint32_t ck[NE];
        bool any_nan = false;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
            if (e < E) {
                const float c = choice(i);
                any_nan |= isnan(c);
                ck[i] = (order_bits(c) & ~kIdMask) | (kIdMask - (uint32_t)e);
                if (n_group > 1) cw[e] = c;
            } else {
                ck[i] = 0u;
            }
        }
        if (__any_sync(0xffffffffu, any_nan)) nan_tokens += (lane == 0);
        uint32_t kept = 0xffffffffu;  // group-limited selection: the kept groups
        int gs = 1;
        if (n_group > 1) {
            __syncwarp();
            gs = E / n_group;
            unsigned long long gk = 0ull;
            if (lane < n_group) {
                unsigned long long k1 = 0ull, k2 = 0ull;
                float c1 = 0.0f, c2 = 0.0f;
                for (int e = lane * gs; e < (lane + 1) * gs; ++e) {
                    const float c = cw[e];
                    const unsigned long long k = select_key(c, e);
                    if (k > k1) { k2 = k1; c2 = c1; k1 = k; c1 = c; }
                    else if (k > k2) { k2 = k; c2 = c; }
                }
                gk = select_key(gs > 1 ? __fadd_rn(c1, c2) : c1, lane);
            }
            __syncwarp();  // the scan is done before the next token overwrites cw
            kept = 0u;
            for (int r = 0; r < topk_group; ++r) {
                const int g = warp_argmax_id(gk);
                kept |= 1u << g;
                if (lane == g) gk = 0ull;
            }
#pragma unroll
            for (int i = 0; i < NE; ++i) {
                const int e = lane + 32 * i;
                if (e < E && ((kept >> (e / gs)) & 1u) == 0u) ck[i] = 0u;
            }
        }
        // cut-key selection, then the strict-decrease test of the kept bits (lane j holds
        // the key of round j; the best key left over is the boundary)
        sort_desc<NE>(ck);
        uint32_t bnd;
        const uint32_t mk = select_rounds<NE, KT>(ck, K, lane, &bnd);
        const uint32_t top = mk & ~kIdMask;
        const uint32_t nxt_lane = __shfl_down_sync(0xffffffffu, top, 1);
        const uint32_t nxt = (lane == K - 1) ? (bnd & ~kIdMask) : nxt_lane;
        int my_id = (int)(kIdMask - (mk & kIdMask));
        if (__any_sync(0xffffffffu, lane < K && top == nxt)) {
            // exact selection on the 64-bit keys
            unsigned long long key[NE];
#pragma unroll
            for (int i = 0; i < NE; ++i) {
                const int e = lane + 32 * i;
                const bool live = e < E && (n_group <= 1 || ((kept >> (e / gs)) & 1u) != 0u);
                key[i] = live ? select_key(choice(i), e) : 0ull;
            }
            sort_desc<NE>(key);
            const unsigned long long m = select_rounds<NE, KT>(key, K, lane, static_cast<unsigned long long*>(nullptr));
            my_id = (int)(0xffffffffu - (uint32_t)m);
        }
        // the unbiased score of this lane's pick: slot my_id / 32 of lane my_id % 32
        float my_s = 0.0f;
        {
            const int src = my_id & 31, slot = my_id >> 5;
#pragma unroll
            for (int i = 0; i < NE; ++i) {
                const float v = __shfl_sync(0xffffffffu, s[i], src);
                if (i == slot) my_s = v;
            }
        }
        // renormalisation denominator: the picks' scores added in rank order
        float den = __shfl_sync(0xffffffffu, my_s, 0);
#pragma unroll
        for (int j = 1; j < (KT > 0 ? KT : K); ++j)
            den = __fadd_rn(den, __shfl_sync(0xffffffffu, my_s, j));
        if (renorm && den == 0.0f) zero_den += (lane == 0);
        if (lane < K) {
            float wv;
            if (renorm)
                wv = (den == 0.0f) ? 0.0f : __fmul_rn(__fdiv_rn(my_s, den), route_scale);
            else
                wv = __fmul_rn(my_s, route_scale);
            ids[(int64_t)t * K + lane] = my_id;
            w[(int64_t)t * K + lane] = wv;
        }
    }
    if (lane == 0) {
        status_add(status, MOE_ST_NAN_TOKENS, nan_tokens);
        status_add(status, MOE_ST_ZERO_DENOM, zero_den);
    }
}

template <int NE, int KT>
cudaError_t launch_nk(const moe_cfg& c, const float* logits, const float* sel_bias,
                      const uint8_t* mask, int32_t* ids, float* w, int32_t* status,
                      cudaStream_t st)
{
    const int threads = 256, wpb = threads / 32;
    int blocks = (c.T + wpb - 1) / wpb;
    const int n_group = c.n_group > 1 ? c.n_group : 0;
    const size_t smem = n_group ? (size_t)wpb * c.E * sizeof(float) : 0;
    // one wave of resident blocks, each warp taking every (grid warps)-th token
    const int cap = resident_blocks((const void*)route_kernel<NE, KT>, threads, smem);
    if (blocks > cap) blocks = cap;
    return launch_pdl(route_kernel<NE, KT>, dim3(blocks), dim3(threads), smem, st, logits, c.T,
                      c.E, c.K, sel_bias, mask, c.score_fn, c.renorm, c.route_scale, n_group,
                      c.topk_group, ids, w, status);
}

// the top-k sizes of the layers this library is built for get unrolled selection rounds
template <int NE>
cudaError_t launch_ne(const moe_cfg& c, const float* logits, const float* sel_bias,
                      const uint8_t* mask, int32_t* ids, float* w, int32_t* status,
                      cudaStream_t st)
{
    switch (c.K) {
    case 1: return launch_nk<NE, 1>(c, logits, sel_bias, mask, ids, w, status, st);
    case 2: return launch_nk<NE, 2>(c, logits, sel_bias, mask, ids, w, status, st);
    case 4: return launch_nk<NE, 4>(c, logits, sel_bias, mask, ids, w, status, st);
    case 6: return launch_nk<NE, 6>(c, logits, sel_bias, mask, ids, w, status, st);
    case 8: return launch_nk<NE, 8>(c, logits, sel_bias, mask, ids, w, status, st);
    default: return launch_nk<NE, 0>(c, logits, sel_bias, mask, ids, w, status, st);
    }
}

}  // namespace

cudaError_t launch_route(const moe_cfg& c, const float* logits, const float* sel_bias,
                         const uint8_t* mask, int32_t* ids, float* w, int32_t* status,
                         cudaStream_t st)
{
    const int ne = (c.E + 31) / 32;
    if (ne <= 1) return launch_ne<1>(c, logits, sel_bias, mask, ids, w, status, st);
    if (ne <= 2) return launch_ne<2>(c, logits, sel_bias, mask, ids, w, status, st);
    if (ne <= 4) return launch_ne<4>(c, logits, sel_bias, mask, ids, w, status, st);
    if (ne <= 8) return launch_ne<8>(c, logits, sel_bias, mask, ids, w, status, st);
    if (ne <= 16) return launch_ne<16>(c, logits, sel_bias, mask, ids, w, status, st);
    return launch_ne<32>(c, logits, sel_bias, mask, ids, w, status, st);
}

}  // namespace moe

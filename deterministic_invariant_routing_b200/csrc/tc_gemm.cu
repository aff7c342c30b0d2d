// Router product on the 5th-generation tensor cores (tcgen05 + TMEM + TMA):
//
//   logits[t, e] = sum_h x[t, h] * W_router[e, h]  (+ logit_bias[e])       fp32
//
// "DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1: the router computes
// logits from hidden states; route.cu then selects the top-k experts. (Routing inside the
// product's epilogue, one thread per token, was measured slower than the separate
// warp-per-token kernel: nothing hides its serial exp/divide/selection chains there.)
//
// Up to 256 experts that are not 256, 384, ... (E a multiple of 128 above 128 runs on the
// CTA-pair kernel of tc_gemm2.cu with an fp32 + bias epilogue) the router runs split along
// K over a cluster of CTAs, each one SM, tile = 128 tokens x BN experts (BN = next power of
// two >= E, at least 32). Roles (192 threads): warp 0 TMA producer (one thread), warp 1
// TMEM allocator + MMA issuer (one thread), warps 2..5 copy the accumulator (warp w reads
// TMEM lanes 32*(w%4) ..) to shared memory, then every thread of the cluster takes part in
// the reduction. Every mbarrier wait is bounded; a give-up records MOE_ST_PIPE_TIMEOUT and
// stops issuing, and the CTA still reaches both cluster barriers, frees TMEM and returns.
//
// Also here: the bounded-wait self-test kernel of moe_pipeline_wait_selftest.
#include "tc_common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;                    // tokens per tile = UMMA M = TMEM lanes
constexpr int kThreads = 192;
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KiB per stage

// ---------------------------------------------------------------------------------------
// Router product split along K over a cluster of KS CTAs. The cluster of tile m owns 128
// tokens x BN experts; CTA q of it multiplies them over k-blocks [q kbs, (q + 1) kbs)
// (kbs = k_blocks / KS) into its own TMEM accumulator, copies that fp32 partial tile into
// its shared memory (over the operand ring, which is idle by then) and, after a cluster
// barrier, sums rows [q 128 / KS, (q + 1) 128 / KS) of the KS partial tiles in rank order
// 0, 1, .., KS - 1 (fp32, round to nearest), adds the logit bias and stores those logits.
// A second cluster barrier keeps every partial tile alive until its readers are done.
//
// Why: a router tile streams its tokens' whole rows of x; one CTA pair per 256 tokens
// left most SMs idle below a few thousand tokens and bound each busy SM by how many bytes
// it can have in flight. Splitting K puts KS SMs on every 128 tokens with a KS-th of the
// bytes each.
//
// Batch invariance: KS depends only on H (router_split_of), each CTA's K order is its
// k-blocks in increasing order with four K=16 steps each, and the partial tiles are added
// in rank order, so a token's logits depend on its row alone.
struct SplitArgs {
    int k_blocks;   // of the whole K
    int n_tiles;    // column tiles of BN experts
    int rows;       // tokens
    float* logits;  // [rows, n_valid] fp32
    int n_valid;    // experts E
    const float* bias;
    int32_t* status;
    int vec4;       // logits rows hold whole 16-byte vectors (E % 4 == 0, 16-byte base)
};

template <int BN>
struct SplitCfg {
    static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "UMMA N / TMEM columns");
    static constexpr int kStages = 3;
    static constexpr uint32_t kBBytes = (uint32_t)BN * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr uint32_t kRingBytes = kStages * kStageBytes;
    static constexpr uint32_t kPartBytes = (uint32_t)BM * BN * 4;
    static constexpr uint32_t kDataBytes = kRingBytes > kPartBytes ? kRingBytes : kPartBytes;
    static constexpr uint32_t kTmemCols = BN;
    static constexpr int kBars = 2 * kStages + 1;  // full, empty, tfull
    static constexpr size_t kSmem = 1024 + (size_t)kDataBytes + kBars * 8 + 16;
};

// DSMEM load of 16 bytes from a cluster shared-memory address
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

template <int BN, int KS>
__global__ void __launch_bounds__(kThreads, 1)
    router_splitk_kernel(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB, SplitArgs args)
{
    using C = SplitCfg<BN>;
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = make_idesc(BM, BN);
    constexpr int kChunks = BN / 4;                // 16-byte chunks per partial row
    constexpr int kRowsPer = (BM + KS - 1) / KS;   // rows this CTA reduces

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sA0 = smem_u32(base);
    const uint32_t sB0 = sA0 + S * kABytes;
    const uint32_t sP = sA0;  // the partial tile: row r, chunk j at chunk slot j ^ (r & 7)
    float4* part = reinterpret_cast<float4*>(base);
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::kDataBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int st) { return bar0 + 8u * (uint32_t)st; };
    auto empty_bar = [&](int st) { return bar0 + 8u * (uint32_t)(S + st); };
    const uint32_t tfull_bar = bar0 + 8u * (uint32_t)(2 * S);
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + C::kBars);  // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t q = cluster_ctarank();
    const int tile = blockIdx.x / KS;
    const int row0 = (tile / args.n_tiles) * BM, col0 = (tile % args.n_tiles) * BN;
    const int kbs = args.k_blocks / KS, kb0 = (int)q * kbs;

    if (threadIdx.x == 0) {
        for (int st = 0; st < S; ++st) {
            mbar_init(full_bar(st), 1);
            mbar_init(empty_bar(st), 1);
        }
        mbar_init(tfull_bar, 1);
        misc[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(misc), C::kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    pdl_wait();  // the previous kernel's writes are visible from here on

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_phase = 0;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
            for (int kb = 0; kb < kbs; ++kb) {
                if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status)) break;
                mbar_expect_tx(full_bar(stage), C::kStageBytes);
                const int kx = (kb0 + kb) * BK;
                tma_load_2d(sA0 + (uint32_t)stage * kABytes, &tmA, kx, row0, full_bar(stage));
                tma_load_2d(sB0 + (uint32_t)stage * C::kBBytes, &tmB, kx, col0, full_bar(stage));
                armed |= 1u << stage;
                armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            pdl_trigger();  // every load is issued: the next kernel may be scheduled
            if (*abort_flag) {
                for (int st = 0; st < S; ++st)
                    if (armed & (1u << st))
                        wait_bounded(full_bar(st), (armed_phase >> st) & 1u, abort_flag,
                                     args.status, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            for (int kb = 0; kb < kbs && !*abort_flag; ++kb) {
                if (!wait_bounded(full_bar(stage), phase, abort_flag, args.status)) break;
                tc_fence_after();
                const uint64_t ad = sw128_desc(sA0 + (uint32_t)stage * kABytes);
                const uint64_t bd = sw128_desc(sB0 + (uint32_t)stage * C::kBBytes);
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                    mma_bf16(tmem_base, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                             (kb | k) != 0 ? 1u : 0u);
                mma_commit(empty_bar(stage));
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // arrives once every MMA issued above has finished (also on a give-up)
            mma_commit(tfull_bar);
        }
    } else {
        // -------------------------------------------------------------- partial tile
        // the commit behind tfull follows the last MMA, which read the last loaded stage:
        // the ring is idle once it fires, and the partial tile may overwrite it
        int ok = 1;
        if (lane == 0) ok = wait_bounded(tfull_bar, 0u, abort_flag, args.status, false);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) {
            tc_fence_after();
            const int qq = warp & 3;
            const int r = qq * 32 + lane;
            const uint32_t tbase = tmem_base + ((uint32_t)(qq * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)c, v);
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int j = (c >> 2) + (m ^ (r & 7));
                    part[r * kChunks + j] =
                        make_float4(__uint_as_float(v[4 * m]), __uint_as_float(v[4 * m + 1]),
                                    __uint_as_float(v[4 * m + 2]), __uint_as_float(v[4 * m + 3]));
                }
            }
        }
    }
    tc_fence_before();
    cluster_sync();  // every partial tile of the cluster is in place

    // ------------------------------------------------------------------ reduction
    {
        const int r_beg = (int)q * kRowsPer;
        uint32_t src[KS];
#pragma unroll
        for (int i = 0; i < KS; ++i) src[i] = mapa_shared(sP, (uint32_t)i);
        for (int idx = threadIdx.x; idx < kRowsPer * kChunks; idx += blockDim.x) {
            const int rr = idx / kChunks, j = idx - rr * kChunks;
            const int r = r_beg + rr;
            const int64_t tok = (int64_t)row0 + r;
            if (r >= BM || tok >= args.rows) continue;
            const uint32_t off = (uint32_t)(r * kChunks + (j ^ (r & 7))) * 16u;
            float4 acc = ld_cluster_f4(src[0] + off);
#pragma unroll
            for (int i = 1; i < KS; ++i) {
                const float4 pv = ld_cluster_f4(src[i] + off);
                acc.x = __fadd_rn(acc.x, pv.x);
                acc.y = __fadd_rn(acc.y, pv.y);
                acc.z = __fadd_rn(acc.z, pv.z);
                acc.w = __fadd_rn(acc.w, pv.w);
            }
            const int col = col0 + 4 * j;
            float o[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (args.bias != nullptr && col + e < args.n_valid)
                    o[e] = __fadd_rn(o[e], args.bias[col + e]);
            float* dst = args.logits + tok * args.n_valid + col;
            if (args.vec4 && col + 3 < args.n_valid) {
                *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (col + e < args.n_valid) dst[e] = o[e];
            }
        }
    }
    cluster_sync();  // no partial tile is released while a peer may still read it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// CTAs per cluster of the split-K router for a hidden size H: the largest power of two up
// to 8 that divides the k-blocks and leaves every CTA at least 16 of them (1 below 32
// k-blocks). Measured on the 30B-A3B router (H = 2048): 8 k-blocks per CTA was faster at
// T <= 4096 (11 against 15 us) but slower at T = 16384 (27 against 19 us), where two CTAs
// per SM with longer main loops keep more bytes in flight.
int router_split_of(int H)
{
    const int kb = H / BK;
    for (int ks = 8; ks >= 2; ks >>= 1)
        if (kb % ks == 0 && kb / ks >= 16) return ks;
    return 1;
}

template <int BN, int KS>
cudaError_t launch_router_splitk_bn(const RouterProblem& p, cudaStream_t st)
{
    using C = SplitCfg<BN>;
    auto kernel = router_splitk_kernel<BN, KS>;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    static bool attr_set[64] = {};
    if (!attr_set[dev]) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   (int)C::kSmem);
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    CUtensorMap ma, mb;
    if (!make_map(&ma, p.x, p.T, p.H, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, p.w_router, p.E, p.H, BN)) return cudaErrorInvalidValue;
    SplitArgs a{};
    a.k_blocks = p.H / BK;
    a.n_tiles = (p.E + BN - 1) / BN;
    a.rows = p.T;
    a.logits = p.logits;
    a.n_valid = p.E;
    a.bias = p.logit_bias;
    a.status = p.status;
    a.vec4 = (p.E % 4 == 0 && (reinterpret_cast<uintptr_t>(p.logits) & 15u) == 0) ? 1 : 0;
    const int64_t tiles = (int64_t)((p.T + BM - 1) / BM) * a.n_tiles;
    if (tiles * KS > 0x7fffffffLL) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)(tiles * KS), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, a);
}

template <int BN>
cudaError_t launch_router_splitk(const RouterProblem& p, cudaStream_t st)
{
    switch (router_split_of(p.H)) {
    case 8: return launch_router_splitk_bn<BN, 8>(p, st);
    case 4: return launch_router_splitk_bn<BN, 4>(p, st);
    case 2: return launch_router_splitk_bn<BN, 2>(p, st);
    default: return launch_router_splitk_bn<BN, 1>(p, st);
    }
}

// One CTA whose thread 0 waits, through the pipelines' bounded wait, on an mbarrier that
// nothing arrives on: after `limit` cycles the wait gives up, raises the CTA's abort flag
// and counts MOE_ST_PIPE_TIMEOUT, as a stuck stage of a tensor-core pipeline would. No
// copy, MMA or tensor memory is involved, so giving up leaves nothing in flight.
__global__ void pipe_wait_selftest_kernel(int32_t* status, long long limit)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        wait_bounded_slow(smem_u32(&bar), 0u, &abort_flag, status, true, limit);
    }
}

}  // namespace

cudaError_t launch_pipe_wait_selftest(int32_t* status, long long limit_cycles, cudaStream_t st)
{
    pipe_wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_cycles);
    return cudaGetLastError();
}

cudaError_t launch_router(const RouterProblem& p, cudaStream_t st)
{
    if (p.H % BK != 0 || p.logits == nullptr) return cudaErrorInvalidValue;
    if (p.E % 128 == 0 && p.E > 128) {
        // 256 or more experts in whole 128-expert column tiles: the CTA-pair kernel, each SM
        // loading half of the router rows per k-block (a split-K tile of 256 experts would
        // need a 128 KB fp32 partial tile and one CTA per SM: 36 against 29 us at H = 4096)
        GemmProblem g{};
        g.epilogue = EPI_F32;
        g.a = p.x;
        g.a_rows = p.T;
        g.a_rows_total = p.T;
        g.b = p.w_router;
        g.b_rows_per_group = p.E;
        g.k = p.H;
        g.n = p.E;
        g.groups = 1;
        g.rows = p.T;
        g.out = p.logits;
        g.ldo = p.E;
        g.bias = p.logit_bias;
        g.status = p.status;
        return launch_tc_gemm_pair(g, st);
    }
    // N = next power of two >= E, at least 32, at most 256 (column tiles beyond)
    if (p.E <= 32) return launch_router_splitk<32>(p, st);
    if (p.E <= 64) return launch_router_splitk<64>(p, st);
    if (p.E <= 128) return launch_router_splitk<128>(p, st);
    return launch_router_splitk<256>(p, st);
}

}  // namespace moe

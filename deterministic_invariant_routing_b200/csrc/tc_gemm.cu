// Router product on the 5th-generation tensor cores (tcgen05 + TMEM + TMA):
//
//   logits[t, e] = sum_h x[t, h] * W_router[e, h]  (+ logit_bias[e])       fp32
//
// "DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1: the router computes
// logits from hidden states; route.cu then selects the top-k experts. Column tiles of BN
// experts (several when E > 256). (Routing inside this epilogue, one thread per token, was
// measured slower than the separate warp-per-token kernel: with one tile per CTA nothing
// hides its serial exp/divide/selection chains.)
//
// Batch invariance: a tile is 128 tokens x BN experts and always runs the full K loop,
// k-block 0 .. KB-1, in 64-wide blocks of four UMMA K=16 steps, fp32 in TMEM. The tile
// shape, instruction shape and K order depend only on (E, H); a token's logits depend only
// on its row. Rows past T are computed and discarded.
//
// Roles (192 threads, one CTA per SM, persistent over tiles): warp 0 TMA producer (one
// thread), warp 1 TMEM allocator + MMA issuer (one thread, two TMEM accumulators so the
// epilogue of tile i overlaps the MMAs of tile i+1), warps 2..5 epilogue (warp w reads
// TMEM lanes 32*(w%4) ..: one thread per token). Every mbarrier wait is bounded; a
// give-up records MOE_ST_PIPE_TIMEOUT, stops issuing, waits (bounded) for the CTA's own
// copies and MMAs, frees TMEM and returns.
#include "tc_common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;                    // tokens per tile = UMMA M = TMEM lanes
constexpr int kThreads = 192;
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KiB per stage

struct TcArgs {
    int k_blocks;
    int n_tiles;    // column tiles of BN experts
    int rows;       // tokens
    float* logits;  // [rows, n_valid] fp32
    int n_valid;    // experts E
    const float* bias;  // logit bias [E] or NULL
    int32_t* status;
};

template <int BN>
struct Cfg {
    static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "UMMA N / TMEM columns");
    static constexpr uint32_t kBBytes = (uint32_t)BN * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages0 = kSmemBudget / (int)kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : (kStages0 < 2 ? 2 : kStages0);
    static constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators, a power of two >= 64
    static constexpr int kBars = 2 * kStages + 5;  // full, empty, tfull[2], tempty[2], drain
    static constexpr size_t kSmem = 1024 + (size_t)kStages * kStageBytes + kBars * 8 + 16;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, TcArgs args)
{
    using C = Cfg<BN>;
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = make_idesc(BM, BN);
    constexpr uint32_t kTx = C::kStageBytes;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sA0 = smem_u32(base);
    const uint32_t sB0 = sA0 + S * kABytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * C::kStageBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(S + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (uint32_t)(2 * S + 4);
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + C::kBars);  // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = ((args.rows + BM - 1) / BM) * args.n_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4 * 32);
        }
        mbar_init(drain_bar, 1);
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
            uint32_t armed = 0, armed_phase = 0;  // stages loaded at least once / their parity
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const int row0 = (t / args.n_tiles) * BM, brow = (t % args.n_tiles) * BN;
                bool ok = true;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full_bar(stage), kTx);
                    tma_load_2d(sA0 + (uint32_t)stage * kABytes, &tmA, kb * BK, row0,
                                full_bar(stage));
                    tma_load_2d(sB0 + (uint32_t)stage * C::kBBytes, &tmB, kb * BK, brow,
                                full_bar(stage));
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            pdl_trigger();  // every load is issued: the next kernel may be scheduled
            if (*abort_flag) {
                // let every copy this thread started land before the CTA exits
                for (int s = 0; s < S; ++s)
                    if (armed & (1u << s))
                        wait_bounded(full_bar(s), (armed_phase >> s) & 1u, abort_flag,
                                     args.status, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int i = 0;
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++i) {
                const int acc = i & 1;
                if (!wait_bounded(tempty_bar(acc), (((uint32_t)i >> 1) & 1u) ^ 1u, abort_flag,
                                  args.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!wait_bounded(full_bar(stage), phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(sA0 + (uint32_t)stage * kABytes);
                    const uint64_t bd = sw128_desc(sB0 + (uint32_t)stage * C::kBBytes);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // +32 bytes along K per UMMA step, inside the 128-byte swizzle row
                        mma_bf16(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                                 (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(empty_bar(stage));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(tfull_bar(acc));
            }
            // every MMA of this CTA has finished before TMEM is released
            mma_commit(drain_bar);
            wait_bounded(drain_bar, 0u, abort_flag, args.status, false);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int i = 0;
        for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++i) {
            const int acc = i & 1;
            int ok = 1;
            if (lane == 0)
                ok = wait_bounded(tfull_bar(acc), ((uint32_t)i >> 1) & 1u, abort_flag, args.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int64_t tok = (int64_t)(t / args.n_tiles) * BM + row;
            const bool valid = tok < args.rows;
#pragma unroll 1
            for (int c = 0; c < BN; c += 32) {
                uint32_t r[32];
                tmem_ld32(tbase + (uint32_t)c, r);
                if (valid) {
                    const int col0 = (t % args.n_tiles) * BN + c;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int col = col0 + j;
                        if (col < args.n_valid) {
                            const float b = args.bias ? args.bias[col] : 0.0f;
                            args.logits[tok * args.n_valid + col] =
                                __fadd_rn(__uint_as_float(r[j]), b);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

template <int BN>
cudaError_t launch_router_variant(const RouterProblem& p, cudaStream_t st)
{
    using C = Cfg<BN>;
    auto kernel = router_gemm_kernel<BN>;
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
    TcArgs a{};
    a.k_blocks = p.H / BK;
    a.n_tiles = (p.E + BN - 1) / BN;
    a.rows = p.T;
    a.logits = p.logits;
    a.n_valid = p.E;
    a.bias = p.logit_bias;
    a.status = p.status;
    const int64_t tiles = (int64_t)((p.T + BM - 1) / BM) * a.n_tiles;
    int grid = num_sms();
    if (tiles < grid) grid = (int)tiles;
    if (grid < 1) grid = 1;
    return launch_pdl(kernel, dim3(grid), dim3(kThreads), C::kSmem, st, ma, mb, a);
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
    if (p.E % 128 == 0) {
        // whole 128-expert column tiles: the CTA-pair kernel, each SM loading half of the
        // router rows per k-block (the rows every tile shares)
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
    if (p.E <= 32) return launch_router_variant<32>(p, st);
    if (p.E <= 64) return launch_router_variant<64>(p, st);
    if (p.E <= 128) return launch_router_variant<128>(p, st);
    return launch_router_variant<256>(p, st);
}

}  // namespace moe

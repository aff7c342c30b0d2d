// The short last tiles of the grouped expert products on single SMs.
//
// A CTA-pair tile is 256 rows; a group (expert) of at most 128 rows would fill only one CTA
// of a pair, so the pair kernel (tc_gemm2.cu, run with skip_tails) leaves such groups here:
// one 128-row tile per group and N tile, on one SM with tcgen05.mma cta_group::1 (M = 128,
// N = 256, K = 16 per instruction). Larger groups stay whole on the pairs, their last tile
// padded: a group split between the two kernels would have its weights read from memory by
// each of them. The operands,
// the k-block order (64 wide, increasing, four K=16 steps each), the fp32 accumulation in
// TMEM and the epilogue arithmetic are the pair kernel's, so a row gets the same bits
// whichever kernel computes it (the batch-sweep and gather-path tests check this).
//
// Roles (192 threads, one CTA per SM, persistent over tail tiles): warp 0 TMA producer
// (one thread: the A tile and two 128-row B boxes per stage), warp 1 TMEM allocator + MMA
// issuer (one thread, two accumulators), warps 2..5 epilogue (warp w reads TMEM lanes
// 32 (w % 4)..). SwiGLU: the B tile is the 128 gate rows then the matching 128 up rows of
// the N tile, so accumulator columns c and 128 + c pair. Every wait is bounded.
#include <cuda_bf16.h>

#include "tc_common.cuh"

namespace moe {
namespace {

constexpr int TM = 128;  // rows per tile = UMMA M = TMEM lanes
constexpr int TN = 256;  // accumulator columns (SwiGLU: 128 gate + 128 up)
constexpr int kTailThreads = 192;
constexpr uint32_t kTA = TM * BK * 2;        // 16 KiB
constexpr uint32_t kTB = TN * BK * 2;        // 32 KiB
constexpr uint32_t kTStage = kTA + kTB;      // 48 KiB
constexpr int kTStages = kSmemBudget / (int)kTStage;  // 4
constexpr uint32_t kTEpi = 4 * 2 * 2048;     // 4 warps x 2 store tiles of 32 x 32 bf16
constexpr int kTQ = 4;                       // tile-index queue from the producer to the others
constexpr int kTBars = 2 * kTStages + 5 + 2 * kTQ;

struct TailArgs {
    int k_blocks;
    int n_tiles;
    int groups;
    const int32_t* offsets;  // [groups + 1], or NULL: one group of `rows` rows
    int rows;
    int b_rows_per_group;
    int half_rows;  // SwiGLU: rows from a gate row to its up row in B
    void* out;
    int64_t ldo;
    int32_t* status;
    int side;  // running beside the pair kernel: no wait at the start, a wait before exiting
    int32_t* tile_ctr;  // tiles taken from this counter (zeroed by the pair launch), or NULL:
                        // tile t on CTA t mod grid
};

struct TailTile {
    int g, n;
    int64_t row0, row_end;
};

template <int EPI>
__global__ void __launch_bounds__(kTailThreads, 1)
    tc_gemm_tail_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO, TailArgs args)
{
    constexpr int S = kTStages;
    constexpr uint32_t kIdesc = make_idesc(TM, TN);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sA0 = smem_u32(base);
    const uint32_t sB0 = sA0 + S * kTA;
    const uint32_t sE0 = sA0 + S * kTStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * kTStage + kTEpi);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(S + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (uint32_t)(2 * S + 4);
    auto qfull_bar = [&](int q) { return bar0 + 8u * (uint32_t)(2 * S + 5 + q); };
    auto qempty_bar = [&](int q) { return bar0 + 8u * (uint32_t)(2 * S + 5 + kTQ + q); };
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + kTBars);  // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    volatile int32_t* tq = reinterpret_cast<volatile int32_t*>(misc + 4);  // [kTQ] tile indices
    int32_t* tprefix = reinterpret_cast<int32_t*>(misc + 8);  // [groups + 1] tail tiles before g
    int32_t* toffs = tprefix + (args.groups + 1);            // [groups + 1] row offsets

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.groups;

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
        for (int q = 0; q < kTQ; ++q) {
            mbar_init(qfull_bar(q), 1);
            mbar_init(qempty_bar(q), 1 + 4);  // the MMA thread and the four epilogue warps
        }
        misc[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(misc), 2 * TN);
    // The previous kernel's writes (offsets, operands) are visible from here on. Beside the
    // pair kernel, that kernel is the pair launch, which started this one only after its own
    // wait (so the dispatch that wrote offsets and operands has completed); this launch then
    // waits for the pair launch before exiting, so the next kernel finds both complete.
    if (!args.side) pdl_wait();
    if (warp == 2) {
        // groups with 1..128 rows past their last full 256-row tile, as a prefix count
        auto row_off = [&](int g) -> int {
            return args.offsets ? args.offsets[g] : (g == 0 ? 0 : args.rows);
        };
        auto has_tail = [&](int n) -> int { return (n > 0 && n <= TM) ? 1 : 0; };
        const int per = (G + 31) / 32;
        const int beg = lane * per < G ? lane * per : G;
        const int end = beg + per < G ? beg + per : G;
        int sum = 0;
        for (int g = beg; g < end; ++g) {
            toffs[g] = row_off(g);
            sum += has_tail(row_off(g + 1) - row_off(g));
        }
        if (lane == 0) toffs[G] = row_off(G);
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        int run = incl - sum;
        for (int g = beg; g < end; ++g) {
            tprefix[g] = run;
            run += has_tail(row_off(g + 1) - row_off(g));
        }
        if (lane == 31) tprefix[G] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int total = tprefix[G] * args.n_tiles;
    auto decode = [&](int t) -> TailTile {
        TailTile ti;
        const int j = t / args.n_tiles;
        ti.n = t - j * args.n_tiles;
        int lo = 0, hi = G - 1;
        while (lo < hi) {  // the group holding the j-th tail: tprefix[g] <= j < tprefix[g+1]
            const int mid = (lo + hi + 1) >> 1;
            if (tprefix[mid] <= j) lo = mid;
            else hi = mid - 1;
        }
        ti.g = lo;
        ti.row0 = (int64_t)toffs[lo];  // the whole group (at most 128 rows)
        ti.row_end = toffs[lo + 1];
        return ti;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0, armed = 0, armed_phase = 0;
            auto b_rows = [&](const TailTile& tt, int& r0, int& r1) {
                if (EPI == EPI_SWIGLU) {
                    r0 = tt.g * args.b_rows_per_group + tt.n * 128;
                    r1 = r0 + args.half_rows;
                } else {
                    r0 = tt.g * args.b_rows_per_group + tt.n * TN;
                    r1 = r0 + 128;
                }
            };
            // every tile index goes through the queue (-1 ends it), taken from the counter
            // when there is one, else this CTA's share t = blockIdx.x + k gridDim.x
            int qi = 0, next = blockIdx.x;
            uint32_t qphase = 0;
            for (;;) {
                int t = -1;
                if (!*abort_flag) {
                    t = args.tile_ctr ? atomicAdd(args.tile_ctr, 1) : next;
                    next += gridDim.x;
                    if (t >= total) t = -1;
                }
                if (!wait_bounded(qempty_bar(qi), qphase ^ 1u, abort_flag, args.status)) break;
                tq[qi] = t;
                mbar_arrive(qfull_bar(qi));
                if (++qi == kTQ) {
                    qi = 0;
                    qphase ^= 1u;
                }
                if (t < 0) break;
                const TailTile ti = decode(t);
                int b0, b1;  // the two 128-row B boxes of the N tile
                b_rows(ti, b0, b1);
                bool ok = true;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx(full_bar(stage), kTStage);
                    const int kx = kb * BK;
                    const uint32_t sb = sB0 + (uint32_t)stage * kTB;
                    tma_load_2d(sA0 + (uint32_t)stage * kTA, &tmA, kx, (int)ti.row0, full_bar(stage));
                    tma_load_2d(sb, &tmB, kx, b0, full_bar(stage));
                    tma_load_2d(sb + kTB / 2, &tmB, kx, b1, full_bar(stage));
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            // beside the pair kernel the next launch is scheduled when this one completes:
            // started earlier, its CTAs could hold SMs that this launch's later CTAs need
            if (!args.side) pdl_trigger();
            if (*abort_flag) {
                for (int s = 0; s < S; ++s)
                    if (armed & (1u << s))
                        wait_bounded(full_bar(s), (armed_phase >> s) & 1u, abort_flag,
                                     args.status, false);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            const uint64_t ad0 = sw128_desc(sA0);
            const uint64_t bd0 = sw128_desc(sB0);
            int stage = 0;
            uint32_t phase = 0;
            int qi = 0;
            uint32_t qphase = 0;
            for (int i = 0;; ++i) {
                if (!wait_bounded(qfull_bar(qi), qphase, abort_flag, args.status)) break;
                const int t = tq[qi];
                mbar_arrive(qempty_bar(qi));
                if (++qi == kTQ) {
                    qi = 0;
                    qphase ^= 1u;
                }
                if (t < 0 || *abort_flag) break;
                const int acc = i & 1;
                if (!wait_bounded(tempty_bar(acc), (((uint32_t)i >> 1) & 1u) ^ 1u, abort_flag,
                                  args.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * TN);
                bool ok = true;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!wait_bounded(full_bar(stage), phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = ad0 + (uint64_t)((uint32_t)stage * (kTA >> 4));
                    const uint64_t bd = bd0 + (uint64_t)((uint32_t)stage * (kTB >> 4));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                                 (kb | k) != 0 ? 1u : 0u);
                    mma_commit(empty_bar(stage));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(tfull_bar(acc));
            }
            mma_commit(drain_bar);
            wait_bounded(drain_bar, 0u, abort_flag, args.status, false);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t ebuf = sE0 + (uint32_t)q * 4096u;
        uint32_t eb = 0;
        const uint32_t erow = (uint32_t)lane * 64u, eswz = ((uint32_t)lane >> 1) & 3u;
        auto store_block = [&](const uint32_t (&pk)[16], bool full_blk, bool valid, int row_blk,
                               int col, uint16_t* dst_row) {
            if (full_blk) {
                const uint32_t b = ebuf + eb * 2048u;
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                                     b + erow + ((((uint32_t)v) ^ eswz) << 4)),
                                 "r"(pk[4 * v]), "r"(pk[4 * v + 1]), "r"(pk[4 * v + 2]),
                                 "r"(pk[4 * v + 3])
                                 : "memory");
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmO, b, col, row_blk);
                    bulk_commit();
                }
                eb ^= 1u;
            } else if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(dst_row);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                    dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
        };
        int qi = 0;
        uint32_t qphase = 0;
        for (int i = 0;; ++i) {
            int t = -1;
            if (lane == 0 && wait_bounded(qfull_bar(qi), qphase, abort_flag, args.status)) {
                t = tq[qi];
                mbar_arrive(qempty_bar(qi));
            }
            t = __shfl_sync(0xffffffffu, t, 0);
            if (++qi == kTQ) {
                qi = 0;
                qphase ^= 1u;
            }
            if (t < 0 || *abort_flag) break;
            const TailTile ti = decode(t);
            const int acc = i & 1;
            int ok = 1;
            if (lane == 0)
                ok = wait_bounded(tfull_bar(acc), ((uint32_t)i >> 1) & 1u, abort_flag, args.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * TN);
            const int64_t grow = ti.row0 + row;
            const bool valid = grow < ti.row_end;
            const int row_blk = (int)(ti.row0 + q * 32);
            const bool full_blk = (int64_t)row_blk + 31 < ti.row_end;
            uint16_t* out = static_cast<uint16_t*>(args.out);
            if (EPI == EPI_SWIGLU) {
#pragma unroll 1
                for (int c = 0; c < TN / 2; c += 32) {
                    uint32_t g[32], u[32];
                    tmem_ld32(tbase + (uint32_t)c, g);
                    tmem_ld32(tbase + (uint32_t)(TN / 2 + c), u);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float hv[2];
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2)
                            hv[h2] = swiglu(__uint_as_float(g[2 * j + h2]),
                                            __uint_as_float(u[2 * j + h2]));
                        pk[j] = bf16x2_rne(hv[0], hv[1]);
                    }
                    const int col = ti.n * (TN / 2) + c;
                    store_block(pk, full_blk, valid, row_blk, col, out + grow * args.ldo + col);
                }
            } else {
#pragma unroll 1
                for (int c = 0; c < TN; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = bf16x2_rne(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                    const int col = ti.n * TN + c;
                    store_block(pk, full_blk, valid, row_blk, col, out + grow * args.ldo + col);
                }
            }
            tc_fence_before();
            mbar_arrive(tempty_bar(acc));
        }
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (args.side) pdl_wait();  // the pair launch beside this one has completed
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 2 * TN);
    }
}

template <int EPI>
cudaError_t launch_tail_variant(const GemmProblem& p, cudaStream_t st)
{
    auto kernel = tc_gemm_tail_kernel<EPI>;
    const int groups = p.offsets ? p.groups : 1;
    const size_t smem = 1024 + (size_t)kTStages * kTStage + kTEpi + kTBars * 8 + 32 +
                        (size_t)2 * (groups + 1) * sizeof(int32_t);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    static bool attr_set[64] = {};
    if (!attr_set[dev]) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    const int64_t rows_total = p.offsets ? p.a_rows_total : p.rows;
    CUtensorMap ma, mb, mo;
    if (!make_map(&ma, p.a, p.a_rows, p.k, TM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, p.b, (int64_t)groups * p.b_rows_per_group, p.k, 128))
        return cudaErrorInvalidValue;
    if (!make_store_map(&mo, p.out, rows_total, p.n, p.ldo)) return cudaErrorInvalidValue;
    TailArgs a{};
    a.k_blocks = p.k / BK;
    a.n_tiles = (EPI == EPI_SWIGLU) ? p.n / (TN / 2) : p.n / TN;
    a.groups = groups;
    a.offsets = p.offsets;
    a.rows = p.rows;
    a.b_rows_per_group = p.b_rows_per_group;
    a.half_rows = (EPI == EPI_SWIGLU) ? p.n : 0;
    a.out = p.out;
    a.ldo = p.ldo;
    a.status = p.status;
    a.side = p.side_sms > 0 ? 1 : 0;
    a.tile_ctr = p.tail_ctr;
    // at most one tail tile per group and N tile. Beside the pair kernel with tiles dealt by
    // CTA index: its side SMs. With the counter: a CTA per SM, the first side_sms of them
    // running beside the pair tiles and the rest taking what is left as pair CTAs finish.
    int64_t grid = (int64_t)groups * a.n_tiles;
    if (a.side && a.tile_ctr == nullptr && grid > p.side_sms) grid = p.side_sms;
    if (grid > num_sms()) grid = num_sms();
    if (grid < 1) grid = 1;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kTailThreads), smem, st, ma, mb, mo, a);
}

}  // namespace

cudaError_t launch_tc_gemm_tail(const GemmProblem& p, cudaStream_t st)
{
    if (p.k % BK != 0 || p.gather_rows != nullptr || p.b_mn || p.a_mn)
        return cudaErrorInvalidValue;
    if (p.epilogue == EPI_SWIGLU) {
        if (p.n % (TN / 2) != 0) return cudaErrorInvalidValue;
        return launch_tail_variant<EPI_SWIGLU>(p, st);
    }
    if (p.epilogue == EPI_BF16) {
        if (p.n % TN != 0) return cudaErrorInvalidValue;
        return launch_tail_variant<EPI_BF16>(p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace moe

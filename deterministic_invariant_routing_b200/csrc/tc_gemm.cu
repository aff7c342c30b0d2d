// Persistent grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
//   out[r, n] = epilogue( sum_k A[r, k] * B[g*Nb + n, k] )   for rows r of group g
//
// Used three ways: the router product (one group, fp32 logits + bias), the expert
// gate_up product with the SwiGLU epilogue (groups = experts, h = silu(gate) * up in bf16)
// and the expert down product (groups = experts, bf16 out). The experts are the grouped
// expert MLP of "DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 2
// (gate_and_up -> down) and SpecForge PR #1003 (grouped_mm_experts).
//
// Batch invariance (the routing/expert contract of the roadmap's Problem 1 and 3 pages):
// a tile is 128 rows x BN columns and always runs the full K loop, k-block 0 .. KB-1, in
// 64-wide blocks of four UMMA K=16 steps, accumulating in TMEM fp32. The tile shape, the
// MMA instruction shape and the K order depend only on the GEMM's (N, K) -- never on the
// number of rows, the rows per group or where a row falls in its tile. No split-K, no
// atomics. Rows of a tile that belong to the next group or lie past the end are computed
// and discarded.
//
// Roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0       TMA producer: A and B k-blocks into a STAGES-deep shared-memory ring
//   warp 1       TMEM allocator and MMA issuer (one thread), two TMEM accumulators so the
//                epilogue of tile i overlaps the MMAs of tile i+1
//   warps 2..5   epilogue: tcgen05.ld the accumulator rows (warp w owns TMEM lanes
//                32*(w%4) ..), apply the epilogue, store rows that belong to the group
// Every mbarrier wait is bounded; when one gives up the CTA records MOE_ST_PIPE_TIMEOUT,
// stops issuing, waits (bounded) for its own copies and MMAs in flight, frees TMEM and
// returns.
#include <cuda_bf16.h>

#include "tc_common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;                   // rows per tile = UMMA M = TMEM lanes
constexpr int kThreads = 192;
constexpr uint32_t kABytes = BM * BK * 2;  // 16 KiB per stage

struct TcArgs {
    int k_blocks;
    int n_tiles;
    int groups;
    const int32_t* offsets;
    int rows;
    int b_rows_per_group;
    int half_rows;  // SWIGLU: rows between a gate row and its up row in B
    void* out;
    int64_t ldo;
    int n_valid;  // columns that exist (F32 epilogue)
    const float* bias;
    int32_t* status;
};

template <int EPI, int BN>
struct Cfg {
    static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "UMMA N / TMEM columns");
    static constexpr uint32_t kBBytes = (uint32_t)BN * BK * 2;
    static constexpr uint32_t kStageBytes = kABytes + kBBytes;
    static constexpr int kStages0 = kSmemBudget / (int)kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : (kStages0 < 2 ? 2 : kStages0);
    static constexpr uint32_t kTmemCols = 2 * BN;  // two accumulators, a power of two >= 64
    static constexpr int kBars = 2 * kStages + 5;  // full, empty, tfull[2], tempty[2], drain
    static size_t smem_bytes(int groups)
    {
        return 1024 + (size_t)kStages * kStageBytes + kBars * 8 + 16 +
               (size_t)2 * (groups + 1) * sizeof(int32_t);
    }
};

struct TileInfo {
    int g, n;
    int64_t row0, row_end;
};

__device__ __forceinline__ TileInfo decode_tile(int t, int n_tiles, int groups,
                                                const int32_t* prefix, const int32_t* offs)
{
    TileInfo ti;
    const int mt = t / n_tiles;
    ti.n = t - mt * n_tiles;
    int lo = 0, hi = groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    ti.g = lo;
    ti.row0 = (int64_t)offs[lo] + (int64_t)(mt - prefix[lo]) * BM;
    ti.row_end = offs[lo + 1];
    return ti;
}

template <int EPI, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   TcArgs args)
{
    using C = Cfg<EPI, BN>;
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
    int32_t* prefix = reinterpret_cast<int32_t*>(misc + 4);  // [groups+1] first tile of group
    int32_t* offs = prefix + (args.groups + 1);              // [groups+1] row offsets

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
        misc[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(smem_u32(misc), C::kTmemCols);
    if (warp == 2) {
        // row offsets and the exclusive scan of the per-group tile-row counts
        auto row_off = [&](int g) -> int {
            return args.offsets ? args.offsets[g] : (g == 0 ? 0 : args.rows);
        };
        const int per = (G + 31) / 32;
        const int beg = lane * per < G ? lane * per : G;
        const int end = beg + per < G ? beg + per : G;
        int sum = 0;
        for (int g = beg; g < end; ++g) {
            const int r0 = row_off(g);
            offs[g] = r0;
            sum += (row_off(g + 1) - r0 + BM - 1) / BM;
        }
        if (lane == 0) offs[G] = row_off(G);
        int incl = sum;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        int run = incl - sum;
        for (int g = beg; g < end; ++g) {
            prefix[g] = run;
            run += (row_off(g + 1) - row_off(g) + BM - 1) / BM;
        }
        if (lane == 31) prefix[G] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    const int total = prefix[G] * args.n_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_phase = 0;  // stages loaded at least once / their parity
            for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
                const TileInfo ti = decode_tile(t, args.n_tiles, G, prefix, offs);
                const int brow = ti.g * args.b_rows_per_group +
                                 ti.n * (EPI == EPI_SWIGLU ? BN / 2 : BN);
                bool ok = true;
                for (int kb = 0; kb < args.k_blocks; ++kb) {
                    if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = sA0 + (uint32_t)stage * kABytes;
                    const uint32_t sb = sB0 + (uint32_t)stage * C::kBBytes;
                    mbar_expect_tx(full_bar(stage), kTx);
                    tma_load_2d(sa, &tmA, kb * BK, (int)ti.row0, full_bar(stage));
                    if (EPI == EPI_SWIGLU) {
                        tma_load_2d(sb, &tmB, kb * BK, brow, full_bar(stage));
                        tma_load_2d(sb + C::kBBytes / 2, &tmB, kb * BK, brow + args.half_rows,
                                    full_bar(stage));
                    } else {
                        tma_load_2d(sb, &tmB, kb * BK, brow, full_bar(stage));
                    }
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
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
            const TileInfo ti = decode_tile(t, args.n_tiles, G, prefix, offs);
            const int acc = i & 1;
            int ok = 1;
            if (lane == 0)
                ok = wait_bounded(tfull_bar(acc), ((uint32_t)i >> 1) & 1u, abort_flag, args.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int64_t grow = ti.row0 + row;
            const bool valid = grow < ti.row_end;
            if (EPI == EPI_SWIGLU) {
                uint16_t* out = static_cast<uint16_t*>(args.out);
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 32) {
                    uint32_t g[32], u[32];
                    tmem_ld32(tbase + (uint32_t)c, g);
                    tmem_ld32(tbase + (uint32_t)(BN / 2 + c), u);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float hv[2];
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const float gv = __uint_as_float(g[2 * j + h2]);
                            const float uv = __uint_as_float(u[2 * j + h2]);
                            hv[h2] = swiglu(gv, uv);
                        }
                        pk[j] = bf16x2_rne(hv[0], hv[1]);
                    }
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(
                            out + grow * args.ldo + (int64_t)ti.n * (BN / 2) + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                                                pk[4 * v + 3]);
                    }
                }
            } else if (EPI == EPI_BF16) {
                uint16_t* out = static_cast<uint16_t*>(args.out);
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = bf16x2_rne(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(out + grow * args.ldo +
                                                              (int64_t)ti.n * BN + c);
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2],
                                                pk[4 * v + 3]);
                    }
                }
            } else {
                float* out = static_cast<float*>(args.out);
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    if (valid) {
                        const int col0 = ti.n * BN + c;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int col = col0 + j;
                            if (col < args.n_valid) {
                                const float b = args.bias ? args.bias[col] : 0.0f;
                                out[grow * args.ldo + col] = __fadd_rn(__uint_as_float(r[j]), b);
                            }
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

// ------------------------------------------------------------------ host side

template <int EPI, int BN>
cudaError_t launch_variant(const GemmProblem& p, cudaStream_t st)
{
    using C = Cfg<EPI, BN>;
    const int groups = p.offsets ? p.groups : 1;
    const size_t smem = C::smem_bytes(groups);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    static bool attr_set[64] = {};
    if (dev < 64 && !attr_set[dev]) {
        err = cudaFuncSetAttribute(tc_gemm_kernel<EPI, BN>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    CUtensorMap ma, mb;
    const int b_box = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    if (!make_map(&ma, p.a, p.a_rows, p.k, BM)) return cudaErrorInvalidValue;
    if (!make_map(&mb, p.b, (int64_t)groups * p.b_rows_per_group, p.k, b_box))
        return cudaErrorInvalidValue;
    TcArgs a;
    a.k_blocks = p.k / BK;
    a.n_tiles = (EPI == EPI_SWIGLU) ? p.n / (BN / 2) : (p.n + BN - 1) / BN;
    a.groups = groups;
    a.offsets = p.offsets;
    a.rows = p.rows;
    a.b_rows_per_group = p.b_rows_per_group;
    a.half_rows = (EPI == EPI_SWIGLU) ? p.n : 0;
    a.out = p.out;
    a.ldo = p.ldo;
    a.n_valid = p.n;
    a.bias = p.bias;
    a.status = p.status;
    const int64_t rows_total = p.offsets ? p.a_rows_total : p.rows;
    const int64_t max_tiles = ((rows_total + BM - 1) / BM + groups) * a.n_tiles;
    int grid = num_sms();
    if (max_tiles < grid) grid = (int)max_tiles;
    if (grid < 1) grid = 1;
    tc_gemm_kernel<EPI, BN><<<grid, kThreads, smem, st>>>(ma, mb, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_gemm(const GemmProblem& p, cudaStream_t st)
{
    if (p.k % BK != 0) return cudaErrorInvalidValue;
    // the expert products run on CTA pairs (tc_gemm2.cu)
    if (p.epilogue == EPI_SWIGLU || p.epilogue == EPI_BF16) return launch_tc_gemm_pair(p, st);
    // fp32 epilogue (router logits): N = next power of two >= E, at least 32, at most 256
    if (p.n <= 32) return launch_variant<EPI_F32, 32>(p, st);
    if (p.n <= 64) return launch_variant<EPI_F32, 64>(p, st);
    if (p.n <= 128) return launch_variant<EPI_F32, 128>(p, st);
    return launch_variant<EPI_F32, 256>(p, st);
}

}  // namespace moe

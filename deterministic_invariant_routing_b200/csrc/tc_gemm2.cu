// Grouped GEMM on CTA pairs: tcgen05.mma.cta_group::2 (M = 256 rows per tile split over
// the two CTAs of a cluster), TMA operand loads, TMEM accumulators. Used for the expert
// products -- gate_up with the SwiGLU epilogue and down -- of "DSV4 Flash MoE
// Train-Inference Consistency Roadmap", Problem 2 (gate_and_up -> down) and SpecForge
// PR #1003 (grouped experts, the always-on shared expert as one more group).
//
// Why a pair: one UMMA of M=128, N=256, K=16 reads 12 KiB of operands from shared memory
// per 128 tensor cycles, and the TMA ring writes as much again -- more than one SM's
// shared-memory bandwidth. With cta_group::2 each SM holds its own 128 rows of A and only
// half of B's columns, so each SM moves 8 KiB per 128 cycles each way.
//
//   leader (even CTA)  A rows [r0, r0+128)       B columns [0, N/2)    TMEM rows r0..
//   peer   (odd CTA)   A rows [r0+128, r0+256)   B columns [N/2, N)    TMEM rows r0+128..
//
// For the SwiGLU product the pair's N = 256 is 128 gate columns (the leader's B half)
// followed by the 128 matching up columns (the peer's B half), so every CTA's accumulator
// row holds gate and up of the same 128 intermediate columns.
//
// Batch invariance: the tile shape (256 x N), the instruction shape and the K order
// (k-blocks of 64 in increasing k, four K=16 steps each) depend only on the GEMM's (N, K);
// rows past the group's end are computed and never stored; no split-K, no atomics.
//
// Protocol (per k-block stage s): both CTAs wait on their own empty[s], load their A and
// B halves with .cta_group::2 TMA whose completion is counted on the LEADER's full[s]
// (the leader posts the byte count of both CTAs); the leader's single MMA thread waits on
// full[s], issues the pair MMAs and commits to empty[s] of both CTAs (multicast commit).
// Accumulators: the commit of the last k-block arrives on tfull[a] of both CTAs; each
// CTA's epilogue drains its own TMEM rows and arrives on the leader's tempty[a] (one
// arrival per epilogue thread of both CTAs). Every wait is bounded and a give-up is
// recorded in MOE_ST_PIPE_TIMEOUT.
//
// Output: each epilogue warp owns 32 accumulator rows and writes them 32 columns at a time.
// Every epilogue but the router's fp32 one runs two warps per 32 rows, each taking every
// other 32-column chunk, so that storing a tile's outputs (and, for the SwiGLU backward,
// reading its gate/up values) keeps pace with the next tile's main loop.
// A block whose 32 rows all lie inside the group goes through a 2 KiB shared-memory tile
// (64-byte swizzle, two per warp, alternating) and one TMA store; the partial block at a
// group's end is stored row by row from registers, so no padding row reaches global memory.
#include <cuda_bf16.h>

#include "tc_common.cuh"

namespace moe {
namespace {

constexpr int PM = 256;                     // rows per pair tile
constexpr int HM = 128;                     // rows per CTA = TMEM lanes
constexpr uint32_t kA2Bytes = HM * BK * 2;  // 16 KiB per stage
constexpr uint16_t kPairMask = 0x3;

struct PairArgs {
    int k_blocks;
    int n_tiles;
    int groups;
    const int32_t* offsets;
    int rows;
    int b_rows_per_group;
    int half_rows;  // SWIGLU: rows between a gate row and its up row in B
    const int32_t* gather_rows;  // A row r is row gather_rows[r] of the A tensor, or NULL
    const uint16_t* a;           // the A tensor (read directly by a gather)
    int k;                       // its row length
    void* out;
    int64_t ldo;
    int32_t* status;
    int m_tiles;                 // EPI_WGRAD: row tiles of A (per group)
    const int32_t* k_offsets;    // EPI_WGRAD: [groups+1] K ranges
    float* gu;                   // EPI_SWIGLU_SAVE / EPI_DSWIGLU: fp32 gate | up values
    int64_t ld_gu;
    int half_out;                // EPI_DSWIGLU, EPI_SWIGLU_SAVE: column of the first up
                                 // value (gradient) in a row
    const float* bias;           // EPI_F32: per-column bias or NULL
    int b_k_rows;                // MN-major B: K rows of each group (0: one shared B)
    int skip_tails;              // leave groups of at most 128 rows to the 1-SM tail kernel
    int early_trigger;           // let the next kernel start on the SMs this launch leaves free
    int32_t* tail_ctr;           // the one-SM launch's tile counter, zeroed here, or NULL
};

// XS = 1: a sixth 32 KB operand stage, taken from the shared memory a CTA has beyond the
// ring's usual budget (fits up to about 170 groups; see launch_pair_variant)
template <int EPI, int NP, int XS = 0>
struct Cfg2 {
    static_assert(NP == 128 || NP == 256, "pair N");
    // epilogue warps: two per TMEM lane quarter (each taking every other 32-column chunk)
    // where the epilogue moves more global bytes than the main loop hides with one
    static constexpr int kEpiWarps =
        (EPI == EPI_DSWIGLU || EPI == EPI_SWIGLU_SAVE || EPI == EPI_WGRAD || EPI == EPI_BF16 ||
         EPI == EPI_SWIGLU)
            ? 8
            : 4;
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    // outputs go through two 2 KiB store tiles per epilogue warp (32 rows of 32 bf16 or 16
    // fp32 values); the router's fp32 logits are written from registers
    static constexpr uint32_t kEpiBytes =
        (EPI == EPI_F32) ? 0u : (uint32_t)kEpiWarps * 2u * 2048u;
    // EPI_DSWIGLU: per epilogue warp a 4 KiB tile of the kept gate and up values (32 rows x
    // 16 fp32 each) loaded by TMA, and its barrier
    static constexpr uint32_t kGuBytes = (EPI == EPI_DSWIGLU) ? (uint32_t)kEpiWarps * 4096u : 0u;
    static constexpr uint32_t kBBytes = (uint32_t)(NP / 2) * BK * 2;  // this CTA's half of B
    static constexpr uint32_t kStageBytes = kA2Bytes + kBBytes;
    // the operand ring gives up what the epilogue tiles take beyond four warps' store tiles
    static constexpr int kEpiAll = (int)(kEpiBytes + kGuBytes);
    static constexpr int kRing =
        kSmemBudget + XS * 32768 - (kEpiAll > 16384 ? kEpiAll - 16384 : 0);
    static constexpr int kStages0 = kRing / (int)kStageBytes;
    static constexpr int kStages = kStages0 > 8 ? 8 : kStages0;
    static constexpr uint32_t kTmemCols = 2 * NP;
    static constexpr int kBars = 2 * kStages + 5 + (EPI == EPI_DSWIGLU ? kEpiWarps : 0);
    static size_t smem_bytes(int groups)
    {
        return 1024 + (size_t)kStages * kStageBytes + kEpiBytes + kGuBytes + kBars * 8 + 16 +
               (size_t)2 * (groups + 1) * sizeof(int32_t) + HM * sizeof(int32_t);
    }
};

struct PairTile {
    int g, n;
    int64_t row0, row_end;  // row0: the pair tile's first row
    int k0, kbs;            // first K column and k-blocks of the tile's reduction
};

// row-grouped products: tiles of 256 rows inside each group's row range, n fastest
__device__ __forceinline__ PairTile decode_pair_tile(int t, int n_tiles, int groups,
                                                     const int32_t* prefix, const int32_t* offs,
                                                     int k_blocks)
{
    PairTile ti;
    const int mt = t / n_tiles;
    ti.n = t - mt * n_tiles;
    int lo = 0, hi = groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= mt) lo = mid;
        else hi = mid - 1;
    }
    ti.g = lo;
    ti.row0 = (int64_t)offs[lo] + (int64_t)(mt - prefix[lo]) * PM;
    ti.row_end = offs[lo + 1];
    ti.k0 = 0;
    ti.kbs = k_blocks;
    return ti;
}

// K-grouped products (EPI_WGRAD): group g owns K columns [k_offsets[g], k_offsets[g+1]);
// tiles are (g, row tile, n), n fastest
__device__ __forceinline__ PairTile decode_wgrad_tile(int t, const PairArgs& a,
                                                     const int32_t* order, int nclusters,
                                                     int total)
{
    // Tiles run in rounds of nclusters (cluster c takes tile c of every round). They are
    // dealt by descending cost -- groups ordered by their K length, longest first -- and
    // every other round in reverse cluster order, so that each cluster's total K is close
    // to the mean however skewed the groups are. Only the schedule changes: a tile's
    // arithmetic is the same wherever it runs.
    const int per = a.m_tiles * a.n_tiles;
    const int k = t / nclusters, j = t - k * nclusters;
    const int base = k * nclusters;
    const int n_here = total - base < nclusters ? total - base : nclusters;
    const int s = base + ((k & 1) ? n_here - 1 - j : j);
    const int r = s / per;
    PairTile ti;
    ti.g = order[r];
    const int rem = s - r * per;
    const int mt = rem / a.n_tiles;
    ti.n = rem - mt * a.n_tiles;
    ti.row0 = (int64_t)mt * PM;
    ti.row_end = a.rows;
    ti.k0 = a.k_offsets[ti.g];
    ti.kbs = (a.k_offsets[ti.g + 1] - ti.k0) / BK;
    return ti;
}

// MN: operand majorness fixed at compile time -- 0 both K-major, 1 B MN-major, 2 A and B
// MN-major (the weight-gradient products)
template <int EPI, int NP, bool GATHER, int MN, int XS>
__global__ void __launch_bounds__(Cfg2<EPI, NP, XS>::kThreads, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO,
                        const __grid_constant__ CUtensorMap tmG, PairArgs args)
{
    using C = Cfg2<EPI, NP, XS>;
    constexpr int S = C::kStages;
    constexpr uint32_t kIdesc = make_idesc(PM, NP);
    constexpr uint32_t kIdescBmn = make_idesc_major(PM, NP, false, true);
    constexpr uint32_t kIdescAB = make_idesc_major(PM, NP, true, true);
    constexpr int kBRows = NP / 2;  // B rows per CTA per stage

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_u32(smem_raw);
    uint8_t* base = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
    const uint32_t sA0 = smem_u32(base);
    const uint32_t sB0 = sA0 + S * kA2Bytes;
    const uint32_t sE0 = sA0 + S * C::kStageBytes;  // epilogue store tiles
    const uint32_t sG0 = sE0 + C::kEpiBytes;          // EPI_DSWIGLU: gate/up tiles
    uint64_t* bars =
        reinterpret_cast<uint64_t*>(base + S * C::kStageBytes + C::kEpiBytes + C::kGuBytes);
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(S + s); };
    auto tfull_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + a); };
    auto tempty_bar = [&](int a) { return bar0 + 8u * (uint32_t)(2 * S + 2 + a); };
    const uint32_t drain_bar = bar0 + 8u * (uint32_t)(2 * S + 4);
    auto gu_bar = [&](int w) { return bar0 + 8u * (uint32_t)(2 * S + 5 + w); };
    uint32_t* misc = reinterpret_cast<uint32_t*>(bars + C::kBars);  // [0] tmem, [1] abort
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
    int32_t* prefix = reinterpret_cast<int32_t*>(misc + 4);
    int32_t* offs = prefix + (args.groups + 1);
    int32_t* gather_tok = offs + (args.groups + 1);  // [HM] source rows of the current tile

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = args.groups;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), GATHER ? 3 : 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 2 * C::kEpiWarps * 32);
        }
        mbar_init(drain_bar, 1);
        if (EPI == EPI_DSWIGLU)
            for (int w = 0; w < C::kEpiWarps; ++w) mbar_init(gu_bar(w), 1);
        misc[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(misc), C::kTmemCols);
    pdl_wait();  // the previous kernel's writes (offsets, operands) are visible from here on
    // the one-SM kernel's tile counter starts at zero: written and fenced before this CTA's
    // trigger, and the one-SM launch starts only once every CTA of this one has triggered
    if (args.tail_ctr != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        *args.tail_ctr = 0;
        __threadfence();
    }
    // the one-SM kernel for small groups may run beside this one from now on (it reads
    // nothing this launch writes, and waits for this launch before it exits)
    if (args.early_trigger && threadIdx.x == 0) pdl_trigger();
    if (warp == 2 && EPI == EPI_WGRAD) {
        // groups by descending K length (ties: lower group first): order[rank] = group
        int32_t* kl = offs;
        int32_t* order = prefix;
        for (int g = lane; g < G; g += 32) kl[g] = args.k_offsets[g + 1] - args.k_offsets[g];
        __syncwarp();
        for (int g = lane; g < G; g += 32) {
            const int kg = kl[g];
            int r = 0;
            for (int h = 0; h < G; ++h) r += (kl[h] > kg || (kl[h] == kg && h < g)) ? 1 : 0;
            order[r] = g;
        }
    } else if (warp == 2) {
        auto row_off = [&](int g) -> int {
            return args.offsets ? args.offsets[g] : (g == 0 ? 0 : args.rows);
        };
        const int per = (G + 31) / 32;
        const int beg = lane * per < G ? lane * per : G;
        const int end = beg + per < G ? beg + per : G;
        // with skip_tails, groups of at most 128 rows are the one-SM tail kernel's
        auto tiles_of = [&](int n) -> int {
            return (args.skip_tails && n <= HM) ? 0 : (n + PM - 1) / PM;
        };
        int sum = 0;
        for (int g = beg; g < end; ++g) {
            const int r0 = row_off(g);
            offs[g] = r0;
            sum += tiles_of(row_off(g + 1) - r0);
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
            run += tiles_of(row_off(g + 1) - row_off(g));
        }
        if (lane == 31) prefix[G] = incl;
    }
    tc_fence_before();
    cluster_sync();  // barriers and TMEM of both CTAs ready before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = misc[0];
    constexpr bool kWgrad = (EPI == EPI_WGRAD);
    constexpr bool kGateUp =
        (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_SAVE);
    const int total = kWgrad ? G * args.m_tiles * args.n_tiles : prefix[G] * args.n_tiles;
    auto decode = [&](int t) -> PairTile {
        if (kWgrad) return decode_wgrad_tile(t, args, prefix, nclusters, total);
        return decode_pair_tile(t, args.n_tiles, G, prefix, offs, args.k_blocks);
    };

    if (warp == 0 && !GATHER) {
        // -------------------------------------------------------------- TMA producer
        // one thread: A and B tiles by TMA, bytes counted on the leader's full[s]
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t armed = 0, armed_phase = 0;
            const uint32_t fb0 = mapa_shared(full_bar(0), 0);  // the leader's full[0]
            // this CTA's B rows of a tile
            auto b_row_of = [&](const PairTile& tt) -> int {
                return kGateUp ? tt.g * args.b_rows_per_group + (leader ? 0 : args.half_rows) +
                                     tt.n * kBRows
                               : tt.g * args.b_rows_per_group + tt.n * NP + (int)rank * kBRows;
            };
            for (int t = cluster; t < total && !*abort_flag; t += nclusters) {
                const PairTile ti = decode(t);
                const int arow = (int)ti.row0 + (int)rank * HM;
                const int brow = kWgrad ? ti.n * NP + (int)rank * kBRows : b_row_of(ti);
                bool ok = true;
                for (int kb = 0; kb < ti.kbs; ++kb) {
                    if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = fb0 + 8u * (uint32_t)stage;
                    if (leader) mbar_expect_tx(full_bar(stage), 2 * C::kStageBytes);
                    const int kx = ti.k0 + kb * BK;
                    if (MN == 2) {
                        // this CTA's 128 A features as two 64-feature boxes of 64 K rows
                        tma_load_2d_pair(sA0 + (uint32_t)stage * kA2Bytes, &tmA, arow, kx, fb);
                        tma_load_2d_pair(sA0 + (uint32_t)stage * kA2Bytes + 8192u, &tmA,
                                         arow + 64, kx, fb);
                    } else {
                        tma_load_2d_pair(sA0 + (uint32_t)stage * kA2Bytes, &tmA, kx, arow, fb);
                    }
                    if (MN >= 1) {
                        // this CTA's B columns [bcol, bcol + kBRows) of rows g * b_k_rows + kx ..
                        const int bcol = ti.n * NP + (int)rank * kBRows;
#pragma unroll
                        for (int q = 0; q < kBRows / 64; ++q)
                            tma_load_2d_pair(sB0 + (uint32_t)stage * C::kBBytes + (uint32_t)q * 8192u,
                                             &tmB, bcol + 64 * q, ti.g * args.b_k_rows + kx, fb);
                    } else {
                        tma_load_2d_pair(sB0 + (uint32_t)stage * C::kBBytes, &tmB, kx, brow, fb);
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
            pdl_trigger();  // every load is issued: the next kernel may be scheduled
            if (*abort_flag && leader) {
                for (int s = 0; s < S; ++s)
                    if (armed & (1u << s))
                        wait_bounded(full_bar(s), (armed_phase >> s) & 1u, abort_flag,
                                     args.status, false);
            }
        }
    } else if (warp == 0) {
        // -------------------------------------------------------------- gathering producer
        // B (and A without a gather): TMA issued by lane 0, bytes counted on the leader's
        // full[s]. With a gather, A row r of this CTA's 128 is token row gather_rows[r] of
        // the A tensor: each lane copies 4 rows with 16-byte cp.async, writing the 128-byte
        // swizzle itself; kLag stages later it waits for those copies, fences them into
        // the async proxy, and lane 0 arrives once for the CTA on the leader's full[s].
        // Loop decisions are lane 0's, broadcast, so the warp stays converged.
        constexpr int kLag = S - 2;
        int stage = 0, sig_stage = 0, pending = 0;
        uint32_t phase = 0;
        uint32_t armed = 0, armed_phase = 0;
        const uint32_t fb0 = mapa_shared(full_bar(0), 0);
        auto signal_oldest = [&](int keep) {
            // all but `keep` of this lane's newest copy groups have landed
            if (keep >= kLag) cp_async_wait_group<kLag>();
            else cp_async_wait_all();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(fb0 + 8u * (uint32_t)sig_stage);
            if (++sig_stage == S) sig_stage = 0;
            --pending;
        };
        for (int t = cluster; t < total; t += nclusters) {
            if (!__shfl_sync(0xffffffffu, lane == 0 ? !*abort_flag : 0, 0)) break;
            const PairTile ti = decode(t);
            const int arow = (int)ti.row0 + (int)rank * HM;
            const int brow = kGateUp ? ti.g * args.b_rows_per_group +
                                           (leader ? 0 : args.half_rows) + ti.n * kBRows
                                     : ti.g * args.b_rows_per_group + ti.n * NP +
                                           (int)rank * kBRows;
            if (GATHER) {
                // source token of each of this CTA's 128 rows; rows past the group's end
                // repeat its last row (computed, never stored)
                const int64_t last = ti.row_end - 1;
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t r = (int64_t)arow + 32 * i + lane;
                    gather_tok[32 * i + lane] = args.gather_rows[r < ti.row_end ? r : last];
                }
                __syncwarp();
            }
            int ok = 1;
            for (int kb = 0; kb < ti.kbs; ++kb) {
                if (lane == 0)
                    ok = wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, args.status);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                const uint32_t fb = fb0 + 8u * (uint32_t)stage;
                const uint32_t sa = sA0 + (uint32_t)stage * kA2Bytes;
                if (lane == 0) {
                    if (leader)
                        mbar_expect_tx(full_bar(stage),
                                       GATHER ? 2 * C::kBBytes : 2 * C::kStageBytes);
                    if (!GATHER) tma_load_2d_pair(sa, &tmA, kb * BK, arow, fb);
                    tma_load_2d_pair(sB0 + (uint32_t)stage * C::kBBytes, &tmB, kb * BK, brow, fb);
                    armed |= 1u << stage;
                    armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                }
                if (GATHER) {
                    // each instruction copies 4 whole 128-byte rows: 8 lanes per row, one
                    // 16-byte chunk each, stored at its swizzled place
                    const int c = lane & 7;
#pragma unroll 8
                    for (int i = 0; i < HM / 4; ++i) {
                        const int r = 4 * i + (lane >> 3);  // row within this CTA's 128
                        const uint16_t* g =
                            args.a + (int64_t)gather_tok[r] * args.k + kb * BK + c * 8;
                        cp_async_16(sa + (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)), g);
                    }
                    cp_async_commit();
                    if (++pending > kLag) signal_oldest(kLag);
                }
                if (++stage == S) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
        }
        if (GATHER)
            while (pending > 0) signal_oldest(0);
        if (lane == 0 && *abort_flag && leader) {
            for (int s = 0; s < S; ++s)
                if (armed & (1u << s))
                    wait_bounded(full_bar(s), (armed_phase >> s) & 1u, abort_flag, args.status,
                                 false);
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------------------------------------------------- MMA issuer
            // K-major operand: +32 bytes per K=16 step inside the swizzle row; MN-major
            // operand: +2048 bytes (16 K rows of 128 bytes)
            const uint64_t ad0 = MN == 2 ? sw128_mn_desc(sA0, 8192u) : sw128_desc(sA0);
            const uint64_t bd0 = MN >= 1 ? sw128_mn_desc(sB0, 8192u) : sw128_desc(sB0);
            constexpr uint64_t astep = MN == 2 ? 128u : 2u;
            constexpr uint64_t bstep = MN >= 1 ? 128u : 2u;
            constexpr uint32_t idesc = MN == 2 ? kIdescAB : (MN == 1 ? kIdescBmn : kIdesc);
            int stage = 0;
            uint32_t phase = 0;
            int i = 0;
            for (int t = cluster; t < total && !*abort_flag; t += nclusters, ++i) {
                const int acc = i & 1;
                if (!wait_bounded(tempty_bar(acc), (((uint32_t)i >> 1) & 1u) ^ 1u, abort_flag,
                                  args.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * NP);
                const int kbs = kWgrad ? decode(t).kbs : args.k_blocks;
                bool ok = true;
                for (int kb = 0; kb < kbs; ++kb) {
                    if (!wait_bounded(full_bar(stage), phase, abort_flag, args.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // stage descriptors: the stage-0 ones plus the stage offset (16-byte units)
                    const uint64_t ad = ad0 + (uint64_t)((uint32_t)stage * (kA2Bytes >> 4));
                    const uint64_t bd = bd0 + (uint64_t)((uint32_t)stage * (C::kBBytes >> 4));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16_pair(d_tmem, ad + astep * (uint64_t)k, bd + bstep * (uint64_t)k,
                                      idesc, (kb | k) != 0 ? 1u : 0u);
                    mma_commit_pair_mc(empty_bar(stage), kPairMask);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair_mc(tfull_bar(acc), kPairMask);
            }
            mma_commit_pair(drain_bar);
            wait_bounded(drain_bar, 0u, abort_flag, args.status, false);
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lanes 32 q .. 32 q + 31 (a warp's lane quarter is warp % 4)
        const int row = q * 32 + lane;
        constexpr bool kTwo = C::kEpiWarps == 8;
        constexpr int cstep = kTwo ? 64 : 32;          // chunk stride of this warp's columns
        const int c0 = kTwo ? 32 * ((warp - 2) >> 2) : 0;  // and its first chunk
        const uint32_t tempty_leader0 = mapa_shared(tempty_bar(0), 0);
        const uint32_t tempty_leader1 = mapa_shared(tempty_bar(1), 0);
        const uint32_t ebuf = sE0 + (uint32_t)(kTwo ? warp - 2 : q) * 4096u;
        uint32_t eb = 0;  // which of the warp's two store tiles is next
        // this lane's row of a store tile: 64 bytes, 16-byte chunks at the swizzled place
        const uint32_t erow = (uint32_t)lane * 64u, eswz = ((uint32_t)lane >> 1) & 3u;
        // 32 x 32 block of rows [row_blk, +32), columns [col, +32): through shared memory
        // and TMA when the whole block is inside the group, else the valid rows directly
        // fp32 weight gradients and the kept gate/up values are not read again soon: their
        // lines go first when L2 needs room, ahead of the operands the tiles share
        const uint64_t evict_first =
            (EPI == EPI_WGRAD || EPI == EPI_SWIGLU_SAVE) ? l2_evict_first_policy() : 0ull;
        auto store_block = [&](const uint32_t (&pk)[16], bool full_blk, bool valid,
                               int row_blk, int col, uint16_t* dst_row,
                               const CUtensorMap* map) {
            if (full_blk) {
                const uint32_t b = ebuf + eb * 2048u;
                if (lane == 0) bulk_wait_read<1>();  // the tile stored two blocks ago is read
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
                    if (EPI == EPI_WGRAD || (EPI == EPI_SWIGLU_SAVE && map == &tmG))
                        tma_store_2d_hint(map, b, col, row_blk, evict_first);
                    else
                        tma_store_2d(map, b, col, row_blk);
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
        // EPI_DSWIGLU: this warp's gate/up tile (g at +0, u at +2 KiB; 64-byte rows, 64-byte
        // swizzle) and its barrier; one 16-column load is in flight at a time
        const uint32_t gbuf = sG0 + (uint32_t)(warp - 2) * 4096u;
        const uint32_t gbar = gu_bar(warp - 2);
        uint32_t gphase = 0;
        bool gu_pending = false, gu_ok = true;
        auto gu_issue = [&](int row_blk_, int col_) {
            mbar_expect_tx(gbar, 4096u);
            tma_load_2d(gbuf, &tmG, col_, row_blk_, gbar);
            tma_load_2d(gbuf + 2048u, &tmG, args.half_out + col_, row_blk_, gbar);
        };
        int i = 0;
        for (int t = cluster; t < total && !*abort_flag; t += nclusters, ++i) {
            const PairTile ti = decode(t);
            const int acc = i & 1;
            if (EPI == EPI_DSWIGLU) {
                // this row's gate and up values of the tile into L2 while the MMAs run, and
                // the warp's first 16-column tile of them into shared memory
                const int64_t r = ti.row0 + (int64_t)rank * HM + row;
                if (r < ti.row_end) {
                    const float* gr = args.gu + r * args.ld_gu + ti.n * NP;
#pragma unroll
                    for (int c = c0; c < NP; c += cstep) {
                        prefetch_l2(gr + c);
                        prefetch_l2(gr + args.half_out + c);
                    }
                }
                if (gu_ok) {
                    if (lane == 0)
                        gu_issue((int)(ti.row0 + (int64_t)rank * HM + q * 32), ti.n * NP + c0);
                    gu_pending = true;
                }
            }
            int ok = 1;
            if (lane == 0)
                ok = wait_bounded(tfull_bar(acc), ((uint32_t)i >> 1) & 1u, abort_flag, args.status);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * NP);
            const int64_t grow = ti.row0 + (int64_t)rank * HM + row;
            const bool valid = grow < ti.row_end;
            const int row_blk = (int)(ti.row0 + (int64_t)rank * HM + q * 32);
            const bool full_blk = (int64_t)row_blk + 31 < ti.row_end;
            uint16_t* out = static_cast<uint16_t*>(args.out);
            if (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_SAVE) {
#pragma unroll 1
                for (int c = c0; c < NP / 2; c += cstep) {
                    uint32_t g[32], u[32];
                    tmem_ld32(tbase + (uint32_t)c, g);
                    tmem_ld32(tbase + (uint32_t)(NP / 2 + c), u);
                    if (EPI == EPI_SWIGLU_SAVE) {
                        // the fp32 gate and up values, for the backward's SwiGLU derivative:
                        // four 16-column store tiles
                        const int gcol = ti.n * (NP / 2) + c;
                        float* gr = args.gu + grow * args.ld_gu + gcol;
#pragma unroll
                        for (int part = 0; part < 4; ++part) {
                            const uint32_t* src = (part < 2 ? g : u) + 16 * (part & 1);
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) pk[j] = src[j];
                            const int off = (part < 2 ? 0 : args.half_out) + 16 * (part & 1);
                            store_block(pk, full_blk, valid, row_blk, gcol + off,
                                        reinterpret_cast<uint16_t*>(gr + off), &tmG);
                        }
                    }
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
                    const int col = ti.n * (NP / 2) + c;
                    store_block(pk, full_blk, valid, row_blk, col, out + grow * args.ldo + col,
                                &tmO);
                }
            } else if (EPI == EPI_DSWIGLU) {
                // dh (fp32, this row's 32 intermediate columns) with the kept gate and up
                // values g, u: dg = dh u silu'(g), du = dh silu(g), where silu(g) = g s,
                // s = 1 / (1 + e^-g), silu'(g) = s (1 + g (1 - s)). g and u come 16 columns
                // at a time through the warp's shared-memory tile; the next 16 are loaded
                // while these are computed.
                const uint32_t grow_s = gbuf + (uint32_t)lane * 64u;
                const uint32_t gswz = ((uint32_t)lane >> 1) & 3u;
                const int row_blk_g = (int)(ti.row0 + (int64_t)rank * HM + q * 32);
#pragma unroll 1
                for (int c = c0; c < NP; c += cstep) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    const int col = ti.n * NP + c;
                    uint32_t pg[16], pu[16];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        // every lane waits: the barrier's completion makes the copy's
                        // bytes visible to the waiting thread
                        if (gu_pending) {
                            if (wait_bounded(gbar, gphase, abort_flag, args.status)) {
                                gphase ^= 1u;
                                gu_pending = false;
                            } else {
                                gu_ok = false;  // still in flight: drained before exit
                            }
                        }
                        uint32_t gw[16], uw[16];
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            const uint32_t off = (((uint32_t)v) ^ gswz) << 4;
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(gw[4 * v]), "=r"(gw[4 * v + 1]),
                                           "=r"(gw[4 * v + 2]), "=r"(gw[4 * v + 3])
                                         : "r"(grow_s + off)
                                         : "memory");
                            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                                         : "=r"(uw[4 * v]), "=r"(uw[4 * v + 1]),
                                           "=r"(uw[4 * v + 2]), "=r"(uw[4 * v + 3])
                                         : "r"(grow_s + 2048u + off)
                                         : "memory");
                        }
                        // the tile is read -- each lane's loads have returned (the values
                        // are used) and are ordered before the copy engine's next writes --
                        // so the next 16 columns may land in it
                        uint32_t used = 0;
#pragma unroll
                        for (int j = 0; j < 16; ++j) used |= gw[j] ^ uw[j];
                        asm volatile("" ::"r"(used));
                        fence_async_smem();
                        __syncwarp();
                        const int ncol = h == 0 ? col + 16 : col + cstep;
                        if (gu_ok && (h == 0 || c + cstep < NP)) {
                            if (lane == 0) gu_issue(row_blk_g, ncol);
                            gu_pending = true;
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            float dg2[2], du2[2];
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const float gv = __uint_as_float(gw[2 * j + h2]);
                                const float uv = __uint_as_float(uw[2 * j + h2]);
                                const float dh = __uint_as_float(r[16 * h + 2 * j + h2]);
                                const float sg = __frcp_rn(1.0f + __expf(-gv));
                                const float dsilu = sg * (1.0f + gv * (1.0f - sg));
                                dg2[h2] = dh * uv * dsilu;
                                du2[h2] = dh * (gv * sg);
                            }
                            pg[8 * h + j] = bf16x2_rne(dg2[0], dg2[1]);
                            pu[8 * h + j] = bf16x2_rne(du2[0], du2[1]);
                        }
                    }
                    store_block(pg, full_blk, valid, row_blk, col, out + grow * args.ldo + col,
                                &tmO);
                    const int ucol = args.half_out + col;
                    store_block(pu, full_blk, valid, row_blk, ucol, out + grow * args.ldo + ucol,
                                &tmO);
                }
            } else if (EPI == EPI_F32) {
                // fp32 rows plus the column bias (the router's logits)
                float* o = static_cast<float*>(args.out);
#pragma unroll 1
                for (int c = c0; c < NP; c += cstep) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    const int col = ti.n * NP + c;
                    if (valid) {
                        float v[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = __fadd_rn(__uint_as_float(r[j]),
                                             args.bias != nullptr ? args.bias[col + j] : 0.0f);
                        float4* dst = reinterpret_cast<float4*>(o + grow * args.ldo + col);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            } else if (EPI == EPI_WGRAD) {
                // fp32 weight gradient rows of group g (rows g * rows + m of the output), 16
                // columns per store tile; a group with no rows gives zeros
                float* o = static_cast<float*>(args.out);
                const int orow_blk = ti.g * args.rows + row_blk;
#pragma unroll 1
                for (int c = c0; c < NP; c += cstep) {
                    uint32_t r[32];
                    if (ti.kbs > 0) {
                        tmem_ld32(tbase + (uint32_t)c, r);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) r[j] = 0u;
                    }
                    uint32_t lo[16], hi[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        lo[j] = r[j];
                        hi[j] = r[16 + j];
                    }
                    const int col = ti.n * NP + c;
                    float* drow = o + ((int64_t)ti.g * args.rows + grow) * args.ldo + col;
                    store_block(lo, full_blk, valid, orow_blk, col,
                                reinterpret_cast<uint16_t*>(drow), &tmO);
                    store_block(hi, full_blk, valid, orow_blk, col + 16,
                                reinterpret_cast<uint16_t*>(drow + 16), &tmO);
                }
            } else {
#pragma unroll 1
                for (int c = c0; c < NP; c += cstep) {
                    uint32_t r[32];
                    tmem_ld32(tbase + (uint32_t)c, r);
                    uint32_t pk[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        pk[j] = bf16x2_rne(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                    const int col = ti.n * NP + c;
                    store_block(pk, full_blk, valid, row_blk, col, out + grow * args.ldo + col,
                                &tmO);
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        }
        if (EPI == EPI_DSWIGLU && gu_pending)
            wait_bounded(gbar, gphase, abort_flag, args.status, false);  // no load in flight
        if (lane == 0) bulk_wait_all();  // the TMA stores have written global memory
    }

    tc_fence_before();
    cluster_sync();  // the peer's last remote arrivals and the leader's MMAs are done
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::kTmemCols);
    }
}

template <int EPI, int NP, bool GATHER, int MN = 0, int XS = 0>
cudaError_t launch_pair_variant(const GemmProblem& p, cudaStream_t st)
{
    using C = Cfg2<EPI, NP, XS>;
    auto kernel = tc_gemm_pair_kernel<EPI, NP, GATHER, MN, XS>;
    const int groups = (p.offsets || EPI == EPI_WGRAD) ? p.groups : 1;
    const size_t smem = C::smem_bytes(groups);
    if (smem > 232448) return cudaErrorInvalidValue;  // more groups than shared memory holds
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    static bool attr_set[64] = {};
    static int max_clusters[64] = {};
    static size_t max_smem[64] = {};
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    if (max_clusters[dev] == 0 || smem > max_smem[dev]) {
        // co-resident clusters at this shared-memory size (one CTA per SM in practice)
        cfg.gridDim = dim3(2 * 74, 1, 1);
        cfg.numAttrs = 1;  // the cluster shape only
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, kernel, &cfg);
        cfg.numAttrs = 2;
        if (err != cudaSuccess) return err;
        if (n <= 0) return cudaErrorInvalidConfiguration;
        max_clusters[dev] = n;
        max_smem[dev] = smem;
    }
    const int64_t rows_total = p.offsets ? p.a_rows_total : p.rows;
    CUtensorMap ma, mb, mo, mg;
    const bool wgrad = (EPI == EPI_WGRAD);
    if (p.a_mn) {
        // [k, a_rows] with the features contiguous: boxes of 64 features x 64 K rows
        if (!wgrad || p.a_rows % 8 != 0) return cudaErrorInvalidValue;
        if (!make_map(&ma, p.a, p.k, p.a_rows, 64)) return cudaErrorInvalidValue;
    } else if (!make_map(&ma, p.a, p.a_rows, p.k, HM)) {
        return cudaErrorInvalidValue;
    }
    if (p.b_mn) {
        // [groups * b_k_rows, n] (EPI_WGRAD: [k, n]) with N contiguous: 64 x 64 boxes
        if (p.n % 64 != 0 || (!wgrad && p.b_k_rows < 1)) return cudaErrorInvalidValue;
        if (!make_map(&mb, p.b, wgrad ? (int64_t)p.k : (int64_t)groups * p.b_k_rows, p.n, 64))
            return cudaErrorInvalidValue;
    } else if (!make_map(&mb, p.b, wgrad ? (int64_t)p.n : (int64_t)groups * p.b_rows_per_group, p.k,
                         NP / 2)) {
        return cudaErrorInvalidValue;
    }
    if (wgrad) {
        // [groups * rows, n] fp32 in 32 x 16 store tiles
        if (!make_store_map_f32(&mo, p.out, (int64_t)groups * p.rows, p.n, p.ldo))
            return cudaErrorInvalidValue;
    } else if (EPI == EPI_F32) {
        mo = mb;  // fp32 rows are stored from registers; the store map is not used
    } else {
        const int out_cols = (EPI == EPI_DSWIGLU) ? 2 * p.n : p.n;
        if (!make_store_map(&mo, p.out, rows_total, out_cols, p.ldo))
            return cudaErrorInvalidValue;
    }
    PairArgs a;
    a.k_blocks = p.k / BK;
    constexpr bool kGateUpL =
        (EPI == EPI_SWIGLU || EPI == EPI_SWIGLU_SAVE);
    a.n_tiles = kGateUpL ? p.n / (NP / 2) : p.n / NP;
    a.groups = groups;
    a.offsets = p.offsets;
    a.rows = p.rows;
    a.b_rows_per_group = p.b_rows_per_group;
    a.half_rows = kGateUpL ? p.n : 0;
    a.m_tiles = wgrad ? (int)((p.rows + PM - 1) / PM) : 0;
    a.k_offsets = p.k_offsets;
    a.half_out =
        (EPI == EPI_DSWIGLU || EPI == EPI_SWIGLU_SAVE) ? p.n : 0;
    a.gu = p.gu;
    a.ld_gu = p.ld_gu;
    a.bias = p.bias;
    a.b_k_rows = wgrad ? 0 : p.b_k_rows;
    a.skip_tails = p.skip_tails;
    a.early_trigger = (p.skip_tails && p.side_sms > 0) ? 1 : 0;
    a.tail_ctr = p.skip_tails ? p.tail_ctr : nullptr;
    a.gather_rows = p.gather_rows;
    a.a = p.a;
    a.k = p.k;
    a.out = p.out;
    a.ldo = p.ldo;
    a.status = p.status;
    const int64_t max_tiles = wgrad ? (int64_t)groups * a.m_tiles * a.n_tiles
                                    : ((rows_total + PM - 1) / PM + groups) * a.n_tiles;
    int64_t clusters = max_clusters[dev];
    if (a.early_trigger) {
        // leave side_sms SMs to the one-SM kernel that runs beside this launch
        const int64_t keep = (num_sms() - p.side_sms) / 2;
        if (keep >= 1 && keep < clusters) clusters = keep;
    }
    if (max_tiles < clusters) clusters = max_tiles;
    if (clusters < 1) clusters = 1;
    cfg.gridDim = dim3((unsigned)(2 * clusters), 1, 1);
    if (EPI == EPI_SWIGLU_SAVE || EPI == EPI_DSWIGLU) {
        // the kept gate | up values: fp32 [rows, ld_gu] in 32 x 16 tiles (stored / loaded)
        if (!make_store_map_f32(&mg, p.gu, rows_total, 2 * (int64_t)p.n, p.ld_gu))
            return cudaErrorInvalidValue;
    } else {
        mg = mo;  // not used
    }
    return cudaLaunchKernelEx(&cfg, kernel, ma, mb, mo, mg, a);
}

// The expert products' main loops wait on operand stages about a sixth of the time (the
// ring full of loads in flight, none landed); a sixth stage cut down's waits from 23 % to
// 19 % of its MMA thread's time. It fits in a CTA's shared memory up to about 170 groups.
template <int EPI>
bool fits_extra_stage(const GemmProblem& p)
{
    const int groups = p.offsets ? p.groups : 1;
    return Cfg2<EPI, 256, 1>::kStages > Cfg2<EPI, 256, 0>::kStages &&
           Cfg2<EPI, 256, 1>::smem_bytes(groups) <= 232448;
}

}  // namespace

cudaError_t launch_tc_gemm_pair(const GemmProblem& p, cudaStream_t st)
{
    // K-major operands are read in 64-wide k-blocks; MN-major weight-gradient operands have
    // any number of K rows (the last block reads zeros past the end)
    if (!(p.epilogue == EPI_WGRAD && p.a_mn && p.b_mn) && p.k % BK != 0)
        return cudaErrorInvalidValue;
    if (p.epilogue == EPI_SWIGLU) {
        if (p.n % 128 != 0) return cudaErrorInvalidValue;
        if (p.gather_rows) return launch_pair_variant<EPI_SWIGLU, 256, true>(p, st);
        if (fits_extra_stage<EPI_SWIGLU>(p)) return launch_pair_variant<EPI_SWIGLU, 256, false, 0, 1>(p, st);
        return launch_pair_variant<EPI_SWIGLU, 256, false>(p, st);
    }
    if (p.gather_rows) return cudaErrorInvalidValue;
    if (p.epilogue == EPI_SWIGLU_SAVE) {
        if (p.n % 128 != 0 || p.gu == nullptr || p.ld_gu < 2 * (int64_t)p.n || p.ld_gu % 4 != 0 ||
            p.b_mn || p.skip_tails)
            return cudaErrorInvalidValue;
        return launch_pair_variant<EPI_SWIGLU_SAVE, 256, false>(p, st);
    }
    if (p.epilogue == EPI_DSWIGLU) {
        // dh = A . B with B MN-major (the down weights as stored), N = the intermediate size
        if (!p.b_mn || p.gu == nullptr || p.ld_gu < 2 * (int64_t)p.n || p.ld_gu % 4 != 0)
            return cudaErrorInvalidValue;
        if (p.n % 256 == 0) return launch_pair_variant<EPI_DSWIGLU, 256, false, 1>(p, st);
        if (p.n % 128 == 0) return launch_pair_variant<EPI_DSWIGLU, 128, false, 1>(p, st);
        return cudaErrorInvalidValue;
    }
    if (p.b_mn && p.epilogue != EPI_BF16 && p.epilogue != EPI_F32 && p.epilogue != EPI_WGRAD)
        return cudaErrorInvalidValue;
    if (p.epilogue == EPI_WGRAD) {
        if (p.k_offsets == nullptr || p.rows < 1) return cudaErrorInvalidValue;
        if (p.a_mn != p.b_mn) return cudaErrorInvalidValue;
        if (p.a_mn) {
            if (p.n % 256 == 0) return launch_pair_variant<EPI_WGRAD, 256, false, 2>(p, st);
            if (p.n % 128 == 0) return launch_pair_variant<EPI_WGRAD, 128, false, 2>(p, st);
            return cudaErrorInvalidValue;
        }
        if (p.n % 256 == 0) return launch_pair_variant<EPI_WGRAD, 256, false>(p, st);
        if (p.n % 128 == 0) return launch_pair_variant<EPI_WGRAD, 128, false>(p, st);
        return cudaErrorInvalidValue;
    }
    if (p.epilogue == EPI_F32) {
        if (p.b_mn) return cudaErrorInvalidValue;
        if (p.n % 256 == 0) return launch_pair_variant<EPI_F32, 256, false>(p, st);
        if (p.n % 128 == 0) return launch_pair_variant<EPI_F32, 128, false>(p, st);
        return cudaErrorInvalidValue;
    }
    if (p.epilogue == EPI_BF16) {
        if (p.b_mn) {
            if (p.n % 256 == 0) return launch_pair_variant<EPI_BF16, 256, false, 1>(p, st);
            if (p.n % 128 == 0) return launch_pair_variant<EPI_BF16, 128, false, 1>(p, st);
            return cudaErrorInvalidValue;
        }
        if (p.n % 256 == 0 && fits_extra_stage<EPI_BF16>(p))
            return launch_pair_variant<EPI_BF16, 256, false, 0, 1>(p, st);
        if (p.n % 256 == 0) return launch_pair_variant<EPI_BF16, 256, false>(p, st);
        if (p.n % 128 == 0) return launch_pair_variant<EPI_BF16, 128, false>(p, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace moe

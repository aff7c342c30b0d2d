// Internal declarations shared by the CUDA translation units of libmoe_b200.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------------------ status helpers

__device__ __forceinline__ void status_add(int32_t* status, int word, int v)
{
    if (status != nullptr && v != 0) atomicAdd(status + word, v);
}

// ------------------------------------------------------------------ dependent launch
// Every kernel of the library is launched with programmatic stream serialization: it may
// be scheduled while the kernel before it on the stream is still finishing, so its launch
// and setup overlap that kernel's tail. pdl_wait() blocks until the preceding grid has
// completed and its memory is visible; every kernel calls it before its first global
// memory access. pdl_trigger() lets the next kernel be scheduled early (a CTA that never
// calls it triggers when it exits).

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ------------------------------------------------------------------ launchers

// routing: one warp per token
cudaError_t launch_route(const moe_cfg& c, const float* logits, const float* sel_bias,
                         const uint8_t* mask, int32_t* ids, float* w, int32_t* status,
                         cudaStream_t st);

// dispatch
size_t permute_ws_bytes(const moe_cfg& c);
cudaError_t launch_permute(const moe_cfg& c, const int32_t* ids, int32_t* offsets,
                           int32_t* perm_token, int32_t* dest_row, int32_t* status, void* ws,
                           cudaStream_t st);
// fixed device scratch for moe_permute_noalloc (ints), and its device address
constexpr int64_t kPermuteFixedScratchInts = 262144;
cudaError_t permute_fixed_scratch(int32_t** out);
// x_perm[dest_row[t, j]] = x[t] for every routed assignment (token-major)
cudaError_t launch_gather_rows(const moe_cfg& c, const uint16_t* x, const int32_t* dest_row,
                               uint16_t* x_perm, cudaStream_t st);

// router statistics (tokens per expert, mean L1-normalised score, load-balance value)
size_t stats_ws_bytes(const moe_cfg& c);
cudaError_t launch_router_stats(const moe_cfg& c, const float* logits, const uint8_t* mask,
                                const int32_t* offsets, int32_t* counts, float* mean_prob,
                                float* aux, void* ws, cudaStream_t st);

// combine
cudaError_t launch_combine(const moe_cfg& c, const uint16_t* y, const float* w,
                           const int32_t* dest_row, const uint16_t* y_shared,
                           const uint8_t* mask, uint16_t* out, cudaStream_t st);

// order-invariant combine (canonical-order double sum of the exact terms)
cudaError_t launch_combine_invariant(const moe_cfg& c, const uint16_t* y, const float* w,
                                     const int32_t* dest_row, const uint16_t* y_shared,
                                     const uint8_t* mask, uint16_t* out, cudaStream_t st);

// backward (backward.cu)
cudaError_t launch_combine_bwd(const moe_cfg& c, const uint16_t* dout, const uint16_t* y,
                               const float* w, const int32_t* dest_row, const uint8_t* mask,
                               float* dw, uint16_t* dy, uint16_t* dy_shared, cudaStream_t st);
cudaError_t launch_router_bwd(const moe_cfg& c, const float* logits, const int32_t* ids,
                              const float* dw, const uint8_t* mask, float* dl, uint16_t* dl_bf,
                              int ld_bf, cudaStream_t st);
cudaError_t launch_unpermute(const moe_cfg& c, const uint16_t* rows, const int32_t* dest_row,
                             const uint16_t* shared, const uint16_t* router, const uint8_t* mask,
                             uint16_t* dx, cudaStream_t st);
cudaError_t launch_padded_offsets(const int32_t* off, int G, int rows, int32_t* poff,
                                  cudaStream_t st);
// split-K of a K-grouped product: koff[s] = min(s * chunk, rows rounded up to 64), s = 0..S
cudaError_t launch_split_offsets(int rows, int chunk, int S, int32_t* koff, cudaStream_t st);
// out[i] = sum over s = 0..S-1 in order of part[s * n + i] (n a multiple of 4)
cudaError_t launch_sum_parts(const float* part, int S, int64_t n, float* out, cudaStream_t st);
// dest_row (dispatch rows) -> rows of the layout whose expert ranges start at poff (each
// padded to 64 rows): r' = poff[e] + (r - off[e]), e = ids[a]; -1 stays -1
cudaError_t launch_pad_rows(const int32_t* ids, const int32_t* dest_row, const int32_t* off,
                            const int32_t* poff, int64_t A, int E, int32_t* dest_pad,
                            cudaStream_t st);
// zero rows [poff[g] + n_g, poff[g+1]) of a [rows, cols] bf16 buffer, n_g = off[g+1] - off[g]
cudaError_t launch_zero_pad_rows(uint16_t* buf, int64_t cols, const int32_t* off,
                                 const int32_t* poff, int G, cudaStream_t st);

// tensor-core GEMMs (tcgen05 / TMEM / TMA)
//   EPI_SWIGLU      out[r, c] = bf16(silu(g) * u) of A . B_g^T (gate and up columns paired)
//   EPI_BF16        out[r, c] = bf16(A . B_g^T)
//   EPI_SWIGLU_SAVE EPI_SWIGLU, also gu[r, c] = g, gu[r, n + c] = u (fp32, as accumulated)
//   EPI_DSWIGLU     dh = A . B_g^T kept in fp32, g = gu[r, c], u = gu[r, n + c]:
//                   out[r, c] = bf16(dh * u * silu'(g)), out[r, n + c] = bf16(dh * silu(g))
//   EPI_WGRAD       grouped over K: out[g][m, c] = fp32(sum over k in [k_offsets[g],
//                   k_offsets[g+1]) of A[m, k] * B[c, k]) -- an expert's rows contracted
//   EPI_F32         out[r, c] = fp32(A . B^T) + bias[c] (one rounded add; bias NULL: + 0)
enum GemmEpilogue {
    EPI_SWIGLU = 0,
    EPI_BF16 = 1,
    EPI_WGRAD = 3,
    EPI_F32 = 4,
    EPI_SWIGLU_SAVE = 5,
    EPI_DSWIGLU = 6
};

struct GemmProblem {
    int epilogue;            // GemmEpilogue
    const uint16_t* a;       // A [a_rows, k] bf16 (row-major, K-major)
    int64_t a_rows;          // rows of the A buffer (TMA bound)
    const int32_t* gather_rows;  // grouped row r reads A row gather_rows[r] (NULL: row r)
    int64_t a_rows_total;    // grouped rows (bound of offsets[groups])
    const uint16_t* b;       // B [groups * b_rows_per_group, k] bf16 (EPI_WGRAD: [n, k])
    int b_rows_per_group;    // SWIGLU: 2*I (gate rows then up rows); else N
    int k;                   // reduction length (multiple of 64; EPI_WGRAD: A's and B's width)
    int n;                   // output columns per group (SWIGLU: I)
    int groups;              // number of row groups (experts)
    const int32_t* offsets;  // device [groups+1] row ranges of A, or NULL: one group [0, rows)
    int rows;                // rows when offsets == NULL (EPI_WGRAD: rows of A = M)
    void* out;               // output [*, ldo]
    int64_t ldo;             // output row stride in elements
    const float* bias;       // EPI_F32: per-column bias or NULL
    int32_t* status;         // device status words (MOE_ST_PIPE_TIMEOUT) or NULL
    float* gu;               // EPI_SWIGLU_SAVE (written) / EPI_DSWIGLU (read): fp32 gate values
    int64_t ld_gu;           //   at columns [0, n), up values at [n, 2n), row stride ld_gu
    const int32_t* k_offsets;  // EPI_WGRAD: device [groups+1] K ranges (multiples of 64)
    int b_mn;                // B given MN-major, [groups * b_k_rows, n] (K rows of each group,
    int b_k_rows;            //   N contiguous), read without transposing (EPI_WGRAD: [k, n])
    int a_mn;                // EPI_WGRAD: A given MN-major, [k, a_rows] (features contiguous)
    int skip_tails;          // EPI_SWIGLU / EPI_BF16, K-major, no gather: the pair kernel leaves
                             // groups of at most 128 rows to launch_tc_gemm_tail
    int32_t* tail_ctr;       // with skip_tails: a device int the pair launch zeroes and the
                             // one-SM launch deals its tiles from, or NULL (dealt by CTA index)
    int side_sms;            // with skip_tails: > 0 runs the two launches side by side -- the
                             // pair kernel on 148 - side_sms SMs signalling its dependents at
                             // once, the one-SM kernel on side_sms SMs, waiting for the pair
                             // kernel only before it exits; 0 runs them one after the other
};

// the grouped expert products on CTA pairs
cudaError_t launch_tc_gemm_pair(const GemmProblem& p, cudaStream_t st);
// the groups a skip_tails pair launch left (those of 1..128 rows): one 128-row tile per
// such group on a single SM (tcgen05 cta_group::1, M = 128)
cudaError_t launch_tc_gemm_tail(const GemmProblem& p, cudaStream_t st);

// the router product: logits[T,E] = x . Wr^T (+ logit_bias), fp32
struct RouterProblem {
    const uint16_t* x;         // [T,H] bf16
    const uint16_t* w_router;  // [E,H] bf16
    int T, H, E;
    const float* logit_bias;   // [E] or NULL
    float* logits;             // [T,E] fp32 out
    int32_t* status;
};
cudaError_t launch_router(const RouterProblem& p, cudaStream_t st);

// diagnostic: one bounded pipeline wait that runs out (see moe_pipeline_wait_selftest)
cudaError_t launch_pipe_wait_selftest(int32_t* status, long long limit_cycles, cudaStream_t st);

// device facts
int num_sms();
bool device_is_sm100();
// blocks of `kernel` resident on the whole GPU at once (grid-stride kernels launched with
// exactly this many run as one wave)
int resident_blocks(const void* kernel, int threads, size_t smem);

}  // namespace moe

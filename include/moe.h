/*
 * moe.h -- C ABI of libmoe_b200: the forward pass of a top-k mixture-of-experts FFN
 * layer with a bitwise consistency contract, as hand-written sm_100a (B200) kernels.
 *
 * The layer (the semantic boundaries named in "DSV4 Flash MoE Train-Inference
 * Consistency Roadmap", Problem 2, and the MoE layer of SpecForge PR #1003):
 *
 *   logits = x . W_router^T (+ logit_bias)                     routing boundary
 *   s      = softmax(logits) or sigmoid(logits)               (unbiased scores)
 *   ids    = top-k of s + sel_bias, ties -> lower expert id
 *   w      = s[ids] / sum(s[ids]) * route_scale   (renorm)   or s[ids] * route_scale
 *   rows   = stable counting sort of the (token, rank) pairs by expert      dispatch
 *   y_r    = W2_e . (silu(W1g_e . x_t) * (W1u_e . x_t))  per dispatched row   experts
 *   out_t  = bf16( sum_j w_j * y_{row(t,j)}  [+ y_shared_t] )  fixed order   reduction
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers of the current CUDA device, row-major,
 *    densely packed, 16-byte aligned. bf16 tensors are passed as uint16_t* (raw bits).
 *  - The caller owns every buffer, including the workspace. The library allocates no
 *    device memory and keeps no per-call state; it caches only immutable per-device
 *    facts (SM count, kernel attributes, the driver's tensor-map encoder).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Calls only enqueue work
 *    on it and never synchronise the host, so they can be captured in a CUDA graph.
 *  - Return value: MOE_OK (0) or a negative MOE_ERR_* code. Arguments are validated on
 *    the host before anything is enqueued; on an error nothing is enqueued.
 *  - Data anomalies found on the device (NaN scores, a zero renormalisation
 *    denominator, expert ids out of range, a tensor-core pipeline wait that gave up)
 *    are counted in `status`, an int32[MOE_STATUS_WORDS] device array that the entry
 *    point clears at its start. Nothing traps or asserts on the device. Callers that
 *    want the fail-closed behaviour of the contract read `status` after the stream
 *    and reject the result when a word is nonzero (the Python binding does).
 *  - Results are bitwise reproducible: for a given build and GPU, a token's routes and
 *    output depend only on its own row and the weights -- never on T, on padding, on
 *    the order of the other tokens or on how a batch is split into calls.
 *
 * Shapes supported: 1 <= E <= 1024, 1 <= K <= min(E, 16), H % 128 == 0 and
 * 128 <= H <= 16384, I % 128 == 0, I_shared % 128 == 0 (0 = no shared expert),
 * 0 <= T and T * K < 2^31. T == 0 is a no-op. Group-limited selection: see moe_cfg.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(_WIN32)
#define MOE_API __declspec(dllexport)
#else
#define MOE_API __attribute__((visibility("default")))
#endif

/* return codes */
#define MOE_OK 0
#define MOE_ERR_ARG (-1)           /* a required pointer is NULL or misaligned */
#define MOE_ERR_SHAPE (-2)         /* a size outside the supported shapes */
#define MOE_ERR_WORKSPACE (-3)     /* ws_bytes smaller than moe_workspace_bytes() */
#define MOE_ERR_CUDA (-4)          /* a CUDA runtime/driver call or a launch failed */
#define MOE_ERR_UNIMPLEMENTED (-5) /* a valid request this build does not serve */
#define MOE_ERR_DEVICE (-6)        /* the current device is not sm_100 */

/* score functions */
#define MOE_SOFTMAX 0
#define MOE_SIGMOID 1
/*
 * sqrtsoftplus score, s = sqrt(softplus(l)) (named beside sigmoid in SpecForge PR #1003,
 * the load-balance commit; the pages give no formula). fp32, every step rounded to
 * nearest: softplus(l) = l for l > 20, else log1p_rl(exp_rl(l)), where log1p_rl(u) is
 * Goldberg's u * ln(1 + u) / ((1 + u) - 1) (u when 1 + u == 1) over a Cody-Waite natural
 * log (odd atanh series through z^9); then the IEEE square root.
 */
#define MOE_SQRTSOFTPLUS 2

/* words of the device status array */
#define MOE_ST_NAN_TOKENS 0     /* tokens with a NaN selection score */
#define MOE_ST_ZERO_DENOM 1     /* tokens whose renormalisation denominator was 0 */
#define MOE_ST_BAD_EXPERT_ID 2  /* expert ids >= E met by the dispatch (not counting -1) */
#define MOE_ST_PIPE_TIMEOUT 3   /* a tensor-core pipeline wait gave up (result invalid) */
#define MOE_STATUS_WORDS 8

/* stages, for moe_workspace_bytes */
#define MOE_STAGE_ROUTE 0
#define MOE_STAGE_PERMUTE 1
#define MOE_STAGE_FFN 2
#define MOE_STAGE_COMBINE 3
#define MOE_STAGE_FORWARD 4
#define MOE_STAGE_STATS 5
#define MOE_STAGE_BACKWARD 6

/* number of CUDA events moe_forward can record (stage boundaries), see moe_forward */
#define MOE_NUM_STAGE_EVENTS 8

typedef struct moe_cfg {
    int32_t T;           /* tokens in this call */
    int32_t H;           /* hidden size */
    int32_t E;           /* routed experts */
    int32_t K;           /* experts per token (top-k) */
    int32_t I;           /* routed expert intermediate size */
    int32_t I_shared;    /* shared (always-on) expert intermediate size, 0 = none */
    int32_t score_fn;    /* MOE_SOFTMAX, MOE_SIGMOID or MOE_SQRTSOFTPLUS */
    int32_t renorm;      /* 1: weights renormalised over the K selected scores */
    float route_scale;   /* weights are multiplied by it (1.0 = unchanged) */
    /*
     * Group-limited selection (the DeepSeek family's override of the selection step,
     * SpecForge PR #1003, "Out of scope"; the pages name it without a formula). 0 or 1 =
     * off. Otherwise the E experts form n_group contiguous groups of E / n_group; a
     * group's score is the fp32 sum of its two best choices (s + sel_bias, best first,
     * the tie rule of the selection; one choice when a group has one expert); the
     * topk_group best groups are kept (higher score, then lower group id) and the K
     * experts are chosen among the kept groups only. Weights still come from the unbiased
     * scores. Needs E % n_group == 0, n_group <= 32, 1 <= topk_group <= n_group and
     * K <= topk_group * (E / n_group); anything else is MOE_ERR_SHAPE.
     */
    int32_t n_group;
    int32_t topk_group;
} moe_cfg;

/*
 * Bytes of workspace the given stage needs for cfg (MOE_STAGE_FORWARD: moe_forward).
 * Returns 0 for an invalid cfg as well as for stages that need none.
 */
MOE_API size_t moe_workspace_bytes(const moe_cfg* cfg, int stage);

/*
 * Routing boundary ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 1
 * "Routing Is A Discrete Decision": router logits, top-k ids, top-k weights and the
 * tie rule; SpecForge PR #1003, the selection-bias commit: the bias shifts only the
 * picks, the weights come from the unbiased scores).
 *
 *  x          [T,H] bf16, or NULL: then `logits` is an INPUT ([T,E] fp32) and the
 *             router product is skipped (replaying or injecting logits).
 *  w_router   [E,H] bf16 (ignored when x is NULL).
 *  logit_bias [E] fp32 or NULL, added to the logits (part of the logits, not of the
 *             selection).
 *  sel_bias   [E] fp32 or NULL: choice = score + sel_bias selects the experts; the
 *             weights still use the unbiased score.
 *  token_mask [T] uint8 or NULL (all tokens real): a 0 marks padding; such tokens get
 *             ids -1 and weights 0 and are skipped by every later stage.
 *  logits     [T,E] fp32: output (x given) or input (x NULL).
 *  topk_ids   [T,K] int32 out, rank order (rank 0 = best).
 *  topk_w     [T,K] fp32 out.
 *  status     int32[MOE_STATUS_WORDS] device, cleared then counted; may be NULL.
 * Score arithmetic is the FP32 contract: exp_rl, the 32-lane softmax tree, IEEE
 * round-to-nearest adds/multiplies/divides, no FMA contraction outside exp_rl.
 * Degenerate rows fail closed through the status words rather than by a made-up value:
 * a softmax row whose logits are all -inf (or that holds a NaN) has no defined
 * distribution -- its max is -inf, so every l - max is NaN -- and every score is NaN;
 * the row counts once in MOE_ST_NAN_TOKENS, NaN keys rank below every number so it
 * takes ids 0..K-1 by the tie rule, and its weights are NaN. A sigmoid or sqrtsoftplus
 * row of all -inf has scores +0: it takes ids 0..K-1, a renormalised row counts in
 * MOE_ST_ZERO_DENOM and its weights are 0.
 */
MOE_API int moe_route(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                      const float* logit_bias, const float* sel_bias,
                      const uint8_t* token_mask, float* logits, int32_t* topk_ids,
                      float* topk_w, int32_t* status, void* stream);

/*
 * Dispatch boundary ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 2:
 * token-to-expert map and valid token counts). A stable counting sort of the T*K
 * assignments a = t*K + j by expert id, ties kept in increasing a.
 *
 *  topk_ids   [T,K] int32 (-1 = not routed, e.g. padding; ids >= E are counted in
 *             status[MOE_ST_BAD_EXPERT_ID] and not routed).
 *  x          [T,H] bf16 or NULL; with x and x_perm given, row r of x_perm receives
 *             x[perm_token[r]].
 *  offsets    [E+1] int32 out: rows of expert e are offsets[e] .. offsets[e+1]-1.
 *  perm_token [T*K] int32 out: row -> token (rows >= offsets[E] are left untouched).
 *  dest_row   [T*K] int32 out: assignment -> row, -1 when not routed.
 *  x_perm     [T*K,H] bf16 out or NULL.
 *  ws         moe_workspace_bytes(cfg, MOE_STAGE_PERMUTE) bytes of device scratch.
 */
MOE_API int moe_permute(const moe_cfg* cfg, const int32_t* topk_ids, const uint16_t* x,
                        int32_t* offsets, int32_t* perm_token, int32_t* dest_row,
                        uint16_t* x_perm, int32_t* status, void* ws, size_t ws_bytes,
                        void* stream);

/*
 * moe_permute without a caller workspace. The source pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory at the point where
 * they dispatch -- for example an engine plug-in that is handed only the tensors of the
 * current step and must not grow or fragment the engine's memory pool, or plain C code
 * that has no device allocator of its own. It computes exactly what moe_permute computes
 * (same arguments minus ws/ws_bytes) and allocates nothing: its per-block histograms live
 * in one fixed 1 MiB device array inside the library (262144 int32), which every GPU that
 * loads the library holds until the process exits.
 *
 *  Limit: ceil(T*K / 2048) * E <= 262144 (e.g. E = 128 allows T*K <= 4,194,304); larger
 *         requests return MOE_ERR_WORKSPACE before anything is enqueued.
 *  Every call looks up the array's device address on the caller's current device (a
 *  host-side query that allocates nothing), so a device reset or a new primary context
 *  between calls does not leave a stale address behind. The first call on a device may
 *  load the library's device code there: make that first call before any stream capture.
 *  All calls share the array and it keeps the last call's contents; nothing in it needs
 *  to start at zero (every call overwrites what it reads). Calls that overlap on the GPU
 *  (other streams, other host threads) race on it: serialise them.
 */
MOE_API int moe_permute_noalloc(const moe_cfg* cfg, const int32_t* topk_ids, const uint16_t* x,
                                int32_t* offsets, int32_t* perm_token, int32_t* dest_row,
                                uint16_t* x_perm, int32_t* status, void* stream);

/*
 * Expert boundary ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 2:
 * gate_and_up -> down; SpecForge PR #1003, experts.py: grouped experts and the
 * always-on shared expert). Grouped SwiGLU GEMMs on the tensor cores:
 *   h_r = bf16( silu(x_r . W13[e, 0:I]^T) * (x_r . W13[e, I:2I]^T) )   (fp32 accumulate)
 *   y_r = bf16( h_r . W2[e]^T )                                        (fp32 accumulate)
 * for every row r of expert e, with a reduction order that is fixed per (H, I): never
 * a function of T, of the rows per expert or of the row's place in a tile.
 *
 *  x          [T,H] bf16 tokens (read by the shared expert, and by the routed experts
 *             through perm_token when x_perm is NULL).
 *  x_perm     [T*K,H] bf16 dispatched rows (from moe_permute), or NULL to gather the
 *             rows from x via perm_token inside the GEMM.
 *  perm_token [T*K] int32 from moe_permute (required when x_perm is NULL).
 *  offsets    [E+1] int32 from moe_permute.
 *  w13        [E, 2I, H] bf16: rows 0..I-1 gate, rows I..2I-1 up (each row K-major).
 *  w2         [E, H, I] bf16.
 *  w13_s, w2_s  shared expert [2*I_shared, H] and [H, I_shared] bf16, or NULL.
 *  y          [T*K, H] bf16 out, row r = output of dispatched row r.
 *  y_shared   [T, H] bf16 out (required when the shared expert is given).
 *  status     as in moe_route (only MOE_ST_PIPE_TIMEOUT is used here), may be NULL.
 *  ws         moe_workspace_bytes(cfg, MOE_STAGE_FFN) bytes.
 */
MOE_API int moe_grouped_ffn(const moe_cfg* cfg, const uint16_t* x, const uint16_t* x_perm,
                            const int32_t* perm_token, const int32_t* offsets,
                            const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                            const uint16_t* w2_s, uint16_t* y, uint16_t* y_shared,
                            int32_t* status, void* ws, size_t ws_bytes, void* stream);

/*
 * Reduction boundary ("DSV4 Flash MoE Train-Inference Consistency Roadmap", Problem 3
 * "Final Reduction Is The Core Drift Point"; "From Expert Reduction to Behavioral
 * Divergence", Abstract: the order of the expert sum is part of the contract).
 * Per token t and column h, in FP32 with IEEE round-to-nearest and no FMA:
 *   acc = w_0 * y[dest_row[t,0], h]; acc += w_j * y[dest_row[t,j], h] for j = 1..K-1
 *   (each product rounded, rank order, terms with dest_row < 0 skipped),
 *   then acc += y_shared[t, h] if given; out = bf16 round-to-nearest-even(acc).
 * Tokens with token_mask[t] == 0 get out = 0.
 *
 *  y [T*K,H] bf16, topk_w [T,K] fp32, dest_row [T,K] int32, y_shared [T,H] bf16 or NULL,
 *  token_mask [T] uint8 or NULL, out [T,H] bf16.
 */
MOE_API int moe_combine(const moe_cfg* cfg, const uint16_t* y, const float* topk_w,
                        const int32_t* dest_row, const uint16_t* y_shared,
                        const uint8_t* token_mask, uint16_t* out, void* stream);

/*
 * Order-invariant combine ("From Expert Reduction to Behavioral Divergence", arXiv
 * 2607.28097, Abstract: scheme C keeps routes and texts because its result does not
 * depend on the order of the expert terms). Same arguments and masking as moe_combine;
 * per output element the terms w_j * y[dest_row[t,j]] (formed exactly in double) and
 * y_shared[t] are summed in double in a canonical order -- ascending magnitude, the
 * negative of two equal magnitudes first -- then rounded to fp32 and to bf16 (nearest
 * even). Any permutation of a token's (topk_w, dest_row) pairs gives the same bits.
 * An alternative to the contract's rank-order combine, not used by moe_forward.
 */
MOE_API int moe_combine_invariant(const moe_cfg* cfg, const uint16_t* y, const float* topk_w,
                                  const int32_t* dest_row, const uint16_t* y_shared,
                                  const uint8_t* token_mask, uint16_t* out, void* stream);

/*
 * The whole layer (SpecForge PR #1003, layer.py: MoELayer = router + routed experts +
 * optional shared expert): moe_route -> moe_permute -> moe_grouped_ffn -> moe_combine
 * on one stream, intermediates in `ws`.
 *
 *  Inputs as in the stages above; out [T,H] bf16.
 *  Optional boundary outputs (NULL = not kept): logits [T,E] fp32, topk_ids [T,K],
 *  topk_w [T,K], offsets [E+1].
 *  status     int32[MOE_STATUS_WORDS] device, required.
 *  ws         moe_workspace_bytes(cfg, MOE_STAGE_FORWARD) bytes.
 *  stage_events NULL, or MOE_NUM_STAGE_EVENTS cudaEvent_t handles recorded on `stream`
 *             at the stage boundaries: [0] start (after the status words are cleared),
 *             [1] after router logits, [2] after routing, [3] after dispatch, [4] after
 *             gate_up, [5] after down, [6] after the shared expert, [7] after the combine
 *             (timing only).
 */
MOE_API int moe_forward(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                        const float* logit_bias, const float* sel_bias,
                        const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                        const uint16_t* w13_s, const uint16_t* w2_s, uint16_t* out,
                        float* logits, int32_t* topk_ids, float* topk_w, int32_t* offsets,
                        int32_t* status, void* ws, size_t ws_bytes, void* const* stage_events,
                        void* stream);

/*
 * Router statistics of one routed batch (SpecForge PR #1003, the load-balance commit: a
 * Switch-style load-balance value E * sum_e load_e * mean_prob_e over the kept tokens,
 * K when balanced, with scores L1-normalised per token). Over the N tokens with
 * token_mask != 0 (all when NULL):
 *   tokens_per_expert[e] = offsets[e+1] - offsets[e]          (from moe_permute/moe_forward)
 *   mean_prob[e] = (1/N) sum_t s[t,e] / sum_e' s[t,e']  (s: unbiased scores of `logits`)
 *   aux = E * sum_e (tokens_per_expert[e] / N) * mean_prob[e]
 * fp32, summed in a fixed order (deterministic for a given T, no atomics); N == 0 gives 0.
 *  logits [T,E] fp32, token_mask [T] uint8 or NULL, offsets [E+1] int32 (device);
 *  tokens_per_expert [E] int32, mean_prob [E] fp32, aux [1] fp32 (device, out);
 *  ws   moe_workspace_bytes(cfg, MOE_STAGE_STATS) bytes.
 */
MOE_API int moe_router_stats(const moe_cfg* cfg, const float* logits, const uint8_t* token_mask,
                             const int32_t* offsets, int32_t* tokens_per_expert,
                             float* mean_prob, float* aux, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * The whole layer from and to HOST memory, overlapping the transfers with the compute
 * (the chunked form is exact: results are bitwise independent of how tokens are split).
 * Tokens are processed in chunks around a nominal `chunk_tokens` = C: up to 2 C tokens in
 * equal chunks of at most C; beyond that a first and a last chunk of C / 2 (a short pipeline
 * fill and drain) with equal chunks of at most 3 C / 2 between them. The host->device copy
 * of chunk i+1 and the device->host copy of chunk i-1 run on two library-owned copy
 * streams while chunk i runs on `stream`, double-buffered in `ws`. When `stream`
 * completes, out_host holds the result. Same output bits as moe_forward on the same tokens.
 *
 *  x_host       [T,H] bf16 in HOST memory (page-locked for the copies to overlap).
 *  out_host     [T,H] bf16 in HOST memory (page-locked).
 *  token_mask   [T] uint8 in DEVICE memory, or NULL.
 *  weights, biases, status: DEVICE, as in moe_forward.
 *  ws           moe_forward_host_workspace_bytes(cfg, chunk_tokens) bytes (device).
 * The copy streams and their events are created on a device's first call and kept until
 * the process exits; calls on one device must not overlap in host threads.
 */
MOE_API size_t moe_forward_host_workspace_bytes(const moe_cfg* cfg, int chunk_tokens);
MOE_API int moe_forward_host(const moe_cfg* cfg, const uint16_t* x_host, const uint16_t* w_router,
                             const float* logit_bias, const float* sel_bias,
                             const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                             const uint16_t* w13_s, const uint16_t* w2_s, uint16_t* out_host,
                             int32_t* status, int chunk_tokens, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * Backward of the whole layer (forward + backward is the contract's scope: "DSV4 Flash MoE
 * Train-Inference Consistency Roadmap", "Why DSV4 Flash MoE Drifts More Easily" and the
 * DSV4-WS1-2 row of "Follow-Up Issue Buckets"; the pages give no backward arithmetic).
 * Gradients of sum(dout * out) for the routes of the forward (selection has no gradient).
 * The forward intermediates (dispatch, h, y and the fp32 gate/up values) are recomputed from
 * x with the forward's kernels (same bits), or taken from `ws` after moe_forward_train.
 *
 *  Inputs (DEVICE): x, w_router, token_mask (or NULL), w13, w2, w13_s/w2_s as in
 *    moe_forward; logits [T,E] fp32, topk_ids [T,K], topk_w [T,K] as the forward returned
 *    them; dout [T,H] bf16.
 *  Outputs (DEVICE, written completely):
 *    dx [T,H] bf16, dw_router [E,H] fp32, dw13 [E,2I,H] fp32, dw2 [E,H,I] fp32,
 *    dw13_s [2I_shared,H] / dw2_s [H,I_shared] fp32 (required when I_shared > 0),
 *    d_topk_w [T,K] fp32 and dlogits [T,E] fp32 (optional boundary outputs, NULL = not kept).
 *  Arithmetic (fixed order, no float atomics: bitwise repeatable; dx of a token depends
 *  only on its own row):
 *    d_topk_w[t,j] = dot32(dout_t, y_row): lane L of 32 sums the rounded products of the
 *      8-element chunks L, L+32, ... in order, then butterfly levels 16..1 (fp32);
 *    dy_row = bf16(topk_w[t,j] * dout_t); dy_shared = dout (0 for masked tokens);
 *    dh = dy . W2_e kept in fp32; [dg | du] = bf16(dh * u * silu'(g) | dh * silu(g)) with
 *      g, u the forward's fp32 gate/up products; dx_row = bf16([dg | du] . W13_e);
 *    dlogits: through the renormalisation and the score function in fp32, each operation
 *      rounded to nearest, rank-order sums (see the router backward of the oracle);
 *    dx_t = bf16(rank-order sum of dx_row + shared term + bf16(dlogits_t) . W_router), +0
 *      for masked tokens;
 *    dW = sum over an expert's rows, ascending, of dy^T h / [dg|du]^T x (fp32 accumulation
 *      on the tensor cores, bf16 operands); dW_router = sum over fixed token chunks (a
 *      function of E, H and T), in chunk order, of the chunks' sums of bf16(dlogits_t)^T x_t.
 *  saved  0: the forward intermediates are recomputed from x; 1: `ws` holds those that
 *         moe_forward_train wrote for the same cfg, inputs and routes (not checked).
 *  ws  moe_workspace_bytes(cfg, MOE_STAGE_BACKWARD) bytes.
 */
MOE_API int moe_backward(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                         const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                         const uint16_t* w13_s, const uint16_t* w2_s, const float* logits,
                         const int32_t* topk_ids, const float* topk_w, const uint16_t* dout,
                         uint16_t* dx, float* dw_router, float* dw13, float* dw2, float* dw13_s,
                         float* dw2_s, float* d_topk_w, float* dlogits, int saved,
                         int32_t* status, void* ws, size_t ws_bytes, void* stream);

/*
 * The forward of a training step: the same output bits as moe_forward, and the dispatch
 * and expert intermediates the backward needs left in `ws` (the backward's workspace,
 * moe_workspace_bytes(cfg, MOE_STAGE_BACKWARD) bytes), so that moe_backward with saved = 1
 * on the same ws, cfg, inputs and routes skips recomputing them. logits, topk_ids and topk_w
 * (device outputs, required) are the routes the backward takes.
 */
MOE_API int moe_forward_train(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                              const float* logit_bias, const float* sel_bias,
                              const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                              const uint16_t* w13_s, const uint16_t* w2_s, uint16_t* out,
                              float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                              void* ws, size_t ws_bytes, void* stream);

/* Text of a return code. */
MOE_API const char* moe_status_string(int code);

/* ABI version of this header (major * 100 + minor). */
MOE_API int moe_abi_version(void);

/*
 * Diagnostic of the fail-closed path ("DSV4 Flash MoE Train-Inference Consistency
 * Roadmap", Follow-Up Issue Buckets: mismatches fail closed). Every pipeline wait of the
 * library's tensor-core and staged-copy kernels is bounded; when one runs out, the kernel
 * stops issuing work, drains what it has in flight, frees its tensor memory, counts
 * MOE_ST_PIPE_TIMEOUT and returns. This call runs that bounded wait once, in a one-CTA
 * kernel, on an mbarrier that nothing arrives on, with the limit shortened to
 * limit_cycles (1000 .. 2e9 SM clock cycles; the kernels use about 2e9): the wait gives up
 * and status[MOE_ST_PIPE_TIMEOUT] becomes 1 instead of the GPU hanging. Nothing else is
 * in flight in that kernel, so it cannot leave the device in a bad state.
 *  status  int32[MOE_STATUS_WORDS] device, cleared first.
 * Returns MOE_ERR_ARG for a NULL status or a limit out of range.
 */
MOE_API int moe_pipeline_wait_selftest(int32_t* status, long long limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

// C ABI of libmoe_b200 (declared in include/moe.h): argument checks, workspace layout,
// tensor-core GEMM set-up and the launch sequence of each boundary. Host code only; the
// kernels live in route.cu, permute.cu, tc_gemm.cu and combine.cu.
#include <math.h>
#include <string.h>

#include <mutex>

#include "moe_internal.cuh"

namespace moe {

// SMs the one-SM kernel of small experts starts on beside the pair kernel: below 192
// routed rows per expert on average, and from 192 to 511. It takes its tiles from a
// counter, so its CTAs past these take the small experts left when pair CTAs finish;
// measured against 64/36 and 32/16 on the 30B-A3B layer (T = 2048 .. 16384) and the
// sigmoid layer (T = 4096, 8192): 48/24 was the fastest or within 1 % everywhere.
constexpr int kSideSmsLow = 48;
constexpr int kSideSmsHigh = 24;

int num_sms()
{
    static int cached[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

int resident_blocks(const void* kernel, int threads, size_t smem)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    return num_sms() * per_sm;
}

bool device_is_sm100()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return false;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return false;
    return major == 10 && minor == 0;
}

namespace {

constexpr size_t kAlign = 256;

size_t up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

int check_cfg(const moe_cfg* c)
{
    if (c == nullptr) return MOE_ERR_ARG;
    if (c->T < 0 || c->E < 1 || c->E > 1024 || c->K < 1 || c->K > 16 || c->K > c->E)
        return MOE_ERR_SHAPE;
    if (c->H < 128 || c->H > 16384 || c->H % 128 != 0) return MOE_ERR_SHAPE;
    if (c->I < 128 || c->I > 16384 || c->I % 128 != 0) return MOE_ERR_SHAPE;
    if (c->I_shared < 0 || c->I_shared > 32768 || c->I_shared % 128 != 0) return MOE_ERR_SHAPE;
    if ((int64_t)c->T * c->K >= ((int64_t)1 << 31)) return MOE_ERR_SHAPE;
    if (c->score_fn != MOE_SOFTMAX && c->score_fn != MOE_SIGMOID &&
        c->score_fn != MOE_SQRTSOFTPLUS)
        return MOE_ERR_SHAPE;
    if (c->renorm != 0 && c->renorm != 1) return MOE_ERR_SHAPE;
    if (!isfinite(c->route_scale)) return MOE_ERR_SHAPE;
    if (c->n_group < 0 || c->n_group > 32) return MOE_ERR_SHAPE;
    if (c->n_group > 1) {
        if (c->E % c->n_group != 0 || c->topk_group < 1 || c->topk_group > c->n_group ||
            c->K > c->topk_group * (c->E / c->n_group))
            return MOE_ERR_SHAPE;
    }
    return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device()
{
    return device_is_sm100() ? MOE_OK : MOE_ERR_DEVICE;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// scratch of moe_grouped_ffn: h [T*K, I] (+ h_shared [T, I_shared]), bf16, and the tile
// counters of the two one-SM launches (gate_up's, down's)
struct FfnLayout {
    size_t h, h_s, ctr, total;
};

FfnLayout ffn_layout(const moe_cfg& c)
{
    FfnLayout L{};
    const size_t A = (size_t)c.T * c.K;
    size_t off = 0;
    L.h = off;
    off += up(A * c.I * 2);
    L.h_s = off;
    off += up((size_t)c.T * c.I_shared * 2);
    L.ctr = off;
    off += up(2 * sizeof(int32_t));
    L.total = off;
    return L;
}

// scratch of moe_forward
struct FwdLayout {
    size_t logits, ids, w, offsets, perm_token, dest_row, perm_ws, x_perm, y, y_s, ffn, total;
};

FwdLayout fwd_layout(const moe_cfg& c)
{
    FwdLayout L{};
    const size_t A = (size_t)c.T * c.K;
    size_t off = 0;
    L.logits = off;     off += up((size_t)c.T * c.E * 4);
    L.ids = off;        off += up(A * 4);
    L.w = off;          off += up(A * 4);
    L.offsets = off;    off += up((size_t)(c.E + 1) * 4);
    L.perm_token = off; off += up(A * 4);
    L.dest_row = off;   off += up(A * 4);
    L.perm_ws = off;    off += up(permute_ws_bytes(c));
    L.x_perm = off;     off += up(A * c.H * 2);
    L.y = off;          off += up(A * c.H * 2);
    L.y_s = off;        off += up(c.I_shared ? (size_t)c.T * c.H * 2 : 0);
    L.ffn = off;        off += ffn_layout(c).total;
    L.total = off;
    return L;
}

template <class T>
T* at(void* ws, size_t off)
{
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

int rec(void* const* ev, int i, cudaStream_t st)
{
    if (ev == nullptr || ev[i] == nullptr) return MOE_OK;
    return cuda_rc(cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st));
}

// router on the tensor cores (logits[T,E] = x . Wr^T + bias, fp32), then the routing kernel
int router_and_route(const moe_cfg& c, const uint16_t* x, const uint16_t* wr,
                     const float* logit_bias, const float* sel_bias, const uint8_t* mask,
                     float* logits, int32_t* ids, float* w, int32_t* status, void* const* ev,
                     cudaStream_t st)
{
    RouterProblem p{};
    p.x = x;
    p.w_router = wr;
    p.T = c.T;
    p.H = c.H;
    p.E = c.E;
    p.logit_bias = logit_bias;
    p.logits = logits;
    p.status = status;
    int rc;
    if ((rc = cuda_rc(launch_router(p, st))) != MOE_OK) return rc;
    if ((rc = rec(ev, 1, st)) != MOE_OK) return rc;
    if ((rc = cuda_rc(launch_route(c, logits, sel_bias, mask, ids, w, status, st))) != MOE_OK)
        return rc;
    return rec(ev, 2, st);
}

// gate_up + SwiGLU over grouped rows: h[r] = silu(a_r . W1g^T) * (a_r . W1u^T), where
// a_r is row gather[r] of a when gather is given (the dispatch fused into the GEMM's
// operand loads) and row r otherwise
// (tail_ctr: a device int for the one-SM launch's tile counter, or NULL)
cudaError_t gate_up(const uint16_t* a, int64_t a_rows, const int32_t* gather, int64_t grouped_rows,
                    const int32_t* offsets, int groups, int rows, const uint16_t* w13, int H, int I,
                    uint16_t* h, int32_t* status, int32_t* tail_ctr, cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_SWIGLU;
    p.a = a;
    p.a_rows = a_rows;
    p.gather_rows = gather;
    p.a_rows_total = grouped_rows;
    p.b = w13;
    p.b_rows_per_group = 2 * I;
    p.k = H;
    p.n = I;
    p.groups = groups;
    p.offsets = offsets;
    p.rows = rows;
    p.out = h;
    p.ldo = I;
    p.status = status;
    if (gather != nullptr) return launch_tc_gemm_pair(p, st);
    if (offsets != nullptr && grouped_rows <= 128) {
        // no expert can have more than 128 rows (decode-sized batches): the one-SM kernel
        // alone, its tiles dealt by CTA index (the pair launch would find no tile)
        p.side_sms = 0;
        p.tail_ctr = nullptr;
        return launch_tc_gemm_tail(p, st);
    }
    // experts of more than 128 rows on CTA pairs (the last tile padded), smaller ones on
    // single SMs: no expert's weights are read by both kernels (the same bits either way).
    // Where small experts are common (about 64 to 512 rows per expert on average) the two
    // launches run side by side: the pair tiles keep the tensor pipes busy while the small
    // experts' tiles, bound by reading their weights, use the SMs left to them. Which SMs
    // run which tiles changes nothing in any row's arithmetic.
    p.skip_tails = 1;
    p.tail_ctr = tail_ctr;
    const int64_t per_expert = groups > 0 ? grouped_rows / groups : 0;
    p.side_sms = (per_expert >= 64 && per_expert < 192) ? kSideSmsLow
                 : (per_expert >= 192 && per_expert < 512) ? kSideSmsHigh
                                                            : 0;
    const cudaError_t e = launch_tc_gemm_pair(p, st);
    if (e != cudaSuccess) return e;
    return launch_tc_gemm_tail(p, st);
}

// down over grouped rows: y[r] = h_r . W2^T
cudaError_t down(const uint16_t* h, int64_t a_rows, const int32_t* offsets, int groups, int rows,
                 const uint16_t* w2, int H, int I, uint16_t* y, int32_t* status, int32_t* tail_ctr,
                 cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_BF16;
    p.a = h;
    p.a_rows = a_rows;
    p.a_rows_total = a_rows;
    p.b = w2;
    p.b_rows_per_group = H;
    p.k = I;
    p.n = H;
    p.groups = groups;
    p.offsets = offsets;
    p.rows = rows;
    p.out = y;
    p.ldo = H;
    p.status = status;
    // Where small experts are common, as for gate_up: their tiles on single SMs side by
    // side with the pair tiles (run one after the other, the one-SM tiles measured no
    // faster here: down's 12-k-block tiles are short).
    const int64_t per_expert = groups > 0 ? a_rows / groups : 0;
    if (offsets != nullptr && H % 256 == 0 && per_expert >= 64 && per_expert < 512) {
        p.skip_tails = 1;
        p.tail_ctr = tail_ctr;
        p.side_sms = per_expert < 192 ? kSideSmsLow : kSideSmsHigh;
        const cudaError_t e = launch_tc_gemm_pair(p, st);
        if (e != cudaSuccess) return e;
        return launch_tc_gemm_tail(p, st);
    }
    return launch_tc_gemm_pair(p, st);
}

// a grouped bf16 product out[r] = a_r . b[g] with b[g] = [b_k_rows, n] (N contiguous): the
// weight as stored, read MN-major by the tensor cores (no transposed copy)
cudaError_t gemm_bf16_mn(const uint16_t* a, int64_t a_rows, const int32_t* offsets, int groups,
                         int rows, const uint16_t* b, int n, int k, int b_k_rows, uint16_t* out,
                         int32_t* status, cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_BF16;
    p.a = a;
    p.a_rows = a_rows;
    p.a_rows_total = a_rows;
    p.b = b;
    p.b_rows_per_group = n;
    p.b_mn = 1;
    p.b_k_rows = b_k_rows;
    p.k = k;
    p.n = n;
    p.groups = groups;
    p.offsets = offsets;
    p.rows = rows;
    p.out = out;
    p.ldo = n;
    p.status = status;
    return launch_tc_gemm_pair(p, st);
}

// the gate/up product recomputed with the SwiGLU backward in its epilogue:
// dgu[r] = [dh * u * silu'(g) | dh * silu(g)] (bf16, 2I columns)
// gate_up + SwiGLU over grouped rows (CTA pairs only) that also keeps the fp32 gate and up
// values: gu[r] = [a_r . W1g^T | a_r . W1u^T], row stride 2 I
cudaError_t gate_up_save(const uint16_t* a, int64_t a_rows, const int32_t* offsets, int groups,
                         int rows, const uint16_t* w13, int H, int I, uint16_t* h, float* gu,
                         int32_t* status, cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_SWIGLU_SAVE;
    p.a = a;
    p.a_rows = a_rows;
    p.a_rows_total = a_rows;
    p.b = w13;
    p.b_rows_per_group = 2 * I;
    p.k = H;
    p.n = I;
    p.groups = groups;
    p.offsets = offsets;
    p.rows = rows;
    p.out = h;
    p.ldo = I;
    p.gu = gu;
    p.ld_gu = 2 * (int64_t)I;
    p.status = status;
    return launch_tc_gemm_pair(p, st);
}

// dgu = SwiGLU backward of dh = a . W2 (W2 [groups, H, I] read MN-major), dh kept in fp32,
// with the gate and up values gu that gate_up_save kept: dgu [rows, 2 I] bf16
cudaError_t gemm_dswiglu(const uint16_t* a, int64_t a_rows, const int32_t* offsets, int groups,
                         int rows, const uint16_t* w2, int I, int H, const float* gu,
                         uint16_t* dgu, int32_t* status, cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_DSWIGLU;
    p.a = a;
    p.a_rows = a_rows;
    p.a_rows_total = a_rows;
    p.b = w2;
    p.b_rows_per_group = I;
    p.b_mn = 1;
    p.b_k_rows = H;
    p.k = H;
    p.n = I;
    p.groups = groups;
    p.offsets = offsets;
    p.rows = rows;
    p.out = dgu;
    p.ldo = 2 * (int64_t)I;
    p.gu = const_cast<float*>(gu);
    p.ld_gu = 2 * (int64_t)I;
    p.status = status;
    return launch_tc_gemm_pair(p, st);
}

int ffn_impl(const moe_cfg& c, const uint16_t* x, const uint16_t* x_perm,
             const int32_t* perm_token, const int32_t* offsets,
             const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s, const uint16_t* w2_s,
             uint16_t* y, uint16_t* y_shared, int32_t* status, void* ws, void* const* ev,
             cudaStream_t st)
{
    const FfnLayout L = ffn_layout(c);
    const int64_t A = (int64_t)c.T * c.K;
    uint16_t* h = at<uint16_t>(ws, L.h);
    int32_t* ctr = at<int32_t>(ws, L.ctr);
    int rc = x_perm != nullptr
                 ? cuda_rc(gate_up(x_perm, A, nullptr, A, offsets, c.E, 0, w13, c.H, c.I, h, status,
                                   ctr, st))
                 : cuda_rc(gate_up(x, c.T, perm_token, A, offsets, c.E, 0, w13, c.H, c.I, h, status,
                                   nullptr, st));
    if (rc != MOE_OK) return rc;
    if ((rc = rec(ev, 4, st)) != MOE_OK) return rc;
    rc = cuda_rc(down(h, A, offsets, c.E, 0, w2, c.H, c.I, y, status, ctr + 1, st));
    if (rc != MOE_OK) return rc;
    if ((rc = rec(ev, 5, st)) != MOE_OK) return rc;
    if (c.I_shared > 0 && w13_s != nullptr) {
        uint16_t* h_s = at<uint16_t>(ws, L.h_s);
        rc = cuda_rc(gate_up(x, c.T, nullptr, c.T, nullptr, 1, c.T, w13_s, c.H, c.I_shared, h_s,
                             status, nullptr, st));
        if (rc != MOE_OK) return rc;
        rc = cuda_rc(down(h_s, c.T, nullptr, 1, c.T, w2_s, c.H, c.I_shared, y_shared, status,
                          nullptr, st));
        if (rc != MOE_OK) return rc;
    }
    return rec(ev, 6, st);
}

int check_forward_args(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                       const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                       const uint16_t* w2_s, const uint16_t* out, const int32_t* status)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (x == nullptr || w_router == nullptr || w13 == nullptr || w2 == nullptr || out == nullptr ||
        status == nullptr)
        return MOE_ERR_ARG;
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(w13) || !aligned16(w2) ||
        !aligned16(out))
        return MOE_ERR_ARG;
    if (cfg->I_shared > 0 &&
        (w13_s == nullptr || w2_s == nullptr || !aligned16(w13_s) || !aligned16(w2_s)))
        return MOE_ERR_ARG;
    return MOE_OK;
}

// the layer on device tensors; status is not cleared (callers clear it once)
int forward_impl(const moe_cfg& c, const uint16_t* x, const uint16_t* w_router,
                 const float* logit_bias, const float* sel_bias, const uint8_t* token_mask,
                 const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                 const uint16_t* w2_s, uint16_t* out, float* logits, int32_t* topk_ids,
                 float* topk_w, int32_t* offsets, int32_t* status, void* ws, void* const* ev,
                 cudaStream_t st)
{
    const FwdLayout L = fwd_layout(c);
    const bool shared = c.I_shared > 0;
    float* lg = logits ? logits : at<float>(ws, L.logits);
    int32_t* ids = topk_ids ? topk_ids : at<int32_t>(ws, L.ids);
    float* w = topk_w ? topk_w : at<float>(ws, L.w);
    int32_t* offs = offsets ? offsets : at<int32_t>(ws, L.offsets);
    int32_t* perm_token = at<int32_t>(ws, L.perm_token);
    int32_t* dest_row = at<int32_t>(ws, L.dest_row);
    uint16_t* x_perm = at<uint16_t>(ws, L.x_perm);
    uint16_t* y = at<uint16_t>(ws, L.y);
    uint16_t* y_s = shared ? at<uint16_t>(ws, L.y_s) : nullptr;
    int rc = router_and_route(c, x, w_router, logit_bias, sel_bias, token_mask, lg, ids, w,
                              status, ev, st);
    if (rc != MOE_OK) return rc;
    rc = cuda_rc(launch_permute(c, ids, offs, perm_token, dest_row, status,
                                at<void>(ws, L.perm_ws), st));
    if (rc != MOE_OK) return rc;
    // materialised dispatch: the gather fused into the GEMM's operand loads is slower here
    if ((rc = cuda_rc(launch_gather_rows(c, x, dest_row, x_perm, st))) != MOE_OK) return rc;
    if ((rc = rec(ev, 3, st)) != MOE_OK) return rc;
    rc = ffn_impl(c, x, x_perm, perm_token, offs, w13, w2, shared ? w13_s : nullptr,
                  shared ? w2_s : nullptr, y, y_s, status, at<void>(ws, L.ffn), ev, st);
    if (rc != MOE_OK) return rc;
    rc = cuda_rc(launch_combine(c, y, w, dest_row, y_s, token_mask, out, st));
    if (rc != MOE_OK) return rc;
    return rec(ev, 7, st);
}

// Token chunks of moe_forward_host for a nominal chunk C: up to 2 C tokens in chunks of at
// most C (equal sizes); beyond that a first and a last chunk of C / 2 -- the pipeline's fill
// (the first copy in) and drain (the last copy out) are only as long as those -- and the
// tokens between them in equal chunks of at most 3 C / 2, since the layer runs faster per
// token on more tokens. Start of chunk i = chunk_start(i), i = 0..n (chunk_start(n) = T).
struct HostChunks {
    int T, n, edge, mid_n, mid_base, mid_rem;
    int64_t start(int i) const
    {
        if (edge == 0) {  // n equal chunks
            const int64_t q = T / n, r = T % n;
            return (int64_t)i * q + (i < r ? i : r);
        }
        if (i == 0) return 0;
        if (i >= n) return T;
        const int k = i - 1;  // middle chunks before chunk i
        return edge + (int64_t)k * mid_base + (k < mid_rem ? k : mid_rem);
    }
    int64_t max_chunk() const
    {
        int64_t m = 0;
        for (int i = 0; i < n; ++i) {
            const int64_t len = start(i + 1) - start(i);
            if (len > m) m = len;
        }
        return m;
    }
};

HostChunks host_chunks(int T, int C)
{
    HostChunks h{};
    h.T = T;
    if (T <= 0) {
        h.n = 0;
        return h;
    }
    if (C < 2 || T <= 2 * (int64_t)C) {
        h.n = (int)((T + (int64_t)C - 1) / C);
        return h;
    }
    h.edge = C / 2;
    const int64_t mid = T - 2 * (int64_t)h.edge;
    const int64_t cap = (int64_t)C + C / 2;
    h.mid_n = (int)((mid + cap - 1) / cap);
    h.mid_base = (int)(mid / h.mid_n);
    h.mid_rem = (int)(mid % h.mid_n);
    h.n = h.mid_n + 2;
    return h;
}

// scratch of moe_forward_host: the forward workspace of the largest chunk, then two x
// chunks and two out chunks (double buffering)
struct HostLayout {
    int chunk;
    size_t fwd, x_buf[2], out_buf[2], total;
};

HostLayout host_layout(const moe_cfg& c, int chunk_tokens)
{
    HostLayout L{};
    const int64_t big = c.T > 0 ? host_chunks(c.T, chunk_tokens).max_chunk() : 1;
    L.chunk = (int)(big > 0 ? big : 1);
    moe_cfg cc = c;
    cc.T = L.chunk;
    const size_t buf = up((size_t)L.chunk * c.H * 2);
    size_t off = 0;
    L.fwd = off;        off += fwd_layout(cc).total;
    L.x_buf[0] = off;   off += buf;
    L.x_buf[1] = off;   off += buf;
    L.out_buf[0] = off; off += buf;
    L.out_buf[1] = off; off += buf;
    L.total = off;
    return L;
}

// copy streams and events of moe_forward_host, created once per device and kept for the
// life of the process (driver objects, no device memory)
struct HostPipe {
    cudaStream_t in, out;
    cudaEvent_t start, done, copied_in[2], computed[2], copied_out[2];
};

cudaError_t host_pipe(HostPipe** out)
{
    static std::mutex mu;
    static HostPipe* pipes[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (pipes[dev] == nullptr) {
        HostPipe* p = new HostPipe();
        if ((e = cudaStreamCreateWithFlags(&p->in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&p->out, cudaStreamNonBlocking)) != cudaSuccess) return e;
        cudaEvent_t* evs[] = {&p->start, &p->done, &p->copied_in[0], &p->copied_in[1],
                              &p->computed[0], &p->computed[1], &p->copied_out[0],
                              &p->copied_out[1]};
        for (cudaEvent_t* ev : evs)
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
        pipes[dev] = p;
    }
    *out = pipes[dev];
    return cudaSuccess;
}

size_t pad64(size_t v) { return (v + 63) / 64 * 64; }

// scratch of moe_backward. The routed rows live in a padded layout: expert e's rows start at
// poff[e] (its count rounded up to 64, the padding rows zero), so that every expert's rows
// form whole 64-row K blocks of the weight-gradient products.
struct BwdLayout {
    size_t offsets, perm_token, dest_row, dest_pad, poff, perm_ws, x_perm, h, y, dy, gu, dgu,
        dx_perm, dw_tk, dl, dl_bf, dx_r, koffT, koffS, wr_part, h_s, gu_s, dgu_s, dx_s, dy_s,
        y_s, total;
    int64_t rp, e_pad;
};

// K splits of the router's weight-gradient product (E x H outputs, K = T tokens): its output
// makes only ceil(E / 256) * H / 256 tiles, too few for the GPU's CTA pairs, so the tokens
// are cut into S chunks of a multiple of 64 (S partial products, then one in-order sum);
// enough chunks for two tiles per pair of a 148-SM B200. A function of (E, H, T) only, so
// the bits do not depend on the device.
int router_wgrad_splits(int E, int H, int T, int* chunk)
{
    constexpr int64_t kPairs = 74;
    const int64_t tiles = ((E + 255) / 256) * (H % 256 == 0 ? H / 256 : H / 128);
    int64_t S = 1;
    if (tiles > 0 && tiles < kPairs) S = (2 * kPairs + tiles - 1) / tiles;
    int64_t ch = (((int64_t)T + S - 1) / S + 63) / 64 * 64;
    if (ch < 64) ch = 64;
    S = ((int64_t)T + ch - 1) / ch;
    if (S < 1) S = 1;
    *chunk = (int)ch;
    return (int)S;
}

BwdLayout bwd_layout(const moe_cfg& c)
{
    BwdLayout L{};
    const size_t A = (size_t)c.T * c.K, H = c.H, I = c.I, Is = c.I_shared, T = c.T;
    L.e_pad = (int64_t)pad64(c.E);
    L.rp = (int64_t)pad64(A + (size_t)63 * c.E);
    const size_t rp = (size_t)L.rp, ep = (size_t)L.e_pad;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += up(bytes);
        return o;
    };
    L.offsets = take((c.E + 1) * 4);
    L.perm_token = take(A * 4);
    L.dest_row = take(A * 4);
    L.dest_pad = take(A * 4);
    L.poff = take((c.E + 1) * 4);
    L.perm_ws = take(permute_ws_bytes(c));
    L.x_perm = take(rp * H * 2);
    L.h = take(rp * I * 2);
    L.y = take(rp * H * 2);
    L.dy = take(rp * H * 2);
    L.gu = take(rp * 2 * I * 4);
    L.dgu = take(rp * 2 * I * 2);
    L.dx_perm = take(rp * H * 2);
    L.dw_tk = take(A * 4);
    L.dl = take(T * c.E * 4);
    L.dl_bf = take(T * ep * 2);
    L.dx_r = take(T * H * 2);
    L.koffT = take(2 * 4);
    int chunk = 0;
    const size_t S = (size_t)router_wgrad_splits(c.E, c.H, c.T, &chunk);
    L.koffS = take((S + 1) * 4);
    L.wr_part = take(S > 1 ? S * c.E * H * 4 : 0);
    L.h_s = take(T * Is * 2);
    L.gu_s = take(T * 2 * Is * 4);
    L.dgu_s = take(T * 2 * Is * 2);
    L.dx_s = take(Is ? T * H * 2 : 0);
    L.dy_s = take(Is ? T * H * 2 : 0);
    L.y_s = take(Is ? T * H * 2 : 0);
    L.total = off;
    return L;
}

// weight gradient with both operands read MN-major in place: out[g] [m, n] = sum over the
// group's K rows of a[k, m] b[k, n]; a [k_rows, a_cols], b [k_rows, n]
cudaError_t gemm_wgrad_mn(const uint16_t* a, int64_t a_cols, int m, const uint16_t* b, int n,
                          int64_t k_rows, const int32_t* k_offsets, int groups, float* out,
                          int32_t* status, cudaStream_t st)
{
    GemmProblem p{};
    p.epilogue = EPI_WGRAD;
    p.a = a;
    p.a_rows = a_cols;
    p.a_mn = 1;
    p.b = b;
    p.b_mn = 1;
    p.k = (int)k_rows;
    p.n = n;
    p.groups = groups;
    p.rows = m;
    p.out = out;
    p.ldo = n;
    p.k_offsets = k_offsets;
    p.status = status;
    return launch_tc_gemm_pair(p, st);
}

#define MOE_TRY(call)                                   \
    do {                                                \
        const int rc_ = cuda_rc(call);                  \
        if (rc_ != MOE_OK) return rc_;                  \
    } while (0)

// Dispatch into the padded layout and the expert intermediates the backward reuses:
// offsets, dest_pad, poff, x_perm (padding rows zero), h, y, and the shared expert's h_s.
// moe_forward_train leaves them in the workspace; moe_backward recomputes them otherwise
// (the same products: a row's bits do not depend on where it sits).
int train_intermediates(const moe_cfg& c, const uint16_t* x, const int32_t* ids,
                        const uint16_t* w13, const uint16_t* w2, const uint16_t* w13s,
                        int32_t* status, void* ws, cudaStream_t st)
{
    const BwdLayout L = bwd_layout(c);
    const int64_t A = (int64_t)c.T * c.K;
    const int H = c.H, I = c.I, Is = c.I_shared, E = c.E, T = c.T;
    const int64_t rp = L.rp;
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* dest_row = at<int32_t>(ws, L.dest_row);
    int32_t* dest_pad = at<int32_t>(ws, L.dest_pad);
    int32_t* poff = at<int32_t>(ws, L.poff);
    uint16_t* x_perm = at<uint16_t>(ws, L.x_perm);
    uint16_t* h = at<uint16_t>(ws, L.h);
    MOE_TRY(launch_permute(c, ids, offsets, at<int32_t>(ws, L.perm_token), dest_row, status,
                           at<void>(ws, L.perm_ws), st));
    MOE_TRY(launch_padded_offsets(offsets, E, 0, poff, st));
    MOE_TRY(launch_pad_rows(ids, dest_row, offsets, poff, A, E, dest_pad, st));
    MOE_TRY(launch_zero_pad_rows(x_perm, H, offsets, poff, E, st));
    MOE_TRY(launch_gather_rows(c, x, dest_pad, x_perm, st));
    MOE_TRY(gate_up_save(x_perm, rp, poff, E, 0, w13, H, I, h, at<float>(ws, L.gu), status, st));
    MOE_TRY(down(h, rp, poff, E, 0, w2, H, I, at<uint16_t>(ws, L.y), status, nullptr, st));
    if (Is > 0)
        MOE_TRY(gate_up_save(x, T, nullptr, 1, T, w13s, H, Is, at<uint16_t>(ws, L.h_s),
                             at<float>(ws, L.gu_s), status, st));
    return MOE_OK;
}

int backward_impl(const moe_cfg& c, const uint16_t* x, const uint16_t* wr, const uint8_t* mask,
                  const uint16_t* w13, const uint16_t* w2, const uint16_t* w13s,
                  const uint16_t* w2s, const float* logits, const int32_t* ids,
                  const float* topk_w, const uint16_t* dout, uint16_t* dx, float* dwr,
                  float* dw13, float* dw2, float* dw13s, float* dw2s, float* d_topk_w,
                  float* dlogits, int saved, int32_t* status, void* ws, cudaStream_t st)
{
    const BwdLayout L = bwd_layout(c);
    const int H = c.H, I = c.I, Is = c.I_shared, E = c.E, T = c.T;
    const int ep = (int)L.e_pad;
    const int64_t rp = L.rp;
    const bool shared = Is > 0;
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* dest_row = at<int32_t>(ws, L.dest_row);
    int32_t* dest_pad = at<int32_t>(ws, L.dest_pad);
    int32_t* poff = at<int32_t>(ws, L.poff);
    uint16_t* x_perm = at<uint16_t>(ws, L.x_perm);
    uint16_t* h = at<uint16_t>(ws, L.h);
    uint16_t* y = at<uint16_t>(ws, L.y);
    uint16_t* dy = at<uint16_t>(ws, L.dy);
    const float* gu = at<float>(ws, L.gu);
    uint16_t* dgu = at<uint16_t>(ws, L.dgu);
    uint16_t* dx_perm = at<uint16_t>(ws, L.dx_perm);
    float* dw_tk = d_topk_w ? d_topk_w : at<float>(ws, L.dw_tk);
    float* dl = dlogits ? dlogits : at<float>(ws, L.dl);
    uint16_t* dl_bf = at<uint16_t>(ws, L.dl_bf);
    uint16_t* dx_r = at<uint16_t>(ws, L.dx_r);
    int32_t* koffT = at<int32_t>(ws, L.koffT);

    // dispatch into the padded layout and the forward intermediates (padding rows give
    // h = 0, y = 0), unless moe_forward_train left them in the workspace
    if (!saved) {
        const int rc = train_intermediates(c, x, ids, w13, w2, w13s, status, ws, st);
        if (rc != MOE_OK) return rc;
    }
    MOE_TRY(launch_zero_pad_rows(dy, H, offsets, poff, E, st));

    // combine backward: routing-weight gradients and the expert-output gradients
    uint16_t* dy_s = shared ? at<uint16_t>(ws, L.dy_s) : nullptr;
    MOE_TRY(launch_combine_bwd(c, dout, y, topk_w, dest_pad, mask, dw_tk, dy, dy_s, st));

    // routed experts: dh = dy . W2 in fp32 and, in the same product's epilogue, the SwiGLU
    // backward dgu from the forward's kept gate/up values; dx rows = dgu . W13; the weights
    // are read MN-major as stored
    MOE_TRY(gemm_dswiglu(dy, rp, poff, E, 0, w2, I, H, gu, dgu, status, st));
    MOE_TRY(gemm_bf16_mn(dgu, rp, poff, E, 0, w13, H, 2 * I, 2 * I, dx_perm, status, st));

    // router: dlogits, then dx_router = bf16(dlogits) . W_router (K padded to 64: the rows
    // of W_router past E read as zeros)
    MOE_TRY(launch_router_bwd(c, logits, ids, dw_tk, mask, dl, dl_bf, ep, st));
    MOE_TRY(gemm_bf16_mn(dl_bf, T, nullptr, 1, T, wr, H, ep, E, dx_r, status, st));

    // shared expert (all kept tokens, dy_shared = dout)
    uint16_t *h_s = nullptr, *dgu_s = nullptr, *dx_s = nullptr;
    if (shared) {
        h_s = at<uint16_t>(ws, L.h_s);
        dgu_s = at<uint16_t>(ws, L.dgu_s);
        dx_s = at<uint16_t>(ws, L.dx_s);
        MOE_TRY(gemm_dswiglu(dy_s, T, nullptr, 1, T, w2s, Is, H, at<float>(ws, L.gu_s), dgu_s,
                             status, st));
        MOE_TRY(gemm_bf16_mn(dgu_s, T, nullptr, 1, T, w13s, H, 2 * Is, 2 * Is, dx_s, status, st));
    }

    // input gradient
    MOE_TRY(launch_unpermute(c, dx_perm, dest_pad, dx_s, dx_r, mask, dx, st));

    // weight gradients, operands read in place (MN-major): an expert's K range is its padded
    // rows; the single-group products take K = T rounded up to 64, the rows past T reading
    // as zeros
    MOE_TRY(gemm_wgrad_mn(dy, H, H, h, I, rp, poff, E, dw2, status, st));
    MOE_TRY(gemm_wgrad_mn(dgu, 2 * I, 2 * I, x_perm, H, rp, poff, E, dw13, status, st));
    MOE_TRY(launch_padded_offsets(nullptr, 1, T, koffT, st));
    int chunk = 0;
    const int S = router_wgrad_splits(E, H, T, &chunk);
    if (S > 1) {
        // the router's product split over K (chunks of tokens), partials summed in order
        int32_t* koffS = at<int32_t>(ws, L.koffS);
        float* part = at<float>(ws, L.wr_part);
        MOE_TRY(launch_split_offsets(T, chunk, S, koffS, st));
        MOE_TRY(gemm_wgrad_mn(dl_bf, ep, E, x, H, T, koffS, S, part, status, st));
        MOE_TRY(launch_sum_parts(part, S, (int64_t)E * H, dwr, st));
    } else {
        MOE_TRY(gemm_wgrad_mn(dl_bf, ep, E, x, H, T, koffT, 1, dwr, status, st));
    }
    if (shared) {
        MOE_TRY(gemm_wgrad_mn(dy_s, H, H, h_s, Is, T, koffT, 1, dw2s, status, st));
        MOE_TRY(gemm_wgrad_mn(dgu_s, 2 * Is, 2 * Is, x, H, T, koffT, 1, dw13s, status, st));
    }
    return MOE_OK;
}

#undef MOE_TRY

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

MOE_API int moe_abi_version(void) { return 104; }

MOE_API int moe_pipeline_wait_selftest(int32_t* status, long long limit_cycles, void* stream)
{
    if (status == nullptr) return MOE_ERR_ARG;
    if (limit_cycles < 1000 || limit_cycles > 2000000000LL) return MOE_ERR_ARG;
    int rc;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK) return rc;
    return cuda_rc(launch_pipe_wait_selftest(status, limit_cycles, st));
}

MOE_API const char* moe_status_string(int code)
{
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_ARG: return "invalid argument (null or misaligned pointer)";
        case MOE_ERR_SHAPE: return "unsupported shape or configuration";
        case MOE_ERR_WORKSPACE: return "workspace too small";
        case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
        case MOE_ERR_UNIMPLEMENTED: return "not implemented in this build";
        case MOE_ERR_DEVICE: return "current device is not an sm_100 (B200) GPU";
        default: return "unknown status";
    }
}

MOE_API size_t moe_workspace_bytes(const moe_cfg* cfg, int stage)
{
    if (check_cfg(cfg) != MOE_OK) return 0;
    switch (stage) {
        case MOE_STAGE_ROUTE: return 0;
        case MOE_STAGE_PERMUTE: return permute_ws_bytes(*cfg);
        case MOE_STAGE_FFN: return ffn_layout(*cfg).total;
        case MOE_STAGE_COMBINE: return 0;
        case MOE_STAGE_FORWARD: return fwd_layout(*cfg).total;
        case MOE_STAGE_STATS: return stats_ws_bytes(*cfg);
        case MOE_STAGE_BACKWARD: return bwd_layout(*cfg).total;
        default: return 0;
    }
}

MOE_API int moe_route(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                      const float* logit_bias, const float* sel_bias, const uint8_t* token_mask,
                      float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                      void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr) return MOE_ERR_ARG;
    if (x != nullptr && (w_router == nullptr || !aligned16(x) || !aligned16(w_router)))
        return MOE_ERR_ARG;
    if (cfg->T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (status && (rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK)
        return rc;
    if (x != nullptr)
        return router_and_route(*cfg, x, w_router, logit_bias, sel_bias, token_mask, logits,
                                topk_ids, topk_w, status, nullptr, st);
    return cuda_rc(launch_route(*cfg, logits, sel_bias, token_mask, topk_ids, topk_w, status, st));
}

MOE_API int moe_permute(const moe_cfg* cfg, const int32_t* topk_ids, const uint16_t* x,
                        int32_t* offsets, int32_t* perm_token, int32_t* dest_row,
                        uint16_t* x_perm, int32_t* status, void* ws, size_t ws_bytes,
                        void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (topk_ids == nullptr || offsets == nullptr || perm_token == nullptr || dest_row == nullptr)
        return MOE_ERR_ARG;
    if (x_perm != nullptr && (x == nullptr || !aligned16(x) || !aligned16(x_perm)))
        return MOE_ERR_ARG;
    if (ws_bytes < permute_ws_bytes(*cfg) || ws == nullptr) return MOE_ERR_WORKSPACE;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (status && (rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK)
        return rc;
    rc = cuda_rc(launch_permute(*cfg, topk_ids, offsets, perm_token, dest_row, status, ws, st));
    if (rc != MOE_OK || x_perm == nullptr) return rc;
    return cuda_rc(launch_gather_rows(*cfg, x, dest_row, x_perm, st));
}

MOE_API int moe_permute_noalloc(const moe_cfg* cfg, const int32_t* topk_ids, const uint16_t* x,
                                int32_t* offsets, int32_t* perm_token, int32_t* dest_row,
                                uint16_t* x_perm, int32_t* status, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (topk_ids == nullptr || offsets == nullptr || perm_token == nullptr || dest_row == nullptr)
        return MOE_ERR_ARG;
    if (x_perm != nullptr && (x == nullptr || !aligned16(x) || !aligned16(x_perm)))
        return MOE_ERR_ARG;
    if (permute_ws_bytes(*cfg) > (size_t)kPermuteFixedScratchInts * sizeof(int32_t))
        return MOE_ERR_WORKSPACE;
    if ((rc = check_device()) != MOE_OK) return rc;
    int32_t* scratch = nullptr;
    if ((rc = cuda_rc(permute_fixed_scratch(&scratch))) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (status && (rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK)
        return rc;
    rc = cuda_rc(launch_permute(*cfg, topk_ids, offsets, perm_token, dest_row, status, scratch,
                                st));
    if (rc != MOE_OK || x_perm == nullptr) return rc;
    return cuda_rc(launch_gather_rows(*cfg, x, dest_row, x_perm, st));
}

MOE_API int moe_grouped_ffn(const moe_cfg* cfg, const uint16_t* x, const uint16_t* x_perm,
                            const int32_t* perm_token, const int32_t* offsets,
                            const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                            const uint16_t* w2_s, uint16_t* y, uint16_t* y_shared,
                            int32_t* status, void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (offsets == nullptr || w13 == nullptr || w2 == nullptr || y == nullptr) return MOE_ERR_ARG;
    if (!aligned16(w13) || !aligned16(w2) || !aligned16(y)) return MOE_ERR_ARG;
    const bool shared = cfg->I_shared > 0;
    if (shared && (x == nullptr || w13_s == nullptr || w2_s == nullptr || y_shared == nullptr ||
                   !aligned16(x) || !aligned16(w13_s) || !aligned16(w2_s) || !aligned16(y_shared)))
        return MOE_ERR_ARG;
    if (x_perm == nullptr && (perm_token == nullptr || x == nullptr || !aligned16(x)))
        return MOE_ERR_ARG;
    if (x_perm != nullptr && !aligned16(x_perm)) return MOE_ERR_ARG;
    if (ws == nullptr || ws_bytes < ffn_layout(*cfg).total) return MOE_ERR_WORKSPACE;
    if (cfg->T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (status && (rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK)
        return rc;
    return ffn_impl(*cfg, x, x_perm, perm_token, offsets, w13, w2, shared ? w13_s : nullptr,
                    shared ? w2_s : nullptr, y, y_shared, status, ws, nullptr, st);
}

MOE_API int moe_combine(const moe_cfg* cfg, const uint16_t* y, const float* topk_w,
                        const int32_t* dest_row, const uint16_t* y_shared,
                        const uint8_t* token_mask, uint16_t* out, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (y == nullptr || topk_w == nullptr || dest_row == nullptr || out == nullptr)
        return MOE_ERR_ARG;
    if (!aligned16(y) || !aligned16(out) || (y_shared != nullptr && !aligned16(y_shared)))
        return MOE_ERR_ARG;
    if (cfg->T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    return cuda_rc(launch_combine(*cfg, y, topk_w, dest_row, y_shared, token_mask, out,
                                  static_cast<cudaStream_t>(stream)));
}

MOE_API int moe_combine_invariant(const moe_cfg* cfg, const uint16_t* y, const float* topk_w,
                                  const int32_t* dest_row, const uint16_t* y_shared,
                                  const uint8_t* token_mask, uint16_t* out, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (y == nullptr || topk_w == nullptr || dest_row == nullptr || out == nullptr)
        return MOE_ERR_ARG;
    if (!aligned16(y) || !aligned16(out) || (y_shared != nullptr && !aligned16(y_shared)))
        return MOE_ERR_ARG;
    if (cfg->T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    return cuda_rc(launch_combine_invariant(*cfg, y, topk_w, dest_row, y_shared, token_mask, out,
                                            static_cast<cudaStream_t>(stream)));
}

MOE_API int moe_forward(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                        const float* logit_bias, const float* sel_bias, const uint8_t* token_mask,
                        const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                        const uint16_t* w2_s, uint16_t* out, float* logits, int32_t* topk_ids,
                        float* topk_w, int32_t* offsets, int32_t* status, void* ws,
                        size_t ws_bytes, void* const* stage_events, void* stream)
{
    int rc = check_forward_args(cfg, x, w_router, w13, w2, w13_s, w2_s, out, status);
    if (rc != MOE_OK) return rc;
    const FwdLayout L = fwd_layout(*cfg);
    if (ws == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (cfg->T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK) return rc;
    if ((rc = rec(stage_events, 0, st)) != MOE_OK) return rc;  // the router stage starts here
    return forward_impl(*cfg, x, w_router, logit_bias, sel_bias, token_mask, w13, w2, w13_s, w2_s,
                        out, logits, topk_ids, topk_w, offsets, status, ws, stage_events, st);
}

MOE_API int moe_router_stats(const moe_cfg* cfg, const float* logits, const uint8_t* token_mask,
                             const int32_t* offsets, int32_t* tokens_per_expert,
                             float* mean_prob, float* aux, void* ws, size_t ws_bytes,
                             void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    if (logits == nullptr || offsets == nullptr || tokens_per_expert == nullptr ||
        mean_prob == nullptr || aux == nullptr)
        return MOE_ERR_ARG;
    if (ws == nullptr || ws_bytes < stats_ws_bytes(*cfg)) return MOE_ERR_WORKSPACE;
    if ((rc = check_device()) != MOE_OK) return rc;
    return cuda_rc(launch_router_stats(*cfg, logits, token_mask, offsets, tokens_per_expert,
                                       mean_prob, aux, ws, static_cast<cudaStream_t>(stream)));
}

MOE_API size_t moe_forward_host_workspace_bytes(const moe_cfg* cfg, int chunk_tokens)
{
    if (check_cfg(cfg) != MOE_OK || chunk_tokens < 1) return 0;
    const HostLayout L = host_layout(*cfg, chunk_tokens);
    return L.total;
}

MOE_API int moe_forward_host(const moe_cfg* cfg, const uint16_t* x_host, const uint16_t* w_router,
                             const float* logit_bias, const float* sel_bias,
                             const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                             const uint16_t* w13_s, const uint16_t* w2_s, uint16_t* out_host,
                             int32_t* status, int chunk_tokens, void* ws, size_t ws_bytes,
                             void* stream)
{
    int rc = check_forward_args(cfg, x_host, w_router, w13, w2, w13_s, w2_s, out_host, status);
    if (rc != MOE_OK) return rc;
    if (chunk_tokens < 1) return MOE_ERR_ARG;
    const moe_cfg& c = *cfg;
    const HostLayout L = host_layout(c, chunk_tokens);
    if (ws == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (c.T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    HostPipe* hp = nullptr;
    if ((rc = cuda_rc(host_pipe(&hp))) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const HostChunks hc = host_chunks(c.T, chunk_tokens);
    const size_t row_bytes = (size_t)c.H * 2;
    if ((rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK) return rc;
    // the copy streams start after everything already queued on the caller's stream
    if ((rc = cuda_rc(cudaEventRecord(hp->start, st))) != MOE_OK) return rc;
    if ((rc = cuda_rc(cudaStreamWaitEvent(hp->in, hp->start, 0))) != MOE_OK) return rc;
    if ((rc = cuda_rc(cudaStreamWaitEvent(hp->out, hp->start, 0))) != MOE_OK) return rc;
    for (int i = 0; i < hc.n; ++i) {
        const int slot = i & 1;
        const int t0 = (int)hc.start(i);
        const int tn = (int)(hc.start(i + 1) - t0);
        uint16_t* xb = at<uint16_t>(ws, L.x_buf[slot]);
        uint16_t* ob = at<uint16_t>(ws, L.out_buf[slot]);
        // H2D of chunk i once the compute of chunk i-2 no longer reads this x buffer
        if (i >= 2 && (rc = cuda_rc(cudaStreamWaitEvent(hp->in, hp->computed[slot], 0))) != MOE_OK)
            return rc;
        rc = cuda_rc(cudaMemcpyAsync(xb, x_host + (size_t)t0 * c.H, (size_t)tn * row_bytes,
                                     cudaMemcpyHostToDevice, hp->in));
        if (rc != MOE_OK) return rc;
        if ((rc = cuda_rc(cudaEventRecord(hp->copied_in[slot], hp->in))) != MOE_OK) return rc;
        // compute of chunk i on the caller's stream, after its input landed and after the
        // D2H of chunk i-2 has read this out buffer
        if ((rc = cuda_rc(cudaStreamWaitEvent(st, hp->copied_in[slot], 0))) != MOE_OK) return rc;
        if (i >= 2 && (rc = cuda_rc(cudaStreamWaitEvent(st, hp->copied_out[slot], 0))) != MOE_OK)
            return rc;
        moe_cfg cc = c;
        cc.T = tn;
        rc = forward_impl(cc, xb, w_router, logit_bias, sel_bias,
                          token_mask ? token_mask + t0 : nullptr, w13, w2, w13_s, w2_s, ob,
                          nullptr, nullptr, nullptr, nullptr, status, at<void>(ws, L.fwd),
                          nullptr, st);
        if (rc != MOE_OK) return rc;
        if ((rc = cuda_rc(cudaEventRecord(hp->computed[slot], st))) != MOE_OK) return rc;
        // D2H of chunk i
        if ((rc = cuda_rc(cudaStreamWaitEvent(hp->out, hp->computed[slot], 0))) != MOE_OK) return rc;
        rc = cuda_rc(cudaMemcpyAsync(out_host + (size_t)t0 * c.H, ob, (size_t)tn * row_bytes,
                                     cudaMemcpyDeviceToHost, hp->out));
        if (rc != MOE_OK) return rc;
        if ((rc = cuda_rc(cudaEventRecord(hp->copied_out[slot], hp->out))) != MOE_OK) return rc;
    }
    // the caller's stream completes only after the last result reached the host
    if ((rc = cuda_rc(cudaEventRecord(hp->done, hp->out))) != MOE_OK) return rc;
    return cuda_rc(cudaStreamWaitEvent(st, hp->done, 0));
}

MOE_API int moe_backward(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                         const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                         const uint16_t* w13_s, const uint16_t* w2_s, const float* logits,
                         const int32_t* topk_ids, const float* topk_w, const uint16_t* dout,
                         uint16_t* dx, float* dw_router, float* dw13, float* dw2, float* dw13_s,
                         float* dw2_s, float* d_topk_w, float* dlogits, int saved,
                         int32_t* status, void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_cfg(cfg);
    if (rc != MOE_OK) return rc;
    const moe_cfg& c = *cfg;
    if (saved != 0 && saved != 1) return MOE_ERR_ARG;
    const void* need[] = {w_router, w13, w2, dw_router, dw13, dw2, status};
    for (const void* q : need)
        if (q == nullptr) return MOE_ERR_ARG;
    const void* per_token[] = {x, logits, topk_ids, topk_w, dout, dx};  // NULL allowed at T == 0
    if (c.T > 0)
        for (const void* q : per_token)
            if (q == nullptr) return MOE_ERR_ARG;
    const void* aligned[] = {x, w_router, w13, w2, logits, topk_ids, topk_w, dout, dx, dw_router,
                             dw13, dw2, d_topk_w, dlogits};
    for (const void* q : aligned)
        if (q != nullptr && !aligned16(q)) return MOE_ERR_ARG;
    if (c.I_shared > 0) {
        if (w13_s == nullptr || w2_s == nullptr || dw13_s == nullptr || dw2_s == nullptr)
            return MOE_ERR_ARG;
        if (!aligned16(w13_s) || !aligned16(w2_s) || !aligned16(dw13_s) || !aligned16(dw2_s))
            return MOE_ERR_ARG;
    }
    const BwdLayout L = bwd_layout(c);
    if (ws == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK) return rc;
    if (c.T == 0) {
        // no tokens: every weight gradient is zero
        const size_t H = c.H, I = c.I, Is = c.I_shared, E = c.E;
        if ((rc = cuda_rc(cudaMemsetAsync(dw_router, 0, E * H * 4, st))) != MOE_OK) return rc;
        if ((rc = cuda_rc(cudaMemsetAsync(dw13, 0, E * 2 * I * H * 4, st))) != MOE_OK) return rc;
        if ((rc = cuda_rc(cudaMemsetAsync(dw2, 0, E * H * I * 4, st))) != MOE_OK) return rc;
        if (Is > 0) {
            if ((rc = cuda_rc(cudaMemsetAsync(dw13_s, 0, 2 * Is * H * 4, st))) != MOE_OK) return rc;
            if ((rc = cuda_rc(cudaMemsetAsync(dw2_s, 0, H * Is * 4, st))) != MOE_OK) return rc;
        }
        return MOE_OK;
    }
    return backward_impl(c, x, w_router, token_mask, w13, w2, w13_s, w2_s, logits, topk_ids,
                         topk_w, dout, dx, dw_router, dw13, dw2, dw13_s, dw2_s, d_topk_w, dlogits,
                         saved, status, ws, st);
}

MOE_API int moe_forward_train(const moe_cfg* cfg, const uint16_t* x, const uint16_t* w_router,
                              const float* logit_bias, const float* sel_bias,
                              const uint8_t* token_mask, const uint16_t* w13, const uint16_t* w2,
                              const uint16_t* w13_s, const uint16_t* w2_s, uint16_t* out,
                              float* logits, int32_t* topk_ids, float* topk_w, int32_t* status,
                              void* ws, size_t ws_bytes, void* stream)
{
    int rc = check_forward_args(cfg, x, w_router, w13, w2, w13_s, w2_s, out, status);
    if (rc != MOE_OK) return rc;
    const moe_cfg& c = *cfg;
    if (c.T > 0 && (logits == nullptr || topk_ids == nullptr || topk_w == nullptr))
        return MOE_ERR_ARG;
    if ((logits && !aligned16(logits)) || (topk_ids && !aligned16(topk_ids)) ||
        (topk_w && !aligned16(topk_w)))
        return MOE_ERR_ARG;
    const BwdLayout L = bwd_layout(c);
    if (ws == nullptr || ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (c.T == 0) return MOE_OK;
    if ((rc = check_device()) != MOE_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((rc = cuda_rc(cudaMemsetAsync(status, 0, MOE_STATUS_WORDS * 4, st))) != MOE_OK) return rc;
    if ((rc = router_and_route(c, x, w_router, logit_bias, sel_bias, token_mask, logits, topk_ids,
                               topk_w, status, nullptr, st)) != MOE_OK)
        return rc;
    if ((rc = train_intermediates(c, x, topk_ids, w13, w2, w13_s, status, ws, st)) != MOE_OK)
        return rc;
    uint16_t* y_s = nullptr;
    if (c.I_shared > 0) {
        y_s = at<uint16_t>(ws, L.y_s);
        if ((rc = cuda_rc(down(at<uint16_t>(ws, L.h_s), c.T, nullptr, 1, c.T, w2_s, c.H,
                               c.I_shared, y_s, status, nullptr, st))) != MOE_OK)
            return rc;
    }
    return cuda_rc(launch_combine(c, at<uint16_t>(ws, L.y), topk_w, at<int32_t>(ws, L.dest_pad),
                                  y_s, token_mask, out, st));
}

}  // extern "C"

// Memory-bound kernels of the layer's backward pass (forward + backward is the consistency
// contract's scope: "DSV4 Flash MoE Train-Inference Consistency Roadmap", "Why DSV4 Flash
// MoE Drifts More Easily", and the DSV4-WS1-2 row of "Follow-Up Issue Buckets"). The
// tensor-core products of the backward are tc_gemm2.cu's; here:
//
//  combine backward   dw[t,j] = dot32(dout_t, y_row) -- lane L owns the 8-element chunks
//                     L, L+32, ... in order, rounded products added in fp32, then butterfly
//                     levels 16..1; dy_row = bf16(w[t,j] * dout_t); dy_shared = dout (0 for
//                     masked tokens)
//  router backward    ds through the renormalisation, dl through the score function, in a
//                     fixed fp32 order (see router_bwd_kernel)
//  un-permute         dx_t = bf16(rank-order sum of the token's row gradients, then the
//                     shared expert's and the router's terms); masked tokens +0
//  padded layout      each expert's dispatch rows start at a multiple of 64 (padding rows
//                     zero), so its rows are whole 64-row K blocks of the weight-gradient
//                     products, which read the row-major activations in place (MN-major)
//
// Nothing here uses float atomics; every reduction has a fixed order, so results are
// bitwise repeatable and a token's input gradient does not depend on the other tokens.
#include "route_math.cuh"

namespace moe {
namespace {

__device__ __forceinline__ uint32_t bf16_bits(float f)
{
    const uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (u >> 16) | 0x40u;
    return (u + 0x7fffu + ((u >> 16) & 1u)) >> 16;
}

__device__ __forceinline__ float lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// one warp per token
__global__ void __launch_bounds__(256) combine_bwd_kernel(const uint4* __restrict__ dout,
                                                          const uint4* __restrict__ y,
                                                          const float* __restrict__ w,
                                                          const int32_t* __restrict__ dest_row,
                                                          const uint8_t* __restrict__ mask,
                                                          int T, int K, int H, float* dw,
                                                          uint4* __restrict__ dy,
                                                          uint4* __restrict__ dy_shared)
{
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int hv = H >> 3;  // 16-byte chunks per row
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
        const bool kept = mask == nullptr || mask[t] != 0;
        const uint4* g = dout + (int64_t)t * hv;
        if (dy_shared != nullptr) {
            const uint4 z = make_uint4(0u, 0u, 0u, 0u);
            for (int c = lane; c < hv; c += 32) dy_shared[(int64_t)t * hv + c] = kept ? g[c] : z;
        }
        for (int j = 0; j < K; ++j) {
            const int64_t a = (int64_t)t * K + j;
            const int32_t r = dest_row[a];
            if (!kept || r < 0) {
                if (lane == 0) dw[a] = 0.0f;
                continue;
            }
            const float wj = w[a];
            const uint4* yr = y + (int64_t)r * hv;
            uint4* dyr = dy + (int64_t)r * hv;
            float acc = 0.0f;
            for (int c = lane; c < hv; c += 32) {
                const uint4 gq = g[c], yq = yr[c];
                const uint32_t gw[4] = {gq.x, gq.y, gq.z, gq.w};
                const uint32_t yw[4] = {yq.x, yq.y, yq.z, yq.w};
                uint32_t o[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float g0 = lo_f(gw[q]), g1 = hi_f(gw[q]);
                    acc = __fadd_rn(acc, __fmul_rn(g0, lo_f(yw[q])));
                    acc = __fadd_rn(acc, __fmul_rn(g1, hi_f(yw[q])));
                    o[q] = bf16_bits(__fmul_rn(wj, g0)) | (bf16_bits(__fmul_rn(wj, g1)) << 16);
                }
                dyr[c] = make_uint4(o[0], o[1], o[2], o[3]);
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1)
                acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, off));
            if (lane == 0) dw[a] = acc;
        }
    }
}

// Router backward, one warp per token (fp32, each operation rounded to nearest):
//   renorm:    D = rank-order sum of s_{id_j}; q = rank-order sum of dw_j * s_{id_j};
//              ds_{id_j} = (route_scale * (dw_j - q / D)) / D  (all 0 when D == 0)
//   no renorm: ds_{id_j} = route_scale * dw_j;  unselected experts ds = 0
//   softmax:   r = rank-order sum of ds_{id_j} * s_{id_j};  dl_e = s_e * (ds_e - r)
//   sigmoid:   dl_e = ds_e * (s_e * (1 - s_e))
//   sqrtsoftplus: dl_e = ds_e * (sigmoid(l_e) / (2 s_e)), 0 where ds_e or s_e is 0
// Writes dl [T,E] fp32 (when given) and its bf16 copy [T, ld_bf] with zero padding columns.
template <int NE>
__global__ void __launch_bounds__(256) router_bwd_kernel(const float* __restrict__ logits,
                                                         const int32_t* __restrict__ ids,
                                                         const float* __restrict__ dw,
                                                         const uint8_t* __restrict__ mask,
                                                         int T, int E, int K, int score_fn,
                                                         int renorm, float route_scale,
                                                         float* dl, uint16_t* dl_bf, int ld_bf)
{
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int warps = (gridDim.x * blockDim.x) >> 5;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
        const float* row = logits + (int64_t)t * E;
        float dlv[NE];
        if (mask != nullptr && mask[t] == 0) {
#pragma unroll
            for (int i = 0; i < NE; ++i) dlv[i] = 0.0f;
        } else {
            float s[NE], ds[NE];
            contract_scores<NE>(row, E, score_fn, lane, s);
#pragma unroll
            for (int i = 0; i < NE; ++i) ds[i] = 0.0f;
            int my_id = -1;
            float my_dw = 0.0f;
            if (lane < K) {
                my_id = ids[(int64_t)t * K + lane];
                my_dw = dw[(int64_t)t * K + lane];
            }
            // the selected scores, broadcast rank by rank (every lane holds them all)
            float D = 0.0f, q = 0.0f;
            float s_sel[16], g_sel[16];
            int id_sel[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j >= K) break;
                const int id = __shfl_sync(0xffffffffu, my_id, j);
                const float g = __shfl_sync(0xffffffffu, my_dw, j);
                float v = 0.0f;
                const int owner = id & 31, slot = id >> 5;
#pragma unroll
                for (int i = 0; i < NE; ++i)
                    if (i == slot) v = s[i];
                v = __shfl_sync(0xffffffffu, v, owner);
                id_sel[j] = (id >= 0 && id < E) ? id : -1;
                s_sel[j] = v;
                g_sel[j] = g;
                if (id_sel[j] >= 0) {
                    D = __fadd_rn(D, v);
                    q = __fadd_rn(q, __fmul_rn(g, v));
                }
            }
            float r = 0.0f;
            const float qd = (renorm && D != 0.0f) ? __fdiv_rn(q, D) : 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j >= K) break;
                if (id_sel[j] < 0) continue;
                float dsj;
                if (renorm)
                    dsj = (D != 0.0f)
                              ? __fdiv_rn(__fmul_rn(route_scale, __fsub_rn(g_sel[j], qd)), D)
                              : 0.0f;
                else
                    dsj = __fmul_rn(route_scale, g_sel[j]);
                r = __fadd_rn(r, __fmul_rn(dsj, s_sel[j]));
                const int owner = id_sel[j] & 31, slot = id_sel[j] >> 5;
#pragma unroll
                for (int i = 0; i < NE; ++i)
                    if (lane == owner && i == slot) ds[i] = dsj;
            }
#pragma unroll
            for (int i = 0; i < NE; ++i) {
                const int e = lane + 32 * i;
                float v = 0.0f;
                if (e < E) {
                    if (score_fn == MOE_SOFTMAX) {
                        v = __fmul_rn(s[i], __fsub_rn(ds[i], r));
                    } else if (score_fn == MOE_SIGMOID) {
                        v = __fmul_rn(ds[i], __fmul_rn(s[i], __fsub_rn(1.0f, s[i])));
                    } else if (ds[i] != 0.0f && s[i] != 0.0f) {
                        const float sig = elementwise_score(row[e], MOE_SIGMOID);
                        v = __fmul_rn(ds[i], __fdiv_rn(sig, __fmul_rn(2.0f, s[i])));
                    }
                }
                dlv[i] = v;
            }
        }
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
            if (e < E && dl != nullptr) dl[(int64_t)t * E + e] = dlv[i];
            if (e < ld_bf) dl_bf[(int64_t)t * ld_bf + e] = (uint16_t)(e < E ? bf16_bits(dlv[i]) : 0u);
        }
        for (int e = 32 * NE + lane; e < ld_bf; e += 32) dl_bf[(int64_t)t * ld_bf + e] = 0;
    }
}

// dx_t = bf16(sum_j rows[dest_row[t,j]] (rank order) + shared_t + router_t), 0 if masked;
// one thread per 16-byte chunk
__global__ void __launch_bounds__(256) unpermute_kernel(const uint4* __restrict__ rows,
                                                        const int32_t* __restrict__ dest_row,
                                                        const uint4* __restrict__ shared,
                                                        const uint4* __restrict__ router,
                                                        const uint8_t* __restrict__ mask,
                                                        int T, int K, int H, uint4* __restrict__ dx)
{
    pdl_wait();
    const int hv = H >> 3;
    const int64_t n = (int64_t)T * hv;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = idx / hv;
        const int64_t c = idx - t * hv;
        if (mask != nullptr && mask[t] == 0) {
            dx[idx] = make_uint4(0u, 0u, 0u, 0u);
            continue;
        }
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        auto add = [&](const uint4 v) {
            const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] = __fadd_rn(acc[2 * e], lo_f(q[e]));
                acc[2 * e + 1] = __fadd_rn(acc[2 * e + 1], hi_f(q[e]));
            }
        };
        for (int j = 0; j < K; ++j) {
            const int32_t r = dest_row[t * K + j];
            if (r >= 0) add(rows[(int64_t)r * hv + c]);
        }
        if (shared != nullptr) add(shared[idx]);
        if (router != nullptr) add(router[idx]);
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = bf16_bits(acc[2 * e]) | (bf16_bits(acc[2 * e + 1]) << 16);
        dx[idx] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// per-group K ranges padded to 64: poff[g] = sum_{g' < g} ceil64(off[g'+1] - off[g']);
// one block of 1024 threads, groups <= 1024 (off == NULL: one group of `rows` rows)
__global__ void __launch_bounds__(1024) padded_offsets_kernel(const int32_t* __restrict__ off,
                                                              int G, int rows, int32_t* poff)
{
    pdl_wait();
    __shared__ int32_t part[1024];
    const int g = threadIdx.x;
    int32_t c = 0;
    if (g < G) {
        const int32_t n = off ? off[g + 1] - off[g] : rows;
        c = (n + 63) / 64 * 64;
    }
    part[g] = c;
    __syncthreads();
    for (int d = 1; d < 1024; d <<= 1) {  // inclusive Hillis-Steele scan
        const int32_t v = g >= d ? part[g - d] : 0;
        __syncthreads();
        part[g] += v;
        __syncthreads();
    }
    if (g < G) poff[g + 1] = part[g];
    if (g == 0) poff[0] = 0;
}

// K ranges of a product over `rows` rows split into chunks of `chunk` rows (a multiple of
// 64): koff[s] = min(s * chunk, rows rounded up to 64), s = 0..S
__global__ void split_offsets_kernel(int rows, int chunk, int S, int32_t* __restrict__ koff)
{
    pdl_wait();
    const int s = blockIdx.x * blockDim.x + threadIdx.x;
    const int end = (rows + 63) / 64 * 64;
    if (s <= S) koff[s] = (int)((int64_t)s * chunk < end ? (int64_t)s * chunk : end);
}

// out[i] = part[0][i] + part[1][i] + ... + part[S-1][i], fp32 adds in chunk order
__global__ void __launch_bounds__(256) sum_parts_kernel(const float4* __restrict__ part, int S,
                                                        int64_t n4, float4* __restrict__ out)
{
    pdl_wait();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 a = part[i];
        for (int s = 1; s < S; ++s) {
            const float4 b = part[(int64_t)s * n4 + i];
            a.x = __fadd_rn(a.x, b.x);
            a.y = __fadd_rn(a.y, b.y);
            a.z = __fadd_rn(a.z, b.z);
            a.w = __fadd_rn(a.w, b.w);
        }
        out[i] = a;
    }
}

__global__ void pad_rows_kernel(const int32_t* __restrict__ ids, const int32_t* __restrict__ dest,
                                const int32_t* __restrict__ off, const int32_t* __restrict__ poff,
                                int64_t A, int E, int32_t* __restrict__ dest_pad)
{
    pdl_wait();
    for (int64_t a = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; a < A;
         a += (int64_t)gridDim.x * blockDim.x) {
        const int32_t r = dest[a];
        const int32_t e = ids[a];
        dest_pad[a] = (r >= 0 && e >= 0 && e < E) ? poff[e] + (r - off[e]) : -1;
    }
}

// block (x, g): 16-byte chunks of group g's padding rows
__global__ void zero_pad_rows_kernel(uint4* __restrict__ buf, int64_t vec_per_row,
                                     const int32_t* __restrict__ off,
                                     const int32_t* __restrict__ poff)
{
    pdl_wait();
    const int g = blockIdx.y;
    const int64_t r0 = (int64_t)poff[g] + (off[g + 1] - off[g]);
    const int64_t n = ((int64_t)poff[g + 1] - r0) * vec_per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        buf[r0 * vec_per_row + i] = make_uint4(0u, 0u, 0u, 0u);
}

template <int NE>
cudaError_t launch_router_bwd_ne(const moe_cfg& c, const float* logits, const int32_t* ids,
                                 const float* dw, const uint8_t* mask, float* dl,
                                 uint16_t* dl_bf, int ld_bf, cudaStream_t st)
{
    int blocks = (c.T + 7) / 8;
    const int cap = num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_pdl(router_bwd_kernel<NE>, dim3(blocks), dim3(256), 0, st, logits, ids, dw, mask,
                      c.T, c.E, c.K, c.score_fn, c.renorm, c.route_scale, dl, dl_bf, ld_bf);
}

int grid_for(int64_t work, int per_block)
{
    int64_t b = (work + per_block - 1) / per_block;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (b > cap) b = cap;
    return (int)(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_combine_bwd(const moe_cfg& c, const uint16_t* dout, const uint16_t* y,
                               const float* w, const int32_t* dest_row, const uint8_t* mask,
                               float* dw, uint16_t* dy, uint16_t* dy_shared, cudaStream_t st)
{
    return launch_pdl(combine_bwd_kernel, dim3(grid_for((int64_t)c.T * 32, 256)), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(dout), reinterpret_cast<const uint4*>(y), w,
                      dest_row, mask, c.T, c.K, c.H, dw, reinterpret_cast<uint4*>(dy),
                      reinterpret_cast<uint4*>(dy_shared));
}

cudaError_t launch_router_bwd(const moe_cfg& c, const float* logits, const int32_t* ids,
                              const float* dw, const uint8_t* mask, float* dl, uint16_t* dl_bf,
                              int ld_bf, cudaStream_t st)
{
    const int ne = (c.E + 31) / 32;
    if (ne <= 1) return launch_router_bwd_ne<1>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
    if (ne <= 2) return launch_router_bwd_ne<2>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
    if (ne <= 4) return launch_router_bwd_ne<4>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
    if (ne <= 8) return launch_router_bwd_ne<8>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
    if (ne <= 16) return launch_router_bwd_ne<16>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
    return launch_router_bwd_ne<32>(c, logits, ids, dw, mask, dl, dl_bf, ld_bf, st);
}

cudaError_t launch_unpermute(const moe_cfg& c, const uint16_t* rows, const int32_t* dest_row,
                             const uint16_t* shared, const uint16_t* router, const uint8_t* mask,
                             uint16_t* dx, cudaStream_t st)
{
    return launch_pdl(unpermute_kernel, dim3(grid_for((int64_t)c.T * (c.H / 8), 256)), dim3(256), 0,
                      st, reinterpret_cast<const uint4*>(rows), dest_row,
                      reinterpret_cast<const uint4*>(shared),
                      reinterpret_cast<const uint4*>(router), mask, c.T, c.K, c.H,
                      reinterpret_cast<uint4*>(dx));
}

cudaError_t launch_padded_offsets(const int32_t* off, int G, int rows, int32_t* poff,
                                  cudaStream_t st)
{
    if (G < 1 || G > 1024) return cudaErrorInvalidValue;
    return launch_pdl(padded_offsets_kernel, dim3(1), dim3(1024), 0, st, off, G, rows, poff);
}

cudaError_t launch_split_offsets(int rows, int chunk, int S, int32_t* koff, cudaStream_t st)
{
    if (S < 1 || chunk < 64 || chunk % 64 != 0) return cudaErrorInvalidValue;
    return launch_pdl(split_offsets_kernel, dim3((unsigned)((S + 1 + 255) / 256)), dim3(256), 0,
                      st, rows, chunk, S, koff);
}

cudaError_t launch_sum_parts(const float* part, int S, int64_t n, float* out, cudaStream_t st)
{
    if (S < 1 || n % 4 != 0) return cudaErrorInvalidValue;
    const int64_t n4 = n / 4;
    if (n4 == 0) return cudaSuccess;
    int64_t blocks = (n4 + 255) / 256;
    const int64_t cap = resident_blocks((const void*)sum_parts_kernel, 256, 0);
    if (blocks > cap) blocks = cap;
    return launch_pdl(sum_parts_kernel, dim3((unsigned)blocks), dim3(256), 0, st,
                      reinterpret_cast<const float4*>(part), S, n4, reinterpret_cast<float4*>(out));
}

cudaError_t launch_pad_rows(const int32_t* ids, const int32_t* dest_row, const int32_t* off,
                            const int32_t* poff, int64_t A, int E, int32_t* dest_pad,
                            cudaStream_t st)
{
    if (A <= 0) return cudaSuccess;
    return launch_pdl(pad_rows_kernel, dim3(grid_for(A, 256)), dim3(256), 0, st, ids, dest_row,
                      off, poff, A, E, dest_pad);
}

cudaError_t launch_zero_pad_rows(uint16_t* buf, int64_t cols, const int32_t* off,
                                 const int32_t* poff, int G, cudaStream_t st)
{
    if (G <= 0 || cols % 8 != 0) return cols % 8 ? cudaErrorInvalidValue : cudaSuccess;
    const int64_t vec = cols / 8;
    int bx = (int)((63 * vec + 255) / 256);
    if (bx > 64) bx = 64;
    if (bx < 1) bx = 1;
    return launch_pdl(zero_pad_rows_kernel, dim3((unsigned)bx, (unsigned)G), dim3(256), 0, st,
                      reinterpret_cast<uint4*>(buf), vec, off, poff);
}

}  // namespace moe

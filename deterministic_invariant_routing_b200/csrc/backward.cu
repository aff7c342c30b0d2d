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
//  transposes         [R, F] -> [F, columns] bf16, rows optionally mapped to padded per-expert
//                     column ranges (the K operand layout of the weight-gradient products),
//                     padding columns zeroed
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

// column of each grouped row in the padded layout (-1 past the last routed row)
__global__ void colmap_kernel(const int32_t* __restrict__ off, const int32_t* __restrict__ poff,
                              int G, int64_t rows_bound, int32_t* __restrict__ col)
{
    pdl_wait();
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows_bound;
         r += (int64_t)gridDim.x * blockDim.x) {
        if (r >= off[G]) {
            col[r] = -1;
            continue;
        }
        int lo = 0, hi = G - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (off[mid] <= r) lo = mid;
            else hi = mid - 1;
        }
        col[r] = (int32_t)(poff[lo] + (r - off[lo]));
    }
}

// out[z][f, col(r)] = in[z][r, f] for a 64 x 64 tile per block; col(r) = colmap[r] (skip
// when < 0) or r. VEC: F and ld_in are multiples of 8 (16-byte loads).
template <bool VEC>
__global__ void __launch_bounds__(256) transpose_kernel(const uint16_t* __restrict__ in,
                                                        int64_t R, int F, int64_t ld_in,
                                                        int64_t in_batch, uint16_t* __restrict__ out,
                                                        int64_t ld_out, int64_t out_batch,
                                                        const int32_t* __restrict__ colmap)
{
    pdl_wait();
    __shared__ uint16_t tile[64][65];
    const int64_t r0 = (int64_t)blockIdx.x * 64;
    const int f0 = blockIdx.y * 64;
    const uint16_t* src = in + (int64_t)blockIdx.z * in_batch;
    uint16_t* dst = out + (int64_t)blockIdx.z * out_batch;
    if (VEC) {
        for (int idx = threadIdx.x; idx < 64 * 8; idx += 256) {
            const int rr = idx >> 3, vv = idx & 7;
            const int64_t r = r0 + rr;
            const int f = f0 + vv * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < R && f < F) v = *reinterpret_cast<const uint4*>(src + r * ld_in + f);
            const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                tile[rr][vv * 8 + 2 * e] = (uint16_t)(q[e] & 0xffffu);
                tile[rr][vv * 8 + 2 * e + 1] = (uint16_t)(q[e] >> 16);
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < 64 * 64; idx += 256) {
            const int rr = idx >> 6, ff = idx & 63;
            const int64_t r = r0 + rr;
            const int f = f0 + ff;
            tile[rr][ff] = (r < R && f < F) ? src[r * ld_in + f] : (uint16_t)0;
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < 64 * 64; idx += 256) {
        const int ff = idx >> 6, rr = idx & 63;
        const int64_t r = r0 + rr;
        const int f = f0 + ff;
        if (r >= R || f >= F) continue;
        const int64_t c = colmap ? (int64_t)colmap[r] : r;
        if (c >= 0) dst[(int64_t)f * ld_out + c] = tile[rr][ff];
    }
}

// zero the padding columns [poff[g] + n_g, poff[g+1]) of every row f < F of out [F, ld_out];
// n_g = off[g+1] - off[g] (off == NULL: one group of `rows` rows)
__global__ void zero_pad_kernel(uint16_t* __restrict__ out, int F, int64_t ld_out,
                                const int32_t* __restrict__ off, const int32_t* __restrict__ poff,
                                int rows)
{
    pdl_wait();
    const int g = blockIdx.y;
    const int64_t n = off ? (int64_t)(off[g + 1] - off[g]) : rows;
    const int64_t c0 = poff[g] + n, c1 = poff[g + 1];
    const int width = (int)(c1 - c0);  // < 64
    if (width <= 0) return;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < F * 64;
         idx += gridDim.x * blockDim.x) {
        const int f = idx >> 6, c = idx & 63;
        if (c < width) out[(int64_t)f * ld_out + c0 + c] = 0;
    }
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

cudaError_t launch_colmap(const int32_t* off, const int32_t* poff, int G, int64_t rows_bound,
                          int32_t* col, cudaStream_t st)
{
    if (rows_bound <= 0) return cudaSuccess;
    return launch_pdl(colmap_kernel, dim3(grid_for(rows_bound, 256)), dim3(256), 0, st, off, poff,
                      G, rows_bound, col);
}

cudaError_t launch_transpose(const uint16_t* in, int64_t R, int F, int64_t ld_in, int64_t in_batch,
                             uint16_t* out, int64_t ld_out, int64_t out_batch, int batches,
                             const int32_t* colmap, cudaStream_t st)
{
    if (R <= 0 || F <= 0 || batches <= 0) return cudaSuccess;
    const dim3 grid((unsigned)((R + 63) / 64), (unsigned)((F + 63) / 64), (unsigned)batches);
    if (grid.x > 2147483647u || grid.y > 65535u || grid.z > 65535u) return cudaErrorInvalidValue;
    const bool vec = (F % 8 == 0) && (ld_in % 8 == 0) &&
                     (reinterpret_cast<uintptr_t>(in) % 16 == 0) && (in_batch % 8 == 0);
    if (vec)
        return launch_pdl(transpose_kernel<true>, grid, dim3(256), 0, st, in, R, F, ld_in, in_batch,
                          out, ld_out, out_batch, colmap);
    return launch_pdl(transpose_kernel<false>, grid, dim3(256), 0, st, in, R, F, ld_in, in_batch,
                      out, ld_out, out_batch, colmap);
}

cudaError_t launch_zero_pad(uint16_t* out, int F, int64_t ld_out, const int32_t* off,
                            const int32_t* poff, int G, int rows, cudaStream_t st)
{
    if (F <= 0 || G <= 0) return cudaSuccess;
    const int bx = (int)((F * 64 + 255) / 256 < 64 ? (F * 64 + 255) / 256 : 64);
    return launch_pdl(zero_pad_kernel, dim3((unsigned)bx, (unsigned)G), dim3(256), 0, st, out, F,
                      ld_out, off, poff, rows);
}

}  // namespace moe

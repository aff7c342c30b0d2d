/*
 * moe_oracle.c -- TEST INFRASTRUCTURE. A plain, slow, single-file CPU oracle of the
 * top-k MoE FFN forward pass. It exists only to check the CUDA library; nothing in the
 * product path may link, load or call it (only the tests, the smoke check and the
 * bench's CPU-baseline leg do). It shares no code, header, table or constant with the
 * CUDA library.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 * (no FMA contraction, IEEE single/double on SSE, default round-to-nearest-even,
 * no flush-to-zero). Every fused multiply-add below is an explicit fmaf().
 *
 * Two parts:
 *  1. The FP32 contract (bit-level): scores, selection, weights, permutation and the
 *     weighted combine exactly as the contract defines them. Results must match the
 *     GPU bit for bit given the same FP32 logits / the same expert outputs.
 *  2. FP64 math: router logits, routing weights of given routes and the SwiGLU
 *     experts in double precision, for the tolerance check of the bf16 layer output.
 *
 * What it follows, by source page:
 *  - "DSV4 Flash MoE Train-Inference Consistency Roadmap" (RL-Kernel blog),
 *    Problem 1 "Routing Is A Discrete Decision": router logits from hidden states, top-k
 *    selection, tie-breaking and expert bias as the routing contract;
 *    Problem 2: the gather -> gate_and_up -> down -> scatter decomposition and the
 *    semantic boundaries (routing / dispatch / expert / shared-expert / reduction);
 *    Problem 3 "Final Reduction Is The Core Drift Point": the weighted combine with a
 *    recorded order, dtype and downcast point.
 *  - "From Expert Reduction to Behavioral Divergence ..." (arXiv 2607.28097), Abstract:
 *    reduction order of the expert sum is observable; 720 orders of a six-term sum fall
 *    into at most 360 exact classes when the first two terms commute.
 *  - SpecForge PR #1003 "MoE FFN support for DFlash-family drafts", Design notes and the
 *    selection-bias commit: the bias shifts the top-k picks only, the weights come from
 *    the unbiased scores; norm_topk_prob renormalisation; route_scale and score_fn are
 *    the DeepSeek seams; the shared expert is always on and added on top.
 *
 * Readings where the pages are silent (the same list is kept with the design notes):
 *  exp_rl (below) is the exponential of the contract; the softmax denominator is the
 *  fixed 32-lane tree (below); selection key = (choice desc, id asc), NaN below -inf,
 *  -0 == +0; weights renormalised by sequential rank-order sum, then x route_scale;
 *  combine = rounded products summed in rank order, shared expert last, one bf16 RNE.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_SOFTMAX 0
#define ORACLE_SIGMOID 1
#define ORACLE_SQRTSOFTPLUS 2

/* ------------------------------------------------------------------ bits & bf16 */

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float oracle_bf16_to_f32(uint16_t h) { return u2f((uint32_t)h << 16); }

/* float -> bf16, round to nearest, ties to even; NaN stays NaN (quieted, sign kept). */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = f2u(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t keep_lsb = (u >> 16) & 1u;
    u += 0x7fffu + keep_lsb;
    return (uint16_t)(u >> 16);
}

void oracle_f32_to_bf16_array(const float* in, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(in[i]);
}

/* ------------------------------------------------------------------ exp_rl */
/*
 * exp_rl(x): the contract's fp32 exponential (the pages fix none; they only name the
 * router softmax as the place to "validate precision and stability first").
 * Cody & Waite (1980) additive range reduction, then a degree-7 Taylor polynomial:
 *   n  = rint(fp32(x * log2e))                         (ties to even)
 *   r  = fma(-n, ln2_hi, x);  r = fma(-n, ln2_lo, r)
 *        ln2_hi = fp32(ln 2) with its 12 low mantissa bits rounded away (n*ln2_hi exact),
 *        ln2_lo = fp32(ln 2 - ln2_hi)
 *   p  = sum_{k=0..7} r^k / k!  by Horner with fma, coefficients fp32(1/k!)
 *   result = p * 2^n  (2^n built from its exponent bits; one rounded multiply)
 * Specials: NaN -> NaN, x < -87 -> +0, x > 88 -> +inf. exp_rl(0) == 1 exactly.
 */
static float ln2_hi_const(void)
{
    uint32_t u = f2u((float)0.69314718055994530942);
    uint32_t low = u & 0xfffu;
    u &= ~0xfffu;
    if (low > 0x800u || (low == 0x800u && (u & 0x1000u))) u += 0x1000u;
    return u2f(u);
}

float oracle_exp_rl(float x)
{
    if (isnan(x)) return x;
    if (x < -87.0f) return 0.0f;
    if (x > 88.0f) return INFINITY;
    const float log2e = (float)1.44269504088896340736;
    const float hi = ln2_hi_const();
    const float lo = (float)(0.69314718055994530942 - (double)hi);
    float t = x * log2e;
    float n = rintf(t);
    float r = fmaf(-n, hi, x);
    r = fmaf(-n, lo, r);
    double fact = 1.0;
    float c[8];
    for (int k = 0; k < 8; ++k) { if (k > 0) fact *= (double)k; c[k] = (float)(1.0 / fact); }
    float p = c[7];
    for (int k = 6; k >= 0; --k) p = fmaf(p, r, c[k]);
    int ni = (int)n;
    float scale = u2f((uint32_t)(ni + 127) << 23);
    return p * scale;
}

void oracle_exp_rl_array(const float* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_exp_rl(in[i]);
}

/* ------------------------------------------------------------------ sqrtsoftplus */
/*
 * The sqrtsoftplus router score, s = sqrt(softplus(l)), named beside sigmoid in SpecForge
 * PR #1003 (the load-balance commit: scores are L1-normalised so that sigmoid and
 * sqrtsoftplus routers share the aux formula). The pages give no formula or precision;
 * the contract here, fp32 with every operation rounded to nearest:
 *
 *   softplus(l) = l                      for l > 20 (log1p(e^l) - l < 2^-28 there)
 *               = log1p_rl(exp_rl(l))    otherwise
 *   s           = sqrt(softplus(l))      (IEEE square root, correctly rounded)
 *
 * log1p_rl(u), u >= 0, is D. Goldberg's formula ("What every computer scientist should
 * know about floating-point arithmetic", 1991, Theorem 4): v = 1 + u; u when v == 1, else
 * (u * ln_rl(v)) / (v - 1), where v - 1 is exact.
 *
 * ln_rl(v), v >= 1 finite: v = m * 2^k with m in [1, 2) from the bits, halved (k + 1)
 * when m > fp32(sqrt 2); f = m - 1 (exact); z = f / (2 + f); ln m = 2 atanh z =
 * 2z + 2 z^3 (1/3 + w/5 + w^2/7 + w^3/9), w = z^2, |z| <= 0.1716 (the next term is below
 * 2^-28 relative); the polynomial by Horner with fma and coefficients fp32(1/k); then
 * ln v = k ln2_hi + (k ln2_lo + ln m), the Cody-Waite split of exp_rl.
 */
float oracle_ln_rl(float v)
{
    uint32_t b = f2u(v);
    int k = (int)(b >> 23) - 127;
    float m = u2f((b & 0x7fffffu) | 0x3f800000u);
    if (m > (float)1.41421356237309504880) { m = m * 0.5f; k += 1; }
    const float f = m - 1.0f;
    const float z = f / (2.0f + f);
    const float w = z * z;
    float q = fmaf(w, (float)(1.0 / 9.0), (float)(1.0 / 7.0));
    q = fmaf(w, q, (float)(1.0 / 5.0));
    q = fmaf(w, q, (float)(1.0 / 3.0));
    const float zw = z * w;
    const float lnm = fmaf(2.0f * zw, q, 2.0f * z);
    const float hi = ln2_hi_const();
    const float lo = (float)(0.69314718055994530942 - (double)hi);
    const float kf = (float)k;
    return fmaf(kf, hi, fmaf(kf, lo, lnm));
}

float oracle_log1p_rl(float u)
{
    const float v = 1.0f + u;
    if (v == 1.0f) return u;
    return (u * oracle_ln_rl(v)) / (v - 1.0f);
}

float oracle_sqrtsoftplus_rl(float l)
{
    const float sp = (l > 20.0f) ? l : oracle_log1p_rl(oracle_exp_rl(l));
    return sqrtf(sp);
}

void oracle_fn_array(int which, const float* in, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = which == 0 ? oracle_ln_rl(in[i])
               : which == 1 ? oracle_log1p_rl(in[i])
                            : oracle_sqrtsoftplus_rl(in[i]);
}

/* ------------------------------------------------------------------ scores */
/*
 * Softmax denominator: the fixed 32-lane tree of the contract. Lane L first sums the
 * terms e = L, L+32, L+64, ... in increasing e (sequential fp32 adds starting from +0);
 * then five butterfly levels with offsets 16, 8, 4, 2, 1, each lane taking
 * v[L] + v[L xor off]. Every lane ends with the same value; lane 0's is returned.
 */
float oracle_tree_sum32(const float* v, int n)
{
    float lane[32], nxt[32];
    for (int l = 0; l < 32; ++l) lane[l] = 0.0f;
    for (int e = 0; e < n; ++e) lane[e & 31] = lane[e & 31] + v[e];
    for (int off = 16; off >= 1; off >>= 1) {
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ off];
        memcpy(lane, nxt, sizeof lane);
    }
    return lane[0];
}

/* Scores of one token (FP32 contract). softmax: m = max, e = exp_rl(l - m), S = tree
 * sum, s = e / S. sigmoid: s = 1 / (1 + exp_rl(-l)). sqrtsoftplus: see above. */
void oracle_scores_fp32(int E, const float* l, int score_fn, float* s)
{
    if (score_fn == ORACLE_SIGMOID) {
        for (int e = 0; e < E; ++e) s[e] = 1.0f / (1.0f + oracle_exp_rl(-l[e]));
        return;
    }
    if (score_fn == ORACLE_SQRTSOFTPLUS) {
        for (int e = 0; e < E; ++e) s[e] = oracle_sqrtsoftplus_rl(l[e]);
        return;
    }
    if (E <= 0) return;
    float m = -INFINITY;
    for (int e = 0; e < E; ++e) if (l[e] > m) m = l[e];
    float* ex = (float*)malloc(sizeof(float) * (size_t)E);
    for (int e = 0; e < E; ++e) ex[e] = oracle_exp_rl(l[e] - m);
    float S = oracle_tree_sum32(ex, E);
    for (int e = 0; e < E; ++e) s[e] = ex[e] / S;
    free(ex);
}

/* ------------------------------------------------------------------ selection */
/*
 * Selection key of (choice, id): higher choice first, then lower id. -0 counts as +0,
 * NaN ranks below -inf. Key = (order-preserving bits of choice) << 32 | (0xffffffff - id).
 */
uint64_t oracle_select_key(float c, int id)
{
    uint32_t ord;
    if (isnan(c)) {
        ord = 0u;
    } else {
        if (c == 0.0f) c = 0.0f;
        uint32_t u = f2u(c);
        ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    return ((uint64_t)ord << 32) | (uint64_t)(0xffffffffu - (uint32_t)id);
}

/*
 * Route T tokens from FP32 logits [T,E] (FP32 contract):
 *   scores s (unbiased); choice = s + sel_bias (if given) -- selection only;
 *   ids = the K largest selection keys, in decreasing key order (rank 0 = best);
 *   renorm: D = s[id0] + s[id1] + ... (rank order), w_j = (s[id_j] / D) * route_scale,
 *           D == 0 -> all w = 0 and one zero-denominator count;
 *   no renorm: w_j = s[id_j] * route_scale.
 * Masked tokens (mask[t] == 0) get ids -1 and weights 0.
 * status[0] += tokens with a NaN choice, status[1] += zero-denominator tokens.
 */
/*
 * Group-limited selection (the DeepSeek family's override of `select` named in SpecForge
 * PR #1003, "Out of scope" and the select() refactor note; the pages give no formula).
 * Reading: the E experts form n_group contiguous groups of E / n_group; a group's score is
 * the fp32 sum of its two best choices (best + second, by the selection key; one choice
 * when the group has one expert); the topk_group groups with the largest (group score,
 * then lower group id) are kept; the K experts are then chosen among the kept groups only.
 * n_group <= 1 turns it off. Weights still come from the unbiased scores.
 */
static void keep_groups(int E, int n_group, int topk_group, const float* c,
                        const uint64_t* key, unsigned char* excluded)
{
    const int gs = E / n_group;
    uint64_t* gkey = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)n_group);
    unsigned char* kept = (unsigned char*)calloc((size_t)n_group, 1);
    for (int g = 0; g < n_group; ++g) {
        int b1 = -1, b2 = -1;
        for (int e = g * gs; e < (g + 1) * gs; ++e) {
            if (b1 < 0 || key[e] > key[b1]) { b2 = b1; b1 = e; }
            else if (b2 < 0 || key[e] > key[b2]) { b2 = e; }
        }
        float score = c[b1];
        if (b2 >= 0) score = score + c[b2];
        gkey[g] = oracle_select_key(score, g);
    }
    for (int r = 0; r < topk_group; ++r) {
        int best = -1;
        for (int g = 0; g < n_group; ++g)
            if (!kept[g] && (best < 0 || gkey[g] > gkey[best])) best = g;
        kept[best] = 1;
    }
    for (int e = 0; e < E; ++e) excluded[e] = !kept[e / gs];
    free(gkey);
    free(kept);
}

void oracle_route_fp32_grouped(int T, int E, int K, const float* logits, const float* sel_bias,
                               const uint8_t* mask, int score_fn, int renorm, float route_scale,
                               int n_group, int topk_group, int32_t* ids, float* w,
                               int64_t* status)
{
    int64_t nan_tokens = 0, zero_den = 0;
#pragma omp parallel for reduction(+ : nan_tokens, zero_den) schedule(static)
    for (int t = 0; t < T; ++t) {
        int32_t* id = ids + (int64_t)t * K;
        float* wt = w + (int64_t)t * K;
        if (mask && !mask[t]) {
            for (int j = 0; j < K; ++j) { id[j] = -1; wt[j] = 0.0f; }
            continue;
        }
        float* s = (float*)malloc(sizeof(float) * (size_t)E);
        float* cv = (float*)malloc(sizeof(float) * (size_t)E);
        uint64_t* key = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)E);
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        oracle_scores_fp32(E, logits + (int64_t)t * E, score_fn, s);
        int has_nan = 0;
        for (int e = 0; e < E; ++e) {
            float c = sel_bias ? s[e] + sel_bias[e] : s[e];
            if (isnan(c)) has_nan = 1;
            cv[e] = c;
            key[e] = oracle_select_key(c, e);
        }
        nan_tokens += has_nan;
        if (n_group > 1) keep_groups(E, n_group, topk_group, cv, key, taken);
        for (int j = 0; j < K; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || key[e] > key[best])) best = e;
            taken[best] = 1;
            id[j] = best;
        }
        if (renorm) {
            float D = s[id[0]];
            for (int j = 1; j < K; ++j) D = D + s[id[j]];
            if (D == 0.0f) {
                for (int j = 0; j < K; ++j) wt[j] = 0.0f;
                zero_den += 1;
            } else {
                for (int j = 0; j < K; ++j) wt[j] = (s[id[j]] / D) * route_scale;
            }
        } else {
            for (int j = 0; j < K; ++j) wt[j] = s[id[j]] * route_scale;
        }
        free(s); free(cv); free(key); free(taken);
    }
    if (status) { status[0] += nan_tokens; status[1] += zero_den; }
}

void oracle_route_fp32(int T, int E, int K, const float* logits, const float* sel_bias,
                       const uint8_t* mask, int score_fn, int renorm, float route_scale,
                       int32_t* ids, float* w, int64_t* status)
{
    oracle_route_fp32_grouped(T, E, K, logits, sel_bias, mask, score_fn, renorm, route_scale, 0,
                              0, ids, w, status);
}

/* ------------------------------------------------------------------ permutation */
/*
 * Dispatch boundary: counting sort of the T*K assignments a = t*K + j by expert,
 * stable in a. ids outside [0,E) (masked tokens carry -1) are not dispatched:
 * dest_row[a] = -1. offsets[E+1] is the exclusive scan of the per-expert counts;
 * perm_token[r] = t for every dispatched row r < offsets[E] (rows past it untouched).
 * Returns the number of ids that were >= E (invalid), not counting the -1s.
 */
int64_t oracle_permute(int T, int K, int E, const int32_t* ids, int32_t* offsets,
                       int32_t* perm_token, int32_t* dest_row)
{
    int64_t A = (int64_t)T * K, bad = 0;
    int64_t* cnt = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    for (int64_t a = 0; a < A; ++a) {
        int32_t e = ids[a];
        if (e >= 0 && e < E) cnt[e] += 1;
        else if (e >= E) bad += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + (int32_t)cnt[e];
    int64_t* next = cnt;
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t a = 0; a < A; ++a) {
        int32_t e = ids[a];
        if (e >= 0 && e < E) {
            int64_t r = next[e]++;
            dest_row[a] = (int32_t)r;
            perm_token[r] = (int32_t)(a / K);
        } else {
            dest_row[a] = -1;
        }
    }
    free(cnt);
    return bad;
}

/* ------------------------------------------------------------------ combine */
/*
 * Reduction boundary (FP32 contract), per token t and hidden column h:
 *   p_j = fp32(w_j * float(y[dest_row[t,j], h]))      (rounded product, no FMA)
 *   acc = first valid p_j; then acc = acc + p_j for the later valid j (rank order)
 *   shared expert given: acc = acc + float(y_shared[t, h])   (added last)
 * A term with dest_row < 0 is skipped; with no valid term acc starts at +0.
 * The accumulator is returned in fp32 (no downcast) -- the combine's one bf16 rounding
 * is applied by oracle_combine_fp32. Masked tokens (mask[t] == 0): acc = 0.
 */
void oracle_combine_acc_fp32(int T, int K, int H, const uint16_t* y, const float* w,
                             const int32_t* dest_row, const uint16_t* y_shared,
                             const uint8_t* mask, float* acc_out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        float* o = acc_out + (int64_t)t * H;
        if (mask && !mask[t]) { for (int h = 0; h < H; ++h) o[h] = 0.0f; continue; }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            int first = 1;
            for (int j = 0; j < K; ++j) {
                int32_t r = dest_row[(int64_t)t * K + j];
                if (r < 0) continue;
                float p = w[(int64_t)t * K + j] * oracle_bf16_to_f32(y[(int64_t)r * H + h]);
                if (first) { acc = p; first = 0; }
                else acc = acc + p;
            }
            if (y_shared) acc = acc + oracle_bf16_to_f32(y_shared[(int64_t)t * H + h]);
            o[h] = acc;
        }
    }
}

void oracle_combine_fp32(int T, int K, int H, const uint16_t* y, const float* w,
                         const int32_t* dest_row, const uint16_t* y_shared,
                         const uint8_t* mask, uint16_t* out)
{
    float* acc = (float*)malloc(sizeof(float) * (size_t)T * (size_t)H);
    oracle_combine_acc_fp32(T, K, H, y, w, dest_row, y_shared, mask, acc);
    for (int64_t i = 0; i < (int64_t)T * H; ++i) out[i] = oracle_f32_to_bf16(acc[i]);
    free(acc);
}

/* ------------------------------------------------------------------ FP64 math */

/* logits[t,e] = sum_h x[t,h] * w_router[e,h] (+ logit_bias[e]), in double. */
void oracle_logits64(int T, int H, int E, const uint16_t* x, const uint16_t* wr,
                     const float* logit_bias, double* logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)oracle_bf16_to_f32(x[(int64_t)t * H + h]) *
                       (double)oracle_bf16_to_f32(wr[(int64_t)e * H + h]);
            if (logit_bias) acc += (double)logit_bias[e];
            logits[(int64_t)t * E + e] = acc;
        }
    }
}

/* sqrt(softplus(x)) in double with libm: softplus = max(x, 0) + log1p(exp(-|x|)) */
double oracle_sqrtsoftplus64(double x)
{
    if (isnan(x)) return x;
    return sqrt(fmax(x, 0.0) + log1p(exp(-fabs(x))));
}
#define sqrtsoftplus64 oracle_sqrtsoftplus64

/* Weights of given routes from double-precision scores of double logits (masked or
 * invalid ids give 0). renorm: w_j = s_j / sum_j s_j * route_scale; else s_j * scale. */
void oracle_weights64(int T, int E, int K, const double* logits, const int32_t* ids,
                      int score_fn, int renorm, double route_scale, double* w)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const double* l = logits + (int64_t)t * E;
        double* s = (double*)malloc(sizeof(double) * (size_t)E);
        if (score_fn == ORACLE_SIGMOID) {
            for (int e = 0; e < E; ++e) s[e] = 1.0 / (1.0 + exp(-l[e]));
        } else if (score_fn == ORACLE_SQRTSOFTPLUS) {
            for (int e = 0; e < E; ++e) s[e] = sqrtsoftplus64(l[e]);
        } else {
            double m = -INFINITY, S = 0.0;
            for (int e = 0; e < E; ++e) if (l[e] > m) m = l[e];
            for (int e = 0; e < E; ++e) { s[e] = exp(l[e] - m); S += s[e]; }
            for (int e = 0; e < E; ++e) s[e] /= S;
        }
        double D = 0.0;
        for (int j = 0; j < K; ++j) {
            int32_t e = ids[(int64_t)t * K + j];
            if (e >= 0 && e < E) D += s[e];
        }
        for (int j = 0; j < K; ++j) {
            int32_t e = ids[(int64_t)t * K + j];
            double v = (e >= 0 && e < E) ? s[e] : 0.0;
            if (renorm) v = (D != 0.0) ? v / D : 0.0;
            w[(int64_t)t * K + j] = v * route_scale;
        }
        free(s);
    }
}

/*
 * One token row through one SwiGLU expert, in double:
 *   g_i = x . W13[i,:], u_i = x . W13[I+i,:]   (gate rows first, then up rows)
 *   a_i = silu(g_i) * u_i,  silu(g) = g / (1 + exp(-g))
 *   y_h = sum_i a_i * W2[h,i]
 * w13 is [2I, H], w2 is [H, I] (bf16 bits). If h_out is given it receives a [I].
 */
void oracle_expert_ffn64(int H, int I, const uint16_t* x_row, const uint16_t* w13,
                         const uint16_t* w2, double* y, double* h_out)
{
    double* a = (double*)malloc(sizeof(double) * (size_t)I);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        const uint16_t* wg = w13 + (int64_t)i * H;
        const uint16_t* wu = w13 + (int64_t)(I + i) * H;
        for (int h = 0; h < H; ++h) {
            double xv = (double)oracle_bf16_to_f32(x_row[h]);
            g += xv * (double)oracle_bf16_to_f32(wg[h]);
            u += xv * (double)oracle_bf16_to_f32(wu[h]);
        }
        a[i] = g / (1.0 + exp(-g)) * u;
        if (h_out) h_out[i] = a[i];
    }
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        const uint16_t* w2r = w2 + (int64_t)h * I;
        for (int i = 0; i < I; ++i) acc += a[i] * (double)oracle_bf16_to_f32(w2r[i]);
        y[h] = acc;
    }
    free(a);
}

/*
 * Layer output in double for the given routes and double weights:
 *   out[t] = sum_j w64[t,j] * FFN_{ids[t,j]}(x_t)  (+ FFN_shared(x_t) when w13_s given)
 * Masked tokens give 0. Only the n_sel tokens listed in sel (or all T when sel is NULL)
 * are computed; out is [n_sel, H].
 */
void oracle_forward64(int T, int H, int E, int K, int I, int I_shared, const uint16_t* x,
                      const int32_t* ids, const double* w64, const uint8_t* mask,
                      const uint16_t* w13, const uint16_t* w2, const uint16_t* w13_s,
                      const uint16_t* w2_s, const int32_t* sel, int n_sel, double* out)
{
    int n = sel ? n_sel : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < n; ++q) {
        int t = sel ? sel[q] : q;
        double* o = out + (int64_t)q * H;
        for (int h = 0; h < H; ++h) o[h] = 0.0;
        if (mask && !mask[t]) continue;
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        const uint16_t* xr = x + (int64_t)t * H;
        for (int j = 0; j < K; ++j) {
            int32_t e = ids[(int64_t)t * K + j];
            if (e < 0 || e >= E) continue;
            oracle_expert_ffn64(H, I, xr, w13 + (int64_t)e * 2 * I * H,
                                w2 + (int64_t)e * H * I, y, NULL);
            double wj = w64[(int64_t)t * K + j];
            for (int h = 0; h < H; ++h) o[h] += wj * y[h];
        }
        if (w13_s && I_shared > 0) {
            oracle_expert_ffn64(H, I_shared, xr, w13_s, w2_s, y, NULL);
            for (int h = 0; h < H; ++h) o[h] += y[h];
        }
        free(y);
    }
}

/*
 * The whole layer on the CPU for n_sel selected tokens (the timed CPU baseline):
 * FP64 logits rounded to fp32, FP32-contract routing, FP64 weights of those routes,
 * FP64 experts. out is [n_sel, H] double; ids/w32 receive the routes of those tokens.
 */
void oracle_layer_forward(int H, int E, int K, int I, int I_shared, int score_fn,
                          int renorm, float route_scale, const uint16_t* x, const uint16_t* wr,
                          const float* logit_bias, const float* sel_bias, const uint16_t* w13,
                          const uint16_t* w2, const uint16_t* w13_s, const uint16_t* w2_s,
                          int n_sel, const int32_t* sel, int32_t* ids, double* out)
{
    uint16_t* xs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n_sel * H);
    for (int q = 0; q < n_sel; ++q)
        memcpy(xs + (int64_t)q * H, x + (int64_t)sel[q] * H, sizeof(uint16_t) * (size_t)H);
    double* l64 = (double*)malloc(sizeof(double) * (size_t)n_sel * E);
    float* l32 = (float*)malloc(sizeof(float) * (size_t)n_sel * E);
    float* w32 = (float*)malloc(sizeof(float) * (size_t)n_sel * K);
    double* w64 = (double*)malloc(sizeof(double) * (size_t)n_sel * K);
    oracle_logits64(n_sel, H, E, xs, wr, logit_bias, l64);
    for (int64_t i = 0; i < (int64_t)n_sel * E; ++i) l32[i] = (float)l64[i];
    oracle_route_fp32(n_sel, E, K, l32, sel_bias, NULL, score_fn, renorm, route_scale, ids,
                      w32, NULL);
    oracle_weights64(n_sel, E, K, l64, ids, score_fn, renorm, (double)route_scale, w64);
    oracle_forward64(n_sel, H, E, K, I, I_shared, xs, ids, w64, NULL, w13, w2, w13_s, w2_s,
                     NULL, n_sel, out);
    free(xs); free(l64); free(l32); free(w32); free(w64);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ router statistics */
/*
 * Router statistics of one forward (SpecForge PR #1003, the load-balance commit: a
 * Switch-style load-balance value E * sum_e load_e * mean_prob_e over the kept tokens,
 * equal to K when balanced; scores L1-normalised per token so sigmoid and softmax routers
 * share the formula; padding skipped through the token mask). Reading: over the N kept
 * tokens, count_e = assignments routed to e, load_e = count_e / N, p_{t,e} = s_{t,e} /
 * sum_e' s_{t,e'} with s the unbiased scores of the fp32 logits (computed here in
 * double), mean_prob_e = sum_t p_{t,e} / N, aux = E * sum_e load_e * mean_prob_e.
 * With N == 0: counts 0, mean_prob 0, aux 0.
 */
void oracle_router_stats(int T, int E, int K, const float* logits, const int32_t* ids,
                         const uint8_t* mask, int score_fn, int64_t* counts, double* mean_prob,
                         double* aux)
{
    int64_t n = 0;
    for (int e = 0; e < E; ++e) { counts[e] = 0; mean_prob[e] = 0.0; }
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        if (mask && !mask[t]) continue;
        n += 1;
        for (int j = 0; j < K; ++j) {
            int32_t e = ids[(int64_t)t * K + j];
            if (e >= 0 && e < E) counts[e] += 1;
        }
        const float* l = logits + (int64_t)t * E;
        double tot = 0.0;
        if (score_fn == ORACLE_SIGMOID) {
            for (int e = 0; e < E; ++e) s[e] = 1.0 / (1.0 + exp(-(double)l[e]));
        } else if (score_fn == ORACLE_SQRTSOFTPLUS) {
            for (int e = 0; e < E; ++e) s[e] = sqrtsoftplus64((double)l[e]);
        } else {
            double m = -INFINITY;
            for (int e = 0; e < E; ++e) if ((double)l[e] > m) m = (double)l[e];
            for (int e = 0; e < E; ++e) s[e] = exp((double)l[e] - m);
        }
        for (int e = 0; e < E; ++e) tot += s[e];
        for (int e = 0; e < E; ++e) mean_prob[e] += s[e] / tot;
    }
    free(s);
    double a = 0.0;
    if (n > 0) {
        for (int e = 0; e < E; ++e) {
            mean_prob[e] /= (double)n;
            a += ((double)counts[e] / (double)n) * mean_prob[e];
        }
        a *= (double)E;
    }
    *aux = a;
}

/* ------------------------------------------------------------------ order-invariant combine */
/*
 * An order-invariant weighted combine ("From Expert Reduction to Behavioral Divergence",
 * arXiv 2607.28097, Abstract: scheme C keeps routes and texts because its result does not
 * depend on the order of the expert terms). Reading: the terms are the products
 * p_j = w_j * float(y_j) formed exactly in double (24 x 8 significant bits) and, when
 * given, the shared expert's float(y_shared); they are added in double in a canonical
 * order -- ascending magnitude, a negative term before the positive one of the same
 * magnitude -- so the sum is a function of the multiset of terms only; out =
 * bf16_rne(fp32_rne(sum)). Terms with dest_row < 0 are skipped; masked tokens give 0;
 * no term gives +0.
 */
static int canon_less(double a, double b)
{
    double fa = fabs(a), fb = fabs(b);
    if (fa != fb) return fa < fb;
    return a < b; /* -x before +x */
}

void oracle_combine_invariant(int T, int K, int H, const uint16_t* y, const float* w,
                              const int32_t* dest_row, const uint16_t* y_shared,
                              const uint8_t* mask, uint16_t* out)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        uint16_t* o = out + (int64_t)t * H;
        if (mask && !mask[t]) { for (int h = 0; h < H; ++h) o[h] = 0; continue; }
        double term[33];
        for (int h = 0; h < H; ++h) {
            int n = 0;
            for (int j = 0; j < K; ++j) {
                int32_t r = dest_row[(int64_t)t * K + j];
                if (r < 0) continue;
                term[n++] = (double)w[(int64_t)t * K + j] *
                            (double)oracle_bf16_to_f32(y[(int64_t)r * H + h]);
            }
            if (y_shared) term[n++] = (double)oracle_bf16_to_f32(y_shared[(int64_t)t * H + h]);
            for (int i = 1; i < n; ++i) { /* insertion sort into the canonical order */
                double v = term[i];
                int k = i - 1;
                while (k >= 0 && canon_less(v, term[k])) { term[k + 1] = term[k]; --k; }
                term[k + 1] = v;
            }
            double s = 0.0;
            for (int i = 0; i < n; ++i) s += term[i];
            o[h] = oracle_f32_to_bf16((float)s);
        }
    }
}

/* ------------------------------------------------------------------ backward: FP32 contract */
/*
 * The backward of the layer (forward + backward is the contract's scope in "DSV4 Flash MoE
 * Train-Inference Consistency Roadmap", "Why DSV4 Flash MoE Drifts More Easily" and the
 * DSV4-WS1-2 row of "Follow-Up Issue Buckets"; the pages fix no backward arithmetic). The
 * reductions whose order decides bits are specified here and reproduced exactly:
 *
 * dot32(a, b), a and b bf16 rows of H: lane L (0..31) owns the 8-element chunks c = L, L+32,
 * ... (elements 8c .. 8c+7) in increasing order and adds each rounded product
 * fp32(a_h * b_h) to its fp32 sum (from +0); then butterfly levels 16, 8, 4, 2, 1.
 */
float oracle_dot32(int H, const uint16_t* a, const uint16_t* b)
{
    float lane[32], nxt[32];
    for (int l = 0; l < 32; ++l) lane[l] = 0.0f;
    for (int h = 0; h < H; ++h) {
        const int L = (h >> 3) & 31;
        const float p = oracle_bf16_to_f32(a[h]) * oracle_bf16_to_f32(b[h]);
        lane[L] = lane[L] + p;
    }
    for (int off = 16; off >= 1; off >>= 1) {
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ off];
        memcpy(lane, nxt, sizeof lane);
    }
    return lane[0];
}

/*
 * Combine backward: for each kept token t and rank j with a row r = dest_row[t,j] >= 0,
 * dw[t,j] = dot32(dout_t, y_r) and dy_r = bf16_rne(fp32(w[t,j] * dout_t)); dw = 0 where there
 * is no row; dy_shared_t = dout_t for kept tokens and +0 for masked ones (their output is 0
 * whatever x is).
 */
void oracle_combine_bwd_fp32(int T, int K, int H, const uint16_t* dout, const uint16_t* y,
                             const float* w, const int32_t* dest_row, const uint8_t* mask,
                             float* dw, uint16_t* dy, uint16_t* dy_shared)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const uint16_t* g = dout + (int64_t)t * H;
        const int kept = !(mask && !mask[t]);
        for (int j = 0; j < K; ++j) {
            const int64_t a = (int64_t)t * K + j;
            const int32_t r = dest_row[a];
            if (!kept || r < 0) { dw[a] = 0.0f; continue; }
            dw[a] = oracle_dot32(H, g, y + (int64_t)r * H);
            for (int h = 0; h < H; ++h)
                dy[(int64_t)r * H + h] = oracle_f32_to_bf16(w[a] * oracle_bf16_to_f32(g[h]));
        }
        if (dy_shared)
            for (int h = 0; h < H; ++h) dy_shared[(int64_t)t * H + h] = kept ? g[h] : 0;
    }
}

/*
 * Router backward, fp32 contract (one token; every operation rounded to nearest):
 *   s = the contract scores of the logits (recomputed exactly as in routing);
 *   renorm:    D = rank-order sum of s_{id_j}; q = rank-order sum of fp32(dw_j * s_{id_j});
 *              ds_{id_j} = ((route_scale * (dw_j - q / D)) / D); all 0 when D == 0;
 *   no renorm: ds_{id_j} = route_scale * dw_j;  ds = 0 for experts not selected;
 *   softmax:      r = rank-order sum of fp32(ds_{id_j} * s_{id_j}); dl_e = s_e * (ds_e - r);
 *   sigmoid:      dl_e = ds_e * (s_e * (1 - s_e));
 *   sqrtsoftplus: dl_e = ds_e * (sig_e / (2 * s_e)) with sig_e = 1 / (1 + exp_rl(-l_e)),
 *                 and 0 where ds_e == 0 or s_e == 0;
 *   masked tokens: dl = 0. Selection (and so the selection bias) has no gradient.
 */
void oracle_router_bwd_fp32(int T, int E, int K, const float* logits, const int32_t* ids,
                            const float* dw, const uint8_t* mask, int score_fn, int renorm,
                            float route_scale, float* dlogits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        float* dl = dlogits + (int64_t)t * E;
        if (mask && !mask[t]) { for (int e = 0; e < E; ++e) dl[e] = 0.0f; continue; }
        const float* l = logits + (int64_t)t * E;
        float* s = (float*)malloc(sizeof(float) * (size_t)E);
        float* ds = (float*)calloc((size_t)E, sizeof(float));
        oracle_scores_fp32(E, l, score_fn, s);
        const int32_t* id = ids + (int64_t)t * K;
        const float* g = dw + (int64_t)t * K;
        if (renorm) {
            float D = 0.0f, q = 0.0f;
            for (int j = 0; j < K; ++j) {
                if (id[j] < 0 || id[j] >= E) continue;
                D = D + s[id[j]];
                q = q + g[j] * s[id[j]];
            }
            if (D != 0.0f) {
                const float qd = q / D;
                for (int j = 0; j < K; ++j)
                    if (id[j] >= 0 && id[j] < E) ds[id[j]] = (route_scale * (g[j] - qd)) / D;
            }
        } else {
            for (int j = 0; j < K; ++j)
                if (id[j] >= 0 && id[j] < E) ds[id[j]] = route_scale * g[j];
        }
        if (score_fn == ORACLE_SOFTMAX) {
            float r = 0.0f;
            for (int j = 0; j < K; ++j)
                if (id[j] >= 0 && id[j] < E) r = r + ds[id[j]] * s[id[j]];
            for (int e = 0; e < E; ++e) dl[e] = s[e] * (ds[e] - r);
        } else if (score_fn == ORACLE_SIGMOID) {
            for (int e = 0; e < E; ++e) dl[e] = ds[e] * (s[e] * (1.0f - s[e]));
        } else {
            for (int e = 0; e < E; ++e) {
                if (ds[e] == 0.0f || s[e] == 0.0f) { dl[e] = 0.0f; continue; }
                const float sig = 1.0f / (1.0f + oracle_exp_rl(-l[e]));
                dl[e] = ds[e] * (sig / (2.0f * s[e]));
            }
        }
        free(s);
        free(ds);
    }
}

/*
 * Un-permute sum of the input gradient: dx_t = bf16_rne(acc), acc from +0 adding, in order,
 * float(dx_rows[dest_row[t,j]]) for j = 0..K-1 (rows >= 0), then float(dx_shared_t), then
 * float(dx_router_t) (each when given). Masked tokens: dx_t = +0.
 */
void oracle_unpermute_fp32(int T, int K, int H, const uint16_t* dx_rows,
                           const int32_t* dest_row, const uint16_t* dx_shared,
                           const uint16_t* dx_router, const uint8_t* mask, uint16_t* dx)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        uint16_t* o = dx + (int64_t)t * H;
        if (mask && !mask[t]) { for (int h = 0; h < H; ++h) o[h] = 0; continue; }
        for (int h = 0; h < H; ++h) {
            float acc = 0.0f;
            for (int j = 0; j < K; ++j) {
                const int32_t r = dest_row[(int64_t)t * K + j];
                if (r >= 0) acc = acc + oracle_bf16_to_f32(dx_rows[(int64_t)r * H + h]);
            }
            if (dx_shared) acc = acc + oracle_bf16_to_f32(dx_shared[(int64_t)t * H + h]);
            if (dx_router) acc = acc + oracle_bf16_to_f32(dx_router[(int64_t)t * H + h]);
            o[h] = oracle_f32_to_bf16(acc);
        }
    }
}

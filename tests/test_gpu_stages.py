"""Level-1 parity of the integer and FP32-contract stages: the CUDA route, dispatch and
combine kernels against the oracle, bit for bit, on the same inputs."""
import numpy as np
import pytest
import torch

import oracle
from deterministic_invariant_routing_b200 import moe, synthetic
from deterministic_invariant_routing_b200 import _native as N
from helpers import DEV, bits

pytestmark = pytest.mark.gpu

SM, SG, SP = moe.SOFTMAX, moe.SIGMOID, moe.SQRTSOFTPLUS


def adversarial_logits(T, E, seed, std=3.0):
    """Random logits with injected exact ties (at every rank), all-equal rows, signed
    zeros, -inf, a NaN row, a row of only -inf and a wide dynamic range (exp_rl's full
    input domain)."""
    l = synthetic.random_logits(T, E, seed, std=std).numpy()
    rng = np.random.default_rng(seed)
    for t in range(0, min(T, 40)):
        i, j = rng.choice(E, 2, replace=False) if E > 1 else (0, 0)
        l[t, j] = l[t, i]
    if T > 45:
        l[41] = 0.5
        l[42, :] = -0.0
        l[42, ::2] = 0.0
        l[43, : max(1, E // 2)] = -np.inf
        l[44] = rng.uniform(-80, 80, E)
        l[45, rng.integers(0, E)] = np.nan
    if T > 46:
        l[46] = -np.inf                   # no defined softmax: NaN scores, fails closed
    return np.ascontiguousarray(l.astype(np.float32))


ROUTE_CASES = [
    # E, K, score_fn, renorm, route_scale, with_bias, T
    (8, 2, SM, 1, 1.0, False, 64),
    (8, 1, SM, 0, 1.0, True, 1000),
    (128, 8, SM, 1, 1.0, False, 3001),
    (256, 6, SG, 1, 2.5, True, 2048),
    (1024, 16, SM, 1, 1.0, True, 517),
    (33, 3, SG, 0, 1.0, False, 700),
    (1, 1, SM, 1, 1.0, False, 50),
    (100, 7, SM, 1, 0.5, True, 999),
    (256, 8, SP, 1, 2.5, True, 2048),   # sqrtsoftplus scores
    (64, 4, SP, 0, 1.0, False, 700),
    (1024, 16, SP, 1, 1.0, True, 300),
]


GROUPED_CASES = [
    # E, K, score_fn, with_bias, n_group, topk_group, T
    (256, 8, SG, True, 8, 4, 4096),     # DeepSeek-V3-like
    (64, 6, SM, False, 8, 3, 2000),
    (1024, 16, SM, True, 32, 4, 517),
    (96, 4, SG, False, 3, 1, 999),
    (32, 2, SM, True, 32, 2, 300),      # one expert per group
    (160, 6, SG, True, 20, 20, 700),    # every group kept: plain top-K
    (256, 8, SP, True, 8, 4, 2048),     # sqrtsoftplus, group-limited
]


@pytest.mark.parametrize("E,K,score_fn,with_bias,n_group,topk_group,T", GROUPED_CASES)
def test_route_group_limited_bit_exact(E, K, score_fn, with_bias, n_group, topk_group, T):
    seed = 300 + E + n_group
    l = adversarial_logits(T, E, seed)
    gs = E // n_group
    rng = np.random.default_rng(seed)
    for t in range(50, min(T, 90)):       # two groups with exactly tied scores
        g0, g1 = rng.choice(n_group, 2, replace=False)
        l[t, g1 * gs:(g1 + 1) * gs] = l[t, g0 * gs:(g0 + 1) * gs]
    bias = synthetic.uniform_f32(E, 0.05, seed, "sel_bias").numpy() if with_bias else None
    if bias is not None:                  # keep the copied groups' choices tied
        bias = np.tile(bias[:gs], n_group).astype(np.float32)
    mask = synthetic.random_mask(T, 0.9, seed).numpy()
    cfg = moe.Config(T=T, H=128, E=E, K=K, I=128, score_fn=score_fn, renorm=True,
                     n_group=n_group, topk_group=topk_group)
    st = moe.new_status(DEV)
    _, ids, w = moe.route(cfg, logits=torch.from_numpy(l).to(DEV),
                          sel_bias=None if bias is None else torch.from_numpy(bias).to(DEV),
                          token_mask=torch.from_numpy(mask).to(DEV), status=st, check=False)
    torch.cuda.synchronize()
    r_ids, r_w, r_st = oracle.route_fp32(l, K, score_fn, True, 1.0, sel_bias=bias, mask=mask,
                                         n_group=n_group, topk_group=topk_group)
    g_ids = ids.cpu().numpy()
    assert np.array_equal(g_ids, r_ids), np.argwhere(g_ids != r_ids)[:5]
    g_w = w.cpu().numpy()
    nan = np.isnan(r_w)
    assert np.array_equal(np.isnan(g_w), nan)
    assert np.array_equal(g_w[~nan].view(np.uint32), r_w[~nan].view(np.uint32))
    s = st.cpu().numpy()
    assert s[N.MOE_ST_NAN_TOKENS] == r_st[0] and s[N.MOE_ST_ZERO_DENOM] == r_st[1]
    live = g_ids[:, 0] >= 0
    assert all(len(set(row // gs)) <= topk_group for row in g_ids[live])


@pytest.mark.parametrize("E,K,score_fn,renorm,scale,with_bias,T", ROUTE_CASES)
def test_route_bit_exact(E, K, score_fn, renorm, scale, with_bias, T):
    seed = 100 + E + K
    l = adversarial_logits(T, E, seed)
    bias = synthetic.uniform_f32(E, 0.05, seed, "sel_bias").numpy() if with_bias else None
    mask = synthetic.random_mask(T, 0.9, seed).numpy()
    cfg = moe.Config(T=T, H=128, E=E, K=K, I=128, score_fn=score_fn, renorm=bool(renorm),
                     route_scale=scale)
    st = moe.new_status(DEV)
    _, ids, w = moe.route(cfg, logits=torch.from_numpy(l).to(DEV),
                          sel_bias=None if bias is None else torch.from_numpy(bias).to(DEV),
                          token_mask=torch.from_numpy(mask).to(DEV), status=st, check=False)
    torch.cuda.synchronize()
    r_ids, r_w, r_st = oracle.route_fp32(l, K, score_fn, renorm, scale, sel_bias=bias, mask=mask)
    g_ids = ids.cpu().numpy()
    g_w = w.cpu().numpy()
    assert np.array_equal(g_ids, r_ids), np.argwhere(g_ids != r_ids)[:5]
    nan = np.isnan(r_w)
    assert np.array_equal(np.isnan(g_w), nan)
    assert np.array_equal(g_w[~nan].view(np.uint32), r_w[~nan].view(np.uint32))
    s = st.cpu().numpy()
    assert s[N.MOE_ST_NAN_TOKENS] == r_st[0] and s[N.MOE_ST_ZERO_DENOM] == r_st[1]


def test_route_golden_two_token(golden):
    g = golden("two_token_route_combine.json")
    l = np.array(g["logits"], np.float32)
    cfg = moe.Config(T=2, H=128, E=g["E"], K=g["K"], I=128, renorm=True)
    _, ids, w = moe.route(cfg, logits=torch.from_numpy(l).to(DEV),
                          sel_bias=torch.tensor(g["sel_bias"], dtype=torch.float32, device=DEV))
    assert ids.cpu().tolist() == g["expect_ids"]
    assert w.cpu().tolist() == g["expect_w"]
    offsets, perm_token, dest_row, _ = moe.permute(cfg, ids)
    assert offsets.cpu().tolist() == g["expect_offsets"]
    assert dest_row.cpu().tolist() == g["expect_dest_row"]
    assert perm_token.cpu().tolist()[:4] == g["expect_perm_token"]
    # combine on 128 columns: the fixture's 4 columns, zeros after them
    y = torch.zeros(4, 128, dtype=torch.bfloat16)
    y[:, :4] = torch.tensor(g["y"])
    ys = torch.zeros(2, 128, dtype=torch.bfloat16)
    ys[:, :4] = torch.tensor(g["y_shared"])
    out = moe.combine(cfg, y.to(DEV), w, dest_row, y_shared=ys.to(DEV))
    ob = bits(out)
    assert [[f"{v:04x}" for v in row[:4]] for row in ob] == g["expect_out_bf16_hex"]
    assert np.all(ob[:, 4:] == 0)


@pytest.mark.parametrize("T,K,E", [(1, 1, 8), (64, 2, 8), (3001, 8, 128), (8192, 1, 8),
                                   (2048, 6, 256), (777, 16, 1024), (20000, 8, 128),
                                   (40000, 8, 256), (5000, 16, 1024), (32768, 8, 128),
                                   (16385, 16, 64)])
def test_permute_bit_exact(T, K, E):
    """Counting sort, bit-exact against the oracle: skewed loads, empty experts, padding and a
    bad id, from one assignment to 320000 (157 blocks of 2048), E up to 1024."""
    rng = np.random.default_rng(T + K + E)
    # skewed expert choice (uneven loads, some experts empty), masked tokens, bad ids
    p = rng.dirichlet(np.full(E, 0.3))
    ids = np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    ids[rng.random(T) < 0.1] = -1
    n_bad = 0
    if T > 10:
        ids[5, 0] = E + 3
        n_bad = 1
    H = 256
    x = synthetic.normal_bf16(T, H, 1.0, 7, "x")
    cfg = moe.Config(T=T, H=H, E=E, K=K, I=128)
    st = moe.new_status(DEV)
    offsets, perm_token, dest_row, x_perm = moe.permute(
        cfg, torch.from_numpy(ids).to(DEV), x=x.to(DEV), status=st, check=False)
    r_off, r_perm, r_dest, r_bad = oracle.permute(ids, E)
    assert np.array_equal(offsets.cpu().numpy(), r_off)
    n = int(r_off[-1])
    assert np.array_equal(perm_token.cpu().numpy()[:n], r_perm[:n])
    assert np.array_equal(dest_row.cpu().numpy(), r_dest)
    assert np.array_equal(bits(x_perm[:n]), bits(x)[r_perm[:n]])
    assert st.cpu().numpy()[N.MOE_ST_BAD_EXPERT_ID] == r_bad == n_bad


@pytest.mark.parametrize("T,K,H,shared,masked", [(1, 1, 128, False, False),
                                                  (64, 2, 128, False, True),
                                                  (1000, 8, 2048, False, True),
                                                  (333, 6, 4096, True, True),
                                                  (4096, 1, 4096, False, False),
                                                  (100, 16, 256, True, False),
                                                  (700, 16, 512, True, True),
                                                  (2000, 3, 1024, True, False),
                                                  (300, 4, 2176, False, True)])
def test_combine_bit_exact(T, K, H, shared, masked):
    """Rank-order combine, bit-exact against the oracle: every K width, a shared expert,
    masks, skipped terms and hidden sizes that are and are not multiples of 256."""
    rng = np.random.default_rng(T * 7 + K)
    rows = T * K
    y = synthetic.normal_bf16(rows, H, 1.5, T + K, "x")
    ys = synthetic.normal_bf16(T, H, 1.0, T + K, "fill") if shared else None
    w = rng.uniform(0, 1, (T, K)).astype(np.float32)
    dest = rng.permutation(rows).astype(np.int32).reshape(T, K)
    mask = (rng.random(T) > 0.2).astype(np.uint8) if masked else None
    if masked:
        dest[mask == 0] = -1
    if T > 3 and K > 1:
        dest[3, K - 1] = -1  # a skipped term inside a live token
    cfg = moe.Config(T=T, H=H, E=max(K, 8), K=K, I=128)
    out = moe.combine(cfg, y.to(DEV), torch.from_numpy(w).to(DEV), torch.from_numpy(dest).to(DEV),
                      y_shared=None if ys is None else ys.to(DEV),
                      token_mask=None if mask is None else torch.from_numpy(mask).to(DEV))
    ref = oracle.combine_fp32(y, w, dest, ys, mask)
    assert np.array_equal(bits(out), ref)


def test_combine_special_values_bit_exact():
    """The combine's single bf16 downcast on values that exercise its rounding: infinities
    (and inf - inf = NaN), sums that overflow only after rounding, fp32 subnormal results,
    bf16 rounding ties (fp32 low halves of exactly 0x8000, odd and even) and signed zeros.
    Finite and infinite outputs must match the oracle bit for bit, NaN outputs be NaN."""
    T, K, H = 257, 8, 256
    rng = np.random.default_rng(91)
    rows = T * K
    yb = synthetic.normal_bf16(rows, H, 1.0, 91, "x").view(torch.int16).numpy().view(np.uint16).copy()
    w = rng.uniform(0, 1, (T, K)).astype(np.float32)
    dest = rng.permutation(rows).astype(np.int32).reshape(T, K)
    bf = lambda v: np.array([v], np.float32).view(np.uint32)[0] >> 16
    # token rows of y by rank: plant specials in the first columns of a few tokens
    for t in range(0, T, 5):
        r = dest[t]
        yb[r[0], 0] = bf(np.inf)
        yb[r[1], 1] = bf(-np.inf)
        yb[r[0], 2] = bf(np.inf)
        yb[r[1], 2] = bf(-np.inf)                       # inf - inf: NaN
        yb[r[:], 3] = 0x7f7f                            # largest bf16: the sum overflows
        w[t, :] = np.maximum(w[t, :], 0.5)
        yb[r[:], 4] = 0x0001                            # bf16 subnormals: fp32 subnormal sums
        yb[r[:], 5] = 0x8000                            # -0
        yb[r[2], 6] = 0x3f81                            # 1 + 2^-7: products near bf16 ties
    for t in range(1, T, 7):                            # exact bf16 ties: 1 + 2^-8 (even
        w[t, :] = 0.0                                   # down) and 1 + 2^-7 + 2^-8 (odd up)
        w[t, 0] = np.float32(1.0 + 2.0 ** -8) if t % 2 else np.float32(1.0 + 2.0 ** -7 + 2.0 ** -8)
        yb[dest[t][0], 7] = 0x3f80
    cfg = moe.Config(T=T, H=H, E=8, K=K, I=128)
    y = torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16)
    out = moe.combine(cfg, y.to(DEV), torch.from_numpy(w).to(DEV), torch.from_numpy(dest).to(DEV))
    ref = oracle.combine_fp32(y, w, dest)
    g = bits(out)
    nan_ref = ((ref & 0x7f80) == 0x7f80) & ((ref & 0x7f) != 0)
    nan_g = ((g & 0x7f80) == 0x7f80) & ((g & 0x7f) != 0)
    assert np.array_equal(nan_g, nan_ref)
    assert nan_ref.any()
    assert np.array_equal(g[~nan_ref], ref[~nan_ref])
    assert ((ref[~nan_ref] & 0x7fff) == 0x7f80).any()        # infinities among them
    assert ((ref[~nan_ref] & 0x7f80) == 0).any()             # and subnormals or zeros
    assert set(ref[1::7, 7].tolist()) == {0x3f80, 0x3f82}    # both ties, rounded to even


def test_combine_cancellation_order(golden):
    c = golden("tree_sum_and_combine_order.json")["combine_case"]
    K, H = c["K"], 128
    y = torch.zeros(K, H, dtype=torch.bfloat16)
    y[:, 0] = torch.tensor([r[0] for r in c["y"]])
    w = torch.tensor(c["w"], dtype=torch.float32)
    d = torch.tensor(c["dest_row"], dtype=torch.int32)
    cfg = moe.Config(T=1, H=H, E=8, K=K, I=128)
    out = moe.combine(cfg, y.to(DEV), w.to(DEV), d.to(DEV))
    assert out.float().cpu()[0, 0].item() == c["expect_acc"][0][0]


@pytest.mark.parametrize("name,T,n_near", [("tiny", 64, 4), ("dsv_sigmoid", 8192, 410),
                                           ("qwen3_30b_a3b", 4096, 205)])
def test_route_injected_near_ties_bit_exact(name, T, n_near):
    """Tied and 1-ulp-apart choices at the K-th/(K+1)-th boundary (the tiny layer's 4 tied
    token pairs; 5% of the DeepSeek-style layer's tokens). Experts 2m and 2m+1 share a
    selection bias, so copying expert a's logit to its partner a^1 ties their choices
    exactly, and the next float below it puts them within an ulp."""
    s = synthetic.shape(name, T=T)
    E, K = s.E, s.K
    l = synthetic.random_logits(T, E, seed=s.seed + 50, std=2.0).numpy().astype(np.float32)
    bias = None
    if s.sel_bias_range is not None:
        bias = synthetic.uniform_f32(E, s.sel_bias_range, s.seed, "sel_bias").numpy()
        bias[1::2] = bias[0::2]
    ids0, _, _ = oracle.route_fp32(l, K, s.score_fn, s.renorm, s.route_scale, sel_bias=bias)
    rng = np.random.default_rng(s.seed)
    for i, t in enumerate(rng.choice(T, n_near, replace=False)):
        a = int(ids0[t, K - 1])
        b = a ^ 1
        if b >= E:
            continue
        l[t, b] = l[t, a] if i % 2 == 0 else np.nextafter(l[t, a], np.float32(-np.inf))
    cfg = moe.Config.of(s)
    _, ids, w = moe.route(cfg, logits=torch.from_numpy(l).to(DEV),
                          sel_bias=None if bias is None else torch.from_numpy(bias).to(DEV))
    r_ids, r_w, _ = oracle.route_fp32(l, K, s.score_fn, s.renorm, s.route_scale, sel_bias=bias)
    assert np.array_equal(ids.cpu().numpy(), r_ids)
    assert np.array_equal(w.cpu().numpy().view(np.uint32), r_w.view(np.uint32))
    from helpers import near_tie_count
    n = near_tie_count(l, s, bias)
    print(f"\n{name}: {n} of {T} tokens with K-th/(K+1)-th choices within 1 ulp")
    assert n >= n_near // 2


def _ulps_below(v, n):
    """The float32 n representable steps below v (towards -inf), for finite v."""
    u = int(np.array([v], np.float32).view(np.uint32)[0])
    if u & 0x80000000:
        u = min(u + n, 0xff7fffff)
    elif u >= n:
        u -= n
    else:
        u = 0x80000000 | (n - u)
    return np.array([u], np.uint32).view(np.float32)[0]


@pytest.mark.parametrize("name,T", [("qwen3_30b_a3b", 4096), ("dsv_sigmoid", 4096),
                                    ("dspark", 2048)])
def test_route_close_choices_every_rank_bit_exact(name, T):
    """Pairs of choices a few ulps apart at every rank and at the K-th/(K+1)-th boundary:
    for each token one expert's logit is set 2^k ulps below the logit of the expert picked
    at rank r (k = 0 .. 12, r = 0 .. K), so their choices land in the same or in
    neighbouring buckets of any fixed number of leading bits. The selection must still
    match the oracle's exact order."""
    s = synthetic.shape(name, T=T)
    E, K = s.E, s.K
    l = synthetic.random_logits(T, E, seed=s.seed + 70, std=2.0).numpy().astype(np.float32)
    bias = None
    if s.sel_bias_range is not None:
        bias = synthetic.uniform_f32(E, s.sel_bias_range, s.seed, "sel_bias").numpy()
        bias[1::2] = bias[0::2]
    ids0, _, _ = oracle.route_fp32(l, min(K + 1, E), s.score_fn, s.renorm, s.route_scale,
                                   sel_bias=bias)
    for t in range(T):
        r = t % min(K + 1, E)
        a = int(ids0[t, r])
        b = a ^ 1
        if b >= E:
            continue
        k = (t // (K + 1)) % 13
        l[t, b] = _ulps_below(l[t, a], 1 << k)
    cfg = moe.Config.of(s)
    _, ids, w = moe.route(cfg, logits=torch.from_numpy(l).to(DEV),
                          sel_bias=None if bias is None else torch.from_numpy(bias).to(DEV))
    r_ids, r_w, _ = oracle.route_fp32(l, K, s.score_fn, s.renorm, s.route_scale, sel_bias=bias)
    assert np.array_equal(ids.cpu().numpy(), r_ids), np.argwhere(ids.cpu().numpy() != r_ids)[:5]
    assert np.array_equal(w.cpu().numpy().view(np.uint32), r_w.view(np.uint32))


@pytest.mark.parametrize("name,T,keep", [("qwen3_30b_a3b", 4096, None), ("qwen3_30b_a3b", 3001, 0.8),
                                         ("dsv_sigmoid", 2048, 0.9), ("tiny", 64, None),
                                         ("dspark", 1000, 0.5), ("dsv_sqrtsoftplus", 2048, 0.9)])
def test_router_stats_against_oracle(name, T, keep):
    """tokens_per_expert exact, mean_prob and the load-balance value within fp32 summation
    error of the FP64 oracle; the same call twice gives the same bits."""
    if name == "dsv_sqrtsoftplus":
        s = synthetic.shape("dsv_sigmoid", T=T, score_fn=synthetic.SQRTSOFTPLUS)
    else:
        s = synthetic.shape(name, T=T)
    l = synthetic.random_logits(T, s.E, seed=T + s.E, std=1.5)
    mask = None if keep is None else synthetic.random_mask(T, keep, 21)
    cfg = moe.Config.of(s)
    _, ids, _ = moe.route(cfg, logits=l.to(DEV), token_mask=None if mask is None else mask.to(DEV))
    offsets, _, _, _ = moe.permute(cfg, ids)
    st1 = moe.router_stats(cfg, l.to(DEV), offsets, None if mask is None else mask.to(DEV))
    st2 = moe.router_stats(cfg, l.to(DEV), offsets, None if mask is None else mask.to(DEV))
    r_counts, r_mp, r_aux = oracle.router_stats(l.numpy(), ids.cpu().numpy(), s.score_fn,
                                                mask=None if mask is None else mask.numpy())
    assert np.array_equal(st1["tokens_per_expert"].cpu().numpy(), r_counts)
    assert np.allclose(st1["mean_prob"].cpu().numpy(), r_mp, rtol=2e-4, atol=1e-7)
    assert abs(float(st1["aux"]) - r_aux) <= 2e-4 * abs(r_aux)
    for k in st1:
        assert np.array_equal(bits(st1[k]), bits(st2[k]))


@pytest.mark.parametrize("T,K,H,shared,masked", [(64, 2, 128, False, True), (1000, 8, 2048, False, True),
                                                  (333, 6, 4096, True, True), (100, 16, 256, True, False),
                                                  (500, 1, 512, False, False)])
@pytest.mark.parametrize("spread", [0.0, 2.0, 12.0])
def test_combine_invariant_bit_exact_and_order_free(T, K, H, shared, masked, spread):
    """The order-invariant combine matches the oracle bit for bit, and permuting each
    token's (weight, row) pairs does not change a bit (the rank-order combine does).
    `spread`: rows scaled by 10^U(-spread, spread) -- 0 keeps nearly every element's terms
    within 16 binary orders (the summed-as-they-come route), 12 sends most elements through
    the sorted route."""
    rng = np.random.default_rng(T * 11 + K)
    rows = T * K
    y = (synthetic.normal_bf16(rows, H, 1.0, T + K, "x").float()
         * torch.from_numpy(10.0 ** rng.uniform(-spread, spread, (rows, 1))).float()
         ).to(torch.bfloat16)
    ys = synthetic.normal_bf16(T, H, 1.0, T + K, "fill") if shared else None
    w = rng.uniform(0, 1, (T, K)).astype(np.float32)
    dest = rng.permutation(rows).astype(np.int32).reshape(T, K)
    mask = (rng.random(T) > 0.2).astype(np.uint8) if masked else None
    if masked:
        dest[mask == 0] = -1
    cfg = moe.Config(T=T, H=H, E=max(K, 8), K=K, I=128)
    dev = lambda a: None if a is None else (a if torch.is_tensor(a) else torch.from_numpy(a)).to(DEV)
    out = moe.combine(cfg, dev(y), dev(w), dev(dest), y_shared=dev(ys), token_mask=dev(mask),
                      order_invariant=True)
    ref = oracle.combine_invariant(y, w, dest, ys, mask)
    assert np.array_equal(bits(out), ref)
    perm = np.argsort(rng.random((T, K)), axis=1)
    w2 = np.take_along_axis(w, perm, 1)
    d2 = np.take_along_axis(dest, perm, 1)
    out2 = moe.combine(cfg, dev(y), dev(w2), dev(d2), y_shared=dev(ys), token_mask=dev(mask),
                       order_invariant=True)
    assert np.array_equal(bits(out2), bits(out))


def _special_bf16(rng, shape):
    """bf16 bits: normals of every exponent, with zeros of both signs, subnormals, infinities
    and NaN mixed in."""
    n = int(np.prod(shape))
    sign = rng.integers(0, 2, n).astype(np.uint16) << 15
    expo = rng.integers(100, 150, n).astype(np.uint16)
    kind = rng.random(n)
    expo[kind < 0.06] = rng.integers(1, 12, int((kind < 0.06).sum()))       # tiny normals
    expo[(kind >= 0.06) & (kind < 0.12)] = rng.integers(200, 255, int(((kind >= 0.06) & (kind < 0.12)).sum()))
    mant = rng.integers(0, 128, n).astype(np.uint16)
    b = sign | (expo << 7) | mant
    b[(kind >= 0.12) & (kind < 0.17)] = sign[(kind >= 0.12) & (kind < 0.17)]            # +-0
    sub = (kind >= 0.17) & (kind < 0.22)
    b[sub] = sign[sub] | rng.integers(1, 128, int(sub.sum())).astype(np.uint16)          # subnormal
    b[(kind >= 0.22) & (kind < 0.225)] = 0x7f80
    b[(kind >= 0.225) & (kind < 0.23)] = 0xff80
    b[(kind >= 0.23) & (kind < 0.235)] = 0x7fc0
    return b.reshape(shape)


@pytest.mark.parametrize("T,K,H,shared", [(300, 8, 256, True), (200, 6, 512, False), (64, 16, 128, True)])
def test_combine_invariant_special_values(T, K, H, shared):
    """The order-invariant combine on terms of every kind -- zeros of both signs, bf16
    subnormals, normals from the bottom to the top of the exponent range, infinities, NaN,
    and weights that are zero, subnormal, negative, huge or infinite -- matches the oracle
    bit for bit wherever the oracle's result is a number (NaN wherever it is NaN), and
    permuting each token's terms changes no bit."""
    rng = np.random.default_rng(T + 7 * K)
    rows = T * K
    y = _special_bf16(rng, (rows, H))
    ys = _special_bf16(rng, (T, H)) if shared else None
    w = rng.uniform(0, 1, (T, K)).astype(np.float32)
    kind = rng.random((T, K))
    w[kind < 0.1] = 0.0
    w[(kind >= 0.1) & (kind < 0.15)] = np.float32(3e-40)
    w[(kind >= 0.15) & (kind < 0.2)] *= -1.0
    w[(kind >= 0.2) & (kind < 0.22)] = np.float32(1e30)
    w[(kind >= 0.22) & (kind < 0.225)] = np.inf
    dest = rng.permutation(rows).astype(np.int32).reshape(T, K)
    dest[rng.random((T, K)) < 0.05] = -1
    cfg = moe.Config(T=T, H=H, E=max(K, 8), K=K, I=128)
    dev = lambda a: None if a is None else torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(DEV)
    bf = lambda a: None if a is None else dev(a).view(torch.bfloat16)
    out = moe.combine(cfg, bf(y), dev(w), dev(dest), y_shared=bf(ys), order_invariant=True)
    ref = oracle.combine_invariant(y, w, dest, ys, None)
    got = bits(out)
    nan_ref = (ref & 0x7fff) > 0x7f80
    nan_got = (got & 0x7fff) > 0x7f80
    assert np.array_equal(nan_got, nan_ref)
    assert np.array_equal(got[~nan_ref], ref[~nan_ref])
    perm = np.argsort(rng.random((T, K)), axis=1)
    out2 = moe.combine(cfg, bf(y), dev(np.take_along_axis(w, perm, 1)),
                       dev(np.take_along_axis(dest, perm, 1)), y_shared=bf(ys),
                       order_invariant=True)
    assert np.array_equal(bits(out2), got)

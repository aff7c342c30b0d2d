"""CPU pins of the oracle: each check compares the oracle with something other than itself
(closed forms, brute force, libm/numpy in float64, torch's bf16 rounding, hand-worked
values), chosen so that a dropped term, a wrong sign or index or a transposed operand in
the oracle fails at least one of them."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from deterministic_invariant_routing_b200 import synthetic

F32 = np.float32


def ulp_f32(x):
    x = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(x, np.finfo(np.float32).tiny)))
    return np.exp2(e - 23)


# ------------------------------------------------------------------ bf16 rounding

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(F32) * F32(1e3),
        (rng.integers(0, 2**32, 200000, dtype=np.uint64).astype(np.uint32)).view(F32),
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0 + 2**-8, 1.0 + 3 * 2**-8,
                  3.3895314e38, -3.3895314e38], F32),
    ])
    x = x[~np.isnan(x)]
    ours = oracle.f32_to_bf16(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    nan = oracle.f32_to_bf16(np.array([np.nan, -np.nan], F32))
    assert np.all(np.isnan(oracle.bf16_to_f32(nan)))


# ------------------------------------------------------------------ exp_rl

def test_exp_rl_exact_at_zero_and_specials():
    v = oracle.exp_rl(np.array([0.0, -0.0, np.nan, -87.0001, -1e30, -np.inf, 88.0001,
                                1e30, np.inf], F32))
    assert v[0] == 1.0 and v[1] == 1.0
    assert np.isnan(v[2])
    assert np.all(v[3:6] == 0.0) and not np.any(np.signbit(v[3:6]))
    assert np.all(np.isinf(v[6:9])) and np.all(v[6:9] > 0)


def test_exp_rl_within_2ulp_of_libm():
    rng = np.random.default_rng(1)
    grid = np.linspace(-87.0, 88.0, 1 << 21, dtype=np.float64).astype(F32)
    near0 = (rng.standard_normal(1 << 18) * 1e-3).astype(F32)
    xs = np.concatenate([grid, near0, rng.uniform(-87, 88, 1 << 18).astype(F32)])
    got = oracle.exp_rl(xs).astype(np.float64)
    ref = np.exp(xs.astype(np.float64))
    err_ulp = np.abs(got - ref) / ulp_f32(ref)
    assert err_ulp.max() <= 2.0, err_ulp.max()
    # monotone on the sorted grid (a wrong range-reduction constant breaks this at the
    # seams between n and n+1)
    g = oracle.exp_rl(grid)
    assert np.all(np.diff(g.astype(np.float64)) >= 0)


# ------------------------------------------------------------------ tree sum

def test_tree_sum_golden(golden):
    for case in golden("tree_sum_and_combine_order.json")["tree_cases"]:
        v = np.zeros(case["n"], F32)
        vals = case["values"]
        if "rest" in vals:
            v[:] = F32(vals["rest"])
        for k, x in vals.items():
            if k != "rest":
                v[int(k)] = F32(x)
        assert oracle.tree_sum32(v) == F32(case["expect"]), case["why"]


def test_tree_sum_exact_integers_and_lanes():
    rng = np.random.default_rng(2)
    for n in (1, 5, 31, 32, 33, 64, 100, 128, 256, 1000):
        v = rng.integers(-1000, 1000, n).astype(F32)
        assert oracle.tree_sum32(v) == F32(v.astype(np.int64).sum())
    # every element reaches the sum (none is dropped or counted twice)
    for n in (8, 128, 256):
        for i in range(n):
            v = np.zeros(n, F32)
            v[i] = 1.0
            assert oracle.tree_sum32(v) == 1.0


# ------------------------------------------------------------------ scores

def softmax64(l):
    l = np.asarray(l, np.float64)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


@pytest.mark.parametrize("E", [8, 128, 256])
def test_softmax_scores_close_to_float64(E):
    rng = np.random.default_rng(E)
    for _ in range(50):
        l = (rng.standard_normal(E) * 3).astype(F32)
        s = oracle.scores_fp32(l, oracle.SOFTMAX).astype(np.float64)
        ref = softmax64(l)
        # error budget of the fp32 contract: rounding of d = l - m (|d| * 2^-24 relative
        # in exp(d)), exp_rl <= 2 ulp, the tree sum (E/32 + 5 rounded adds), one division
        d = np.abs(l.astype(np.float64) - l.max())
        rel = d * 2.0**-24 + 2 * 2.0**-23 + (E / 32 + 5) * 2.0**-24 + 2.0**-24
        assert np.all(np.abs(s - ref) <= rel * ref + 1e-45)
        assert abs(s.sum() - 1.0) <= E * 2.0**-23


@pytest.mark.parametrize("E", [8, 16, 128, 256])
def test_softmax_all_equal_closed_form(E):
    for c in (0.0, -3.5, 17.25):
        s = oracle.scores_fp32(np.full(E, c, F32), oracle.SOFTMAX)
        assert np.all(s == F32(1.0 / E))


def test_sigmoid_scores():
    s = oracle.scores_fp32(np.array([0.0, -0.0], F32), oracle.SIGMOID)
    assert np.all(s == 0.5)
    rng = np.random.default_rng(3)
    l = (rng.standard_normal(10000) * 4).astype(F32)
    s = oracle.scores_fp32(l, oracle.SIGMOID).astype(np.float64)
    ref = 1.0 / (1.0 + np.exp(-l.astype(np.float64)))
    assert np.all(np.abs(s - ref) <= 4 * ulp_f32(ref))
    # symmetry s(l) + s(-l) ~= 1
    s2 = oracle.scores_fp32(-l, oracle.SIGMOID).astype(np.float64)
    assert np.all(np.abs(s + s2 - 1.0) <= 2.0**-22)


# ------------------------------------------------------------------ selection

def py_key(c, idx):
    c = float(c)
    return (0, 0.0, -idx) if math.isnan(c) else (1, c, -idx)


def test_select_key_order_matches_python_sort():
    rng = np.random.default_rng(4)
    vals = np.concatenate([rng.standard_normal(200).astype(F32),
                           np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 1e-40, -1e-40], F32)])
    items = [(F32(v), int(i)) for i, v in enumerate(vals)]
    ours = sorted(items, key=lambda it: oracle.select_key(it[0], it[1]), reverse=True)
    ref = sorted(items, key=lambda it: py_key(it[0], it[1]), reverse=True)
    assert [i for _, i in ours] == [i for _, i in ref]


def brute_force_topk(choice, K):
    """Lexicographic max over every ordered K-tuple of distinct experts of the
    per-rank keys (choice, -id); NaN ranks below everything."""
    E = len(choice)
    best, best_key = None, None
    for tup in itertools.permutations(range(E), K):
        key = tuple(py_key(choice[e], e) for e in tup)
        if best_key is None or key > best_key:
            best, best_key = tup, key
    return list(best)


@pytest.mark.parametrize("score_fn", [oracle.SOFTMAX, oracle.SIGMOID, oracle.SQRTSOFTPLUS])
def test_route_ids_brute_force(score_fn):
    rng = np.random.default_rng(5 + score_fn)
    cases = []
    for E in (2, 3, 5, 8, 10):
        for K in (1, 2, 3):
            if K > E:
                continue
            for _ in range(12):
                l = (rng.standard_normal(E) * 2).astype(F32)
                mode = rng.integers(0, 5)
                if mode == 1:
                    l[:] = F32(0.7)                       # all equal
                elif mode == 2:
                    i, j = rng.choice(E, 2, replace=False)
                    l[j] = l[i]                           # one exact tie
                elif mode == 3:
                    l[rng.integers(0, E)] = -0.0          # signed zeros
                    l[rng.integers(0, E)] = 0.0
                elif mode == 4 and score_fn != oracle.SOFTMAX:
                    l[rng.integers(0, E)] = np.nan        # a NaN logit
                bias = None
                if rng.integers(0, 2):
                    bias = rng.uniform(-0.05, 0.05, E).astype(F32)
                    if mode == 2:
                        bias[j] = bias[i]
                cases.append((E, K, l, bias))
    for E, K, l, bias in cases:
        ids, w, st = oracle.route_fp32(l[None], K, score_fn, True, 1.0, sel_bias=bias)
        s = oracle.scores_fp32(l, score_fn)
        choice = s if bias is None else (s + bias).astype(F32)
        assert list(ids[0]) == brute_force_topk(choice, K), (l, bias)
        assert st[0] == int(np.any(np.isnan(choice)))


def test_route_all_equal_logits_gives_lowest_ids_and_uniform_weights():
    for E, K in ((8, 2), (128, 8), (256, 6)):
        ids, w, _ = oracle.route_fp32(np.zeros((3, E), F32), K, oracle.SOFTMAX, True)
        assert np.all(ids == np.arange(K)) and np.all(w == F32(1.0 / K))
        ids, w, _ = oracle.route_fp32(np.zeros((1, E), F32), 1, oracle.SOFTMAX, True)
        assert np.all(w == 1.0)  # K=1 renormalised: s/s = 1 exactly


def test_route_weights_renorm_and_scale():
    rng = np.random.default_rng(6)
    for score_fn, scale, K, E in ((oracle.SOFTMAX, 1.0, 8, 128),
                                  (oracle.SIGMOID, 2.5, 6, 256),
                                  (oracle.SQRTSOFTPLUS, 2.5, 6, 256)):
        l = (rng.standard_normal((200, E)) * 2).astype(F32)
        bias = rng.uniform(-0.05, 0.05, E).astype(F32)
        ids, w, st = oracle.route_fp32(l, K, score_fn, True, scale, sel_bias=bias)
        tot = w.astype(np.float64).sum(1)
        assert np.all(np.abs(tot - scale) <= K * scale * 2.0**-23), np.abs(tot - scale).max()
        # weights are the unbiased float64 scores of the chosen ids, renormalised
        lf = l.astype(np.float64)
        ref_s = {oracle.SOFTMAX: lambda: softmax64(l),
                 oracle.SIGMOID: lambda: 1 / (1 + np.exp(-lf)),
                 oracle.SQRTSOFTPLUS: lambda: np.sqrt(np.logaddexp(0.0, lf))}[score_fn]()
        sel = np.take_along_axis(ref_s, ids.astype(np.int64), 1)
        ref_w = sel / sel.sum(1, keepdims=True) * scale
        assert np.allclose(w, ref_w, rtol=1e-6, atol=0)
        assert st.tolist() == [0, 0]


def test_route_no_renorm_weight_is_unbiased_score():
    rng = np.random.default_rng(7)
    E, K = 8, 1
    l = (rng.standard_normal((500, E))).astype(F32)
    bias = np.zeros(E, F32)
    bias[3] = 0.5  # large: expert 3 wins far more often, but its weight stays its prob
    ids, w, _ = oracle.route_fp32(l, K, oracle.SOFTMAX, False, 1.0, sel_bias=bias)
    p = softmax64(l)
    assert np.mean(ids[:, 0] == 3) > 0.5
    ref = p[np.arange(500), ids[:, 0]]
    assert np.all(np.abs(w[:, 0] - ref) <= 8 * ulp_f32(ref))
    for t in range(20):  # bit-equal to the contract score of that expert
        s = oracle.scores_fp32(l[t], oracle.SOFTMAX)
        assert w[t, 0] == s[ids[t, 0]]


def test_route_ranking_agrees_with_float64_away_from_ties():
    rng = np.random.default_rng(8)
    E, K = 128, 8
    l = (rng.standard_normal((400, E)) * 1.3).astype(F32)
    ids, _, _ = oracle.route_fp32(l, K, oracle.SOFTMAX, True)
    p = softmax64(l)
    order = np.argsort(-p, axis=1, kind="stable")[:, :K]
    srt = -np.sort(-p, axis=1)
    gaps = np.min(srt[:, :K] - srt[:, 1:K + 1], axis=1)
    clear = gaps > 1e-6 * srt[:, 0]
    assert clear.sum() > 300
    assert np.array_equal(ids[clear], order[clear])


def test_route_mask_and_zero_denominator():
    l = np.zeros((4, 8), F32)
    mask = np.array([1, 0, 1, 0], np.uint8)
    ids, w, st = oracle.route_fp32(l, 2, oracle.SOFTMAX, True, mask=mask)
    assert np.all(ids[1] == -1) and np.all(w[1] == 0) and np.all(ids[3] == -1)
    assert np.all(ids[0] == [0, 1])
    # sigmoid scores underflow to 0 for logits below -88: D == 0 -> weights 0, counted
    l = np.full((2, 8), -100.0, F32)
    ids, w, st = oracle.route_fp32(l, 2, oracle.SIGMOID, True)
    assert np.all(w == 0) and st[1] == 2 and np.all(ids == [0, 1])
    # a NaN logit under softmax makes every score NaN: counted, ids by the lowest id
    l = np.zeros((1, 8), F32)
    l[0, 5] = np.nan
    ids, w, st = oracle.route_fp32(l, 2, oracle.SOFTMAX, True)
    assert st[0] == 1 and list(ids[0]) == [0, 1] and np.all(np.isnan(w))


def test_route_all_minus_inf_row_fails_closed():
    """A row whose logits are all -inf has no softmax (max = -inf, every l - max is NaN):
    every score is NaN, the row is counted once as a NaN token and takes ids 0..K-1 by the
    tie rule with NaN weights. Sigmoid and sqrtsoftplus scores of -inf are exactly +0:
    ids 0..K-1, the renormalisation denominator is 0, weights 0, counted there instead."""
    l = np.full((3, 8), -np.inf, F32)
    l[1, 6] = 0.0                          # one finite logit: p = 1 on expert 6
    s = oracle.scores_fp32(l[0], oracle.SOFTMAX)
    assert np.all(np.isnan(s))
    ids, w, st = oracle.route_fp32(l, 3, oracle.SOFTMAX, True)
    assert list(st) == [2, 0]
    assert list(ids[0]) == [0, 1, 2] and np.all(np.isnan(w[0]))
    assert list(ids[1]) == [6, 0, 1] and list(w[1]) == [1.0, 0.0, 0.0]
    for fn in (oracle.SIGMOID, oracle.SQRTSOFTPLUS):
        assert np.all(oracle.scores_fp32(l[0], fn) == 0.0)
        ids, w, st = oracle.route_fp32(l[[0, 2]], 3, fn, True)
        assert list(st) == [0, 2] and np.all(ids == [0, 1, 2]) and np.all(w == 0.0)


# ------------------------------------------------------------------ permutation

def test_permute_properties():
    rng = np.random.default_rng(9)
    for T, K, E in ((1, 1, 4), (64, 2, 8), (300, 8, 128), (50, 6, 256)):
        ids = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
        ids[rng.random(T) < 0.2] = -1  # masked tokens
        offsets, perm_token, dest_row, bad = oracle.permute(ids, E)
        assert bad == 0
        valid = ids >= 0
        cnt = np.bincount(ids[valid], minlength=E)
        assert np.array_equal(np.diff(offsets), cnt) and offsets[0] == 0
        assert offsets[E] == valid.sum()
        assert np.all(dest_row[~valid] == -1)
        t_idx = np.repeat(np.arange(T), K).reshape(T, K)
        # unpermute o permute = identity on the token index
        assert np.array_equal(perm_token[dest_row[valid]], t_idx[valid])
        rows = dest_row[valid]
        assert np.array_equal(np.sort(rows), np.arange(offsets[E]))
        # rows of one expert are ordered by the flat assignment index a = t*K + j
        a_of_row = np.empty(offsets[E], np.int64)
        a_of_row[rows] = np.flatnonzero(valid.reshape(-1))
        for e in range(E):
            seg = a_of_row[offsets[e]:offsets[e + 1]]
            assert np.all(np.diff(seg) > 0)
            assert np.all(ids.reshape(-1)[seg] == e)
        # permuting rows of x then gathering back is the identity
        x = rng.integers(0, 2**16, (T, 16)).astype(np.uint16)
        x_perm = x[perm_token[:offsets[E]]]
        assert np.array_equal(x_perm[dest_row[valid]], np.repeat(x, K, 0).reshape(T, K, 16)[valid])


def test_permute_counts_invalid_ids():
    ids = np.array([[0, 9], [3, -1]], np.int32)
    offsets, perm_token, dest_row, bad = oracle.permute(ids, 8)
    assert bad == 1 and dest_row.tolist() == [[0, -1], [1, -1]]
    assert offsets.tolist() == [0, 1, 1, 1, 2, 2, 2, 2, 2]


# ------------------------------------------------------------------ combine

def test_combine_720_orders_at_most_360_classes():
    rng = np.random.default_rng(10)
    K, H = 6, 64
    live = 0
    for trial in range(4):
        w = rng.uniform(0.05, 0.4, (1, K)).astype(F32)
        y = oracle.f32_to_bf16(rng.standard_normal((K, H)).astype(F32) * 3)
        d = np.arange(K, dtype=np.int32)[None]
        res = {}
        for perm in itertools.permutations(range(K)):
            p = list(perm)
            acc = oracle.combine_acc_fp32(y[p], w[:, p], d)
            res[perm] = acc.tobytes()
        classes = set(res.values())
        assert len(classes) <= 360
        for perm, r in res.items():  # swapping the first two terms is exact
            sw = (perm[1], perm[0]) + perm[2:]
            assert res[sw] == r
        live += len(classes) > 1
    assert live == 4  # the order is observable on random data


def test_combine_golden_cancellation(golden):
    c = golden("tree_sum_and_combine_order.json")["combine_case"]
    w = np.array(c["w"], F32)
    y = oracle.f32_to_bf16(np.array(c["y"], F32))
    d = np.array(c["dest_row"], np.int32)
    acc = oracle.combine_acc_fp32(y, w, d)
    assert acc.tolist() == c["expect_acc"]
    acc2 = oracle.combine_acc_fp32(y[[0, 2, 1]], w, d)
    assert acc2.tolist() == c["expect_acc_order_021"]


def test_combine_matches_float64_within_rounding():
    rng = np.random.default_rng(11)
    T, K, H = 40, 8, 96
    w = rng.uniform(0, 0.3, (T, K)).astype(F32)
    y = oracle.f32_to_bf16(rng.standard_normal((T * K, H)).astype(F32))
    ys = oracle.f32_to_bf16(rng.standard_normal((T, H)).astype(F32))
    d = rng.permutation(T * K).astype(np.int32).reshape(T, K)
    mask = (rng.random(T) > 0.1).astype(np.uint8)
    out = oracle.bf16_to_f32(oracle.combine_fp32(y, w, d, ys, mask)).astype(np.float64)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    ref = np.einsum("tk,tkh->th", w.astype(np.float64), yf[d]) + oracle.bf16_to_f32(ys)
    ref[mask == 0] = 0
    assert np.all(out[mask == 0] == 0)
    tol = 2.0**-8 * np.abs(ref) + 1e-5 * (np.abs(w[..., None] * yf[d]).sum(1) + 1)
    assert np.all(np.abs(out - ref) <= tol)


# ------------------------------------------------------------------ FP64 math

def test_fp64_layer_matches_dense_numpy():
    s, d = synthetic.make_layer("tiny")
    x = oracle.bf16_to_f32(synthetic.bf16_bits(d["x"])).astype(np.float64)
    wr = oracle.bf16_to_f32(synthetic.bf16_bits(d["w_router"])).astype(np.float64)
    w13 = oracle.bf16_to_f32(synthetic.bf16_bits(d["w13"])).astype(np.float64)
    w2 = oracle.bf16_to_f32(synthetic.bf16_bits(d["w2"])).astype(np.float64)
    l64 = oracle.logits64(d["x"], d["w_router"])
    assert np.allclose(l64, x @ wr.T, rtol=1e-12, atol=1e-15)
    ids, _, _ = oracle.route_fp32(l64.astype(F32), s.K, s.score_fn, s.renorm)
    w64 = oracle.weights64(l64, ids, s.score_fn, s.renorm)
    p = softmax64(x @ wr.T)
    sel = np.take_along_axis(p, ids.astype(np.int64), 1)
    assert np.allclose(w64, sel / sel.sum(1, keepdims=True), rtol=1e-12)
    # dense evaluation: every expert on every token, then keep the routed ones
    I = s.I
    g = np.einsum("th,eih->tei", x, w13[:, :I])
    u = np.einsum("th,eih->tei", x, w13[:, I:])
    a = g / (1 + np.exp(-g)) * u
    y_all = np.einsum("tei,ehi->teh", a, w2)
    ref = np.einsum("tk,tkh->th", w64, np.take_along_axis(y_all, ids[..., None].astype(np.int64), 1))
    out = oracle.forward64(d["x"], ids, w64, d["w13"], d["w2"])
    assert np.allclose(out, ref, rtol=1e-10, atol=1e-14 * np.abs(ref).max())
    # single-expert entry point agrees with the dense evaluation too, h included
    y0, h0 = oracle.expert_ffn64(d["x"][5], d["w13"][3], d["w2"][3], return_h=True)
    assert np.allclose(y0, y_all[5, 3], rtol=1e-10, atol=1e-15)
    assert np.allclose(h0, a[5, 3], rtol=1e-10, atol=1e-15)


def test_fp64_shared_expert_and_sigmoid_weights():
    rng = np.random.default_rng(12)
    T, H, E, K, I, Is = 6, 64, 16, 3, 128, 256
    bf = lambda *sh: oracle.f32_to_bf16((rng.standard_normal(sh) * 0.05).astype(F32))
    x, wr = bf(T, H), bf(E, H)
    w13, w2, w13s, w2s = bf(E, 2 * I, H), bf(E, H, I), bf(2 * Is, H), bf(H, Is)
    f = lambda b: oracle.bf16_to_f32(b).astype(np.float64)
    l64 = oracle.logits64(x, wr)
    ids, _, _ = oracle.route_fp32(l64.astype(F32), K, oracle.SIGMOID, True, 2.5)
    w64 = oracle.weights64(l64, ids, oracle.SIGMOID, True, 2.5)
    sg = 1 / (1 + np.exp(-(f(x) @ f(wr).T)))
    sel = np.take_along_axis(sg, ids.astype(np.int64), 1)
    assert np.allclose(w64, sel / sel.sum(1, keepdims=True) * 2.5, rtol=1e-12)
    mask = np.array([1, 1, 0, 1, 1, 1], np.uint8)
    out = oracle.forward64(x, ids, w64, w13, w2, w13s, w2s, mask=mask)

    def ffn(xr, a13, a2, n):
        g, u = a13[:n] @ xr, a13[n:] @ xr
        return a2 @ (g / (1 + np.exp(-g)) * u)

    for t in range(T):
        ref = np.zeros(H)
        if mask[t]:
            for j in range(K):
                ref += w64[t, j] * ffn(f(x[t]), f(w13[ids[t, j]]), f(w2[ids[t, j]]), I)
            ref += ffn(f(x[t]), f(w13s), f(w2s), Is)
        assert np.allclose(out[t], ref, rtol=1e-10, atol=1e-14)
    sel_rows = np.array([4, 0], np.int32)
    out2 = oracle.forward64(x, ids, w64, w13, w2, w13s, w2s, mask=mask, sel=sel_rows)
    assert np.array_equal(out2, out[sel_rows])


def test_layer_forward_consistent_with_pieces():
    s, d = synthetic.make_layer("tiny")
    sel = np.array([0, 7, 63], np.int32)
    ids, out = oracle.layer_forward(s, d, sel)
    l64 = oracle.logits64(d["x"], d["w_router"])
    ids2, _, _ = oracle.route_fp32(l64.astype(F32), s.K, s.score_fn, s.renorm)
    assert np.array_equal(ids, ids2[sel])
    w64 = oracle.weights64(l64, ids2, s.score_fn, s.renorm)
    ref = oracle.forward64(d["x"], ids2, w64, d["w13"], d["w2"], sel=sel)
    assert np.allclose(out, ref, rtol=1e-14, atol=0)


# ------------------------------------------------------------------ router statistics

def test_router_stats_balanced_is_K():
    # every token routed to K distinct experts, expert loads and mean scores uniform
    E, K, T = 8, 2, 16
    l = np.zeros((T, E), F32)  # uniform scores: mean_prob = 1/E
    ids = np.array([[(2 * t) % E, (2 * t + 1) % E] for t in range(T)], np.int32)
    counts, mp, aux = oracle.router_stats(l, ids, oracle.SOFTMAX)
    assert counts.tolist() == [4] * E and np.allclose(mp, 1 / E)
    assert aux == pytest.approx(K, abs=1e-12)


def test_router_stats_hand_worked():
    # E=2, K=1, two kept tokens and one padding token. Token 0: sigmoid scores of logits
    # (0, 0) -> (1/2, 1/2), routed to 0; token 1: logits (+inf-ish 20, -20) -> p ~ (1, 0),
    # routed to 0. load = (1, 0); mean_prob_0 = (1/2 + p) / 2 ~ 3/4; aux = 2 * 1 * 3/4 = 1.5
    l = np.array([[0, 0], [20, -20], [5, 5]], F32)
    ids = np.array([[0], [0], [1]], np.int32)
    mask = np.array([1, 1, 0], np.uint8)
    counts, mp, aux = oracle.router_stats(l, ids, oracle.SIGMOID, mask=mask)
    p1 = (1 / (1 + np.exp(-20.0))) / (1 / (1 + np.exp(-20.0)) + 1 / (1 + np.exp(20.0)))
    assert counts.tolist() == [2, 0]
    assert mp[0] == pytest.approx((0.5 + p1) / 2, rel=1e-14)
    assert aux == pytest.approx(2 * 1.0 * (0.5 + p1) / 2, rel=1e-14)


def test_router_stats_matches_numpy():
    rng = np.random.default_rng(13)
    T, E, K = 300, 16, 3
    l = (rng.standard_normal((T, E)) * 2).astype(F32)
    ids, _, _ = oracle.route_fp32(l, K, oracle.SOFTMAX, True)
    mask = (rng.random(T) > 0.2).astype(np.uint8)
    counts, mp, aux = oracle.router_stats(l, ids, oracle.SOFTMAX, mask=mask)
    keep = mask == 1
    p = softmax64(l[keep])
    ref_counts = np.bincount(ids[keep].reshape(-1), minlength=E)
    assert np.array_equal(counts, ref_counts)
    assert np.allclose(mp, p.mean(0), rtol=1e-12)
    assert aux == pytest.approx(E * np.sum(ref_counts / keep.sum() * p.mean(0)), rel=1e-12)
    assert counts.sum() == K * keep.sum() and mp.sum() == pytest.approx(1.0)


# ------------------------------------------------------------------ order-invariant combine

def test_combine_invariant_all_720_orders_identical():
    rng = np.random.default_rng(14)
    K, H = 6, 64
    for trial in range(3):
        w = rng.uniform(0.05, 0.4, (1, K)).astype(F32)
        y = oracle.f32_to_bf16((rng.standard_normal((K, H)) * 10 ** rng.uniform(-3, 3, (K, 1)))
                               .astype(F32))
        d = np.arange(K, dtype=np.int32)[None]
        ref = oracle.combine_invariant(y, w, d)
        for perm in itertools.permutations(range(K)):
            p = list(perm)
            assert np.array_equal(oracle.combine_invariant(y[p], w[:, p], d), ref)
        # while the rank-order contract combine does depend on the order here
        outs = {oracle.combine_acc_fp32(y[list(pp)], w[:, list(pp)], d).tobytes()
                for pp in itertools.permutations(range(K))}
        assert len(outs) > 1


def test_combine_invariant_cancellation_and_accuracy(golden):
    c = golden("tree_sum_and_combine_order.json")["combine_case"]
    w = np.array(c["w"], F32)
    y = oracle.f32_to_bf16(np.array(c["y"], F32))
    d = np.array(c["dest_row"], np.int32)
    # terms 2^24, 1, -2^24: the canonical order adds 1 first, then -2^24 + 2^24 exactly
    out = oracle.bf16_to_f32(oracle.combine_invariant(y, w, d))
    assert out.tolist() == [[1.0]]
    # random rows: within one bf16 rounding (plus fp32) of the float64 sum
    rng = np.random.default_rng(15)
    T, K, H = 30, 8, 64
    w = rng.uniform(0, 0.3, (T, K)).astype(F32)
    y = oracle.f32_to_bf16(rng.standard_normal((T * K, H)).astype(F32))
    ys = oracle.f32_to_bf16(rng.standard_normal((T, H)).astype(F32))
    d = rng.permutation(T * K).astype(np.int32).reshape(T, K)
    got = oracle.bf16_to_f32(oracle.combine_invariant(y, w, d, ys)).astype(np.float64)
    yf = oracle.bf16_to_f32(y).astype(np.float64)
    ref = np.einsum("tk,tkh->th", w.astype(np.float64), yf[d]) + oracle.bf16_to_f32(ys)
    assert np.all(np.abs(got - ref) <= 2.0**-8 * np.abs(ref) + 1e-30)


# ------------------------------------------------------------------ group-limited selection

def brute_force_grouped(choice, K, n_group, topk_group):
    """Group scores = best + second-best choice of each group (by the selection key), the
    topk_group best groups kept (higher score, then lower group), then the brute-force
    top-K over the kept experts (excluded experts never chosen)."""
    E = len(choice)
    gs = E // n_group
    gkeys = []
    for g in range(n_group):
        members = sorted(range(g * gs, (g + 1) * gs), key=lambda e: py_key(choice[e], e),
                         reverse=True)
        sc = np.float32(choice[members[0]])
        if gs > 1:
            sc = np.float32(sc + np.float32(choice[members[1]]))
        gkeys.append((py_key(sc, g), g))
    kept = {g for _, g in sorted(gkeys, reverse=True)[:topk_group]}
    masked = [choice[e] if e // gs in kept else None for e in range(E)]
    best, best_key = None, None
    for tup in itertools.permutations([e for e in range(E) if masked[e] is not None], K):
        key = tuple(py_key(choice[e], e) for e in tup)
        if best_key is None or key > best_key:
            best, best_key = tup, key
    return list(best)


@pytest.mark.parametrize("E,K,n_group,topk_group", [(8, 2, 4, 2), (9, 3, 3, 1), (10, 3, 5, 3),
                                                    (8, 2, 8, 3), (6, 2, 2, 2)])
def test_grouped_route_brute_force(E, K, n_group, topk_group):
    rng = np.random.default_rng(E * 100 + K * 10 + n_group)
    for trial in range(25):
        l = (rng.standard_normal(E) * 2).astype(F32)
        if trial % 5 == 1:
            l[:] = F32(0.3)                      # all tied: lowest groups, lowest ids
        if trial % 5 == 2:
            i, j = rng.choice(E, 2, replace=False)
            l[j] = l[i]
        bias = rng.uniform(-0.05, 0.05, E).astype(F32) if trial % 2 else None
        score_fn = oracle.SIGMOID if trial % 3 == 0 else oracle.SOFTMAX
        ids, w, _ = oracle.route_fp32(l[None], K, score_fn, True, 1.0, sel_bias=bias,
                                      n_group=n_group, topk_group=topk_group)
        s = oracle.scores_fp32(l, score_fn)
        choice = s if bias is None else (s + bias).astype(F32)
        assert list(ids[0]) == brute_force_grouped(list(choice), K, n_group, topk_group)
    # n_group = 1 or topk_group = n_group leaves plain top-K
    l = (rng.standard_normal((20, E)) * 2).astype(F32)
    a = oracle.route_fp32(l, K, oracle.SOFTMAX, True)[0]
    assert np.array_equal(oracle.route_fp32(l, K, oracle.SOFTMAX, True, n_group=1)[0], a)
    assert np.array_equal(oracle.route_fp32(l, K, oracle.SOFTMAX, True, n_group=n_group,
                                            topk_group=n_group)[0], a)


# ------------------------------------------------------------------ sqrtsoftplus score

def test_ln_rl_within_2ulp_of_libm():
    rng = np.random.default_rng(21)
    v = np.concatenate([
        np.linspace(1.0, 4.0, 1 << 19, dtype=np.float64),
        np.exp(rng.uniform(0, np.log(4.9e8), 1 << 19)),
        2.0 ** np.arange(0, 29),                                   # k ln2 exactly
        np.nextafter(np.float32(np.sqrt(2)), [0, 3]).astype(np.float64),  # the halving seam
    ]).astype(F32)
    got = oracle.ln_rl(v).astype(np.float64)
    ref = np.log(v.astype(np.float64))
    err = np.abs(got - ref) / ulp_f32(np.maximum(ref, 1e-30))
    err[ref == 0] = np.abs(got[ref == 0])
    assert oracle.ln_rl(np.array([1.0], F32))[0] == 0.0
    assert err.max() <= 2.0, err.max()
    assert np.all(np.diff(oracle.ln_rl(np.sort(v)).astype(np.float64)) >= 0)


def test_log1p_rl_within_2ulp_of_libm_and_exact_for_tiny():
    rng = np.random.default_rng(22)
    u = np.concatenate([np.exp(rng.uniform(np.log(1e-12), np.log(4.85e8), 1 << 19)),
                        np.linspace(0, 2, 1 << 16)]).astype(F32)
    got = oracle.log1p_rl(u).astype(np.float64)
    ref = np.log1p(u.astype(np.float64))
    nz = ref > 0
    err = np.abs(got[nz] - ref[nz]) / ulp_f32(ref[nz])
    # Goldberg's bound: the log's error (<= 2 ulp, above) plus three roundings of half an
    # ulp (1 + u, the product, the quotient; v - 1 is exact)
    assert err.max() <= 3.5, err.max()
    tiny = np.array([0.0, 2.0 ** -30, 1e-9, 2.0 ** -25], F32)   # 1 + u rounds to 1
    assert np.array_equal(oracle.log1p_rl(tiny), tiny)


def test_sqrtsoftplus_within_3ulp_closed_forms_and_specials():
    rng = np.random.default_rng(23)
    x = np.concatenate([np.linspace(-87, 40, 1 << 20), rng.normal(0, 3, 1 << 17)]).astype(F32)
    got = oracle.sqrtsoftplus_rl(x).astype(np.float64)
    ref = np.sqrt(np.logaddexp(0.0, x.astype(np.float64)))
    err = np.abs(got - ref) / ulp_f32(ref)
    # softplus carries exp_rl's 2 ulp (scaled by u / ((1 + u) log1p u) <= 1) and log1p's
    # 3.5; the square root halves a relative error and rounds once: <= 3 ulp
    assert err.max() <= 3.0, err.max()
    # Goldberg's log1p is not monotone at the ulp level (1 + u and v - 1 step while u
    # moves): on sorted inputs a score may dip by an ulp or two, never more
    srt = oracle.sqrtsoftplus_rl(np.sort(x)).astype(np.float64)
    assert np.all(np.diff(srt) >= -2 * ulp_f32(srt[1:]))
    # the FP64 reference used by the level-2 weights agrees with numpy's form
    assert np.allclose(oracle.sqrtsoftplus64(x[:2000].astype(np.float64)), ref[:2000],
                       rtol=1e-15, atol=0)
    # above the threshold softplus is l itself: squares give exact roots
    big = np.array([25, 36, 400, 20.25, 1e30], F32)
    assert np.array_equal(oracle.sqrtsoftplus_rl(big), np.sqrt(big))
    s0 = oracle.sqrtsoftplus_rl(np.array([0.0, -0.0], F32)).astype(np.float64)
    assert np.all(np.abs(s0 - np.sqrt(np.log(2.0))) <= ulp_f32(np.sqrt(np.log(2.0))))
    sp = oracle.sqrtsoftplus_rl(np.array([-87.5, -1e30, -np.inf, np.inf, np.nan], F32))
    assert np.all(sp[:3] == 0.0) and sp[3] == np.inf and np.isnan(sp[4])
    assert np.array_equal(oracle.scores_fp32(x[:999], oracle.SQRTSOFTPLUS),
                          oracle.sqrtsoftplus_rl(x[:999]))


def test_router_stats_sqrtsoftplus_l1_normalised():
    rng = np.random.default_rng(24)
    T, E, K = 200, 12, 2
    l = (rng.standard_normal((T, E)) * 2).astype(F32)
    ids, _, _ = oracle.route_fp32(l, K, oracle.SQRTSOFTPLUS, True)
    counts, mp, aux = oracle.router_stats(l, ids, oracle.SQRTSOFTPLUS)
    s = np.sqrt(np.logaddexp(0.0, l.astype(np.float64)))
    p = s / s.sum(1, keepdims=True)
    assert np.allclose(mp, p.mean(0), rtol=1e-12) and mp.sum() == pytest.approx(1.0)
    assert aux == pytest.approx(E * np.sum(counts / T * p.mean(0)), rel=1e-12)

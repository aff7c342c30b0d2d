"""Pins of the oracle's backward (CPU): the FP64 gradients against central differences of
the FP64 forward, the numpy FP64 forward against the C oracle's, and the FP32-contract
pieces (dot32, the router backward, the combine backward, the un-permute sum) against
hand-worked values, exact sums and the FP64 gradients."""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward64 as B

F32 = np.float32


def tiny_problem(seed, score_fn, renorm, shared, masked, T=6, H=12, E=6, K=2, I=4, Is=3):
    rng = np.random.default_rng(seed)
    p = dict(x=rng.standard_normal((T, H)), wr=rng.standard_normal((E, H)) * 0.5,
             w13=rng.standard_normal((E, 2 * I, H)) * 0.4,
             w2=rng.standard_normal((E, H, I)) * 0.4,
             w13_s=rng.standard_normal((2 * Is, H)) * 0.4 if shared else None,
             w2_s=rng.standard_normal((H, Is)) * 0.4 if shared else None)
    lg = p["x"] @ p["wr"].T
    ids = np.argsort(-B.scores64(lg, score_fn), axis=1, kind="stable")[:, :K]
    mask = (rng.random(T) > 0.3).astype(np.uint8) if masked else None
    if masked:
        mask[0] = 1
    dout = rng.standard_normal((T, H))
    kw = dict(score_fn=score_fn, renorm=renorm, route_scale=1.7, mask=mask)
    return p, ids, dout, kw


def loss(p, ids, dout, kw, logits=None):
    out = B.layer_forward64(p["x"], p["wr"], p["w13"], p["w2"], ids, w13_s=p["w13_s"],
                            w2_s=p["w2_s"], logits=logits, **kw)
    return float((dout * out).sum())


@pytest.mark.parametrize("score_fn,renorm,shared,masked", [
    (B.SOFTMAX, True, False, False), (B.SIGMOID, True, True, True),
    (B.SQRTSOFTPLUS, True, False, True), (B.SOFTMAX, False, True, False),
    (B.SIGMOID, False, False, False)])
def test_backward64_matches_central_differences(score_fn, renorm, shared, masked):
    p, ids, dout, kw = tiny_problem(3 + score_fn, score_fn, renorm, shared, masked)
    g = B.layer_backward64(dout, p["x"], p["wr"], p["w13"], p["w2"], ids, w13_s=p["w13_s"],
                           w2_s=p["w2_s"], **kw)
    rng = np.random.default_rng(9)
    eps = 1e-6

    def fd(name, idx):
        a = p[name]
        old = a[idx]
        a[idx] = old + eps
        lp = loss(p, ids, dout, kw)
        a[idx] = old - eps
        lm = loss(p, ids, dout, kw)
        a[idx] = old
        return (lp - lm) / (2 * eps)

    def check(name, ana, n=12):
        a = p[name]
        for _ in range(n):
            idx = tuple(int(rng.integers(0, d)) for d in a.shape)
            num = fd(name, idx)
            assert abs(num - ana[idx]) <= 1e-6 * (1 + abs(num)), (name, idx, num, ana[idx])

    check("x", g["dx"])
    check("wr", g["dwr"])
    if shared:
        check("w13_s", g["dw13_s"])
        check("w2_s", g["dw2_s"])
    for e in list(g["dw13"])[:3]:
        dense13 = np.zeros_like(p["w13"])
        dense13[e] = g["dw13"][e]
        dense2 = np.zeros_like(p["w2"])
        dense2[e] = g["dw2"][e]
        for _ in range(6):
            i = (e, int(rng.integers(0, p["w13"].shape[1])), int(rng.integers(0, p["w13"].shape[2])))
            assert abs(fd("w13", i) - dense13[i]) <= 1e-6 * (1 + abs(dense13[i]))
            i = (e, int(rng.integers(0, p["w2"].shape[1])), int(rng.integers(0, p["w2"].shape[2])))
            assert abs(fd("w2", i) - dense2[i]) <= 1e-6 * (1 + abs(dense2[i]))
    # dlogits: differentiate the forward that takes the logits directly
    lg = p["x"] @ p["wr"].T
    for _ in range(8):
        t, e = int(rng.integers(0, lg.shape[0])), int(rng.integers(0, lg.shape[1]))
        lp, lm = lg.copy(), lg.copy()
        lp[t, e] += eps
        lm[t, e] -= eps
        num = (loss(p, ids, dout, kw, lp) - loss(p, ids, dout, kw, lm)) / (2 * eps)
        assert abs(num - g["dlogits"][t, e]) <= 1e-6 * (1 + abs(num))
    if masked:
        dead = kw["mask"] == 0
        assert np.all(g["dx"][dead] == 0) and np.all(g["dlogits"][dead] == 0)


def test_numpy_forward64_matches_c_forward64():
    from deterministic_invariant_routing_b200 import synthetic
    s, d = synthetic.make_layer("tiny", T=32)
    def bits(t):
        return t.view(torch.int16).numpy().view(np.uint16)

    x = bits(d["x"])
    lg = oracle.logits64(d["x"], d["w_router"])
    ids, _, _ = oracle.route_fp32(lg.astype(F32), s.K, s.score_fn, s.renorm)
    w64 = oracle.weights64(lg, ids, s.score_fn, s.renorm)
    ref = oracle.forward64(d["x"], ids, w64, d["w13"], d["w2"])
    got = B.layer_forward64(B.bf16_to_f64(x), B.bf16_to_f64(bits(d["w_router"])),
                            B.bf16_to_f64(bits(d["w13"])), B.bf16_to_f64(bits(d["w2"])), ids,
                            s.score_fn, s.renorm)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-15)


def bf(v):
    return oracle.f32_to_bf16(np.asarray(v, F32))


def test_dot32_lane_order_is_observable():
    # H = 16: elements 0..7 are lane 0's, 8..15 lane 1's. a = 1. With b0 = 2^24, b1 = 1 and
    # b8 = -2^24, lane 0 rounds 2^24 + 1 to 2^24 and the butterfly gives 0; with the 1 moved
    # to element 9 lane 1 holds -(2^24 - 1) exactly and the result is 1.
    a = bf(np.ones(16))
    b = np.zeros(16, F32)
    b[0], b[1], b[8] = 2.0 ** 24, 1.0, -(2.0 ** 24)
    assert oracle.dot32(a, bf(b)) == 0.0
    b[1], b[9] = 0.0, 1.0
    assert oracle.dot32(a, bf(b)) == 1.0


def test_dot32_exact_on_integers_and_within_bound():
    rng = np.random.default_rng(4)
    a = bf(rng.integers(-8, 9, 2048))
    b = bf(rng.integers(-8, 9, 2048))
    exact = (oracle.bf16_to_f32(a).astype(np.int64) * oracle.bf16_to_f32(b).astype(np.int64)).sum()
    assert oracle.dot32(a, b) == exact
    for H in (128, 2048, 4096):
        a = bf(rng.standard_normal(H))
        b = bf(rng.standard_normal(H))
        fa = oracle.bf16_to_f32(a).astype(np.float64)
        fb = oracle.bf16_to_f32(b).astype(np.float64)
        # products of bf16 are exact in fp32; H/32 + 5 sequential roundings per path
        bound = (H / 32 + 5) * 2.0 ** -24 * np.abs(fa * fb).sum()
        assert abs(float(oracle.dot32(a, b)) - (fa * fb).sum()) <= bound


def test_combine_bwd_hand_worked_and_fp64():
    T, K, H = 3, 2, 256
    rng = np.random.default_rng(5)
    dout = bf(rng.standard_normal((T, H)))
    y = bf(rng.standard_normal((T * K, H)))
    w = np.array([[0.5, 0.25], [0.75, 0.125], [1.0, 0.0]], F32)
    dest = np.array([[1, 0], [3, 2], [5, -1]], np.int32)
    mask = np.array([1, 1, 0], np.uint8)
    dw, dy, dys = oracle.combine_bwd_fp32(dout, y, w, dest, T * K, mask=mask, shared=True)
    # dy rows: w * dout is exact here (power-of-two weights, 0.75 = 3/4 of a bf16 value
    # may round once), compare with fp32 numpy products rounded to bf16
    g = oracle.bf16_to_f32(dout)
    assert np.array_equal(dy[1], bf(F32(0.5) * g[0]))
    assert np.array_equal(dy[0], bf(F32(0.25) * g[0]))
    assert np.array_equal(dy[3], bf(F32(0.75) * g[1]))
    assert dw[2].tolist() == [0.0, 0.0] and np.all(dys[2] == 0) and np.array_equal(dys[0], dout[0])
    for t, j in ((0, 0), (0, 1), (1, 0), (1, 1)):
        ref = (g[t].astype(np.float64) * oracle.bf16_to_f32(y[dest[t, j]]).astype(np.float64)).sum()
        assert abs(dw[t, j] - ref) <= 1e-5 * np.abs(g[t]).sum() * 4


@pytest.mark.parametrize("score_fn,renorm,scale", [(oracle.SOFTMAX, True, 1.0),
                                                   (oracle.SIGMOID, True, 2.5),
                                                   (oracle.SQRTSOFTPLUS, True, 2.5),
                                                   (oracle.SOFTMAX, False, 1.0),
                                                   (oracle.SIGMOID, False, 1.0)])
def test_router_bwd_fp32_close_to_fp64(score_fn, renorm, scale):
    rng = np.random.default_rng(6 + score_fn)
    T, E, K = 300, 64, 6
    l = (rng.standard_normal((T, E)) * 2).astype(F32)
    ids, _, _ = oracle.route_fp32(l, K, score_fn, renorm, scale)
    dw = rng.standard_normal((T, K)).astype(F32)
    mask = (rng.random(T) > 0.1).astype(np.uint8)
    got = oracle.router_bwd_fp32(l, ids, dw, score_fn, renorm, scale, mask=mask)
    ref = B.router_grad64(l.astype(np.float64), ids, dw.astype(np.float64), score_fn, renorm,
                          scale, mask)
    tol = 1e-5 * np.abs(ref).max(axis=1, keepdims=True) + 1e-30
    assert np.all(np.abs(got - ref) <= tol)
    assert np.all(got[mask == 0] == 0)
    if score_fn == oracle.SOFTMAX:   # a softmax gradient sums to zero over the experts
        assert np.all(np.abs(got.astype(np.float64).sum(1)) <= 1e-5 * np.abs(got).sum(1) + 1e-30)
    if score_fn != oracle.SOFTMAX:   # elementwise scores: unselected experts get nothing
        sel = np.zeros((T, E), bool)
        np.put_along_axis(sel, ids, True, axis=1)
        assert np.all(got[~sel] == 0)


def test_unpermute_hand_worked():
    T, K, H = 2, 2, 128
    rows = np.zeros((4, H), F32)
    rows[2] = 1.0
    rows[0] = 2.0 ** -8           # 1 + 2^-8 is exact in fp32; alone it would round to 1 in bf16
    rows[1] = 3.0
    rows[3] = -3.0
    dest = np.array([[2, 0], [1, 3]], np.int32)
    shared = np.full((T, H), 2.0 ** -8, F32)
    out = oracle.unpermute_fp32(bf(rows), dest, dx_shared=bf(shared))
    # token 0: 1 + 2^-8 + 2^-8 = 1 + 2^-7, exactly a bf16 value (one rounding at the end);
    # token 1: 3 - 3 + 2^-8
    assert np.all(oracle.bf16_to_f32(out[0]) == F32(1 + 2.0 ** -7))
    assert np.all(oracle.bf16_to_f32(out[1]) == F32(2.0 ** -8))
    out = oracle.unpermute_fp32(bf(rows), dest)
    assert np.all(oracle.bf16_to_f32(out[0]) == 1.0)   # the tie 1 + 2^-8 rounds to even
    out = oracle.unpermute_fp32(bf(rows), dest, mask=np.array([0, 1], np.uint8))
    assert np.all(out[0] == 0) and np.all(oracle.bf16_to_f32(out[1]) == 0.0)

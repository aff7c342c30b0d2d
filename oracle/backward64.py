"""FP64 forward and backward of the layer for given routes, in numpy (test infrastructure).

The backward pass is in the consistency contract's scope ("DSV4 Flash MoE Train-Inference
Consistency Roadmap", "Why DSV4 Flash MoE Drifts More Easily": forward + backward; the
DSV4-WS1-2 row of "Follow-Up Issue Buckets"). The pages give the forward only, so this is
the plain calculus of it, in double precision with no intermediate rounding:

    logits = x Wr^T (+ b);  s = score(logits);  w_j = route_scale * s_{id_j} / D  (renorm,
    D = sum_j s_{id_j}) or route_scale * s_{id_j};
    y_{t,j} = W2_e (silu(g) * u),  [g; u] = W13_e x_t,  e = id_{t,j};
    out_t = sum_j w_j y_{t,j} + y_shared(x_t)

with the routes (ids) held fixed: selection is discrete and has no gradient. Masked tokens
output 0 whatever x is, so every gradient through them is 0. The float64 arrays are the
exact values of the bf16 / fp32 inputs. Matrix products are numpy's (a library primitive
applied as the step the formula names). Pinned by central differences of layer_forward64
and by agreement with the C oracle's forward64.
"""
from __future__ import annotations

import numpy as np

SOFTMAX, SIGMOID, SQRTSOFTPLUS = 0, 1, 2


def bf16_to_f64(bits) -> np.ndarray:
    b = np.asarray(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def scores64(l: np.ndarray, score_fn: int) -> np.ndarray:
    l = np.asarray(l, np.float64)
    if score_fn == SIGMOID:
        return 1.0 / (1.0 + np.exp(-l))
    if score_fn == SQRTSOFTPLUS:
        return np.sqrt(np.logaddexp(0.0, l))
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


def _sigma(z):
    return 1.0 / (1.0 + np.exp(-z))


def _route_weights(s, ids, renorm, route_scale):
    """(w [T,K], D [T]) from scores s [T,E] and ids [T,K] (-1 = no route)."""
    valid = ids >= 0
    sel = np.where(valid, np.take_along_axis(s, np.maximum(ids, 0), axis=1), 0.0)
    D = sel.sum(axis=1)
    if renorm:
        with np.errstate(divide="ignore", invalid="ignore"):
            w = np.where(D[:, None] != 0, sel / D[:, None], 0.0) * route_scale
    else:
        w = sel * route_scale
    return w, D, sel


def _experts_forward(xr, w13_e, w2_e):
    """Rows xr [n,H] through one expert: (g, u, a, y)."""
    I = w13_e.shape[0] // 2
    gu = xr @ w13_e.T
    g, u = gu[:, :I], gu[:, I:]
    a = g * _sigma(g) * u
    return g, u, a, a @ w2_e.T


def layer_forward64(x, wr, w13, w2, ids, score_fn, renorm, route_scale=1.0, mask=None,
                    w13_s=None, w2_s=None, logits=None, logit_bias=None):
    """out [T,H] in double for the given routes. `logits` replaces x Wr^T (+ bias) when
    given (for differentiating with respect to the logits)."""
    x = np.asarray(x, np.float64)
    T, H = x.shape
    ids = np.asarray(ids, np.int64)
    kept = np.ones(T, bool) if mask is None else np.asarray(mask) != 0
    if logits is None:
        logits = x @ np.asarray(wr, np.float64).T
        if logit_bias is not None:
            logits = logits + np.asarray(logit_bias, np.float64)
    s = scores64(logits, score_fn)
    w, _, _ = _route_weights(s, ids, renorm, route_scale)
    out = np.zeros((T, H))
    for e in np.unique(ids[ids >= 0]):
        tt, jj = np.nonzero((ids == e) & kept[:, None])
        if tt.size == 0:
            continue
        _, _, _, y = _experts_forward(x[tt], np.asarray(w13[e], np.float64),
                                      np.asarray(w2[e], np.float64))
        np.add.at(out, tt, w[tt, jj][:, None] * y)
    if w13_s is not None:
        _, _, _, ys = _experts_forward(x, np.asarray(w13_s, np.float64),
                                       np.asarray(w2_s, np.float64))
        out = out + ys
    out[~kept] = 0.0
    return out


def router_grad64(logits, ids, dw, score_fn, renorm, route_scale=1.0, mask=None):
    """dlogits [T,E] from the routing weights' gradient dw [T,K]: through the
    renormalisation w_j = route_scale * s_j / D (or w_j = route_scale * s_j) and the score
    function; only selected experts carry a score gradient."""
    logits = np.asarray(logits, np.float64)
    ids = np.asarray(ids, np.int64)
    dw = np.asarray(dw, np.float64)
    T, K = ids.shape
    kept = np.ones(T, bool) if mask is None else np.asarray(mask) != 0
    s = scores64(logits, score_fn)
    _, D, sel = _route_weights(s, ids, renorm, route_scale)
    valid = ids >= 0
    ds = np.zeros_like(s)
    if renorm:
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (dw * sel).sum(axis=1)
            dsel = np.where(D[:, None] != 0,
                            route_scale * (dw - (q / D)[:, None]) / D[:, None], 0.0)
    else:
        dsel = route_scale * dw
    for j in range(K):
        t = np.nonzero(valid[:, j] & kept)[0]
        ds[t, ids[t, j]] += dsel[t, j]
    if score_fn == SOFTMAX:
        dl = s * (ds - (ds * s).sum(axis=1, keepdims=True))
    elif score_fn == SIGMOID:
        dl = ds * s * (1.0 - s)
    else:
        with np.errstate(divide="ignore", invalid="ignore"):
            dl = np.where((ds != 0) & (s != 0), ds * _sigma(logits) / (2.0 * s), 0.0)
    dl[~kept] = 0.0
    return dl


def layer_backward64(dout, x, wr, w13, w2, ids, score_fn, renorm, route_scale=1.0, mask=None,
                     w13_s=None, w2_s=None, logits=None, logit_bias=None, experts=None):
    """Gradients of sum(dout * out) for the given routes, in double:
    {dx [T,H], dwr [E,H], dw13 {e: [2I,H]}, dw2 {e: [H,I]}, dw13_s, dw2_s, dlogits [T,E],
    dw [T,K] (gradient of the routing weights)}. `experts` limits dw13/dw2 to some experts
    (the others' contributions to dx are still computed)."""
    x = np.asarray(x, np.float64)
    g_out = np.asarray(dout, np.float64)
    T, H = x.shape
    wr = np.asarray(wr, np.float64)
    ids = np.asarray(ids, np.int64)
    K = ids.shape[1]
    kept = np.ones(T, bool) if mask is None else np.asarray(mask) != 0
    g_out = np.where(kept[:, None], g_out, 0.0)
    if logits is None:
        logits = x @ wr.T
        if logit_bias is not None:
            logits = logits + np.asarray(logit_bias, np.float64)
    logits = np.asarray(logits, np.float64)
    s = scores64(logits, score_fn)
    w, _, _ = _route_weights(s, ids, renorm, route_scale)

    dx = np.zeros((T, H))
    dw = np.zeros((T, K))
    dw13, dw2 = {}, {}
    for e in np.unique(ids[ids >= 0]):
        tt, jj = np.nonzero((ids == e) & kept[:, None])
        if tt.size == 0:
            continue
        w13_e = np.asarray(w13[e], np.float64)
        w2_e = np.asarray(w2[e], np.float64)
        g, u, a, y = _experts_forward(x[tt], w13_e, w2_e)
        dw[tt, jj] = np.einsum("nh,nh->n", g_out[tt], y)
        dy = w[tt, jj][:, None] * g_out[tt]
        da = dy @ w2_e
        sg = _sigma(g)
        dg = da * u * sg * (1.0 + g * (1.0 - sg))
        du = da * g * sg
        dgu = np.concatenate([dg, du], axis=1)
        np.add.at(dx, tt, dgu @ w13_e)
        if experts is None or e in experts:
            dw2[int(e)] = dy.T @ a
            dw13[int(e)] = dgu.T @ x[tt]
    res = {"dw13": dw13, "dw2": dw2, "dw13_s": None, "dw2_s": None}
    if w13_s is not None:
        w13s = np.asarray(w13_s, np.float64)
        w2s = np.asarray(w2_s, np.float64)
        g, u, a, _ = _experts_forward(x, w13s, w2s)
        da = g_out @ w2s
        sg = _sigma(g)
        dgu = np.concatenate([da * u * sg * (1.0 + g * (1.0 - sg)), da * g * sg], axis=1)
        dx += dgu @ w13s
        res["dw2_s"] = g_out.T @ a
        res["dw13_s"] = dgu.T @ x

    dl = router_grad64(logits, ids, dw, score_fn, renorm, route_scale, mask)
    dx += dl @ wr
    dx[~kept] = 0.0
    res.update(dx=dx, dwr=dl.T @ x, dlogits=dl, dw=np.where(kept[:, None], dw, 0.0))
    return res

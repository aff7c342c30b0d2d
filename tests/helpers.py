"""Shared helpers of the GPU tests: building layers on the device, reference values from
the oracle for sampled tokens, and the error metrics of the parity levels."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from deterministic_invariant_routing_b200 import moe, synthetic

DEV = "cuda:0"

# Level-2 bar: per token row, max|gpu - ref| / max|ref| (bf16 output vs the FP64 layer)
LEVEL2_ROW_REL = 1e-2

# Lines the parity tests report (errors, near-tie counts); printed at the end of the run.
REPORT: list = []


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bits of a tensor as an unsigned numpy array (bf16 -> uint16, fp32 -> uint32)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.numpy()


def layer(name: str, T=None, device=DEV, **over):
    s, d = synthetic.make_layer(name, T=T, device=device, **over)
    return s, d, moe.Config.of(s)


def expert_subset(d, ids_rows: np.ndarray):
    """CPU copies of only the experts that the given routes use, and the routes remapped
    onto that subset (keeps oracle inputs small for layers with GBs of weights)."""
    used = np.unique(ids_rows[ids_rows >= 0])
    remap = np.full(int(d["w13"].shape[0]), -1, np.int32)
    remap[used] = np.arange(used.size, dtype=np.int32)
    sel = torch.from_numpy(used.astype(np.int64)).to(d["w13"].device)
    w13 = d["w13"].index_select(0, sel).cpu()
    w2 = d["w2"].index_select(0, sel).cpu()
    ids_sub = np.where(ids_rows >= 0, remap[np.maximum(ids_rows, 0)], -1).astype(np.int32)
    return w13, w2, ids_sub


def reference_rows(s, d, x_rows_cpu, logits64_rows, ids_rows, mask_rows=None):
    """FP64 layer output of some tokens for the given routes (the FP32-contract routes),
    with weights recomputed in FP64 from FP64 scores."""
    w64 = oracle.weights64(logits64_rows, ids_rows, s.score_fn, s.renorm, s.route_scale)
    w13, w2, ids_sub = expert_subset(d, ids_rows)
    w13s = d["w13_s"].cpu() if d.get("w13_s") is not None else None
    w2s = d["w2_s"].cpu() if d.get("w2_s") is not None else None
    return oracle.forward64(x_rows_cpu, ids_sub, w64, w13, w2, w13s, w2s, mask=mask_rows)


def row_rel_err(gpu_bf16: torch.Tensor, ref64: np.ndarray) -> np.ndarray:
    g = gpu_bf16.detach().float().cpu().numpy().astype(np.float64)
    den = np.maximum(np.abs(ref64).max(axis=1), 1e-30)
    return np.abs(g - ref64).max(axis=1) / den


def mean_abs_err(gpu_bf16: torch.Tensor, ref64: np.ndarray) -> float:
    g = gpu_bf16.detach().float().cpu().numpy().astype(np.float64)
    return float(np.abs(g - ref64).mean())


def near_tie_count(logits_f32: np.ndarray, s, sel_bias=None) -> int:
    """Tokens whose K-th and (K+1)-th selection choices are within 1 fp32 ulp (by the
    oracle's contract scores)."""
    if s.K >= s.E:
        return 0
    n = 0
    b = None if sel_bias is None else np.asarray(sel_bias, np.float32)
    for row in logits_f32:
        sc = oracle.scores_fp32(row, s.score_fn)
        c = sc if b is None else (sc + b).astype(np.float32)
        c = c[~np.isnan(c)]
        if c.size <= s.K:
            continue
        top = np.sort(c)[::-1]
        a, z = np.float32(top[s.K - 1]), np.float32(top[s.K])
        if a - z <= np.spacing(a):
            n += 1
    return n


# ------------------------------------------------------------------ backward bounds
#
# Element-wise error bounds of the weight gradients against the FP64 backward (given the
# same logits and routes). Every gradient element is a sum of products
# G[m, c] = sum_r A[r, m] * B[r, c] whose operands the GPU computes in fp32 and holds in
# bf16 (8 significant bits: a rounding is off by at most u = 2^-8 of the value), summed in
# fp32 (n terms: at most g(n) = n * 2^-24 of the sum of their magnitudes). The bound follows
# each operand's chain with first-order error propagation, in double:
#   g, u = x . Wg, x . Wu (fp32 over H)     e_g = g(H) |x|.|Wg|,  e_u = g(H) |x|.|Wu|
#   h = bf16(silu(g) u)                     e_h = u |h| + |u silu'(g)| e_g + |silu(g)| e_u
#   y = bf16(h . W2^T) (fp32 over I)        e_y = (u + g(I)) |h|.|W2|^T + e_h.|W2|^T
#   dw_j = dot32(dout, y)                   e_dw = |dout|.e_y + g(H) |dout|.|y|
#   dy = bf16(w dout)                       e_dy = (u + 2^-20) |w dout|
#   dh = dy . W2 (fp32 over H)              e_dh = (u + 2^-20 + g(H)) |dy|.|W2|   (= ... DH)
#   dg = bf16(dh u silu'(g)),               e_dg = (u + ...) DH |u silu'| + DH (|silu'| e_u +
#   du = bf16(dh silu(g))                          |u silu''| e_g), e_du likewise
#   dW13 = [dg | du]^T . x, dW2 = dy^T . h, dW_router = bf16(dlogits)^T . x (fp32 over the
#   rows, in fixed chunks for the router), dlogits carrying e_dw through the score and
#   renormalisation steps linearly.
# The test allows twice that bound (second-order terms). A bound of this worst-case kind is
# loose where an expert has many rows and the terms cancel, so a wrong element of typical
# size could hide below it; a second, statistical check uses root-sum-squares over the
# rows, whose rounding errors are independent: Q = sqrt(sum_r t_r^2) of typical term sizes
# t_r (each operand's value plus the root-sum-square of the product that made it), each
# rounding within 2^-7 of its typical size with a standard deviation below 2^-7 / sqrt(3),
# so the sum's standard deviation is below 0.0046 Q, and allowed 2^-3 Q (2^-2 Q for the
# router, three roundings deep); plus 8 root-sum-squares of the rows' typical gate/up
# errors (fp32 sums of H products, taken as 4 x 2^-24 sqrt(H) times their root-sum-square),
# which cancellation in g or u makes large relative to h. An element taken from the wrong
# row or column is off by about Q.
WGRAD_EXPERT_CQ = 2.0 ** -3
WGRAD_ROUTER_CQ = 2.0 ** -2
_U8 = 2.0 ** -8


def _g(n):
    return n * 2.0 ** -24


def _sigma64(z):
    return 1.0 / (1.0 + np.exp(-z))


def _silu_parts(g):
    """silu(g), silu'(g), silu''(g) in double."""
    s = _sigma64(g)
    d1 = s * (1.0 + g * (1.0 - s))
    d2 = s * (1.0 - s) * (2.0 + g * (1.0 - 2.0 * s))
    return g * s, d1, d2


def _rss(a, b):
    return np.sqrt((a * a).T @ (b * b))


def _expert_bounds(xr, dsgn_r, w_r, w13_e, w2_e, ad_r, shared):
    """(bound13, bound2, Q13, Q2, G13, G2, e_dw, Y, typical e_dw) for one expert's rows:
    error bounds, root-sum-squares of typical term sizes and of typical gate/up-induced
    term errors, and the routing-weight gradient's error bound, magnitude and typical
    gate/up-induced error per row."""
    H = xr.shape[1]
    I = w13_e.shape[0] // 2
    R = xr.shape[0]
    ax = np.abs(xr)
    aw13 = np.abs(w13_e)
    gu = xr @ w13_e.T
    g, u = gu[:, :I], gu[:, I:]
    mag = ax @ aw13.T
    e_g, e_u = _g(H) * mag[:, :I], _g(H) * mag[:, I:]
    rss = 4.0 * 2.0 ** -24 * np.sqrt(H) * np.sqrt((xr * xr) @ (w13_e * w13_e).T)
    t_g, t_u = rss[:, :I], rss[:, I:]
    sl, d1, d2 = _silu_parts(g)
    a = sl * u
    aa = np.abs(a)
    gu_a = np.abs(u * d1) * e_g + np.abs(sl) * e_u        # g/u part of e_h
    gu_a_t = np.abs(u * d1) * t_g + np.abs(sl) * t_u      # and its typical size
    aw2 = np.abs(w2_e)
    # rows of the forward's y: its magnitude and error (for the routing-weight gradient)
    Y = aa @ aw2.T
    e_y = (2 * _U8 + _g(I)) * Y + gu_a @ aw2.T
    e_dw = np.einsum("nh,nh->n", ad_r, e_y) + _g(H) * np.einsum("nh,nh->n", ad_r, Y)
    e_y_t = np.sqrt((gu_a_t * gu_a_t) @ (w2_e * w2_e).T)
    e_dw_t = np.sqrt(np.einsum("nh,nh->n", ad_r ** 2, e_y_t ** 2))
    # dy: exact for the shared expert (dy = dout), else one rounding of w dout
    dy = (1.0 if shared else np.abs(w_r)[:, None]) * ad_r
    r_dy = 0.0 if shared else _U8 + 2.0 ** -20
    DH = dy @ aw2
    f_g, f_u = np.abs(u * d1), np.abs(sl)
    DGU = np.concatenate([DH * f_g, DH * f_u], axis=1)
    gu_dgu = np.concatenate([DH * (np.abs(d1) * e_u + np.abs(u * d2) * e_g),
                             DH * np.abs(d1) * e_g], axis=1)
    e_dgu = (_U8 + r_dy + _g(H)) * DGU + gu_dgu
    b13 = e_dgu.T @ ax + _g(R) * (DGU.T @ ax)
    S2 = dy.T @ aa
    b2 = (r_dy + _U8 + _g(R)) * S2 + dy.T @ gu_a
    # typical sizes: the value plus the root-sum-square of the product that made it
    sgn_dy = (1.0 if shared else w_r[:, None]) * dsgn_r
    dht = np.abs(sgn_dy @ w2_e) + np.sqrt((dy * dy) @ (w2_e * w2_e))
    t = np.concatenate([dht * f_g, dht * f_u], axis=1)
    Q13 = _rss(t, ax)
    Q2 = _rss(dy, aa)
    tg = np.concatenate([dht * (np.abs(d1) * t_u + np.abs(u * d2) * t_g),
                         dht * np.abs(d1) * t_g], axis=1)
    G13 = _rss(tg, ax)
    G2 = _rss(dy, gu_a_t)
    return b13, b2, Q13, Q2, G13, G2, e_dw, Y, e_dw_t


def wgrad_bounds64(dout, x, logits, w13, w2, ids, score_fn, renorm, route_scale, mask=None,
                   w13_s=None, w2_s=None, experts=()):
    """Error bounds of the weight gradients (see above), in double, for the given logits
    and routes: {name: (bound, Q, Qg)} (Qg: root-sum-square of the typical gate/up-induced
    term errors) for "dw13[e]", "dw2[e]" (e in
    `experts`), "dw_router" and, with a shared expert, "dw13_s", "dw2_s". w13/w2 are
    indexable per expert (float64 arrays); the router's bound needs every routed row."""
    from oracle import backward64 as B
    x = np.asarray(x, np.float64)
    ids = np.asarray(ids, np.int64)
    T, H = x.shape
    K = ids.shape[1]
    kept = np.ones(T, bool) if mask is None else np.asarray(mask) != 0
    dsgn = np.where(kept[:, None], np.asarray(dout, np.float64), 0.0)
    ad = np.abs(dsgn)
    ax = np.abs(x)
    logits = np.asarray(logits, np.float64)
    s = B.scores64(logits, score_fn)
    valid = ids >= 0
    sel = np.where(valid, np.take_along_axis(s, np.maximum(ids, 0), axis=1), 0.0)
    D = sel.sum(axis=1)
    if renorm:
        with np.errstate(divide="ignore", invalid="ignore"):
            w = np.where(D[:, None] != 0, sel / D[:, None], 0.0) * route_scale
    else:
        w = sel * route_scale
    dwmag = np.zeros((T, K))     # |dout| . |y|: the routing-weight gradient's magnitude
    dwerr = np.zeros((T, K))     # its error bound
    dwtyp = np.zeros((T, K))     # its typical size
    res = {}
    for e in np.unique(ids[valid]):
        tt, jj = np.nonzero((ids == e) & kept[:, None])
        if tt.size == 0:
            continue
        w13_e, w2_e = np.asarray(w13[e], np.float64), np.asarray(w2[e], np.float64)
        b13, b2, Q13, Q2, G13, G2, e_dw, Y, e_dw_t = _expert_bounds(
            x[tt], dsgn[tt], w[tt, jj], w13_e, w2_e, ad[tt], False)
        dwmag[tt, jj] = np.einsum("nh,nh->n", ad[tt], Y)
        dwerr[tt, jj] = e_dw
        I = w13_e.shape[0] // 2
        gu = x[tt] @ w13_e.T
        a = _silu_parts(gu[:, :I])[0] * gu[:, I:]
        yv = a @ w2_e.T
        yt = np.abs(yv) + np.sqrt((a * a) @ (w2_e * w2_e).T)
        dwtyp[tt, jj] = (np.abs(np.einsum("nh,nh->n", dsgn[tt], yv))
                         + np.sqrt(np.einsum("nh,nh->n", ad[tt] ** 2, yt ** 2))
                         + 2.0 ** 7 * e_dw_t)
        if int(e) in experts:
            res[f"dw13[{int(e)}]"] = (b13, Q13, G13)
            res[f"dw2[{int(e)}]"] = (b2, Q2, G2)

    # router: magnitudes and errors through the renormalisation and the score function
    def dlogits_mag(dwm):
        if renorm:
            with np.errstate(divide="ignore", invalid="ignore"):
                q = (dwm * sel).sum(axis=1)
                dsel = np.where(D[:, None] != 0,
                                abs(route_scale) * (dwm + (q / np.abs(D))[:, None])
                                / np.abs(D)[:, None], 0.0)
        else:
            dsel = abs(route_scale) * dwm
        ds = np.zeros_like(s)
        for j in range(K):
            t = np.nonzero(valid[:, j] & kept)[0]
            ds[t, ids[t, j]] += dsel[t, j]
        if score_fn == B.SOFTMAX:
            dl = s * (ds + (ds * s).sum(axis=1, keepdims=True))
        elif score_fn == B.SIGMOID:
            dl = ds * s * (1.0 - s)
        else:
            with np.errstate(divide="ignore", invalid="ignore"):
                dl = np.where((ds != 0) & (s != 0), ds * _sigma64(logits) / (2.0 * s), 0.0)
        dl[~kept] = 0.0
        return dl

    DL = dlogits_mag(dwmag)
    e_dl = dlogits_mag(dwerr) + _U8 * DL
    dl_typ = dlogits_mag(dwtyp)
    res["dw_router"] = (e_dl.T @ ax + _g(T) * (DL.T @ ax), _rss(dl_typ, ax), 0.0)
    if w13_s is not None:
        b13, b2, Q13, Q2, G13, G2, _, _, _ = _expert_bounds(
            x, dsgn, None, np.asarray(w13_s, np.float64), np.asarray(w2_s, np.float64), ad, True)
        res["dw13_s"] = (b13, Q13, G13)
        res["dw2_s"] = (b2, Q2, G2)
    return res


def assert_within_bounds(gpu, ref, bounds, cq, what):
    """|gpu - ref| <= 2 * bound and <= cq * Q + 8 * Qg, element by element. Returns the
    largest fraction of either allowance used."""
    bound, Q, Qg = bounds
    g = np.asarray(gpu, np.float64)
    err = np.abs(g - ref)
    used = 0.0
    for lim, name in ((2.0 * bound + 1e-30, "twice the error bound"),
                      (cq * Q + 8.0 * Qg + 1e-30, f"{cq:.3g} x root-sum-square")):
        r = err / lim
        i = np.unravel_index(np.argmax(r), r.shape)
        if r[i] > 1.0:
            raise AssertionError(f"{what}: {int((r > 1).sum())} of {r.size} elements beyond "
                                 f"{name}; worst {i}: gpu {g[i]:.6g} ref {ref[i]:.6g}")
        used = max(used, float(r[i]))
    return used

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
# Element-wise bounds of the weight gradients. Every weight gradient is a sum of products
# G[m, c] = sum_r A[r, m] * B[r, c] whose operands the GPU holds in bf16 (8 significant
# bits: each rounding is off by at most 2^-8 of the value), each rounded once from a value
# that is itself a rounded product chain, accumulated in fp32. Its error against the FP64
# backward (given the same logits and routes) is bounded with every operand replaced by
# the magnitude of its own chain:
#   dy = bf16(w * dout)            |dy| <= |w| |dout|
#   dh = dy . W2 (fp32)             mag(dh) = |dy| . |W2|
#   dg = bf16(dh * u * silu'(g)),   mag(dg) = mag(dh) |u silu'(g)|,  mag(du) = mag(dh) |silu(g)|
#   du = bf16(dh * silu(g))
#   dW13 = [dg | du]^T . x          terms mag(dgu)[r, m] |x[r, c]|
#   dW2  = dy^T . h, h = bf16(a)    terms |dy[r, m]| |a[r, c]|
# (1) Worst case: two bf16 roundings on the chain (2 * 2^-8) plus fp32 accumulation over R
#     rows (R * 2^-24, 1.2e-4 at R = 2000) stay below 2^-7 (1 + 2 %) of the linear sum
#     S = sum_r |terms|: the bound 2^-6 S leaves a factor of two.
# (2) Cancellation makes S loose where an expert has many rows (a wrong element of typical
#     size can hide below it), so a second bound uses root-sum-squares Q = sqrt(sum_r
#     t_r^2) of "typical" term sizes t_r, whose operands are the value itself plus the
#     root-sum-square of the product that made it (e.g. typ(dh) = |dh| + sqrt(dy^2 .
#     W2^2)): rounding errors of different terms are independent, each within 2^-7 of its
#     typical size with a standard deviation below 2^-7 / sqrt(3), so the error sum has a
#     standard deviation below 0.0046 Q; the bound 2^-3 Q is 27 of those, while an element
#     taken from the wrong row or column is off by about Q.
# The router's chain starts from the routing-weight gradient dw_j = dot32(dout, y): y is a
# bf16 product of the bf16 h (its error <= 2^-7 of mag(y) = |h| . |W2|^T), so dw carries
# 2^-7 of mag(dw) = |dout| . mag(y); the score and renormalisation steps carry it linearly
# into mag(dlogits), which is rounded to bf16 once (2^-8) and contracted with x over T
# tokens in fixed chunks (T * 2^-24): below 0.012 S at T = 4096, so the bound 2^-5 S; the
# typical sizes follow the same chain (typ(y) = |y| + sqrt(h^2 . W2^2), typ(dw) = |dw| +
# sqrt(dout^2 . typ(y)^2)) and the bound is 2^-2 Q (three roundings deep).
WGRAD_EXPERT_C = 2.0 ** -6
WGRAD_EXPERT_CQ = 2.0 ** -3
WGRAD_ROUTER_C = 2.0 ** -5
WGRAD_ROUTER_CQ = 2.0 ** -2


def _sigma64(z):
    return 1.0 / (1.0 + np.exp(-z))


def _lin_rss(a, b):
    """(sum_r |a[r, m]| |b[r, c]|, sqrt(sum_r a[r, m]^2 b[r, c]^2)) for a, b >= 0."""
    return a.T @ b, np.sqrt((a * a).T @ (b * b))


def wgrad_scales64(dout, x, logits, w13, w2, ids, score_fn, renorm, route_scale, mask=None,
                   w13_s=None, w2_s=None, experts=()):
    """Magnitude sums of the weight gradients' terms (see above), in double, for the given
    logits and routes: {name: (S, Q)} for names "dw13[e]", "dw2[e]" (e in `experts`),
    "dw_router" and, with a shared expert, "dw13_s", "dw2_s". w13/w2 are indexable per
    expert (float64 arrays); the router's sums need every routed row."""
    from oracle import backward64 as B
    x = np.asarray(x, np.float64)
    ids = np.asarray(ids, np.int64)
    T, H = x.shape
    K = ids.shape[1]
    kept = np.ones(T, bool) if mask is None else np.asarray(mask) != 0
    ad = np.where(kept[:, None], np.abs(np.asarray(dout, np.float64)), 0.0)
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
    dwmag = np.zeros((T, K))     # linear magnitude of dw
    dwtyp = np.zeros((T, K))     # typical size of dw
    dsgn = np.where(kept[:, None], np.asarray(dout, np.float64), 0.0)
    res = {}
    for e in np.unique(ids[valid]):
        tt, jj = np.nonzero((ids == e) & kept[:, None])
        if tt.size == 0:
            continue
        w13_e, w2_e = np.asarray(w13[e], np.float64), np.asarray(w2[e], np.float64)
        I = w13_e.shape[0] // 2
        gu = x[tt] @ w13_e.T
        g, u = gu[:, :I], gu[:, I:]
        sg = _sigma64(g)
        a = g * sg * u
        aa = np.abs(a)
        aw2 = np.abs(w2_e)
        dwmag[tt, jj] = np.einsum("nh,nh->n", ad[tt], aa @ aw2.T)
        ytyp = np.abs(a @ w2_e.T) + np.sqrt((a * a) @ (w2_e * w2_e).T)
        dwtyp[tt, jj] = (np.abs(np.einsum("nh,nh->n", dsgn[tt], a @ w2_e.T))
                         + np.sqrt(np.einsum("nh,nh->n", ad[tt] ** 2, ytyp ** 2)))
        if int(e) in experts:
            dy = np.abs(w[tt, jj])[:, None] * ad[tt]
            dh = dy @ aw2
            dht = np.abs((w[tt, jj][:, None] * dsgn[tt]) @ w2_e) + np.sqrt((dy * dy) @ (w2_e * w2_e))
            fg, fu = np.abs(u * sg * (1.0 + g * (1.0 - sg))), np.abs(g * sg)
            S13 = np.concatenate([dh * fg, dh * fu], axis=1).T @ ax[tt]
            t = np.concatenate([dht * fg, dht * fu], axis=1)
            Q13 = np.sqrt((t * t).T @ (ax[tt] * ax[tt]))
            res[f"dw13[{int(e)}]"] = (S13, Q13)
            res[f"dw2[{int(e)}]"] = (dy.T @ aa, np.sqrt((dy * dy).T @ (aa * aa)))
    # router: magnitudes through the renormalisation and the score function
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

    dl_lin, dl_typ = dlogits_mag(dwmag), dlogits_mag(dwtyp)
    res["dw_router"] = (dl_lin.T @ ax, np.sqrt((dl_typ * dl_typ).T @ (ax * ax)))
    if w13_s is not None:
        w13s, w2s = np.asarray(w13_s, np.float64), np.asarray(w2_s, np.float64)
        Is = w13s.shape[0] // 2
        gu = x @ w13s.T
        g, u = gu[:, :Is], gu[:, Is:]
        sg = _sigma64(g)
        dh = ad @ np.abs(w2s)
        dht = np.abs(dsgn @ w2s) + np.sqrt((ad * ad) @ (w2s * w2s))
        fg, fu = np.abs(u * sg * (1.0 + g * (1.0 - sg))), np.abs(g * sg)
        t = np.concatenate([dht * fg, dht * fu], axis=1)
        res["dw13_s"] = (np.concatenate([dh * fg, dh * fu], axis=1).T @ ax,
                         np.sqrt((t * t).T @ (ax * ax)))
        aa = np.abs(g * sg * u)
        res["dw2_s"] = (ad.T @ aa, np.sqrt((ad * ad).T @ (aa * aa)))
    return res


def assert_within_scales(gpu, ref, scales, c, cq, what):
    """|gpu - ref| <= c * S and <= cq * Q element by element (S, Q = linear and
    root-sum-square magnitude sums of the element's terms). Returns the largest fraction
    of either bound used."""
    g = np.asarray(gpu, np.float64)
    err = np.abs(g - ref)
    used = 0.0
    for lim, name in ((c * scales[0] + 1e-30, f"{c:.3g} x linear sum"),
                      (cq * scales[1] + 1e-30, f"{cq:.3g} x root-sum-square")):
        r = err / lim
        i = np.unravel_index(np.argmax(r), r.shape)
        if r[i] > 1.0:
            raise AssertionError(f"{what}: {int((r > 1).sum())} of {r.size} elements beyond "
                                 f"{name}; worst {i}: gpu {g[i]:.6g} ref {ref[i]:.6g}")
        used = max(used, float(r[i]))
    return used
